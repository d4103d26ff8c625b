"""ctypes binding of ``libdcp.so`` (the C ABI declared in ``include/dcp.h``).

Argument marshalling only: every computation runs in the CUDA library.  The
functions carry the C names.  Device buffers are passed as torch tensors (or
raw integer addresses); host arrays as numpy arrays or Python sequences.
``stream`` defaults to torch's current CUDA stream.

Importing this module fails loudly if the compiled library is missing: there
is no fallback implementation.
"""
from __future__ import annotations

import ctypes as C
import os
from typing import Optional, Sequence, Tuple

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libdcp.so")

DCP_OK, DCP_ERR_INVALID_ARG, DCP_ERR_UNSUPPORTED, DCP_ERR_CAPACITY, DCP_ERR_CUDA, DCP_ERR_DEVICE = range(6)
DCP_LAYOUT_GQA, DCP_LAYOUT_MLA = 0, 1
DCP_KV_BF16, DCP_KV_FP8_E4M3 = 0, 1
DCP_SHARD_INTERLEAVED, DCP_SHARD_CONTIGUOUS = 0, 1

EXPORTED = ["dcp_version", "dcp_status_string", "dcp_block_table_extent", "dcp_build_block_table",
            "dcp_block_table_extent_rule", "dcp_build_block_table_rule",
            "dcp_kv_page_bytes", "dcp_place_kv", "dcp_decode_workspace_bytes", "dcp_workspace_init",
            "dcp_decode_partial", "dcp_decode_partial_all", "dcp_lse_merge", "dcp_read_device_error",
            "dcp_validate_config", "dcp_decode_partial_all_noalloc", "dcp_noalloc_read_device_error",
            "dcp_grow_block_table", "dcp_append_kv", "dcp_host_step_staging_bytes", "dcp_decode_step_host",
            "dcp_owner_chunk_floats", "dcp_decode_partial_owner_major", "dcp_check_wait_timeout",
            "dcp_decode_partial_to_owners", "dcp_ipc_handle_bytes", "dcp_ipc_export", "dcp_ipc_open",
            "dcp_ipc_close"]


class DcpError(RuntimeError):
    def __init__(self, fn: str, status: int):
        super().__init__(f"{fn} failed: {status_string(status)} ({status})")
        self.status = status


class dcp_attn_desc(C.Structure):
    _fields_ = [("layout", C.c_int32), ("batch", C.c_int32), ("num_q_heads", C.c_int32),
                ("num_kv_heads", C.c_int32), ("head_dim_qk", C.c_int32), ("head_dim_v", C.c_int32),
                ("block_size", C.c_int32), ("max_local_blocks", C.c_int32), ("softmax_scale", C.c_float),
                ("q_len", C.c_int32), ("kv_dtype", C.c_int32), ("k_scale", C.c_float), ("v_scale", C.c_float),
                ("shard_rule", C.c_int32)]


def _load() -> C.CDLL:
    if not os.path.exists(LIB_PATH):
        raise ImportError(f"{LIB_PATH} is missing: build it with `python -m sequence_sharded_decode_paged_b200.build`"
                          " (there is no non-CUDA fallback)")
    lib = C.CDLL(LIB_PATH)
    p, i32, u64, sz = C.c_void_p, C.c_int32, C.c_uint64, C.c_size_t
    sig = {
        "dcp_version": (i32, []),
        "dcp_status_string": (C.c_char_p, [C.c_int]),
        "dcp_block_table_extent": (C.c_int, [p, i32, i32, i32, p, p]),
        "dcp_build_block_table": (C.c_int, [p, i32, i32, i32, u64, i32, p, p]),
        "dcp_block_table_extent_rule": (C.c_int, [p, i32, i32, i32, i32, p, p]),
        "dcp_build_block_table_rule": (C.c_int, [p, i32, i32, i32, i32, u64, i32, p, p]),
        "dcp_kv_page_bytes": (sz, [p]),
        "dcp_place_kv": (C.c_int, [p, i32, p, p, p, p, p, p, p, p]),
        "dcp_decode_workspace_bytes": (sz, [p, i32]),
        "dcp_workspace_init": (C.c_int, [p, sz, p]),
        "dcp_decode_partial": (C.c_int, [p, p, p, i32, p, p, i32, i32, p, p, p, sz, p]),
        "dcp_decode_partial_all": (C.c_int, [p, p, p, p, p, p, i32, p, p, p, sz, p]),
        "dcp_lse_merge": (C.c_int, [p, p, i32, i32, i32, p, p, p]),
        "dcp_read_device_error": (C.c_int, [p, p, p]),
        "dcp_check_wait_timeout": (C.c_int, [p, p]),
        "dcp_validate_config": (C.c_int, [i32, i32, i32, i32]),
        "dcp_decode_partial_all_noalloc": (C.c_int, [p, p, p, p, p, p, i32, p, p, p]),
        "dcp_noalloc_read_device_error": (C.c_int, [p, p]),
        "dcp_host_step_staging_bytes": (sz, [p, i32]),
        "dcp_owner_chunk_floats": (sz, [p, i32]),
        "dcp_decode_partial_owner_major": (C.c_int, [p, p, p, i32, p, p, i32, i32, i32, p, p, sz, p]),
        "dcp_decode_partial_to_owners": (C.c_int, [p, p, p, i32, p, p, i32, i32, i32, p, p, sz, p]),
        "dcp_ipc_handle_bytes": (sz, []),
        "dcp_ipc_export": (C.c_int, [p, p, p]),
        "dcp_ipc_open": (C.c_int, [p, p]),
        "dcp_ipc_close": (C.c_int, [p]),
        "dcp_decode_step_host": (C.c_int, [p, i32, p, p, p, p, p, p, sz, p, sz, p, p, p]),
        "dcp_grow_block_table": (C.c_int, [p, p, i32, i32, i32, i32, p, p, p, p]),
        "dcp_append_kv": (C.c_int, [p, i32, p, p, p, p, p, p, p, p]),
    }
    for name, (res, args) in sig.items():
        fn = getattr(lib, name)
        fn.restype = res
        fn.argtypes = args
    return lib


_lib = _load()


def status_string(status: int) -> str:
    return _lib.dcp_status_string(status).decode()


def _check(fn: str, status: int) -> None:
    if status != DCP_OK:
        raise DcpError(fn, status)


def _addr(x) -> Optional[int]:
    if x is None:
        return None
    if isinstance(x, int):
        return x
    return int(x.data_ptr())


def _stream(stream) -> Optional[int]:
    if stream is not None:
        return int(stream) if isinstance(stream, int) else int(stream.cuda_stream)
    import torch
    return int(torch.cuda.current_stream().cuda_stream) if torch.cuda.is_available() else None


def _haddr(x) -> Optional[int]:
    """Address of a host buffer: a numpy array, a CPU torch tensor or a raw integer address."""
    if x is None:
        return None
    if isinstance(x, int):
        return x
    if isinstance(x, np.ndarray):
        if not x.flags.c_contiguous:
            raise TypeError("host arrays must be C-contiguous")
        return int(x.ctypes.data)
    if x.is_cuda:
        raise TypeError("expected a host buffer, got a CUDA tensor")
    return int(x.data_ptr())


def _ptr_array(xs):
    return (C.c_void_p * len(xs))(*[_addr(x) for x in xs])


def _i32(a) -> np.ndarray:
    return np.ascontiguousarray(a, dtype=np.int32)


def make_desc(layout: int, batch: int, num_q_heads: int, num_kv_heads: int, head_dim_qk: int, head_dim_v: int,
              block_size: int, max_local_blocks: int, softmax_scale: float, q_len: int = 1,
              kv_dtype: int = 0, k_scale: float = 1.0, v_scale: float = 1.0, shard_rule: int = 0) -> dcp_attn_desc:
    return dcp_attn_desc(layout, batch, num_q_heads, num_kv_heads, head_dim_qk, head_dim_v, block_size,
                         max_local_blocks, softmax_scale, q_len, kv_dtype, k_scale, v_scale, shard_rule)


# --------------------------------------------------------------------------- host calls
def dcp_version() -> int:
    return _lib.dcp_version()


def dcp_block_table_extent(seq_lens: Sequence[int], block_size: int, D: int, shard_rule: int = 0):
    sl = _i32(seq_lens)
    mlb = C.c_int32(0)
    pages = np.zeros(D, dtype=np.int32)
    if shard_rule == DCP_SHARD_INTERLEAVED:
        rc = _lib.dcp_block_table_extent(sl.ctypes.data, sl.shape[0], block_size, D, C.addressof(mlb),
                                         pages.ctypes.data)
    else:
        rc = _lib.dcp_block_table_extent_rule(sl.ctypes.data, sl.shape[0], block_size, D, shard_rule,
                                              C.addressof(mlb), pages.ctypes.data)
    _check("dcp_block_table_extent", rc)
    return int(mlb.value), pages


def dcp_build_block_table(seq_lens: Sequence[int], block_size: int, D: int, perm_seed: int = 0,
                          max_local_blocks: Optional[int] = None, shard_rule: int = 0):
    """Returns ``(tables int32[D][B][max_local_blocks], local_len int32[D][B])``."""
    sl = _i32(seq_lens)
    if max_local_blocks is None:
        max_local_blocks = max(1, dcp_block_table_extent(sl, block_size, D, shard_rule)[0])
    tables = np.empty((D, sl.shape[0], max_local_blocks), dtype=np.int32)
    local_len = np.empty((D, sl.shape[0]), dtype=np.int32)
    if shard_rule == DCP_SHARD_INTERLEAVED:
        rc = _lib.dcp_build_block_table(sl.ctypes.data, sl.shape[0], block_size, D, perm_seed, max_local_blocks,
                                        tables.ctypes.data, local_len.ctypes.data)
    else:
        rc = _lib.dcp_build_block_table_rule(sl.ctypes.data, sl.shape[0], block_size, D, shard_rule, perm_seed,
                                             max_local_blocks, tables.ctypes.data, local_len.ctypes.data)
    _check("dcp_build_block_table", rc)
    return tables, local_len


def dcp_grow_block_table(old_seq_lens, new_seq_lens, block_size: int, D: int, tables: np.ndarray,
                         local_len: Optional[np.ndarray], next_page: np.ndarray, pool_pages) -> None:
    """Grow ``tables`` (int32[D][B][mlb]), ``local_len`` and ``next_page`` (int32[D]) in place."""
    o, n, pp = _i32(old_seq_lens), _i32(new_seq_lens), _i32(pool_pages)
    for a in (tables, next_page) + ((local_len,) if local_len is not None else ()):
        if a.dtype != np.int32 or not a.flags.c_contiguous:
            raise TypeError("tables, local_len and next_page must be C-contiguous int32 arrays")
    _check("dcp_grow_block_table", _lib.dcp_grow_block_table(
        o.ctypes.data, n.ctypes.data, o.shape[0], block_size, D, tables.shape[2], tables.ctypes.data,
        None if local_len is None else local_len.ctypes.data, next_page.ctypes.data, pp.ctypes.data))


def dcp_kv_page_bytes(desc: dcp_attn_desc) -> int:
    return int(_lib.dcp_kv_page_bytes(C.byref(desc)))


def dcp_decode_workspace_bytes(desc: dcp_attn_desc, D: int) -> int:
    return int(_lib.dcp_decode_workspace_bytes(C.byref(desc), D))


def dcp_validate_config(tp: int, dcp: int, num_kv_heads: int, layout: int) -> int:
    """Returns the raw status: DCP_OK (allowed), DCP_ERR_UNSUPPORTED (not allowed) or DCP_ERR_INVALID_ARG."""
    return _lib.dcp_validate_config(tp, dcp, num_kv_heads, layout)


# --------------------------------------------------------------------------- device calls
def dcp_place_kv(desc: dcp_attn_desc, D: int, kv_src, cu_seqlens, seq_lens, tables, kv_pools, pool_pages,
                 device_error=None, stream=None) -> None:
    pp = _i32(pool_pages)
    _check("dcp_place_kv", _lib.dcp_place_kv(
        C.byref(desc), D, _addr(kv_src), _addr(cu_seqlens), _addr(seq_lens), _ptr_array(tables),
        _ptr_array(kv_pools), pp.ctypes.data, _addr(device_error), _stream(stream)))


def dcp_append_kv(desc: dcp_attn_desc, D: int, kv_new, cu_rows, first_pos, tables, kv_pools, pool_pages,
                  device_error=None, stream=None) -> None:
    pp = _i32(pool_pages)
    _check("dcp_append_kv", _lib.dcp_append_kv(
        C.byref(desc), D, _addr(kv_new), _addr(cu_rows), _addr(first_pos), _ptr_array(tables), _ptr_array(kv_pools),
        pp.ctypes.data, _addr(device_error), _stream(stream)))


def dcp_workspace_init(workspace, workspace_bytes: Optional[int] = None, stream=None) -> None:
    n = workspace_bytes if workspace_bytes is not None else workspace.numel() * workspace.element_size()
    _check("dcp_workspace_init", _lib.dcp_workspace_init(_addr(workspace), n, _stream(stream)))


def dcp_decode_partial(desc: dcp_attn_desc, q, kv_pool, pool_pages: int, table, seq_lens, shard: int, D: int, O_i,
                       LSE_i, workspace, workspace_bytes: Optional[int] = None, stream=None) -> None:
    n = workspace_bytes if workspace_bytes is not None else workspace.numel() * workspace.element_size()
    _check("dcp_decode_partial", _lib.dcp_decode_partial(
        C.byref(desc), _addr(q), _addr(kv_pool), pool_pages, _addr(table), _addr(seq_lens), shard, D, _addr(O_i),
        _addr(LSE_i), _addr(workspace), n, _stream(stream)))


def dcp_owner_chunk_floats(desc: dcp_attn_desc, n_owners: int) -> int:
    return int(_lib.dcp_owner_chunk_floats(C.byref(desc), n_owners))


def dcp_decode_partial_owner_major(desc: dcp_attn_desc, q, kv_pool, pool_pages: int, table, seq_lens, shard: int,
                                   D: int, n_owners: int, send, workspace, workspace_bytes: Optional[int] = None,
                                   stream=None) -> None:
    n = workspace_bytes if workspace_bytes is not None else workspace.numel() * workspace.element_size()
    _check("dcp_decode_partial_owner_major", _lib.dcp_decode_partial_owner_major(
        C.byref(desc), _addr(q), _addr(kv_pool), pool_pages, _addr(table), _addr(seq_lens), shard, D, n_owners,
        _addr(send), _addr(workspace), n, _stream(stream)))


def dcp_decode_partial_to_owners(desc: dcp_attn_desc, q, kv_pool, pool_pages: int, table, seq_lens, shard: int,
                                 D: int, owner_chunks, workspace, workspace_bytes: Optional[int] = None,
                                 stream=None) -> None:
    """``owner_chunks``: one chunk per owner, each a device tensor or a raw device address (int), e.g. a
    peer GPU's buffer mapped with ``dcp_ipc_open``."""
    n = workspace_bytes if workspace_bytes is not None else workspace.numel() * workspace.element_size()
    ptrs = (C.c_void_p * len(owner_chunks))(*[c if isinstance(c, int) else _addr(c) for c in owner_chunks])
    _check("dcp_decode_partial_to_owners", _lib.dcp_decode_partial_to_owners(
        C.byref(desc), _addr(q), _addr(kv_pool), pool_pages, _addr(table), _addr(seq_lens), shard, D,
        len(owner_chunks), ptrs, _addr(workspace), n, _stream(stream)))


def dcp_ipc_handle_bytes() -> int:
    return int(_lib.dcp_ipc_handle_bytes())


def dcp_ipc_export(device_tensor) -> Tuple[bytes, int]:
    """(handle of the allocation holding the tensor's first byte, byte offset inside it)."""
    h = C.create_string_buffer(dcp_ipc_handle_bytes())
    off = C.c_uint64(0)
    _check("dcp_ipc_export", _lib.dcp_ipc_export(_addr(device_tensor), h, C.byref(off)))
    return h.raw, int(off.value)


def dcp_ipc_open(handle: bytes) -> int:
    """Maps another process's allocation; returns its base address in this process."""
    h = C.create_string_buffer(handle, len(handle))
    base = C.c_void_p(0)
    _check("dcp_ipc_open", _lib.dcp_ipc_open(h, C.byref(base)))
    return int(base.value)


def dcp_ipc_close(base: int) -> None:
    _check("dcp_ipc_close", _lib.dcp_ipc_close(C.c_void_p(base)))


def dcp_decode_partial_all(desc: dcp_attn_desc, q, kv_pools, pool_pages, tables, seq_lens, D: int, O_parts,
                           LSE_parts, workspace, workspace_bytes: Optional[int] = None, stream=None) -> None:
    n = workspace_bytes if workspace_bytes is not None else workspace.numel() * workspace.element_size()
    pp = _i32(pool_pages)
    _check("dcp_decode_partial_all", _lib.dcp_decode_partial_all(
        C.byref(desc), _addr(q), _ptr_array(kv_pools), pp.ctypes.data, _ptr_array(tables), _addr(seq_lens), D,
        _ptr_array(O_parts), _ptr_array(LSE_parts), _addr(workspace), n, _stream(stream)))


def dcp_decode_partial_all_noalloc(desc: dcp_attn_desc, q, kv_pools, pool_pages, tables, seq_lens, D: int,
                                   O_parts, LSE_parts, stream=None) -> None:
    """GQA all-shard partials without a workspace (the library's own fixed scratch; see include/dcp.h)."""
    pp = _i32(pool_pages)
    _check("dcp_decode_partial_all_noalloc", _lib.dcp_decode_partial_all_noalloc(
        C.byref(desc), _addr(q), _ptr_array(kv_pools), pp.ctypes.data, _ptr_array(tables), _addr(seq_lens), D,
        _ptr_array(O_parts), _ptr_array(LSE_parts), _stream(stream)))


def dcp_noalloc_read_device_error(stream=None) -> int:
    """Read and clear the status word of the allocation-free call's scratch (synchronous)."""
    err = C.c_int32(0)
    _check("dcp_noalloc_read_device_error", _lib.dcp_noalloc_read_device_error(C.addressof(err), _stream(stream)))
    return int(err.value)


def dcp_host_step_staging_bytes(desc: dcp_attn_desc, D: int) -> int:
    return int(_lib.dcp_host_step_staging_bytes(C.byref(desc), D))


def dcp_decode_step_host(desc: dcp_attn_desc, D: int, host_q, host_seq_lens, host_tables, kv_pools, pool_pages,
                         staging, workspace, host_O, host_LSE=None, staging_bytes: Optional[int] = None,
                         workspace_bytes: Optional[int] = None, stream=None) -> None:
    """One decode step with host inputs and outputs (see include/dcp.h); asynchronous on ``stream``."""
    sb = staging_bytes if staging_bytes is not None else staging.numel() * staging.element_size()
    wb = workspace_bytes if workspace_bytes is not None else workspace.numel() * workspace.element_size()
    pp = _i32(pool_pages)
    _check("dcp_decode_step_host", _lib.dcp_decode_step_host(
        C.byref(desc), D, _haddr(host_q), _haddr(host_seq_lens), _haddr(host_tables), _ptr_array(kv_pools),
        pp.ctypes.data, _addr(staging), sb, _addr(workspace), wb, _haddr(host_O), _haddr(host_LSE),
        _stream(stream)))


def dcp_lse_merge(O_parts, LSE_parts, D: int, rows: int, d_v: int, O, LSE_out=None, stream=None) -> None:
    _check("dcp_lse_merge", _lib.dcp_lse_merge(
        _ptr_array(O_parts), _ptr_array(LSE_parts), D, rows, d_v, _addr(O), _addr(LSE_out), _stream(stream)))


def dcp_check_wait_timeout(workspace, stream=None) -> None:
    """Launch the bounded-wait diagnostic: sets the timeout bit of the workspace status word after
    the wait limit (asynchronous; read it back with dcp_read_device_error)."""
    _check("dcp_check_wait_timeout", _lib.dcp_check_wait_timeout(_addr(workspace), _stream(stream)))


def dcp_read_device_error(workspace, stream=None) -> int:
    err = C.c_int32(0)
    _check("dcp_read_device_error", _lib.dcp_read_device_error(_addr(workspace), C.addressof(err), _stream(stream)))
    return int(err.value)
