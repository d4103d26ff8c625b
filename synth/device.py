"""Device-side filler for the seeded synthetic inputs (see ``synth/__init__.py``).

Fills multi-gigabyte unsharded KV sources and queries directly in HBM with
values bit-identical to the numpy generator.  Used by the GPU tests and the
benchmark; it draws numbers only.
"""
from __future__ import annotations

import ctypes as C
import os
import subprocess

import torch

from . import GQA, Workload

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "synth_fill.cu")
_LIB = os.path.join(_HERE, "libdcp_synth.so")
_lib = None


def build(force: bool = False) -> str:
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        tmp = _LIB + f".tmp{os.getpid()}"
        subprocess.check_call(["/usr/local/cuda/bin/nvcc", "-gencode", "arch=compute_100a,code=sm_100a", "-O3",
                               "-std=c++17", "-Xcompiler", "-fPIC", "-Xcompiler", "-fvisibility=hidden", "-shared",
                               "-o", tmp, _SRC])
        os.replace(tmp, _LIB)
    return _LIB


def _load():
    global _lib
    if _lib is None:
        if not os.path.exists(_LIB):
            raise ImportError(f"{_LIB} missing; build it with synth.device.build()")
        lib = C.CDLL(_LIB)
        lib.synth_fill.restype = C.c_int
        lib.synth_fill.argtypes = [C.c_void_p, C.c_void_p, C.c_int, C.c_int, C.c_int, C.c_int, C.c_uint64,
                                   C.c_double, C.c_int64, C.c_int, C.c_void_p]
        _lib = lib
    return _lib


def _fill(dst: torch.Tensor, cu, B, kind, H, d, seed, amp, rows):
    sms = torch.cuda.get_device_properties(dst.device).multi_processor_count
    rc = _load().synth_fill(dst.data_ptr(), 0 if cu is None else cu.data_ptr(), B, kind, H, d, seed, amp, rows,
                            sms, torch.cuda.current_stream(dst.device).cuda_stream)
    if rc != 0:
        raise RuntimeError("synth_fill launch failed")


def cu_seqlens(w: Workload, device) -> torch.Tensor:
    cu = [0]
    for n in w.seq_lens:
        cu.append(cu[-1] + int(n))
    return torch.tensor(cu, dtype=torch.int64, device=device)


def query(w: Workload, device) -> torch.Tensor:
    """q[B][Hq][d_qk] bf16 on the device; q[B][q_len][Hq][d_qk] when the workload has q_len > 1."""
    rows = w.q_len * w.num_q_heads  # per request, in the order of Workload.queries
    shape = (w.batch, w.num_q_heads, w.head_dim_qk) if w.q_len == 1 else \
        (w.batch, w.q_len, w.num_q_heads, w.head_dim_qk)
    q = torch.empty(shape, dtype=torch.bfloat16, device=device)
    _fill(q, None, w.batch, 2, rows, w.head_dim_qk, w.seed, w.q_amp, w.batch * rows)
    return q


def kv_source(w: Workload, device, cu: torch.Tensor = None) -> torch.Tensor:
    """Unsharded KV rows of all requests: GQA [T][2][Hkv][d], MLA [T][d_qk] (bf16)."""
    if cu is None:
        cu = cu_seqlens(w, device)
    T = w.total_tokens
    if w.layout == GQA:
        src = torch.empty((T, 2, w.num_kv_heads, w.head_dim_qk), dtype=torch.bfloat16, device=device)
        _fill(src, cu, w.batch, 0, w.num_kv_heads, w.head_dim_qk, w.seed, w.kv_amp, T)
    else:
        src = torch.empty((T, w.head_dim_qk), dtype=torch.bfloat16, device=device)
        _fill(src, cu, w.batch, 1, 1, w.head_dim_qk, w.seed, w.kv_amp, T)
    return src
