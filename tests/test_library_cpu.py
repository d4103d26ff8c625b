"""Host-side checks of the C-ABI library (no GPU needed).

The shard tables built by the library are compared bit for bit with the
oracle's independent construction; the library must export every symbol that
include/dcp.h declares; argument errors must come back as status codes.
"""
import ctypes
import os
import re

import numpy as np
import pytest

import oracle
from helpers import ROOT, golden
from sequence_sharded_decode_paged_b200 import dcp

HEADER = os.path.join(ROOT, "include", "dcp.h")


def declared_symbols():
    text = open(HEADER, encoding="utf-8").read()
    return sorted(set(re.findall(r"DCP_API\s+[\w\s\*]*?\b(dcp_\w+)\s*\(", text)))


def test_header_declares_the_binding_surface():
    assert declared_symbols() == sorted(dcp.EXPORTED)


def test_library_exports_every_declared_symbol():
    lib = ctypes.CDLL(dcp.LIB_PATH)
    for name in declared_symbols():
        assert hasattr(lib, name), name
    assert dcp.dcp_version() >= 100


def test_owner_calls_check_their_arguments_on_the_host():
    # refused before anything is launched (fake, aligned device addresses; no GPU needed): more than 16
    # owners, a null or misaligned owner chunk
    lib = ctypes.CDLL(dcp.LIB_PATH)
    desc = dcp.make_desc(dcp.DCP_LAYOUT_GQA, 2, 32, 4, 64, 64, 16, 8, 0.125)
    fake = [0x10000 * (i + 1) for i in range(8)]
    args = lambda n_owners, chunks: (ctypes.byref(desc), fake[0], fake[1], 4, fake[2], fake[3], 0, 1, n_owners,
                                     chunks, fake[4], 1 << 40, None)
    to_owners = lib.dcp_decode_partial_to_owners
    to_owners.argtypes = [ctypes.c_void_p] * 3 + [ctypes.c_int32] + [ctypes.c_void_p] * 2 + [ctypes.c_int32] * 3 + \
        [ctypes.c_void_p, ctypes.c_void_p, ctypes.c_size_t, ctypes.c_void_p]
    ptrs = lambda xs: (ctypes.c_void_p * len(xs))(*xs)
    assert to_owners(*args(32, ptrs([fake[5]] * 32))) == dcp.DCP_ERR_INVALID_ARG   # 32 owners > 16
    assert to_owners(*args(2, ptrs([fake[5], 0]))) == dcp.DCP_ERR_INVALID_ARG       # null chunk
    assert to_owners(*args(2, ptrs([fake[5], fake[6] + 4]))) == dcp.DCP_ERR_INVALID_ARG  # misaligned chunk
    assert to_owners(*args(3, ptrs([fake[5]] * 3))) == dcp.DCP_ERR_INVALID_ARG      # 3 does not divide 32 heads
    major = lib.dcp_decode_partial_owner_major
    major.argtypes = to_owners.argtypes
    assert major(*args(32, fake[5])) == dcp.DCP_ERR_INVALID_ARG                      # 32 owners > 16


def test_ipc_helpers_check_their_arguments_on_the_host():
    # a CUDA IPC handle is 64 bytes; null arguments come back as status codes before any CUDA call
    assert dcp.dcp_ipc_handle_bytes() == 64
    lib = ctypes.CDLL(dcp.LIB_PATH)
    off = ctypes.c_uint64(0)
    buf = ctypes.create_string_buffer(64)
    assert lib.dcp_ipc_export(None, buf, ctypes.byref(off)) == dcp.DCP_ERR_INVALID_ARG
    assert lib.dcp_ipc_open(None, ctypes.byref(ctypes.c_void_p())) == dcp.DCP_ERR_INVALID_ARG
    assert lib.dcp_ipc_close(None) == dcp.DCP_ERR_INVALID_ARG


@pytest.mark.parametrize("D", [1, 2, 3, 4, 8, 16])
@pytest.mark.parametrize("bs", [16, 64])
@pytest.mark.parametrize("perm", [0, 99])
def test_tables_bit_exact_vs_oracle(D, bs, perm):
    rng = np.random.default_rng(D * 1000 + bs + perm)
    seq_lens = list(rng.integers(0, 3000, size=9)) + [0, 1, bs, bs + 1, D * bs, D * bs + 1]
    t_lib, l_lib = dcp.dcp_build_block_table(seq_lens, bs, D, perm)
    mlb, pages = dcp.dcp_block_table_extent(seq_lens, bs, D)
    t_or, l_or, p_or = oracle.block_tables(seq_lens, bs, D, perm_seed=perm, max_local_blocks=t_lib.shape[2])
    np.testing.assert_array_equal(t_lib, t_or)
    np.testing.assert_array_equal(l_lib, l_or)
    np.testing.assert_array_equal(pages, p_or)
    assert mlb == int((t_or >= 0).sum(axis=2).max())


@pytest.mark.parametrize("name", ["gqa_tiny", "gqa_70b", "mla_b32", "mla_long", "mla_mix"])
def test_tables_bit_exact_on_workloads(name):
    import synth
    w = synth.workload(name)
    for D in w.shards:
        t_lib, l_lib = dcp.dcp_build_block_table(w.seq_lens, w.block_size, D)
        t_or, l_or, _ = oracle.block_tables(w.seq_lens, w.block_size, D, max_local_blocks=t_lib.shape[2])
        np.testing.assert_array_equal(t_lib, t_or)
        np.testing.assert_array_equal(l_lib, l_or)


def test_table_capacity_and_argument_errors():
    with pytest.raises(dcp.DcpError) as e:
        dcp.dcp_build_block_table([100], 16, 2, 0, max_local_blocks=3)
    assert e.value.status == dcp.DCP_ERR_CAPACITY
    for args in [([5], 0, 2), ([5], 16, 0), ([5], 16, 17), ([-1], 16, 2)]:
        with pytest.raises(dcp.DcpError) as e:
            dcp.dcp_build_block_table(*args)
        assert e.value.status == dcp.DCP_ERR_INVALID_ARG


def test_validate_config_matches_page_examples():
    for row in golden("validate_config.txt"):
        layout, tp, dcp_, kvh, want = map(int, row)
        got = dcp.dcp_validate_config(tp, dcp_, kvh, layout)
        assert got == (dcp.DCP_OK if want else dcp.DCP_ERR_UNSUPPORTED), row
    assert dcp.dcp_validate_config(0, 1, 1, 0) == dcp.DCP_ERR_INVALID_ARG


def test_page_bytes_and_supported_shapes():
    d = dcp.make_desc(dcp.DCP_LAYOUT_GQA, 64, 64, 8, 128, 128, 16, 10, 0.1)
    assert dcp.dcp_kv_page_bytes(d) == 16 * oracle.kv_bytes_per_token(8, 128, 2)
    m = dcp.make_desc(dcp.DCP_LAYOUT_MLA, 4, 64, 1, 576, 512, 64, 10, 0.07)
    assert dcp.dcp_kv_page_bytes(m) == 64 * 576 * 2
    for bad in [dcp.make_desc(0, 1, 8, 2, 96, 96, 16, 1, 0.1),    # head_dim 96
                dcp.make_desc(0, 1, 8, 3, 64, 64, 16, 1, 0.1),    # Hq % Hkv != 0
                dcp.make_desc(0, 1, 64, 2, 64, 64, 16, 1, 0.1),   # G = 32 > 16
                dcp.make_desc(0, 1, 8, 2, 64, 64, 24, 1, 0.1),    # block 24
                dcp.make_desc(0, 1, 8, 2, 128, 128, 256, 1, 0.1),  # block 256 at head_dim 128
                dcp.make_desc(1, 1, 32, 1, 576, 512, 64, 1, 0.1)]:  # MLA with 32 heads
        assert dcp.dcp_kv_page_bytes(bad) == 0
        assert dcp.dcp_decode_workspace_bytes(bad, 2) == 0
    assert dcp.dcp_decode_workspace_bytes(d, 0) == 0
    assert dcp.dcp_decode_workspace_bytes(d, 4) > 0


def test_device_calls_reject_bad_arguments_before_launch():
    d = dcp.make_desc(dcp.DCP_LAYOUT_GQA, 2, 8, 2, 64, 64, 16, 9, 0.125)
    lib = ctypes.CDLL(dcp.LIB_PATH)
    lib.dcp_decode_partial.restype = ctypes.c_int
    null = ctypes.c_void_p(0)
    st = lib.dcp_decode_partial(ctypes.byref(d), null, null, 0, null, null, 0, 2, null, null, null,
                                ctypes.c_size_t(0), null)
    assert st == dcp.DCP_ERR_INVALID_ARG
    lib.dcp_lse_merge.restype = ctypes.c_int
    assert lib.dcp_lse_merge(null, null, 2, 4, 64, null, null, null) == dcp.DCP_ERR_INVALID_ARG
    lib.dcp_check_wait_timeout.restype = ctypes.c_int
    assert lib.dcp_check_wait_timeout(null, null) == dcp.DCP_ERR_INVALID_ARG


@pytest.mark.parametrize("D", [1, 2, 3, 4, 8])
def test_grow_block_table_bit_exact_vs_oracle(D):
    rng = np.random.default_rng(D + 40)
    bs, B, mlb = 16, 7, 64
    lens = rng.integers(0, 300, size=B).astype(np.int32)
    t_lib = np.full((D, B, mlb), -1, np.int32)
    l_lib = np.zeros((D, B), np.int32)
    n_lib = np.zeros(D, np.int32)
    t_or, l_or, n_or = t_lib.copy(), l_lib.copy(), n_lib.copy()
    pool = [10 ** 6] * D
    dcp.dcp_grow_block_table([0] * B, lens, bs, D, t_lib, l_lib, n_lib, pool)
    assert oracle.grow_tables([0] * B, lens, bs, D, t_or, l_or, n_or, pool) == 0
    for step in range(25):
        new = lens + rng.integers(0, 50, size=B).astype(np.int32) * (rng.random(B) < 0.7)
        dcp.dcp_grow_block_table(lens, new, bs, D, t_lib, l_lib, n_lib, pool)
        assert oracle.grow_tables(lens, new, bs, D, t_or, l_or, n_or, pool) == 0
        np.testing.assert_array_equal(t_lib, t_or)
        np.testing.assert_array_equal(l_lib, l_or)
        np.testing.assert_array_equal(n_lib, n_or)
        lens = new


def test_grow_from_empty_equals_build():
    lens = [100, 257, 0, 64, 1, 3000]
    for D in (1, 2, 4):
        t_b, l_b = dcp.dcp_build_block_table(lens, 16, D)
        t = np.full(t_b.shape, -1, np.int32)
        l = np.zeros(l_b.shape, np.int32)
        nxt = np.zeros(D, np.int32)
        dcp.dcp_grow_block_table([0] * len(lens), lens, 16, D, t, l, nxt, [10 ** 6] * D)
        np.testing.assert_array_equal(t, t_b)
        np.testing.assert_array_equal(l, l_b)
        assert list(nxt) == list(dcp.dcp_block_table_extent(lens, 16, D)[1])


def test_grow_errors_leave_tables_untouched():
    t = np.full((2, 1, 3), -1, np.int32)
    l = np.zeros((2, 1), np.int32)
    nxt = np.zeros(2, np.int32)
    with pytest.raises(dcp.DcpError) as e:
        dcp.dcp_grow_block_table([5], [3], 16, 2, t, l, nxt, [9, 9])
    assert e.value.status == dcp.DCP_ERR_INVALID_ARG
    with pytest.raises(dcp.DcpError) as e:
        dcp.dcp_grow_block_table([0], [16 * 3], 16, 2, t, l, nxt, [1, 9])  # shard 0 needs 2 pages, has 1
    assert e.value.status == dcp.DCP_ERR_CAPACITY
    with pytest.raises(dcp.DcpError) as e:
        dcp.dcp_grow_block_table([0], [16 * 7], 16, 2, t, l, nxt, [9, 9])  # local block 3 >= 3
    assert e.value.status == dcp.DCP_ERR_CAPACITY
    assert (t == -1).all() and (l == 0).all() and (nxt == 0).all()


def test_q_len_validation_and_workspace_growth():
    # q_len outside 1..4 is refused; a multi-token workspace holds q_len times the rows
    for ql in (0, 5, -1):
        desc = dcp.make_desc(dcp.DCP_LAYOUT_GQA, 1, 8, 2, 64, 64, 16, 4, 0.125, ql)
        assert dcp.dcp_decode_workspace_bytes(desc, 2) == 0
    base = dcp.dcp_decode_workspace_bytes(dcp.make_desc(dcp.DCP_LAYOUT_GQA, 4, 8, 2, 64, 64, 16, 4, 0.125, 1), 2)
    multi = dcp.dcp_decode_workspace_bytes(dcp.make_desc(dcp.DCP_LAYOUT_GQA, 4, 8, 2, 64, 64, 16, 4, 0.125, 4), 2)
    assert base > 0 and multi > base
    mla = dcp.dcp_decode_workspace_bytes(dcp.make_desc(dcp.DCP_LAYOUT_MLA, 4, 64, 1, 576, 512, 64, 4, 0.07, 3), 2)
    assert mla > 0


def test_descriptor_layout_matches_header():
    import ctypes
    assert ctypes.sizeof(dcp.dcp_attn_desc) == 14 * 4
    assert dcp.dcp_attn_desc.q_len.offset == 36
    assert dcp.dcp_attn_desc.v_scale.offset == 48


def test_fp8_page_bytes_and_rejections():
    # FP8 pools: GQA (head_dim 64 and 128) and MLA; a page is one byte per value.  The MLA latent is one
    # tensor, so its key and value scales must be the same number.
    assert dcp.dcp_kv_page_bytes(dcp.make_desc(dcp.DCP_LAYOUT_MLA, 1, 64, 1, 576, 512, 64, 1, 0.07, 1,
                                               dcp.DCP_KV_FP8_E4M3, 0.5, 0.5)) == 64 * 576
    unequal = dcp.make_desc(dcp.DCP_LAYOUT_MLA, 1, 64, 1, 576, 512, 64, 1, 0.07, 1, dcp.DCP_KV_FP8_E4M3, 1.0, 0.5)
    assert dcp.dcp_kv_page_bytes(unequal) == 0
    assert dcp.dcp_decode_workspace_bytes(unequal, 2) == 0
    assert dcp.dcp_kv_page_bytes(dcp.make_desc(dcp.DCP_LAYOUT_GQA, 1, 8, 2, 64, 64, 16, 1, 0.1, 1, dcp.DCP_KV_FP8_E4M3, 1.0, 1.0)) == \
        2 * 2 * 16 * 64
    assert dcp.dcp_kv_page_bytes(dcp.make_desc(dcp.DCP_LAYOUT_GQA, 1, 8, 2, 128, 128, 16, 1, 0.1, 1, dcp.DCP_KV_FP8_E4M3, 1.0, 1.0)) == \
        2 * 2 * 16 * 128
    for ks, vs in ((0.0, 1.0), (1.0, float("inf")), (-1.0, 1.0), (float("nan"), 1.0)):
        assert dcp.dcp_kv_page_bytes(dcp.make_desc(dcp.DCP_LAYOUT_GQA, 1, 8, 2, 128, 128, 16, 1, 0.1, 1,
                                                   dcp.DCP_KV_FP8_E4M3, ks, vs)) == 0
    assert dcp.dcp_kv_page_bytes(dcp.make_desc(dcp.DCP_LAYOUT_GQA, 1, 8, 2, 128, 128, 16, 1, 0.1, 1, 7)) == 0


@pytest.mark.parametrize("D", [1, 2, 3, 4, 8, 16])
@pytest.mark.parametrize("bs", [16, 64])
@pytest.mark.parametrize("perm", [0, 99])
def test_contiguous_tables_bit_exact_vs_oracle(D, bs, perm):
    rng = np.random.default_rng(D * 2000 + bs + perm)
    seq_lens = list(rng.integers(0, 3000, size=9)) + [0, 1, bs, bs + 1, D * bs, D * bs + 1, (D - 1) * bs + 1]
    C = dcp.DCP_SHARD_CONTIGUOUS
    t_lib, l_lib = dcp.dcp_build_block_table(seq_lens, bs, D, perm, shard_rule=C)
    mlb, pages = dcp.dcp_block_table_extent(seq_lens, bs, D, C)
    t_or, l_or, p_or = oracle.block_tables(seq_lens, bs, D, perm_seed=perm, max_local_blocks=t_lib.shape[2],
                                           rule=oracle.CONTIGUOUS)
    np.testing.assert_array_equal(t_lib, t_or)
    np.testing.assert_array_equal(l_lib, l_or)
    np.testing.assert_array_equal(pages, p_or)
    assert mlb == int((t_or >= 0).sum(axis=2).max())


def test_contiguous_rule_argument_checks():
    with pytest.raises(dcp.DcpError) as e:
        dcp.dcp_build_block_table([100], 16, 2, 0, shard_rule=2)
    assert e.value.status == dcp.DCP_ERR_INVALID_ARG
    bad = dcp.make_desc(dcp.DCP_LAYOUT_GQA, 1, 8, 2, 64, 64, 16, 4, 0.125, shard_rule=5)
    assert dcp.dcp_decode_workspace_bytes(bad, 2) == 0
    ok = dcp.make_desc(dcp.DCP_LAYOUT_GQA, 1, 8, 2, 64, 64, 16, 4, 0.125, shard_rule=dcp.DCP_SHARD_CONTIGUOUS)
    assert dcp.dcp_decode_workspace_bytes(ok, 2) > 0
    # contiguous tables cannot grow: appending is refused before anything runs
    with pytest.raises(dcp.DcpError) as e:
        dcp.dcp_append_kv(ok, 2, 16, 16, 16, [16, 16], [16, 16], [1, 1])
    assert e.value.status == dcp.DCP_ERR_UNSUPPORTED


@pytest.mark.parametrize("q_len", [1, 2, 3, 4])
@pytest.mark.parametrize("rule", [0, 1])
def test_descriptor_option_matrix(q_len, rule):
    # every supported combination of draft length, pool type and shard rule sizes its buffers; the shard
    # rule never changes them, and an FP8 page is half a bf16 page
    def desc(layout, kv_dtype, Hq=64, Hkv=8, d=128, bs=16):
        dv = 512 if layout == dcp.DCP_LAYOUT_MLA else d
        return dcp.make_desc(layout, 8, Hq, Hkv, d, dv, bs, 32, 0.1, q_len, kv_dtype, 0.5, 0.25, rule)
    g16, g8 = desc(0, 0), desc(0, 1)
    mla = desc(1, 0, 64, 1, 576, 64)
    assert dcp.dcp_kv_page_bytes(g8) * 2 == dcp.dcp_kv_page_bytes(g16) > 0
    assert dcp.dcp_kv_page_bytes(mla) == 64 * 576 * 2
    for dsc in (g16, g8, mla):
        ws = dcp.dcp_decode_workspace_bytes(dsc, 4)
        assert ws > 0
        other = dcp.dcp_attn_desc.from_buffer_copy(dsc)
        other.shard_rule = 1 - rule
        assert dcp.dcp_decode_workspace_bytes(other, 4) == ws
    # FP8 MLA (one scale for the latent): half a bf16 page, the same workspace
    m8 = dcp.make_desc(1, 8, 64, 1, 576, 512, 64, 32, 0.1, q_len, 1, 0.5, 0.5, rule)
    assert dcp.dcp_kv_page_bytes(m8) * 2 == dcp.dcp_kv_page_bytes(mla)
    assert dcp.dcp_decode_workspace_bytes(m8, 4) == dcp.dcp_decode_workspace_bytes(mla, 4)
    assert dcp.dcp_kv_page_bytes(desc(1, 1, 64, 1, 576, 64)) == 0  # FP8 MLA with unequal scales
    assert dcp.dcp_kv_page_bytes(desc(0, 1, 16, 2, 64)) == 2 * 2 * 16 * 64  # FP8 head_dim 64: one byte per value
