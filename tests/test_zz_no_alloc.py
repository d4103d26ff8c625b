"""The allocation-free GQA entry point against the workspace entry point.

dcp_decode_partial_all_noalloc serves callers that cannot allocate device
memory (plugins handed only their buffers, serving loops that forbid
allocation after start-up): it runs the same decode kernel on a fixed
scratch array inside the library.  Its outputs must match
dcp_decode_partial_all on the same inputs, on two calls in a row (the second
call reuses the scratch the first one left behind), bit for bit, since it is
the same kernel on the same grid; once they are also checked against the
float64 oracle.  This file is collected last so that a run stopping at the
first failure has run everything else.
"""
import numpy as np
import pytest
import torch

import synth
from gpu_cases import (LSE_TOL, O_TOL, assert_lse_close, assert_o_close, build_cache, host_kv, host_q,
                       oracle_request)
from sequence_sharded_decode_paged_b200 import dcp

pytestmark = pytest.mark.gpu


def _run_noalloc(cache, q):
    O = torch.full_like(cache.O_parts, float("nan"))
    L = torch.full_like(cache.LSE_parts, float("nan"))
    dcp.dcp_decode_partial_all_noalloc(cache.desc, q, cache.pools, cache.pool_pages, cache.tables,
                                       cache.seq_lens_dev, cache.D, list(O), list(L))
    torch.cuda.synchronize()
    return O, L


def _same(a_O, a_L, b_O, b_L):
    # the same kernel on the same grid and inputs as the workspace call: bit for bit
    assert torch.isfinite(a_O).all()
    assert torch.equal(a_O, b_O)
    assert torch.equal(a_L, b_L)


@pytest.mark.parametrize("case", [
    ("gqa_tiny", None, 2),
    ("mixed", ([5000, 33, 12000, 0, 700], 64, 8, 128, 16), 4),  # splits across CTAs, an empty request
])
def test_noalloc_matches_workspace_entry_point_twice(case):
    name, shape, D = case
    if shape is None:
        w = synth.workload(name)
    else:
        seq_lens, Hq, Hkv, d, bs = shape
        w = synth.custom(synth.GQA, seq_lens, Hq, Hkv, d, d, bs, seed=41)
    cache, q = build_cache(w, D)
    cache.partials(q)
    torch.cuda.synchronize()
    ref_O, ref_L = cache.O_parts.clone(), cache.LSE_parts.clone()
    for _ in range(2):
        O, L = _run_noalloc(cache, q)
        _same(O, L, ref_O, ref_L)
        assert dcp.dcp_noalloc_read_device_error() == 0
    # and against the float64 oracle directly, shard by shard
    On, Ln = O.cpu().numpy(), L.cpu().numpy()
    for b in range(w.batch):
        _, _, Op, Lp = oracle_request(w, b, D)
        for s in range(D):
            assert_o_close(On[s, b], Op[s], O_TOL, f"O_{s}[{b}]")
            assert_lse_close(Ln[s, b], Lp[s], LSE_TOL, f"LSE_{s}[{b}]")


def test_noalloc_contiguous_chunk_rule():
    # the kernel instantiated for the contiguous-chunk shard rule, through the allocation-free call
    from sequence_sharded_decode_paged_b200.cache import ShardedPagedCache
    w = synth.custom(synth.GQA, [3000, 40, 7000, 500], 32, 4, 128, 128, 16, seed=44, kv_amp=0.5)
    cache = ShardedPagedCache(w.layout, w.num_q_heads, w.num_kv_heads, w.head_dim_qk, w.head_dim_v, w.block_size, 3,
                              w.seq_lens, w.softmax_scale, 5, "cuda", pool_fill=0xFFFF,
                              shard_rule=dcp.DCP_SHARD_CONTIGUOUS)
    cache.place(torch.from_numpy(host_kv(w).view(np.int16)).cuda())
    q = torch.from_numpy(host_q(w).view(np.int16)).cuda()
    cache.partials(q)
    torch.cuda.synchronize()
    ref_O, ref_L = cache.O_parts.clone(), cache.LSE_parts.clone()
    for _ in range(2):
        O, L = _run_noalloc(cache, q)
        _same(O, L, ref_O, ref_L)


def test_noalloc_reports_out_of_range_pages():
    w = synth.custom(synth.GQA, [300, 130], 8, 2, 64, 64, 16, seed=45)
    cache, q = build_cache(w, 2)
    good = cache.tables[0].clone()
    cache.tables[0][1, 0] = int(cache.pool_pages[0]) + 7
    O, _ = _run_noalloc(cache, q)
    assert torch.isfinite(O).all()
    assert dcp.dcp_noalloc_read_device_error() == 1
    assert dcp.dcp_noalloc_read_device_error() == 0  # read-and-clear
    cache.tables[0].copy_(good)
    _run_noalloc(cache, q)
    assert dcp.dcp_noalloc_read_device_error() == 0  # each call starts from a clear status


@pytest.mark.parametrize("q_len,kv_dtype", [(3, dcp.DCP_KV_BF16), (1, dcp.DCP_KV_FP8_E4M3), (3, dcp.DCP_KV_FP8_E4M3)])
def test_noalloc_with_draft_tokens_and_fp8_cache(q_len, kv_dtype):
    # the same kernel variants as the workspace entry point: draft rows, FP8 pools, paired pages
    from sequence_sharded_decode_paged_b200.cache import ShardedPagedCache
    w = synth.custom(synth.GQA, [4000, 17, 9000, 1], 64, 8, 128, 128, 16, seed=43, q_len=q_len, kv_amp=0.5)
    cache = ShardedPagedCache(w.layout, w.num_q_heads, w.num_kv_heads, w.head_dim_qk, w.head_dim_v, w.block_size, 3,
                              w.seq_lens, w.softmax_scale, 0, "cuda", pool_fill=0xFFFF, q_len=q_len,
                              kv_dtype=kv_dtype, k_scale=2.0 ** -7, v_scale=2.0 ** -7)
    cache.place(torch.from_numpy(host_kv(w).view(np.int16)).cuda())
    q = torch.from_numpy(host_q(w).view(np.int16)).cuda()
    cache.partials(q)
    torch.cuda.synchronize()
    ref_O, ref_L = cache.O_parts.clone(), cache.LSE_parts.clone()
    for _ in range(2):
        O, L = _run_noalloc(cache, q)
        _same(O, L, ref_O, ref_L)


def test_noalloc_rejects_problems_larger_than_its_scratch():
    # 16 query heads per KV head and 8 KV heads per CTA: the split partials need more than 16 MiB.
    w = synth.custom(synth.GQA, [64], 128, 8, 128, 128, 16, seed=3)
    cache, q = build_cache(w, 1)
    assert cache.ws_bytes > 16 << 20
    with pytest.raises(dcp.DcpError) as e:
        _run_noalloc(cache, q)
    assert e.value.status == dcp.DCP_ERR_CAPACITY


def test_noalloc_rejects_mla():
    d = dcp.make_desc(dcp.DCP_LAYOUT_MLA, 1, 64, 1, 576, 512, 64, 1, 0.07)
    x = torch.zeros(64 * 576, dtype=torch.int16, device="cuda")
    o = torch.zeros(64 * 512, dtype=torch.float32, device="cuda")
    l = torch.zeros(64, dtype=torch.float32, device="cuda")
    t = torch.zeros(1, dtype=torch.int32, device="cuda")
    with pytest.raises(dcp.DcpError) as e:
        dcp.dcp_decode_partial_all_noalloc(d, x, [x], [1], [t], t, 1, [o], [l])
    assert e.value.status == dcp.DCP_ERR_UNSUPPORTED
