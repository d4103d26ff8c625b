"""Multi-token decode (q_len 2..4 query tokens per request, causal within the draft) on the GPU:
CUDA path through the C ABI vs the float64 oracle, per shard and merged."""
import numpy as np
import pytest
import torch

import oracle
import synth
from gpu_cases import D_INVARIANCE_TOL, LSE_TOL, O_TOL, assert_lse_close, assert_o_close, build_cache

pytestmark = pytest.mark.gpu


def _check(w, D, cache, requests=None):
    Op = cache.O_parts.cpu().numpy()
    Lp = cache.LSE_parts.cpu().numpy()
    O = cache.O.cpu().numpy()
    L = cache.LSE.cpu().numpy()
    for b in (range(w.batch) if requests is None else requests):
        Ob, Lb, Opb, Lpb = oracle.sharded_mtp(w.layout, w.num_q_heads, w.num_kv_heads, w.head_dim_qk, w.head_dim_v,
                                              w.queries(b), w.kv_source(b), w.softmax_scale, w.q_len,
                                              w.block_size, D)
        for s in range(D):
            assert_o_close(Op[s, b], Opb[s], O_TOL, f"O_{s}[{b}]")
            assert_lse_close(Lp[s, b], Lpb[s], LSE_TOL, f"LSE_{s}[{b}]")
        assert_o_close(O[b], Ob, O_TOL, f"O[{b}]")
        assert_lse_close(L[b], Lb, LSE_TOL, f"LSE[{b}]")


# lengths: shorter than the draft, block boundaries on both sides, several pages, a few CTAs' worth
GQA_LENS = [1, 2, 3, 16, 17, 33, 300, 1000]


@pytest.mark.parametrize("q_len", [2, 3, 4])
@pytest.mark.parametrize("D", [1, 3])
def test_gqa_small_heads(q_len, D):
    w = synth.custom(synth.GQA, GQA_LENS, 8, 2, 64, 64, 16, seed=40 + q_len, q_len=q_len)
    cache, q = build_cache(w, D, perm_seed=D)
    cache.step(q)
    torch.cuda.synchronize()
    _check(w, D, cache)
    assert cache.device_error() == 0


@pytest.mark.parametrize("q_len", [2, 4])
def test_gqa_70b_heads(q_len):
    # G = 8: q_len 2 fills one 16-row tile per KV head, q_len 4 takes two tiles (two warps per head)
    w = synth.custom(synth.GQA, [5, 129, 2000, 4097], 64, 8, 128, 128, 16, seed=7 * q_len, q_len=q_len,
                     kv_amp=0.5)
    cache, q = build_cache(w, 4)
    cache.step(q)
    torch.cuda.synchronize()
    _check(w, 4, cache)


@pytest.mark.parametrize("q_len", [2, 3, 4])
def test_gqa_two_pages_per_step(q_len):
    # 8 KV heads, block 16: one warp per (head, row tile), pages taken two at a time; the draft
    # straddles page boundaries and odd page counts leave a single page
    w = synth.custom(synth.GQA, [1, 2, 16, 17, 18, 33, 47, 300, 1001], 64, 8, 128, 128, 16, seed=70 + q_len,
                     q_len=q_len, kv_amp=0.5)
    for D in (1, 3):
        cache, q = build_cache(w, D)
        cache.step(q)
        torch.cuda.synchronize()
        _check(w, D, cache)


def test_gqa_sixteen_heads_per_kv_head():
    # G = 16, q_len 4: 64 rows per KV head, four row tiles
    w = synth.custom(synth.GQA, [4, 70, 513], 32, 2, 128, 128, 32, seed=5, q_len=4)
    cache, q = build_cache(w, 2)
    cache.step(q)
    torch.cuda.synchronize()
    _check(w, 2, cache)


@pytest.mark.parametrize("q_len", [2, 4])
@pytest.mark.parametrize("D", [1, 2])
def test_mla(q_len, D):
    w = synth.custom(synth.MLA, [1, 3, 64, 65, 130, 700], 64, 1, 576, 512, 64, seed=60 + q_len, q_len=q_len)
    cache, q = build_cache(w, D)
    cache.step(q)
    torch.cuda.synchronize()
    _check(w, D, cache)
    assert cache.device_error() == 0


@pytest.mark.parametrize("layout", [synth.GQA, synth.MLA])
def test_last_draft_token_is_single_token_decode(layout):
    # the last draft token sees the whole cache: it must agree with a q_len = 1 call on that token
    shape = (16, 2, 128, 128, 16) if layout == synth.GQA else (64, 1, 576, 512, 64)
    lens = [37, 500, 1200]
    wm = synth.custom(layout, lens, *shape, seed=9, q_len=3)
    cm, qm = build_cache(wm, 2)
    cm.step(qm)
    c1, _ = build_cache(synth.custom(layout, lens, *shape, seed=9), 2)
    q_last = qm[:, 2].contiguous()
    c1.step(q_last)
    torch.cuda.synchronize()
    np.testing.assert_allclose(cm.O[:, 2].cpu().numpy(), c1.O.cpu().numpy(), rtol=0, atol=D_INVARIANCE_TOL)
    np.testing.assert_allclose(cm.LSE[:, 2].cpu().numpy(), c1.LSE.cpu().numpy(), rtol=0, atol=D_INVARIANCE_TOL)


@pytest.mark.parametrize("layout", [synth.GQA, synth.MLA])
def test_d_invariance(layout):
    shape = (8, 2, 64, 64, 16) if layout == synth.GQA else (64, 1, 576, 512, 64)
    w = synth.custom(layout, [3, 150, 2100], *shape, seed=12, q_len=4)
    outs = []
    for D in (1, 2, 4):
        cache, q = build_cache(w, D)
        cache.step(q)
        outs.append((cache.O.cpu().numpy(), cache.LSE.cpu().numpy()))
    for O, L in outs[1:]:
        np.testing.assert_allclose(O, outs[0][0], rtol=0, atol=D_INVARIANCE_TOL)
        np.testing.assert_allclose(L, outs[0][1], rtol=0, atol=D_INVARIANCE_TOL)



def _oracle_mtp_heads(w, b, D, heads):
    """Merged multi-token result of request b for a head range (oracle, float64)."""
    hb, he = heads
    parts = [oracle.attend_mtp(w.layout, w.num_q_heads, w.num_kv_heads, w.head_dim_qk, w.head_dim_v, w.queries(b),
                               w.kv_source(b), w.softmax_scale, w.q_len, w.block_size, D, s, heads)
             for s in range(D)]
    Op = np.stack([p[0][:, hb:he] for p in parts])
    Lp = np.stack([p[1][:, hb:he] for p in parts])
    rows = w.q_len * (he - hb)
    O, L = oracle.merge(Op.reshape(D, rows, -1), Lp.reshape(D, rows))
    return O.reshape(w.q_len, he - hb, -1), L.reshape(w.q_len, he - hb)


@pytest.mark.parametrize("name,q_len,heads", [("gqa_70b", 4, (0, 64)), ("mla_b32", 2, (0, 4))])
def test_full_size_workload_sampled(name, q_len, heads):
    """Full-size workloads with draft tokens, in the benchmark's launch configuration: sampled
    requests (and, for MLA, a head range) against the oracle, every row finite."""
    w = synth.workload(name)
    w.q_len = q_len
    D = max(w.shards)
    cache, q = build_cache(w, D, device_kv=True)
    cache.step(q)
    torch.cuda.synchronize()
    assert cache.device_error() == 0
    assert torch.isfinite(cache.O).all() and torch.isfinite(cache.LSE).all()
    lens = np.array(w.seq_lens)
    sample = sorted({int(lens.argmin()), int(np.argsort(lens)[len(lens) // 2])})
    O, L = cache.O.cpu().numpy(), cache.LSE.cpu().numpy()
    hb, he = heads
    for b in sample:
        Ob, Lb = _oracle_mtp_heads(w, b, D, heads)
        assert_o_close(O[b][:, hb:he], Ob, O_TOL, f"O[{b}]")
        assert_lse_close(L[b][:, hb:he], Lb, LSE_TOL, f"LSE[{b}]")
    del cache
    torch.cuda.empty_cache()


@pytest.mark.parametrize("layout,kv_dtype", [(synth.GQA, 0), (synth.GQA, 1), (synth.MLA, 0)])
def test_per_shard_calls_agree_with_one_launch(layout, kv_dtype):
    """D single-shard dcp_decode_partial calls and one dcp_decode_partial_all launch agree to rounding
    (different CTA splits), with draft tokens and, for GQA, either cache type."""
    from sequence_sharded_decode_paged_b200.cache import ShardedPagedCache
    from gpu_cases import host_kv, host_q
    shape = (64, 8, 128, 128, 16) if layout == synth.GQA else (64, 1, 576, 512, 64)
    w = synth.custom(layout, [300, 17, 1000, 64], *shape, seed=29, q_len=2, kv_amp=0.5)
    cache = ShardedPagedCache(w.layout, w.num_q_heads, w.num_kv_heads, w.head_dim_qk, w.head_dim_v, w.block_size, 3,
                              w.seq_lens, w.softmax_scale, 5, "cuda", pool_fill=0xFFFF, q_len=2, kv_dtype=kv_dtype,
                              k_scale=2.0 ** -7, v_scale=2.0 ** -7)
    cache.place(torch.from_numpy(host_kv(w).view(np.int16)).cuda())
    q = torch.from_numpy(host_q(w).view(np.int16)).cuda()
    cache.partials(q, per_shard=False)
    a = (cache.O_parts.clone(), cache.LSE_parts.clone())
    cache.partials(q, per_shard=True)
    torch.cuda.synchronize()
    assert (cache.O_parts - a[0]).abs().max().item() <= 1e-4
    inf = torch.isinf(a[1])
    assert torch.equal(torch.isinf(cache.LSE_parts), inf)
    assert (cache.LSE_parts[~inf] - a[1][~inf]).abs().max().item() <= 1e-4


def test_mla_wide_score_range():
    # query amplitude 8: reference raises (and O^T rescales) inside pieces of several pairs, per draft token
    w = synth.custom(synth.MLA, [40000, 9000], 64, 1, 576, 512, 64, seed=95, q_len=2, q_amp=8.0)
    cache, q = build_cache(w, 1, device_kv=True)
    cache.step(q)
    torch.cuda.synchronize()
    assert cache.device_error() == 0
    _check(w, 1, cache)
