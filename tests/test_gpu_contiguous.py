"""Contiguous-chunk shard rule on the GPU: shard s holds a request's blocks floor(s*nblk/D) ..
floor((s+1)*nblk/D) - 1.  Placement must equal the oracle's byte for byte; decoding must match the
oracle per shard and merged, and the merged result must agree with the interleaved rule's."""
import numpy as np
import pytest
import torch

import oracle
import synth
from gpu_cases import D_INVARIANCE_TOL, LSE_TOL, O_TOL, assert_lse_close, assert_o_close, host_kv, host_q
from sequence_sharded_decode_paged_b200 import dcp
from sequence_sharded_decode_paged_b200.cache import ShardedPagedCache

pytestmark = pytest.mark.gpu

CONTIG = dcp.DCP_SHARD_CONTIGUOUS
SCALE = 2.0 ** -7


def _cache(w, D, rule=CONTIG, kv_dtype=0, perm_seed=0, device_kv=False):
    cache = ShardedPagedCache(w.layout, w.num_q_heads, w.num_kv_heads, w.head_dim_qk, w.head_dim_v, w.block_size, D,
                              w.seq_lens, w.softmax_scale, perm_seed, "cuda", pool_fill=0xFFFF, q_len=w.q_len,
                              kv_dtype=kv_dtype, k_scale=SCALE, v_scale=SCALE, shard_rule=rule)
    if device_kv:
        import synth.device as sdev
        kv = sdev.kv_source(w, "cuda", cache.cu_seqlens)
        q = sdev.query(w, "cuda")
    else:
        kv = torch.from_numpy(host_kv(w).view(np.int16)).cuda()
        q = torch.from_numpy(host_q(w).view(np.int16)).cuda()
    cache.place(kv)
    del kv
    return cache, q


def _oracle(w, b, D, kv_dtype, heads=None):
    """(O, LSE, O_parts, LSE_parts) of request b under the contiguous rule, float64."""
    src = w.kv_source(b)
    vals = (oracle.dequantize_kv_gqa(oracle.quantize_kv_gqa(src, SCALE, SCALE), SCALE, SCALE) if kv_dtype
            else synth.bf16_bits_to_f64(src))
    q = w.queries(b) if w.q_len > 1 else w.query(b)
    qs = q.reshape(w.q_len, w.num_q_heads, w.head_dim_qk)
    L = src.shape[0]
    Op = np.full((D, w.q_len, w.num_q_heads, w.head_dim_v), np.nan)
    Lp = np.full((D, w.q_len, w.num_q_heads), np.nan)
    for s in range(D):
        for j in range(w.q_len):
            n = oracle.visible_tokens(L, w.q_len, j)
            Op[s, j], Lp[s, j] = oracle.attend_values(w.layout, w.num_q_heads, w.num_kv_heads, w.head_dim_qk,
                                                      w.head_dim_v, qs[j], vals[:n], w.softmax_scale, w.block_size,
                                                      D, s, heads, oracle.CONTIGUOUS, L)
    hb, he = heads if heads is not None else (0, w.num_q_heads)
    rows = w.q_len * (he - hb)
    O, LSE = oracle.merge(Op[:, :, hb:he].reshape(D, rows, -1), Lp[:, :, hb:he].reshape(D, rows))
    O, LSE = O.reshape(w.q_len, he - hb, -1), LSE.reshape(w.q_len, he - hb)
    if w.q_len == 1:
        return O[0], LSE[0], Op[:, 0], Lp[:, 0]
    return O, LSE, Op, Lp


def _check(w, D, cache, kv_dtype=0, requests=None, heads=None):
    Op, Lp = cache.O_parts.cpu().numpy(), cache.LSE_parts.cpu().numpy()
    O, L = cache.O.cpu().numpy(), cache.LSE.cpu().numpy()
    hb, he = heads if heads is not None else (0, w.num_q_heads)
    for b in (range(w.batch) if requests is None else requests):
        Ob, Lb, Opb, Lpb = _oracle(w, b, D, kv_dtype, heads)
        for s in range(D):
            assert_o_close(Op[s, b][..., hb:he, :], Opb[s][..., hb:he, :], O_TOL, f"O_{s}[{b}]")
            assert_lse_close(Lp[s, b][..., hb:he], Lpb[s][..., hb:he], LSE_TOL, f"LSE_{s}[{b}]")
        assert_o_close(O[b][..., hb:he, :], Ob, O_TOL, f"O[{b}]")
        assert_lse_close(L[b][..., hb:he], Lb, LSE_TOL, f"LSE[{b}]")


LENS = [1, 15, 16, 17, 40, 300, 1000, 2500]


@pytest.mark.parametrize("layout,kv_dtype", [(synth.GQA, 0), (synth.GQA, 1), (synth.MLA, 0)])
@pytest.mark.parametrize("D,perm", [(3, 0), (4, 11)])
def test_placement_is_byte_exact(layout, kv_dtype, D, perm):
    shape = (16, 2, 128, 128, 16) if layout == synth.GQA else (64, 1, 576, 512, 64)
    w = synth.custom(layout, LENS, *shape, seed=5 + D)
    cache, _ = _cache(w, D, kv_dtype=kv_dtype, perm_seed=perm)
    t, _, pages = oracle.block_tables(w.seq_lens, w.block_size, D, perm_seed=perm,
                                      max_local_blocks=cache.max_local_blocks, rule=oracle.CONTIGUOUS)
    if kv_dtype:
        codes = [oracle.quantize_kv_gqa(w.kv_source(b), SCALE, SCALE) for b in range(w.batch)]
        want = oracle.place_u8(w.num_kv_heads, w.head_dim_qk, w.block_size, D, t, codes, pages, fill=0xFF,
                               rule=oracle.CONTIGUOUS)
        got = [p.cpu().numpy().view(np.uint8) for p in cache.pools]
    else:
        want = oracle.place(w.layout, w.num_kv_heads, w.head_dim_qk, w.block_size, D, t,
                            [w.kv_source(b) for b in range(w.batch)], pages, fill=0xFFFF, rule=oracle.CONTIGUOUS)
        got = [p.cpu().numpy().view(np.uint16) for p in cache.pools]
    for s in range(D):
        np.testing.assert_array_equal(got[s][:want[s].size], want[s])


@pytest.mark.parametrize("layout,kv_dtype,q_len", [(synth.GQA, 0, 1), (synth.GQA, 0, 3), (synth.GQA, 1, 1),
                                                   (synth.GQA, 1, 2), (synth.MLA, 0, 1), (synth.MLA, 0, 2)])
@pytest.mark.parametrize("D", [2, 5])
def test_decode_parity(layout, kv_dtype, q_len, D):
    shape = (64, 8, 128, 128, 16) if layout == synth.GQA else (64, 1, 576, 512, 64)
    w = synth.custom(layout, LENS, *shape, seed=60 + D + q_len, q_len=q_len, kv_amp=0.5)
    cache, q = _cache(w, D, kv_dtype=kv_dtype)
    cache.step(q)
    torch.cuda.synchronize()
    assert cache.device_error() == 0
    heads = None if layout == synth.GQA else (0, 8)
    _check(w, D, cache, kv_dtype, heads=heads)


@pytest.mark.parametrize("layout", [synth.GQA, synth.MLA])
def test_rules_agree_after_the_merge(layout):
    shape = (16, 2, 64, 64, 16) if layout == synth.GQA else (64, 1, 576, 512, 64)
    if layout == synth.MLA:
        shape = (64, 1, 576, 512, 64)
    w = synth.custom(layout, [3, 150, 2100, 777], *shape, seed=8)
    outs = []
    for rule in (dcp.DCP_SHARD_INTERLEAVED, CONTIG):
        cache, q = _cache(w, 4, rule=rule)
        cache.step(q)
        outs.append((cache.O.cpu().numpy(), cache.LSE.cpu().numpy()))
    np.testing.assert_allclose(outs[1][0], outs[0][0], rtol=0, atol=D_INVARIANCE_TOL)
    np.testing.assert_allclose(outs[1][1], outs[0][1], rtol=0, atol=D_INVARIANCE_TOL)


def test_70b_class_layer_sampled():
    """Full-size GQA layer (5.2 GB) under the contiguous rule at D = 4 in the benchmark's launch
    configuration: sampled requests against the oracle, every row finite."""
    w = synth.workload("gqa_70b")
    cache, q = _cache(w, 4, device_kv=True)
    cache.step(q)
    torch.cuda.synchronize()
    assert cache.device_error() == 0
    assert torch.isfinite(cache.O).all() and torch.isfinite(cache.LSE).all()
    lens = np.array(w.seq_lens)
    _check(w, 4, cache, requests=sorted({int(lens.argmin()), int(lens.argmax())}))
    del cache
    torch.cuda.empty_cache()
