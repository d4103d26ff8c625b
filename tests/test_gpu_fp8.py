"""FP8 (E4M3) GQA KV cache on the GPU (head_dim 128 and 64): the cache write's codes must equal
the oracle's byte for byte, and decoding the FP8 cache must match the oracle's attention over the
values the codes stand for (scale * e4m3(code)), per shard and merged."""
import numpy as np
import pytest
import torch

import oracle
import synth
from gpu_cases import D_INVARIANCE_TOL, LSE_TOL, O_TOL, assert_lse_close, assert_o_close, host_kv, host_q
from sequence_sharded_decode_paged_b200 import dcp
from sequence_sharded_decode_paged_b200.cache import ShardedPagedCache

pytestmark = pytest.mark.gpu

FP8 = dcp.DCP_KV_FP8_E4M3


def _cache(w, D, k_scale, v_scale, perm_seed=0):
    cache = ShardedPagedCache(w.layout, w.num_q_heads, w.num_kv_heads, w.head_dim_qk, w.head_dim_v, w.block_size, D,
                              w.seq_lens, w.softmax_scale, perm_seed, "cuda", pool_fill=0xFFFF, q_len=w.q_len,
                              kv_dtype=FP8, k_scale=k_scale, v_scale=v_scale)
    cache.place(torch.from_numpy(host_kv(w).view(np.int16)).cuda())
    q = torch.from_numpy(host_q(w).view(np.int16)).cuda()
    return cache, q


def _pools_u8(cache):
    return [p.cpu().numpy().view(np.uint8) for p in cache.pools]


def _oracle_pools(w, D, k_scale, v_scale, max_local_blocks, perm_seed=0):
    t, _, pages = oracle.block_tables(w.seq_lens, w.block_size, D, perm_seed=perm_seed,
                                      max_local_blocks=max_local_blocks)
    codes = [oracle.quantize_kv_gqa(w.kv_source(b), k_scale, v_scale) for b in range(w.batch)]
    return oracle.place_u8(w.num_kv_heads, w.head_dim_qk, w.block_size, D, t, codes, pages, fill=0xFF)


def _check(w, D, cache, k_scale, v_scale):
    Op, Lp = cache.O_parts.cpu().numpy(), cache.LSE_parts.cpu().numpy()
    O, L = cache.O.cpu().numpy(), cache.LSE.cpu().numpy()
    for b in range(w.batch):
        vals = oracle.dequantize_kv_gqa(oracle.quantize_kv_gqa(w.kv_source(b), k_scale, v_scale), k_scale, v_scale)
        if w.q_len == 1:
            Ob, Lb, Opb, Lpb = oracle.sharded_values(w.layout, w.num_q_heads, w.num_kv_heads, w.head_dim_qk,
                                                     w.head_dim_v, w.query(b), vals, w.softmax_scale, w.block_size, D)
        else:
            parts = []
            for s in range(D):
                O_s = np.empty((w.q_len, w.num_q_heads, w.head_dim_v))
                L_s = np.empty((w.q_len, w.num_q_heads))
                for j in range(w.q_len):
                    n = oracle.visible_tokens(vals.shape[0], w.q_len, j)
                    O_s[j], L_s[j] = oracle.attend_values(w.layout, w.num_q_heads, w.num_kv_heads, w.head_dim_qk,
                                                          w.head_dim_v, w.queries(b)[j], vals[:n], w.softmax_scale,
                                                          w.block_size, D, s)
                parts.append((O_s, L_s))
            Opb = np.stack([p[0] for p in parts])
            Lpb = np.stack([p[1] for p in parts])
            rows = w.q_len * w.num_q_heads
            Ob, Lb = oracle.merge(Opb.reshape(D, rows, -1), Lpb.reshape(D, rows))
            Ob, Lb = Ob.reshape(w.q_len, w.num_q_heads, -1), Lb.reshape(w.q_len, w.num_q_heads)
        for s in range(D):
            assert_o_close(Op[s, b], Opb[s], O_TOL, f"O_{s}[{b}]")
            assert_lse_close(Lp[s, b], Lpb[s], LSE_TOL, f"LSE_{s}[{b}]")
        assert_o_close(O[b], Ob, O_TOL, f"O[{b}]")
        assert_lse_close(L[b], Lb, LSE_TOL, f"LSE[{b}]")


LENS = [1, 15, 16, 17, 300, 1000, 2500]


@pytest.mark.parametrize("hd", [128, 64])
@pytest.mark.parametrize("D,perm", [(1, 0), (3, 7), (4, 0)])
@pytest.mark.parametrize("scales", [(0.05, 0.02), (1.0, 1.0), (0.001, 0.5)])  # the last one saturates K
def test_cache_write_is_byte_exact(D, perm, scales, hd):
    w = synth.custom(synth.GQA, LENS, 16, 2, hd, hd, 16, seed=80 + D)
    cache, _ = _cache(w, D, *scales, perm_seed=perm)
    want = _oracle_pools(w, D, *scales, cache.max_local_blocks, perm)
    got = _pools_u8(cache)
    for s in range(D):
        np.testing.assert_array_equal(got[s][:want[s].size], want[s])


@pytest.mark.parametrize("hd", [128, 64])
@pytest.mark.parametrize("D", [1, 3, 4])
@pytest.mark.parametrize("bs", [16, 32])
def test_decode_parity(D, bs, hd):
    w = synth.custom(synth.GQA, LENS, 16, 2, hd, hd, bs, seed=90 + D + bs)
    cache, q = _cache(w, D, 0.05, 0.02)
    cache.step(q)
    torch.cuda.synchronize()
    _check(w, D, cache, 0.05, 0.02)
    assert cache.device_error() == 0


def test_head_dim_64_wide_blocks_and_contiguous_rule():
    # head_dim 64 allows blocks up to 256 tokens; the contiguous-chunk rule through the FP8 kernel
    w = synth.custom(synth.GQA, [1, 255, 256, 257, 3000], 8, 2, 64, 64, 256, seed=33)
    cache, q = _cache(w, 2, 0.05, 0.05)
    cache.step(q)
    torch.cuda.synchronize()
    _check(w, 2, cache, 0.05, 0.05)
    wc = synth.custom(synth.GQA, [5, 700, 1600], 16, 2, 64, 64, 16, seed=34)
    cc = ShardedPagedCache(wc.layout, wc.num_q_heads, wc.num_kv_heads, wc.head_dim_qk, wc.head_dim_v, wc.block_size,
                           3, wc.seq_lens, wc.softmax_scale, 0, "cuda", pool_fill=0xFFFF, kv_dtype=FP8, k_scale=0.05,
                           v_scale=0.05, shard_rule=dcp.DCP_SHARD_CONTIGUOUS)
    cc.place(torch.from_numpy(host_kv(wc).view(np.int16)).cuda())
    cc.step(torch.from_numpy(host_q(wc).view(np.int16)).cuda())
    torch.cuda.synchronize()
    O, L = cc.O.cpu().numpy(), cc.LSE.cpu().numpy()
    for b in range(wc.batch):
        vals = oracle.dequantize_kv_gqa(oracle.quantize_kv_gqa(wc.kv_source(b), 0.05, 0.05), 0.05, 0.05)
        Ob, Lb, _, _ = oracle.sharded_values(wc.layout, 16, 2, 64, 64, wc.query(b), vals, wc.softmax_scale, 16, 3,
                                             oracle.CONTIGUOUS)
        assert_o_close(O[b], Ob, O_TOL, f"O[{b}]")
        assert_lse_close(L[b], Lb, LSE_TOL, f"LSE[{b}]")


def test_decode_parity_70b_heads():
    w = synth.custom(synth.GQA, [5, 129, 4100, 9000], 64, 8, 128, 128, 16, seed=31, kv_amp=0.5)
    cache, q = _cache(w, 4, 0.01, 0.01)
    cache.step(q)
    torch.cuda.synchronize()
    _check(w, 4, cache, 0.01, 0.01)


@pytest.mark.parametrize("hd", [128, 64])
@pytest.mark.parametrize("q_len", [2, 4])
def test_multi_token_decode(q_len, hd):
    w = synth.custom(synth.GQA, [2, 17, 333, 1500], 16, 2, hd, hd, 16, seed=50 + q_len, q_len=q_len)
    cache, q = _cache(w, 3, 0.05, 0.05)
    cache.step(q)
    torch.cuda.synchronize()
    _check(w, 3, cache, 0.05, 0.05)


@pytest.mark.parametrize("hd", [128, 64])
def test_d_invariance(hd):
    w = synth.custom(synth.GQA, [3, 700, 5000], 16, 2, hd, hd, 16, seed=13)
    outs = []
    for D in (1, 2, 5):
        cache, q = _cache(w, D, 0.05, 0.05)
        cache.step(q)
        outs.append((cache.O.cpu().numpy(), cache.LSE.cpu().numpy()))
    for O, L in outs[1:]:
        np.testing.assert_allclose(O, outs[0][0], rtol=0, atol=D_INVARIANCE_TOL)
        np.testing.assert_allclose(L, outs[0][1], rtol=0, atol=D_INVARIANCE_TOL)


def test_append_writes_the_same_codes_as_placement():
    w = synth.custom(synth.GQA, [40, 3, 70], 16, 2, 128, 128, 16, seed=66)
    D = 2
    cache, _ = _cache(w, D, 0.05, 0.02)  # placement of the full lengths
    want = _pools_u8(cache)
    for s in range(D):
        cache.pools[s].fill_(-1)
    # append every request's rows in two steps at their positions
    for lo_frac, hi_frac in ((0.0, 0.5), (0.5, 1.0)):
        lo = [int(n * lo_frac) for n in w.seq_lens]
        hi = [int(n * hi_frac) for n in w.seq_lens]
        rows = [w.kv_source(b)[lo[b]:hi[b]] for b in range(w.batch)]
        cu = np.zeros(w.batch + 1, np.int64)
        cu[1:] = np.cumsum([r.shape[0] for r in rows])
        kv = torch.from_numpy(np.concatenate(rows).view(np.int16)).cuda()
        dcp.dcp_append_kv(cache.desc, D, kv, torch.from_numpy(cu).cuda(),
                          torch.tensor(lo, dtype=torch.int32, device="cuda"), cache.tables, cache.pools,
                          cache.pool_pages)
    torch.cuda.synchronize()
    got = _pools_u8(cache)
    for s in range(D):
        np.testing.assert_array_equal(got[s], want[s])



@pytest.mark.parametrize("D,q_len,hd", [(1, 1, 128), (2, 1, 128), (3, 1, 128), (3, 2, 128), (2, 4, 128),
                                        (1, 1, 64), (3, 1, 64), (3, 2, 64)])
def test_two_pages_per_step_path(D, q_len, hd):
    # eight KV heads at block 16 (one warp per head and row tile, one chunk per page): pages go two
    # at a time, odd page counts leave a single page, partial last pages and one-token requests included
    w = synth.custom(synth.GQA, [1, 16, 17, 31, 32, 33, 48, 500, 1111], 64, 8, hd, hd, 16, seed=17 + D,
                     kv_amp=0.5, q_len=q_len)
    cache, q = _cache(w, D, 0.01, 0.01)
    cache.step(q)
    torch.cuda.synchronize()
    _check(w, D, cache, 0.01, 0.01)
    assert cache.device_error() == 0


def test_70b_class_layer_sampled():
    """Full-size GQA layer with an FP8 cache (2.6 GB of codes) in the benchmark's launch configuration
    (D = 4, scales 2^-7): a sample of requests against the oracle over the dequantised values, every
    row finite."""
    import synth.device as sdev
    w = synth.workload("gqa_70b")
    D, scale = 4, 2.0 ** -7
    cache = ShardedPagedCache(w.layout, w.num_q_heads, w.num_kv_heads, w.head_dim_qk, w.head_dim_v, w.block_size, D,
                              w.seq_lens, w.softmax_scale, 0, "cuda", kv_dtype=FP8, k_scale=scale, v_scale=scale)
    kv = sdev.kv_source(w, "cuda", cache.cu_seqlens)
    cache.place(kv)
    del kv
    q = sdev.query(w, "cuda")
    cache.step(q)
    torch.cuda.synchronize()
    assert cache.device_error() == 0
    assert torch.isfinite(cache.O).all() and torch.isfinite(cache.LSE).all()
    lens = np.array(w.seq_lens)
    sample = sorted({int(lens.argmin()), int(lens.argmax())})
    O, L = cache.O.cpu().numpy(), cache.LSE.cpu().numpy()
    for b in sample:
        vals = oracle.dequantize_kv_gqa(oracle.quantize_kv_gqa(w.kv_source(b), scale, scale), scale, scale)
        Ob, Lb, _, _ = oracle.sharded_values(w.layout, w.num_q_heads, w.num_kv_heads, w.head_dim_qk, w.head_dim_v,
                                             w.query(b), vals, w.softmax_scale, w.block_size, D)
        assert_o_close(O[b], Ob, O_TOL, f"O[{b}]")
        assert_lse_close(L[b], Lb, LSE_TOL, f"LSE[{b}]")
    del cache
    torch.cuda.empty_cache()
