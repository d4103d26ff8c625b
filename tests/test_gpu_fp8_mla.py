"""FP8 (E4M3) MLA latent cache on the GPU.  The cache write must produce the oracle's codes byte for
byte, and decoding the FP8 cache must match the oracle's attention over the values the codes stand
for (scale * e4m3(code); one scale for the whole 576-wide latent row), per shard and merged, under
both shard rules, with draft tokens, and in the benchmark's launch configuration."""
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
CONTIG = dcp.DCP_SHARD_CONTIGUOUS


def _cache(w, D, scale, perm_seed=0, rule=0, kv_dev=None):
    cache = ShardedPagedCache(w.layout, w.num_q_heads, w.num_kv_heads, w.head_dim_qk, w.head_dim_v, w.block_size, D,
                              w.seq_lens, w.softmax_scale, perm_seed, "cuda", pool_fill=0xFFFF, q_len=w.q_len,
                              kv_dtype=FP8, k_scale=scale, v_scale=scale, shard_rule=rule)
    if kv_dev is None and w.total_tokens > 0:
        kv_dev = torch.from_numpy(host_kv(w).view(np.int16)).cuda()
    if kv_dev is not None:
        cache.place(kv_dev)
    q = torch.from_numpy(host_q(w).view(np.int16)).cuda()
    return cache, q


def _values(w, b, scale):
    return oracle.dequantize_kv_mla(oracle.quantize_kv_mla(w.kv_source(b), scale), scale)


def _oracle_parts(w, b, vals, D, rule=0, heads=None):
    """Per-shard (O, LSE) of request b over the dequantised latent `vals`, [D][q_len][Hq](...)."""
    n_all = vals.shape[0]
    Op = np.empty((D, w.q_len, w.num_q_heads, w.head_dim_v))
    Lp = np.empty((D, w.q_len, w.num_q_heads))
    for s in range(D):
        for j in range(w.q_len):
            q = w.query(b) if w.q_len == 1 else w.queries(b)[j]
            n = oracle.visible_tokens(n_all, w.q_len, j)
            Op[s, j], Lp[s, j] = oracle.attend_values(w.layout, w.num_q_heads, w.num_kv_heads, w.head_dim_qk,
                                                      w.head_dim_v, q, vals[:n], w.softmax_scale, w.block_size, D,
                                                      s, heads, rule, n_all)
    return Op, Lp


def _check(w, D, cache, scale, rule=0, requests=None, head_ranges=None):
    Op, Lp = cache.O_parts.cpu().numpy(), cache.LSE_parts.cpu().numpy()
    O, L = cache.O.cpu().numpy(), cache.LSE.cpu().numpy()
    if w.q_len == 1:  # give every array a q_len axis
        Op, Lp, O, L = Op[:, :, None], Lp[:, :, None], O[:, None], L[:, None]
    for b in (range(w.batch) if requests is None else requests):
        vals = _values(w, b, scale)
        for hb, he in (head_ranges or [(0, w.num_q_heads)]):
            Opb, Lpb = _oracle_parts(w, b, vals, D, rule, (hb, he))
            Opb, Lpb = Opb[:, :, hb:he], Lpb[:, :, hb:he]
            rows = w.q_len * (he - hb)
            Ob, Lb = oracle.merge(Opb.reshape(D, rows, -1), Lpb.reshape(D, rows))
            for s in range(D):
                assert_o_close(Op[s, b, :, hb:he], Opb[s], O_TOL, f"O_{s}[{b}]")
                assert_lse_close(Lp[s, b, :, hb:he], Lpb[s], LSE_TOL, f"LSE_{s}[{b}]")
            assert_o_close(O[b, :, hb:he].reshape(rows, -1), Ob, O_TOL, f"O[{b}]")
            assert_lse_close(L[b, :, hb:he].reshape(rows), Lb, LSE_TOL, f"LSE[{b}]")
        del vals


LENS = [1, 63, 64, 65, 129, 700, 2500]


@pytest.mark.parametrize("D,perm,rule", [(1, 0, 0), (3, 7, 0), (4, 0, CONTIG)])
@pytest.mark.parametrize("scale", [0.05, 1.0, 0.002])  # the last one saturates
def test_cache_write_is_byte_exact(D, perm, rule, scale):
    w = synth.custom(synth.MLA, LENS, 64, 1, 576, 512, 64, seed=120 + D)
    cache, _ = _cache(w, D, scale, perm_seed=perm, rule=rule)
    t, _, pages = oracle.block_tables(w.seq_lens, 64, D, perm_seed=perm, max_local_blocks=cache.max_local_blocks,
                                      rule=rule)
    codes = [oracle.quantize_kv_mla(w.kv_source(b), scale) for b in range(w.batch)]
    want = oracle.place_mla_u8(64, D, t, codes, pages, fill=0xFF, rule=rule)
    got = [p.cpu().numpy().view(np.uint8) for p in cache.pools]
    for s in range(D):
        np.testing.assert_array_equal(got[s][:want[s].size], want[s])


@pytest.mark.parametrize("case", [
    ([1], 1), ([64], 1), ([65], 2), ([70, 3, 200], 2), ([0, 130, 64, 129], 4),
    ([1000, 31, 257], 3), ([4097, 64], 8), ([300] * 5, 16),
])
def test_decode_parity(case):
    # one-token and empty requests, a pair's missing second page, partial last pages, segments cut
    # across several CTAs, up to 16 shards
    seq_lens, D = case
    w = synth.custom(synth.MLA, seq_lens, 64, 1, 576, 512, 64, seed=sum(seq_lens) + D + 1)
    cache, q = _cache(w, D, 0.05, perm_seed=11)
    cache.step(q)
    torch.cuda.synchronize()
    _check(w, D, cache, 0.05)
    assert cache.device_error() == 0


def test_decode_parity_unit_scale_and_contiguous_rule():
    w = synth.custom(synth.MLA, [5, 640, 1500, 64], 64, 1, 576, 512, 64, seed=77)
    for rule in (0, CONTIG):
        cache, q = _cache(w, 3, 1.0, rule=rule)
        cache.step(q)
        torch.cuda.synchronize()
        _check(w, 3, cache, 1.0, rule)


def test_decode_parity_with_saturated_codes():
    # scale 2^-9: values past 448 * 2^-9 = 0.875 saturate to the largest code, as the oracle's cache
    # write does -- the decode must see exactly those values
    w = synth.custom(synth.MLA, [700, 64, 2000], 64, 1, 576, 512, 64, seed=93)
    scale = 2.0 ** -9
    cache, q = _cache(w, 2, scale)
    codes = np.concatenate([p.cpu().numpy().view(np.uint8) for p in cache.pools])
    assert ((codes & 0x7F) == 0x7E).sum() > 1000  # many saturated codes
    cache.step(q)
    torch.cuda.synchronize()
    _check(w, 2, cache, scale)


def test_out_of_pool_page_is_flagged_and_skipped():
    # one table entry of request 1 names a page past its pool: the page is never loaded or widened,
    # status bit 0 is set, every output stays finite and the other requests are exact
    w = synth.custom(synth.MLA, [900, 600, 1300], 64, 1, 576, 512, 64, seed=94)
    D = 2
    cache, q = _cache(w, D, 0.05)
    t = cache.tables[1]
    t[1, 2] = int(cache.pool_pages[1]) + 7
    cache.step(q)
    torch.cuda.synchronize()
    assert cache.device_error() == 1
    assert torch.isfinite(cache.O).all() and torch.isfinite(cache.LSE).all()
    _check(w, D, cache, 0.05, requests=[0, 2])


def test_wide_score_range():
    # query amplitude 8: scores spread far, so reference raises and O^T rescales happen mid-piece
    w = synth.custom(synth.MLA, [3000, 900], 64, 1, 576, 512, 64, seed=91, q_amp=8.0)
    cache, q = _cache(w, 2, 0.03)
    cache.step(q)
    torch.cuda.synchronize()
    _check(w, 2, cache, 0.03)


@pytest.mark.parametrize("q_len,rule", [(2, 0), (3, CONTIG)])
def test_multi_token_decode(q_len, rule):
    w = synth.custom(synth.MLA, [2, 65, 333, 1500], 64, 1, 576, 512, 64, seed=60 + q_len, q_len=q_len)
    cache, q = _cache(w, 3, 0.05, rule=rule)
    cache.step(q)
    torch.cuda.synchronize()
    _check(w, 3, cache, 0.05, rule)


def test_d_invariance():
    w = synth.custom(synth.MLA, [3, 700, 5000], 64, 1, 576, 512, 64, seed=14)
    outs = []
    for D in (1, 2, 4, 8):
        cache, q = _cache(w, D, 0.05)
        cache.step(q)
        outs.append((cache.O.cpu().numpy(), cache.LSE.cpu().numpy()))
    for O, L in outs[1:]:
        np.testing.assert_allclose(O, outs[0][0], rtol=0, atol=D_INVARIANCE_TOL)
        np.testing.assert_allclose(L, outs[0][1], rtol=0, atol=D_INVARIANCE_TOL)


def test_per_shard_calls_equal_one_launch():
    w = synth.custom(synth.MLA, [900, 77, 2000], 64, 1, 576, 512, 64, seed=15)
    cache, q = _cache(w, 3, 0.05)
    cache.partials(q)
    ref_O, ref_L = cache.O_parts.clone(), cache.LSE_parts.clone()
    cache.partials(q, per_shard=True)
    torch.cuda.synchronize()
    torch.testing.assert_close(cache.O_parts, ref_O, rtol=0, atol=1e-4)
    torch.testing.assert_close(cache.LSE_parts, ref_L, rtol=0, atol=1e-4)


def test_append_writes_the_same_codes_as_placement():
    w = synth.custom(synth.MLA, [40, 3, 130], 64, 1, 576, 512, 64, seed=67)
    D = 2
    cache, _ = _cache(w, D, 0.05)
    want = [p.cpu().numpy().view(np.uint8).copy() for p in cache.pools]
    for s in range(D):
        cache.pools[s].fill_(-1)
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
    for s in range(D):
        np.testing.assert_array_equal(cache.pools[s].cpu().numpy().view(np.uint8), want[s])


def test_mla_b32_sampled():
    """The 32-request MLA layer (lognormal lengths, median 67K) with an FP8 latent cache in the
    benchmark's launch configuration (D = 4, scale 2^-4): the shortest, a middle-length and the
    longest request against the oracle on one head per quarter of the 64, every row finite."""
    import synth.device as sdev
    w = synth.workload("mla_b32")
    D, scale = 4, 2.0 ** -4
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
    lens = np.asarray(w.seq_lens)
    order = np.argsort(lens, kind="stable")
    sample = sorted({int(order[0]), int(order[len(lens) // 2]), int(order[-1])})
    _check(w, D, cache, scale, requests=sample, head_ranges=[(0, 1), (21, 22), (42, 43), (63, 64)])
    del cache
    torch.cuda.empty_cache()
