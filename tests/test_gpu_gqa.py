"""GQA parity on the GPU: CUDA path through the C ABI vs the float64 oracle."""
import numpy as np
import pytest
import torch

import oracle
import synth
from gpu_cases import (D_INVARIANCE_TOL, LSE_TOL, O_BOUND_UNIT_AMP, O_TOL, assert_lse_close, assert_o_close, build_cache, host_kv,
                       host_q, oracle_request)

pytestmark = pytest.mark.gpu


def _check_against_oracle(w, D, cache, requests=None):
    reqs = range(w.batch) if requests is None else requests
    Op = cache.O_parts.cpu().numpy()
    Lp = cache.LSE_parts.cpu().numpy()
    O = cache.O.cpu().numpy()
    L = cache.LSE.cpu().numpy()
    worst = 0.0
    for b in reqs:
        Ob, Lb, Opb, Lpb = oracle_request(w, b, D)
        for s in range(D):
            worst = max(worst, assert_o_close(Op[s, b], Opb[s], O_TOL, f"O_{s}[{b}]"))
            assert_lse_close(Lp[s, b], Lpb[s], LSE_TOL, f"LSE_{s}[{b}]")
        worst = max(worst, assert_o_close(O[b], Ob, O_TOL, f"O[{b}]"))
        assert_lse_close(L[b], Lb, LSE_TOL, f"LSE[{b}]")
    return worst


def test_device_generator_matches_host_generator():
    import synth.device as sdev
    w = synth.workload("gqa_tiny")
    cache, _ = build_cache(w, 1)
    kv = sdev.kv_source(w, "cuda", cache.cu_seqlens).view(torch.int16).cpu().numpy().view(np.uint16)
    np.testing.assert_array_equal(kv, host_kv(w))
    q = sdev.query(w, "cuda").view(torch.int16).cpu().numpy().view(np.uint16)
    np.testing.assert_array_equal(q, host_q(w))
    m = synth.custom(synth.MLA, [70, 3], 64, 1, 576, 512, 64, seed=77)
    cu = torch.tensor([0, 70, 73], dtype=torch.int64, device="cuda")
    src = sdev.kv_source(m, "cuda", cu).view(torch.int16).cpu().numpy().view(np.uint16)
    np.testing.assert_array_equal(src, host_kv(m))


@pytest.mark.parametrize("D,perm", [(1, 0), (2, 0), (2, 31), (3, 5), (8, 0)])
def test_placement_is_byte_exact(D, perm):
    w = synth.workload("gqa_tiny")
    cache, _ = build_cache(w, D, perm_seed=perm)
    t_or, _, pages = oracle.block_tables(w.seq_lens, w.block_size, D, perm_seed=perm,
                                         max_local_blocks=cache.max_local_blocks)
    pools = oracle.place(synth.GQA, w.num_kv_heads, w.head_dim_qk, w.block_size, D, t_or,
                         [w.kv_source(b) for b in range(w.batch)], pages, fill=0xFFFF)
    for s in range(D):
        got = cache.pools[s].cpu().numpy().view(np.uint16)[:pools[s].size]
        np.testing.assert_array_equal(got, pools[s])


def test_tiny_workload_parity():
    w = synth.workload("gqa_tiny")
    cache, q = build_cache(w, 2)
    cache.step(q)
    torch.cuda.synchronize()
    err = _check_against_oracle(w, 2, cache)
    assert err < O_BOUND_UNIT_AMP  # bf16 rounding of the weights only
    assert cache.device_error() == 0


@pytest.mark.parametrize("D", [1, 2, 3, 4, 8, 16])
def test_tiny_workload_all_D(D):
    w = synth.workload("gqa_tiny")
    cache, q = build_cache(w, D, perm_seed=D)
    cache.step(q)
    _check_against_oracle(w, D, cache)


def test_per_shard_calls_agree_with_one_launch():
    w = synth.custom(synth.GQA, [300, 17, 1000, 64], 16, 2, 128, 128, 16, seed=21)
    cache, q = build_cache(w, 4, perm_seed=3)
    cache.partials(q, per_shard=False)
    a = (cache.O_parts.clone(), cache.LSE_parts.clone())
    cache.partials(q, per_shard=True)
    # different launches split the page lists differently; with integral softmax
    # reference maxima the bf16 P values do not depend on the split, so the two
    # agree to fp32 accumulation order
    assert (a[0] - cache.O_parts).abs().max().item() <= 1e-4
    inf = torch.isinf(a[1])
    assert torch.equal(inf, torch.isinf(cache.LSE_parts))
    assert (a[1][~inf] - cache.LSE_parts[~inf]).abs().max().item() <= LSE_TOL


def test_repeated_steps_are_identical():
    w = synth.custom(synth.GQA, [5000, 33, 12000], 64, 8, 128, 128, 16, seed=22)
    cache, q = build_cache(w, 2)
    O1, L1 = [t.clone() for t in cache.step(q)]
    O2, L2 = cache.step(q)
    assert torch.equal(O1, O2) and torch.equal(L1, L2)


def test_d_invariance_tiny_and_mixed():
    for w in [synth.workload("gqa_tiny"), synth.custom(synth.GQA, [4097, 900, 16, 3], 64, 8, 128, 128, 16, seed=5)]:
        outs = []
        for D in (1, 2, 4, 8):
            cache, q = build_cache(w, D)
            O, _ = cache.step(q)
            outs.append(O.cpu().numpy())
        for o in outs[1:]:
            assert np.abs(o - outs[0]).max() <= D_INVARIANCE_TOL


@pytest.mark.parametrize("case", [
    # seq_lens, Hq, Hkv, d, bs, D
    ([0, 1, 15, 16, 17, 33, 100], 8, 2, 64, 16, 4),     # empty requests and shards, partial pages
    ([1, 2, 3], 4, 4, 128, 16, 8),                      # G = 1, most shards empty
    ([700, 31], 16, 1, 128, 16, 2),                     # G = 16 (full mma rows), one KV head
    ([129, 64, 500], 12, 3, 64, 32, 3),                 # Hkv = 3, block 32
    ([333, 1024], 8, 8, 128, 64, 2),                    # block 64
    ([2000], 64, 8, 64, 128, 4),                        # block 128, head_dim 64
    ([5], 128, 16, 128, 16, 1),                         # two head groups
])
def test_edge_cases(case):
    seq_lens, Hq, Hkv, d, bs, D = case
    w = synth.custom(synth.GQA, seq_lens, Hq, Hkv, d, d, bs, seed=sum(seq_lens) + Hq)
    cache, q = build_cache(w, D, perm_seed=7)
    cache.step(q)
    _check_against_oracle(w, D, cache)
    assert cache.device_error() == 0


def test_out_of_range_page_is_reported_and_skipped():
    w = synth.custom(synth.GQA, [64, 40], 8, 2, 64, 64, 16, seed=9)
    cache, q = build_cache(w, 2)
    bad = cache.tables[1].clone()
    bad[0, 0] = int(cache.pool_pages[1]) + 5  # outside shard 1's pool
    cache.tables[1].copy_(bad)
    cache.step(q)
    torch.cuda.synchronize()
    assert cache.device_error() == 1
    assert cache.device_error() == 0  # reading clears the word
    assert torch.isfinite(cache.O).all()


@pytest.mark.parametrize("D", [1, 2, 4])
def test_70b_class_layer_sampled(D):
    """Full-size GQA layer (batch 64, 8K-32K tokens, 5.4 GB of KV) in the benchmark's launch
    configuration; a sample of requests is checked against the oracle, all rows for finiteness."""
    w = synth.workload("gqa_70b")
    cache, q = build_cache(w, D, device_kv=True)
    cache.step(q)
    torch.cuda.synchronize()
    assert cache.device_error() == 0
    assert torch.isfinite(cache.O).all() and torch.isfinite(cache.LSE).all()
    lens = np.array(w.seq_lens)
    sample = sorted({int(lens.argmin()), int(lens.argmax()), 17})
    _check_against_oracle(w, D, cache, requests=sample)
    del cache
    torch.cuda.empty_cache()
