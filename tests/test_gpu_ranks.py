"""The multi-GPU form's device side on one GPU.

dcp_decode_partial_owner_major runs the same decode kernels as
dcp_decode_partial with the rows written in head-owner order; on the same
inputs its chunks must be the standard partial's rows, permuted, bit for bit.
RankShardedDecode's step (owner-major partial, all-to-all, merge) on a
one-rank NCCL group must equal the single-shard step.  The exchange between
several ranks is covered on CPU ranks (tests/test_ranks_cpu.py); runs here
have one GPU.
"""

import numpy as np
import pytest
import torch

import synth
from gpu_cases import build_cache
from sequence_sharded_decode_paged_b200 import dcp

pytestmark = pytest.mark.gpu


FP8_SCALE = 2.0 ** -6


def _cases():
    # (name, workload, D, FP8 cache)
    return [
        ("gqa", synth.custom(synth.GQA, [3000, 17, 900, 0, 1], 32, 4, 128, 128, 16, seed=61, kv_amp=0.5), 3, False),
        ("gqa_draft", synth.custom(synth.GQA, [2000, 5, 700], 16, 2, 64, 64, 16, seed=62, q_len=3), 2, False),
        ("mla", synth.custom(synth.MLA, [5000, 65, 1, 3000], 64, 1, 576, 512, 64, seed=63), 4, False),
        ("mla_draft", synth.custom(synth.MLA, [1500, 130], 64, 1, 576, 512, 64, seed=64, q_len=2), 2, False),
        ("mla_fp8", synth.custom(synth.MLA, [2500, 65, 1], 64, 1, 576, 512, 64, seed=69), 2, True),
        ("gqa64_fp8", synth.custom(synth.GQA, [1800, 40, 3], 16, 2, 64, 64, 16, seed=70), 3, True),
    ]


def _fp8_cache(w, D):
    from gpu_cases import host_kv, host_q
    from sequence_sharded_decode_paged_b200.cache import ShardedPagedCache
    cache = ShardedPagedCache(w.layout, w.num_q_heads, w.num_kv_heads, w.head_dim_qk, w.head_dim_v, w.block_size, D,
                              w.seq_lens, w.softmax_scale, 0, "cuda", pool_fill=0xFFFF, q_len=w.q_len,
                              kv_dtype=dcp.DCP_KV_FP8_E4M3, k_scale=FP8_SCALE, v_scale=FP8_SCALE)
    cache.place(torch.from_numpy(host_kv(w).view(np.int16)).cuda())
    return cache, torch.from_numpy(host_q(w).view(np.int16)).cuda()


@pytest.mark.parametrize("idx", range(6))
@pytest.mark.parametrize("n_owners", [1, 2, 4, 8])
def test_owner_major_partial_is_the_standard_partial_permuted(idx, n_owners):
    name, w, D, fp8 = _cases()[idx]
    if w.num_q_heads % n_owners != 0:
        pytest.skip("owners must split the query heads evenly")
    cache, q = _fp8_cache(w, D) if fp8 else build_cache(w, D)
    d = cache.desc
    Hq, dv, B, ql = w.num_q_heads, w.head_dim_v, w.batch, w.q_len
    Hk = Hq // n_owners
    rows = B * ql * Hk
    chunk = dcp.dcp_owner_chunk_floats(d, n_owners)
    for s in range(D):
        O = torch.empty((B, ql, Hq, dv), dtype=torch.float32, device="cuda")
        L = torch.empty((B, ql, Hq), dtype=torch.float32, device="cuda")
        dcp.dcp_decode_partial(d, q, cache.pools[s], int(cache.pool_pages[s]), cache.tables[s], cache.seq_lens_dev,
                               s, D, O, L, cache.workspace)
        send = torch.full((n_owners * chunk,), float("nan"), dtype=torch.float32, device="cuda")
        dcp.dcp_decode_partial_owner_major(d, q, cache.pools[s], int(cache.pool_pages[s]), cache.tables[s],
                                           cache.seq_lens_dev, s, D, n_owners, send, cache.workspace)
        torch.cuda.synchronize()
        for k in range(n_owners):
            c = send[k * chunk:(k + 1) * chunk]
            want_O = O[:, :, k * Hk:(k + 1) * Hk, :].reshape(-1)
            want_L = L[:, :, k * Hk:(k + 1) * Hk].reshape(-1)
            assert torch.equal(c[:rows * dv], want_O), f"{name} shard {s} owner {k}: O rows"
            assert torch.equal(c[rows * dv:rows * dv + rows], want_L), f"{name} shard {s} owner {k}: LSE rows"
    assert cache.device_error() == 0


@pytest.mark.parametrize("idx", [0, 1, 2, 3, 4])
@pytest.mark.parametrize("n_owners", [2, 4])
def test_partial_to_owners_writes_the_owner_major_chunks(idx, n_owners):
    # each owner's chunk in its own allocation (on a multi-GPU run: another GPU's buffer); the rows
    # must be the owner-major chunks, bit for bit, and nothing outside a chunk may be written
    name, w, D, fp8 = _cases()[idx]
    cache, q = _fp8_cache(w, D) if fp8 else build_cache(w, D)
    d = cache.desc
    chunk = dcp.dcp_owner_chunk_floats(d, n_owners)
    for s in range(D):
        send = torch.empty((n_owners * chunk,), dtype=torch.float32, device="cuda")
        dcp.dcp_decode_partial_owner_major(d, q, cache.pools[s], int(cache.pool_pages[s]), cache.tables[s],
                                           cache.seq_lens_dev, s, D, n_owners, send, cache.workspace)
        # guard bands around every chunk
        bufs = [torch.full((chunk + 128,), float("nan"), dtype=torch.float32, device="cuda") for _ in range(n_owners)]
        dcp.dcp_decode_partial_to_owners(d, q, cache.pools[s], int(cache.pool_pages[s]), cache.tables[s],
                                         cache.seq_lens_dev, s, D, [b[64:64 + chunk] for b in bufs], cache.workspace)
        torch.cuda.synchronize()
        rows = w.batch * w.q_len * (w.num_q_heads // n_owners)
        used = rows * w.head_dim_v + rows  # O rows, then LSE rows (the padding is never written)
        for k in range(n_owners):
            got = bufs[k][64:64 + used]
            assert torch.equal(got, send[k * chunk:k * chunk + used]), f"{name} shard {s} owner {k}"
            assert torch.isnan(bufs[k][:64]).all() and torch.isnan(bufs[k][64 + used:]).all()
    assert cache.device_error() == 0


def test_partial_to_owners_rejects_misaligned_chunks():
    w = synth.custom(synth.GQA, [100], 8, 2, 64, 64, 16, seed=71)
    cache, q = build_cache(w, 1)
    chunk = dcp.dcp_owner_chunk_floats(cache.desc, 2)
    buf = torch.empty(2 * chunk + 8, dtype=torch.float32, device="cuda")
    with pytest.raises(dcp.DcpError) as e:
        dcp.dcp_decode_partial_to_owners(cache.desc, q, cache.pools[0], int(cache.pool_pages[0]), cache.tables[0],
                                         cache.seq_lens_dev, 0, 1, [buf[1:], buf[chunk + 4:]], cache.workspace)
    assert e.value.status == dcp.DCP_ERR_INVALID_ARG


def test_owner_major_rejects_uneven_owners():
    w = synth.custom(synth.GQA, [100], 8, 2, 64, 64, 16, seed=65)
    cache, q = build_cache(w, 1)
    send = torch.empty(4096, dtype=torch.float32, device="cuda")
    with pytest.raises(dcp.DcpError) as e:
        dcp.dcp_decode_partial_owner_major(cache.desc, q, cache.pools[0], int(cache.pool_pages[0]), cache.tables[0],
                                           cache.seq_lens_dev, 0, 1, 3, send, cache.workspace)
    assert e.value.status == dcp.DCP_ERR_INVALID_ARG


@pytest.mark.parametrize("layout,fp8", [(synth.GQA, False), (synth.MLA, False), (synth.MLA, True)])
def test_rank_step_on_a_one_rank_nccl_group(layout, fp8, tmp_path):
    import torch.distributed as dist
    from sequence_sharded_decode_paged_b200.ranks import RankShardedDecode
    if layout == synth.GQA:
        w = synth.custom(synth.GQA, [2500, 40, 0, 800], 16, 2, 128, 128, 16, seed=66, kv_amp=0.5)
    else:
        w = synth.custom(synth.MLA, [3000, 70, 900], 64, 1, 576, 512, 64, seed=67)
    cache, q = _fp8_cache(w, 1) if fp8 else build_cache(w, 1)
    O_ref, L_ref = [t.clone() for t in cache.step(q)]
    store = dist.FileStore(str(tmp_path / "store"), 1)
    dist.init_process_group("nccl", store=store, rank=0, world_size=1)
    try:
        extra = dict(kv_dtype=dcp.DCP_KV_FP8_E4M3, k_scale=FP8_SCALE, v_scale=FP8_SCALE) if fp8 else {}
        r = RankShardedDecode(w.layout, w.num_q_heads, w.num_kv_heads, w.head_dim_qk, w.head_dim_v, w.block_size,
                              w.seq_lens, w.softmax_scale, device="cuda", **extra)
        from gpu_cases import host_kv
        kv = torch.from_numpy(host_kv(w).view(np.int16)).cuda()
        r.place(kv, cache.cu_seqlens)
        O, L = r.step(q)
        torch.cuda.synchronize()
        assert torch.equal(O.reshape(O_ref.shape), O_ref)
        assert torch.equal(L.reshape(L_ref.shape), L_ref)
        assert r.device_error() == 0
    finally:
        dist.destroy_process_group()


def test_placement_of_one_shard_leaves_the_others_untouched():
    """RankShardedDecode.place writes one shard: the other shards' pools get 0 pages, so their rows
    are skipped -- the placed pool must equal that shard's pool of a full placement, byte for byte."""
    w = synth.custom(synth.MLA, [700, 65, 300], 64, 1, 576, 512, 64, seed=68)
    D = 3
    cache, q = build_cache(w, D, pool_fill=0)
    from gpu_cases import host_kv
    kv = torch.from_numpy(host_kv(w).view(np.int16)).cuda()
    for r in range(D):
        pool = torch.zeros_like(cache.pools[r])
        pools = [None] * D
        pages = [0] * D
        pools[r], pages[r] = pool, int(cache.pool_pages[r])
        dcp.dcp_place_kv(cache.desc, D, kv, cache.cu_seqlens, cache.seq_lens_dev, [cache.tables[r]] * D, pools, pages)
        torch.cuda.synchronize()
        assert torch.equal(pool, cache.pools[r])
