"""The one-shard-per-GPU form with the exchange folded into the decode kernel (exchange="p2p").

Each rank maps the other ranks' receive buffers with CUDA IPC and its decode kernel stores
every owner's rows straight into that owner's buffer; a barrier then orders the stores before
the merge.  Runs here have one GPU, so the two ranks are two processes on the same GPU (gloo for
the handle exchange and the barrier).  Their kernels never wait on one another -- the only
synchronisation is on the host -- so sharing a GPU does not change what is tested: the IPC
mapping, the owner pointers of both receive buffers, and the stores from another process's
kernel.  Every rank's merged heads must equal the same heads of the single-process D = 2 step
with one launch per shard, bit for bit (the same kernels and the same merge over the same values).
"""
import numpy as np
import pytest
import torch
import torch.multiprocessing as mp

pytestmark = pytest.mark.gpu


def _workload(case):
    import synth
    if case == "gqa":
        return synth.custom(synth.GQA, [2500, 40, 0, 800], 16, 2, 128, 128, 16, seed=66, kv_amp=0.5)
    if case == "mla":
        return synth.custom(synth.MLA, [3000, 70, 900], 64, 1, 576, 512, 64, seed=67)
    return synth.custom(synth.MLA, [1200, 64], 64, 1, 576, 512, 64, seed=72, q_len=2)


def _worker(rank, world, store_path, case, q_out):
    import torch.distributed as dist
    from gpu_cases import host_kv, host_q
    from sequence_sharded_decode_paged_b200.ranks import RankShardedDecode
    torch.cuda.set_device(0)
    store = dist.FileStore(store_path, world)
    dist.init_process_group("gloo", store=store, rank=rank, world_size=world)
    try:
        w = _workload(case)
        r = RankShardedDecode(w.layout, w.num_q_heads, w.num_kv_heads, w.head_dim_qk, w.head_dim_v, w.block_size,
                              w.seq_lens, w.softmax_scale, device="cuda", q_len=w.q_len, exchange="p2p")
        kv = torch.from_numpy(host_kv(w).view(np.int16)).cuda()
        cu = np.zeros(w.batch + 1, np.int64)
        cu[1:] = np.cumsum(w.seq_lens)
        r.place(kv, torch.from_numpy(cu).cuda())
        q = torch.from_numpy(host_q(w).view(np.int16)).cuda()
        outs = []
        for _ in range(3):  # both receive buffers, and the first one again
            O, L = r.step(q)
            torch.cuda.synchronize()
            outs.append((O.cpu().numpy().copy(), L.cpu().numpy().copy()))
        err = r.device_error()
        r.close()
        dist.barrier()
        q_out.put((rank, outs, err))
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("case", ["gqa", "mla", "mla_draft"])
def test_p2p_exchange_two_ranks(case, tmp_path):
    from gpu_cases import build_cache
    w = _workload(case)
    cache, q = build_cache(w, 2)
    cache.partials(q, per_shard=True)  # one launch per shard, as each rank runs its own
    cache.merge()
    O_ref, L_ref = cache.O.cpu().numpy(), cache.LSE.cpu().numpy()
    if w.q_len == 1:  # rank outputs carry a q_len axis
        O_ref, L_ref = O_ref[:, None], L_ref[:, None]
    ctx = mp.get_context("spawn")
    q_out = ctx.Queue()
    store = str(tmp_path / "store")
    procs = [ctx.Process(target=_worker, args=(r, 2, store, case, q_out)) for r in range(2)]
    for p in procs:
        p.start()
    res = sorted(q_out.get(timeout=300) for _ in procs)
    for p in procs:
        p.join(timeout=120)
        assert p.exitcode == 0
    Hk = w.num_q_heads // 2
    for rank, outs, err in res:
        assert err == 0
        for O, L in outs:
            np.testing.assert_array_equal(O, O_ref[:, :, rank * Hk:(rank + 1) * Hk])
            np.testing.assert_array_equal(L, L_ref[:, :, rank * Hk:(rank + 1) * Hk])
