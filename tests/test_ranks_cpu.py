"""The multi-GPU form of the method on CPU ranks: the exchange of owner-major partials.

"Efficient Decode Context Parallelism with vLLM for Long Context Workloads",
A2 方法细节, step 3: the D ranks exchange their partials (O_i, LSE_i) so that each
ends with the merged output of its own slice of query heads.  Here every rank of
a gloo group (2 or 4 spawned processes, no GPU) plays shard r: it takes its
partial from the float64 oracle, lays it out in the owner-major order that
include/dcp.h specifies for dcp_decode_partial_owner_major (written out again
here from that specification), and runs the product's ``exchange``.  Checked:
each rank receives, bit for bit, every shard's partial for its own heads, and
merging them gives the direct (unsharded) attention of those heads to 1e-12.
"""
import os
import socket

import numpy as np
import pytest
import torch
import torch.multiprocessing as mp

import oracle
import synth


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def _chunk_floats(rows, d_v):
    return rows * d_v + (rows + 63) // 64 * 64


def _pack(Op, Lp, D, Hk, d_v, dtype):
    """Owner-major send buffer of one shard: Op [B][q_len][Hq][d_v], Lp [B][q_len][Hq] -> D chunks of
    (O rows [B][q_len][Hk][d_v], LSE rows [B][q_len][Hk], zero padding)."""
    rows = Op.shape[0] * Op.shape[1] * Hk
    chunk = _chunk_floats(rows, d_v)
    buf = np.zeros(D * chunk, dtype=dtype)
    for k in range(D):
        c = buf[k * chunk:(k + 1) * chunk]
        c[:rows * d_v] = Op[:, :, k * Hk:(k + 1) * Hk, :].reshape(-1)
        c[rows * d_v:rows * d_v + rows] = Lp[:, :, k * Hk:(k + 1) * Hk].reshape(-1)
    return buf


def _case(name):
    if name == "gqa":
        return synth.custom(synth.GQA, [130, 17, 300, 1], 8, 2, 64, 64, 16, seed=51)
    if name == "gqa_draft":  # three draft tokens per request, causal within the draft
        return synth.custom(synth.GQA, [150, 3, 260], 8, 2, 64, 64, 16, seed=53, q_len=3)
    return synth.custom(synth.MLA, [200, 64, 500], 64, 1, 576, 512, 64, seed=52)


def _partials(w, D):
    """Per request: (O_parts [D][q_len][Hq][d_v], LSE_parts [D][q_len][Hq]) and the direct
    attention (O [q_len][Hq][d_v], LSE [q_len][Hq]) over the unsharded cache."""
    out = []
    for b in range(w.batch):
        args = (w.layout, w.num_q_heads, w.num_kv_heads, w.head_dim_qk, w.head_dim_v)
        if w.q_len == 1:
            _, _, Op, Lp = oracle.sharded(*args, w.query(b), w.kv_source(b), w.softmax_scale, w.block_size, D)
            Od, Ld = oracle.attend(*args, w.query(b), w.kv_source(b), w.softmax_scale, w.block_size, 1, 0)
            out.append((Op[:, None], Lp[:, None], Od[None], Ld[None]))
        else:
            _, _, Op, Lp = oracle.sharded_mtp(*args, w.queries(b), w.kv_source(b), w.softmax_scale, w.q_len,
                                              w.block_size, D)
            Od, Ld = oracle.attend_mtp(*args, w.queries(b), w.kv_source(b), w.softmax_scale, w.q_len,
                                       w.block_size, 1, 0)
            out.append((Op, Lp, Od, Ld))
    return out


def _worker(rank, world, port, name, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    import torch.distributed as dist
    from sequence_sharded_decode_paged_b200 import ranks
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        w = _case(name)
        D, Hq, d_v, ql = world, w.num_q_heads, w.head_dim_v, w.q_len
        Hk = Hq // D
        res = _partials(w, D)
        Op = np.stack([r[0] for r in res])          # [B][D][q_len][Hq][d_v]
        Lp = np.stack([r[1] for r in res])          # [B][D][q_len][Hq]
        rows = w.batch * ql * Hk
        mine = slice(rank * Hk, (rank + 1) * Hk)
        Od = np.stack([r[2][:, mine] for r in res]).reshape(rows, d_v)
        Ld = np.stack([r[3][:, mine] for r in res]).reshape(rows)
        out = {}
        for dtype, tname in ((np.float32, "f32"), (np.float64, "f64")):
            send = torch.from_numpy(_pack(Op[:, rank], Lp[:, rank], D, Hk, d_v, dtype))
            recv = torch.full_like(send, float("nan"))
            ranks.exchange(send, recv)
            Os, Ls = ranks.split_chunks(recv, D, rows, d_v)
            exact = all(
                np.array_equal(Os[j].numpy(), Op[:, j, :, mine, :].astype(dtype).reshape(rows, d_v)) and
                np.array_equal(Ls[j].numpy(), Lp[:, j, :, mine].astype(dtype).reshape(rows))
                for j in range(D))
            O, L = oracle.merge(np.stack([o.numpy() for o in Os]).astype(np.float64),
                                np.stack([l.numpy() for l in Ls]).astype(np.float64))
            fin = ~np.isneginf(Ld)
            dL = float(np.abs(L[fin] - Ld[fin]).max()) if fin.any() else 0.0
            same_inf = bool(np.array_equal(np.isneginf(L), np.isneginf(Ld)))
            out[tname] = (exact and same_inf, float(np.abs(O - Od).max()), dL)
        q.put((rank, out))
    finally:
        dist.destroy_process_group()


def _run(world, name):
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, world, port, name, q)) for r in range(world)]
    for p in procs:
        p.start()
    import queue as _queue
    import time
    out, t0 = {}, time.time()
    while len(out) < world:
        try:
            r, res = q.get(timeout=2)
            out[r] = res
        except _queue.Empty:
            dead = [p.exitcode for p in procs if p.exitcode not in (None, 0)]
            assert not dead, f"a rank exited with {dead}"
            assert time.time() - t0 < 300, "ranks did not finish"
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    return out


@pytest.mark.parametrize("world,name", [(2, "gqa"), (2, "mla"), (4, "gqa"), (2, "gqa_draft")])
def test_exchange_gives_each_rank_its_heads(world, name):
    out = _run(world, name)
    assert sorted(out) == list(range(world))
    for r, res in out.items():
        exact32, dO32, dL32 = res["f32"]
        exact64, dO64, dL64 = res["f64"]
        assert exact32 and exact64, f"rank {r}: received partials differ from the shards' partials"
        assert dO64 <= 1e-12 and dL64 <= 1e-12, f"rank {r}: merged float64 parts {dO64}, {dL64}"
        assert dO32 <= 1e-6 and dL32 <= 1e-5, f"rank {r}: merged float32 parts {dO32}, {dL32}"


def test_chunk_size_matches_the_library():
    from sequence_sharded_decode_paged_b200 import dcp, ranks
    for (B, ql, Hq, d_v, n) in [(2, 1, 8, 64, 2), (256, 1, 64, 512, 8), (3, 4, 64, 512, 4), (5, 2, 32, 128, 1)]:
        desc = dcp.make_desc(dcp.DCP_LAYOUT_GQA, B, Hq, 8, d_v, d_v, 16, 4, 0.1, ql)
        assert dcp.dcp_owner_chunk_floats(desc, n) == ranks.owner_chunk_floats(B, ql, Hq, d_v, n)
        assert dcp.dcp_owner_chunk_floats(desc, n) % 64 == 0 or (B * ql * Hq // n * d_v) % 4 == 0
    desc = dcp.make_desc(dcp.DCP_LAYOUT_GQA, 2, 8, 2, 64, 64, 16, 4, 0.1)
    assert dcp.dcp_owner_chunk_floats(desc, 3) == 0  # 3 owners do not split 8 heads


def test_folded_exchange_addresses_assemble_the_owner_layout():
    # emulate D ranks' receive buffers as numpy arrays at fake base addresses: every rank "stores"
    # its owner-major chunks at the addresses owner_chunk_addresses gives; each owner's buffer must
    # then hold, chunk by chunk in shard order, the rows it merges -- for both step parities
    from sequence_sharded_decode_paged_b200.ranks import owner_chunk_addresses, split_chunks
    D, rows, dv = 3, 5, 4
    chunk = rows * dv + 64  # O rows, then LSE rows padded to 64 floats
    bases = [(1 << 40) * (r + 1) for r in range(D)]
    bufs = [np.full(2 * D * chunk, np.nan, dtype=np.float32) for _ in range(D)]
    for parity in (0, 1):
        for shard in range(D):
            for owner, addr in enumerate(owner_chunk_addresses(bases, shard, chunk, parity)):
                r = next(k for k in range(D) if bases[k] <= addr < bases[k] + bufs[k].nbytes)
                assert r == owner
                off = (addr - bases[r]) // 4
                vals = np.arange(chunk, dtype=np.float32) + 1000 * shard + 100 * owner + 10 * parity
                bufs[r][off:off + chunk] = vals
        for owner in range(D):
            half = torch.from_numpy(bufs[owner][parity * D * chunk:(parity + 1) * D * chunk].copy())
            Os, Ls = split_chunks(half, D, rows, dv)
            for shard in range(D):
                base = 1000 * shard + 100 * owner + 10 * parity
                assert torch.equal(Os[shard].reshape(-1), torch.arange(rows * dv, dtype=torch.float32) + base)
                assert torch.equal(Ls[shard], torch.arange(rows * dv, rows * dv + rows, dtype=torch.float32) + base)
