"""The benchmark's multi-rank plumbing on CPU with two gloo ranks.

Under torchrun every rank runs an independent replica of the workload; the only
collectives are the timing barrier and the max-over-ranks reduction of the
step time.  These tests run that plumbing in two spawned processes (no GPU).
"""
import os
import socket

import pytest
import torch
import torch.multiprocessing as mp

import bench


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def _worker(rank, world, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world),
                      LOCAL_RANK=str(rank))
    r, w, _ = bench.dist_env()
    bench.dist_init(w, "gloo")
    slow = bench.reduce_max(1.5 * (r + 1), w, torch.device("cpu"))
    bench.barrier(w)
    value = bench.job_value(w, 10 ** 9, slow)
    q.put((r, slow, value))
    torch.distributed.destroy_process_group()


def test_max_over_two_gloo_ranks_and_job_value():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    out = sorted(q.get(timeout=180) for _ in procs)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    # both ranks see the slowest rank's time; the job moved 2 replicas' bytes in that time
    assert [o[1] for o in out] == [3.0, 3.0]
    assert out[0][2] == pytest.approx(2 * 1e9 / 3.0 / 1e6)


def test_single_rank_needs_no_process_group():
    assert bench.reduce_max(2.5, 1, torch.device("cpu")) == 2.5
    bench.barrier(1)
    assert bench.job_value(1, 5 * 10 ** 9, 1.0) == pytest.approx(5000.0)


def test_reference_arm_runs_on_rank_zero_only():
    args = bench.parse(["--impl", "reference", "--steps", "1", "--warmup", "0", "--batch-limit", "2"])
    assert bench.run_reference(args, rank=1, world=2) is None
