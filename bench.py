#!/usr/bin/env python
"""Benchmark of the sharded paged decode-attention hot path on B200.

One step = the whole hot path for one decode token of every request of the
workload: all D shard partials (one ``dcp_decode_partial_all`` launch)
followed by the LSE merge (``dcp_lse_merge``), through the C ABI.  Inputs are
seeded synthetic tensors resident in HBM; L2 is flushed (a write of twice its
size) before every timed step, outside the timed events.

Default: the GQA 70B-class layer (batch 64, 64 q / 8 KV heads, head_dim 128,
block 16, lengths 8K-32K) at D = 4; the other D values of the workload are
measured in the same run and reported under ``other_D``.

``--impl reference`` times the float64 CPU oracle (the reference arm of this
build) on a bounded sample of the same workload.  Under torchrun every rank
runs an independent replica (weak scaling, no data-path collective); times
are reduced as the max over ranks.

Prints ONE JSON line on rank 0.
"""
from __future__ import annotations

import argparse
import datetime
import hashlib
import json
import os
import statistics
import subprocess
import sys
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

METRIC = "decode-attn KV GB/s & % of HBM/tensor roofline; merge GB/s; µs/step/layer"
DEFAULT_WORKLOAD = "gqa_70b"


def parse(argv=None):
    ap = argparse.ArgumentParser(description=__doc__, formatter_class=argparse.RawDescriptionHelpFormatter)
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=1000)
    ap.add_argument("--warmup", type=int, default=10)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", default=DEFAULT_WORKLOAD)
    ap.add_argument("--shards", type=int, default=None, help="D (default: the largest of the workload's list)")
    ap.add_argument("--other-d-steps", type=int, default=200, help="steps for the workload's other D values (0: skip)")
    ap.add_argument("--e2e-steps", type=int, default=100)
    ap.add_argument("--cpu-seconds", type=float, default=12.0, help="CPU baseline time budget")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--q-len", type=int, default=1,
                    help="query tokens per request (multi-token decode, causal within the draft; 1..4)")
    ap.add_argument("--kv-dtype", choices=["bf16", "fp8"], default="bf16",
                    help="cache element type (fp8: E4M3 codes, per-tensor scales 2^-7; GQA head_dim 128)")
    ap.add_argument("--batch-limit", type=int, default=None,
                    help="keep only the first N requests (small cases for profiling)")
    return ap.parse_args(argv)


# ----------------------------------------------------------------------------- distributed plumbing
def dist_env():
    return int(os.environ.get("RANK", "0")), int(os.environ.get("WORLD_SIZE", "1")), int(
        os.environ.get("LOCAL_RANK", "0"))


def dist_init(world: int, backend: str):
    import torch.distributed as dist
    if world > 1 and not dist.is_initialized():
        dist.init_process_group(backend=backend, timeout=datetime.timedelta(seconds=300))


def reduce_max(value: float, world: int, device) -> float:
    """Max of a float over ranks (identity at world size 1)."""
    if world == 1:
        return value
    import torch
    import torch.distributed as dist
    t = torch.tensor([value], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def job_value(world: int, bytes_per_replica: int, ms_max: float) -> float:
    """Whole-job throughput in GB/s: every rank runs one replica of the workload (weak
    scaling), and the job takes as long as its slowest rank."""
    return world * bytes_per_replica / ms_max / 1e6


def barrier(world: int):
    if world > 1:
        import torch.distributed as dist
        dist.barrier()


# ----------------------------------------------------------------------------- clocks
class ClockSampler:
    FIELDS = ("clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")
    REASONS = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]

    def __init__(self, device_index: int):
        import torch
        self.proc = None
        try:
            props = torch.cuda.get_device_properties(device_index)
            bus = f"{props.pci_domain_id:08X}:{props.pci_bus_id:02X}:{props.pci_device_id:02X}.0"
            self.proc = subprocess.Popen(["nvidia-smi", f"--id={bus}", f"--query-gpu={self.FIELDS}",
                                          "--format=csv,noheader,nounits", "-lms", "100"],
                                         stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except Exception:
            self.proc = None

    def stop(self):
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["unavailable"], "samples": 0}
        self.proc.terminate()
        try:
            out, _ = self.proc.communicate(timeout=10)
        except subprocess.TimeoutExpired:
            self.proc.kill()
            out, _ = self.proc.communicate()
        sm, mx, power, reasons = [], None, [], set()
        for line in out.splitlines():
            f = [x.strip() for x in line.split(",")]
            if len(f) < 8:
                continue
            try:
                sm.append(float(f[0]))
                mx = float(f[1])
                power.append(float(f[2]))
            except ValueError:
                continue
            for name, val in zip(self.REASONS, f[4:8]):
                if val.lower() == "active":
                    reasons.add(name)
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": mx,
                "reasons": sorted(reasons), "samples": len(sm),
                "power_w_max": max(power) if power else None}


# ----------------------------------------------------------------------------- helpers
def measured_peaks():
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as f:
            return json.load(f), "measured"
    except OSError:
        return {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}, "fallback"


def kernel_source_hash(layout: int) -> str:
    csrc = os.path.join(ROOT, "sequence_sharded_decode_paged_b200", "csrc")
    names = ["dcp_gqa.cu", "dcp_device.cuh"] if layout == 0 else ["dcp_mla.cu", "dcp_device.cuh"]
    h = hashlib.sha256()
    for n in names:
        with open(os.path.join(csrc, n), "rb") as f:
            h.update(f.read())
    return h.hexdigest()[:16]


def recorded_traffic(workload: str, D: int, layout: int):
    """DRAM bytes per launch of the decode kernel from a committed ncu summary, if it matches this source."""
    try:
        with open(os.path.join(ROOT, "profiles", "traffic.json")) as f:
            rec = json.load(f)
    except OSError:
        return None
    ent = rec.get(f"{workload}/D{D}")
    if not ent or ent.get("source_hash") != kernel_source_hash(layout):
        return None
    return ent.get("dram_bytes_per_launch")


def load_workload(args):
    import synth
    w = synth.workload(args.workload)
    if args.batch_limit is not None and args.batch_limit < w.batch:
        w.seq_lens = w.seq_lens[:args.batch_limit]
        w.batch = args.batch_limit
        w.name = f"{w.name}[:{args.batch_limit}]"
    if args.q_len != 1:
        w.q_len = args.q_len
        w.name = f"{w.name} q_len={args.q_len}"
    w.extra["kv_dtype"] = args.kv_dtype
    if args.kv_dtype == "fp8":
        w.name = f"{w.name} fp8"
    return w


FP8_SCALE = 2.0 ** -7  # per-tensor K and V scale of the FP8 cache: |x| <= 3.5 maps inside E4M3's 448


def cache_elem_bytes(w) -> int:
    return 1 if w.extra.get("kv_dtype") == "fp8" else 2


def tensor_figures(w, decode_ms: float, peaks: dict, peaks_kind: str):
    """Tensor-pipe side of the roofline: the method's flops per launch vs the dense bf16 peak.

    Per context token, query token and query head: 2*d_qk (q.k) + 2*d_v (p*v) flops (the few
    draft tokens a causal row does not see are not subtracted)."""
    flops = w.total_tokens * w.q_len * w.num_q_heads * 2 * (w.head_dim_qk + w.head_dim_v)
    tf = flops / decode_ms / 1e9
    peak = peaks["bf16_tflops"]
    bytes_time = w.total_tokens * w.kv_bytes_per_token * cache_elem_bytes(w) / 2 / (peaks["hbm_gbs"] * 1e9)
    flop_time = flops / (peak * 1e12)
    return {"flops_per_launch": flops, "achieved_tflops": round(tf, 1), "peak_tflops": peak,
            "frac": round(tf / peak, 4), "peak_kind": f"{peaks_kind} dense bf16 (burst)",
            "roofline_bound": "hbm" if bytes_time >= flop_time else "tensor",
            "roofline_us": round(max(bytes_time, flop_time) * 1e6, 2)}


def algorithmic_bytes(w, D: int):
    """(KV bytes, decode-kernel bytes, merge bytes) the method must move per step."""
    rows = w.batch * w.q_len * w.num_q_heads
    kv = w.total_tokens * w.kv_bytes_per_token * cache_elem_bytes(w) // 2
    q = rows * w.head_dim_qk * 2
    partial_out = rows * (w.head_dim_v + 1) * 4
    decode = kv + D * q + D * partial_out
    merge = D * partial_out + partial_out
    return kv, decode, merge


# ----------------------------------------------------------------------------- CPU oracle baseline
def run_oracle_sample(w, D: int, sample) -> float:
    """Seconds the float64 oracle takes for one sample: D shard partials + their merge."""
    import oracle
    _, q, src, hq, _ = sample
    t0 = time.perf_counter()
    oracle.sharded(w.layout, hq, 1, w.head_dim_qk, w.head_dim_v, q, src, w.softmax_scale, w.block_size, D)
    return time.perf_counter() - t0


def cpu_baseline(w, D: int, budget_s: float):
    """Time the oracle on (request, KV head) samples until ``budget_s`` seconds of oracle work.

    Returns (GB/s of KV processed, seconds, description)."""
    spent, kv_bytes, n = 0.0, 0, 0
    i = 0
    while spent < budget_s and i < 4 * w.batch:
        s = _sample_at(w, i)
        spent += run_oracle_sample(w, D, s)
        kv_bytes += s[4]
        n += 1
        i += 1
    what = "(request, KV head) pairs" if w.layout == 0 else "(request, 4 of 64 heads) pairs"
    desc = f"{n} {what} of {w.name}, D={D}: float64 shard partials + merge, single thread"
    return kv_bytes / spent / 1e9, spent, desc


def _sample_at(w, i: int, max_tokens: int = None):
    import synth
    order = sorted(range(w.batch), key=lambda b: (b * 7919) % w.batch)
    b = order[i % w.batch]
    if w.layout == synth.GQA:
        h = (i // w.batch + b) % w.num_kv_heads
        G = w.num_q_heads // w.num_kv_heads
        src = w.kv_source_head(b, h, max_tokens)
        return (b, w.query(b)[h * G:(h + 1) * G], src, G, src.shape[0] * 2 * w.head_dim_qk * 2)
    src = w.kv_source(b, max_tokens)
    return (b, w.query(b)[:4], src, 4, src.shape[0] * w.head_dim_qk * 2)


# ----------------------------------------------------------------------------- our arm
def run_ours(args, rank, world, local):
    import numpy as np
    import torch

    import synth
    import synth.device as sdev
    from sequence_sharded_decode_paged_b200.cache import ShardedPagedCache

    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    dist_init(world, "nccl")
    w = load_workload(args)
    D = args.shards or max(w.shards)
    peaks, peaks_kind = measured_peaks()
    l2 = torch.cuda.get_device_properties(local).L2_cache_size
    flush = torch.empty(2 * l2, dtype=torch.uint8, device=dev)

    def build(Dx):
        cache = ShardedPagedCache(w.layout, w.num_q_heads, w.num_kv_heads, w.head_dim_qk, w.head_dim_v,
                                  w.block_size, Dx, w.seq_lens, w.softmax_scale, device=dev, q_len=w.q_len,
                                  kv_dtype=1 if cache_elem_bytes(w) == 1 else 0, k_scale=FP8_SCALE,
                                  v_scale=FP8_SCALE)
        kv = sdev.kv_source(w, dev, cache.cu_seqlens)
        cache.place(kv)
        del kv
        torch.cuda.synchronize()
        return cache

    q = sdev.query(w, dev)

    def timed(cache, steps, warmup):
        for i in range(warmup):
            flush.fill_(i & 0xFF)
            cache.step(q)
        torch.cuda.synchronize()
        ev = [[torch.cuda.Event(enable_timing=True) for _ in range(3)] for _ in range(steps)]
        barrier(world)
        torch.cuda.synchronize()
        for i in range(steps):
            flush.fill_(i & 0xFF)
            ev[i][0].record()
            cache.partials(q)
            ev[i][1].record()
            cache.merge()
            ev[i][2].record()
        torch.cuda.synchronize()
        barrier(world)
        part = [e[0].elapsed_time(e[1]) for e in ev]
        merge = [e[1].elapsed_time(e[2]) for e in ev]
        step = [e[0].elapsed_time(e[2]) for e in ev]
        return sum(step) / steps, sum(part) / steps, sum(merge) / steps, statistics.median(step)

    cache = build(D)
    sampler = ClockSampler(local)
    time.sleep(0.3)
    step_ms, part_ms, merge_ms, step_med = timed(cache, args.steps, args.warmup)
    clocks = sampler.stop()
    err = cache.device_error()
    if err != 0:
        raise RuntimeError(f"device status {err} during the timed run")

    # end to end through the public API: every step uploads its packed inputs (query,
    # lengths, block tables) from pinned host memory and reads its results (O, LSE)
    # back; neighbouring steps' copies overlap the current step's compute
    from sequence_sharded_decode_paged_b200.cache import HostStepPipeline
    pipe = HostStepPipeline(cache)
    host_in = pipe.pack_inputs(q.view(torch.int16).cpu().numpy(), w.seq_lens, cache.tables_host)
    host_out = [pipe.host_output(), pipe.host_output()]
    for i in range(2):
        pipe.step(i, host_in, host_out[i & 1])
    pipe.synchronize()
    barrier(world)
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(pipe.s_in)
    for i in range(args.e2e_steps):
        pipe.step(i, host_in, host_out[i & 1])
    e1.record(pipe.s_out)
    pipe.synchronize()
    torch.cuda.synchronize()
    barrier(world)
    e2e_ms = e0.elapsed_time(e1) / max(1, args.e2e_steps)
    h2d, d2h = pipe.in_bytes, pipe.out_bytes
    assert np.isfinite(pipe.unpack_output(host_out[0])[0].numpy()).all()

    # cache write of one new token per request (the append that precedes each decode step),
    # timed on its own; it rewrites each request's last slot, after which the cache is not reused
    from sequence_sharded_decode_paged_b200 import dcp
    row_elems = w.kv_bytes_per_token // 2
    kv_row = torch.zeros((w.batch, row_elems), dtype=torch.int16, device=dev)
    cu_rows = torch.arange(w.batch + 1, dtype=torch.int64, device=dev)
    last_pos = (cache.seq_lens_dev - 1).clamp_min(0).contiguous()
    # 20 appends captured in one CUDA graph, so the events time the kernels, not the host calls
    side = torch.cuda.Stream(dev)
    with torch.cuda.stream(side):
        for _ in range(3):
            dcp.dcp_append_kv(cache.desc, D, kv_row, cu_rows, last_pos, cache.tables, cache.pools,
                              cache.pool_pages, stream=side)
    side.synchronize()
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph, stream=side):
        for _ in range(20):
            dcp.dcp_append_kv(cache.desc, D, kv_row, cu_rows, last_pos, cache.tables, cache.pools,
                              cache.pool_pages, stream=side)
    graph.replay()
    torch.cuda.synchronize()
    a0, a1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    a0.record()
    for _ in range(5):
        graph.replay()
    a1.record()
    torch.cuda.synchronize()
    append_ms = a0.elapsed_time(a1) / 100
    del graph

    kv_b, dec_b, mrg_b = algorithmic_bytes(w, D)
    step_ms_max = reduce_max(step_ms, world, dev)
    append_ms_max = reduce_max(append_ms, world, dev)
    part_ms_max = reduce_max(part_ms, world, dev)
    merge_ms_max = reduce_max(merge_ms, world, dev)
    e2e_ms_max = reduce_max(e2e_ms, world, dev)

    other = {}
    if args.other_d_steps > 0:
        for Dx in w.shards:
            if Dx == D:
                continue
            del cache
            torch.cuda.empty_cache()
            cache = build(Dx)
            s_ms, p_ms, m_ms, _ = timed(cache, args.other_d_steps, max(3, args.warmup // 2))
            s_ms, p_ms, m_ms = (reduce_max(x, world, dev) for x in (s_ms, p_ms, m_ms))
            kb, db, mb = algorithmic_bytes(w, Dx)
            other[str(Dx)] = {"kv_gbs": round(world * kb / s_ms / 1e6, 1), "us_per_step_per_layer": round(s_ms * 1e3, 2),
                              "decode_kernel_gbs": round(db / p_ms / 1e6, 1), "merge_gbs": round(mb / m_ms / 1e6, 1),
                              "decode_us": round(p_ms * 1e3, 2), "merge_us": round(m_ms * 1e3, 2),
                              "steps": args.other_d_steps}

    if rank != 0:
        return None
    peak = peaks["hbm_gbs"]
    achieved = dec_b / part_ms_max / 1e6
    line = {
        "metric": METRIC,
        "value": round(job_value(world, kv_b, step_ms_max), 1),
        "unit": "GB/s",
        "n_gpus": world,
        "steps": args.steps,
        "warmup": args.warmup,
        "ms_per_step": round(step_ms_max, 4),
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": "bf16" if cache_elem_bytes(w) == 2 else "fp8-e4m3 cache, f16 products, f32 accumulate",
        "data": "synthetic",
        "config": {"workload": f"{w.name}: {w.note}", "D": D, "batch": w.batch, "q_len": w.q_len,
                   "context_tokens": w.total_tokens, "kv_bytes_per_step": kv_b,
                   "l2": "flushed before every step (write of 2x L2), outside the timed events",
                   "parallelism": "replicas" if world > 1 else "single GPU (D shard pools in one HBM)"},
        "roofline": {"bound": "hbm", "achieved": round(achieved, 1), "peak": peak, "unit": "GB/s",
                     "frac": round(achieved / peak, 4), "traffic": recorded_traffic(w.name, D, w.layout),
                     "kernel": "gqa_decode_kernel" if w.layout == 0 else "mla_decode_kernel",
                     "peak_kind": f"{peaks_kind} HBM copy (burst)",
                     "algorithmic_bytes_per_launch": dec_b},
        "us_per_step_per_layer": round(step_ms_max * 1e3, 2),
        "decode_kernel_us": round(part_ms_max * 1e3, 2),
        "merge_kernel_us": round(merge_ms_max * 1e3, 2),
        "merge_gbs": round(mrg_b / merge_ms_max / 1e6, 1),
        "append_kernel_us": round(append_ms_max * 1e3, 2),
        "append_bytes_per_step": w.batch * w.kv_bytes_per_token * (2 + cache_elem_bytes(w)) // 2,
        "context_tokens_per_s": round(world * w.total_tokens / step_ms_max * 1e3, 1),
        "query_tokens_per_s": round(world * w.batch * w.q_len / step_ms_max * 1e3, 1),
        "frac_of_8tbs_spec": round(achieved / 8000.0, 4),
        "tensor": tensor_figures(w, part_ms_max, peaks, peaks_kind),
        "median_step_ms": round(step_med, 4),
        "gpu_launches": 2 * args.steps,
        "clocks": clocks,
        "e2e": {"value": round(job_value(world, kv_b, e2e_ms_max), 1), "unit": "GB/s",
                "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h, "ms_per_step": round(e2e_ms_max, 4),
                "steps": args.e2e_steps, "api": "HostStepPipeline (one packed upload and one download per step, "
                                                "overlapped with neighbouring steps)"},
        "other_D": other,
    }
    if world == 1 and not args.no_cpu_baseline and w.q_len == 1 and cache_elem_bytes(w) == 2:
        gbs, secs, desc = cpu_baseline(w, D, args.cpu_seconds)
        line["cpu_baseline"] = {"value": round(gbs, 4), "unit": "GB/s", "cores": 1, "kind": "oracle",
                                "sample": desc, "seconds": round(secs, 2)}
    return line


# ----------------------------------------------------------------------------- reference arm (the oracle)
def run_reference(args, rank, world):
    import synth
    if rank != 0:  # the oracle runs once, on rank 0; other ranks have no work
        return None
    w = load_workload(args)
    D = args.shards or max(w.shards)
    total_budget = 150.0  # seconds of oracle work for warm-up + timed steps
    per_step = total_budget / max(1, args.steps + args.warmup)
    probe = _sample_at(w, 0, 2048)
    tok_rate = probe[2].shape[0] / run_oracle_sample(w, D, probe)
    max_tok = max(64, int(tok_rate * per_step))
    pool = [_sample_at(w, i, max_tok) for i in range(8)]
    for i in range(args.warmup):
        run_oracle_sample(w, D, pool[i % len(pool)])
    t0 = time.perf_counter()
    kv_total, secs_total = 0, 0.0
    for i in range(args.steps):
        s = pool[i % len(pool)]
        secs_total += run_oracle_sample(w, D, s)
        kv_total += s[4]
    wall = time.perf_counter() - t0
    value = kv_total / secs_total / 1e9
    line = {
        "impl": "reference", "metric": METRIC, "value": round(value, 4), "unit": "GB/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(secs_total / args.steps * 1e3, 3),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": {"workload": f"{w.name}: {w.note}", "D": D, "batch": w.batch, "context_tokens": w.total_tokens},
        "cpu_baseline": {"value": round(value, 4), "unit": "GB/s", "cores": 1, "kind": "oracle",
                         "sample": f"each step: one (request, KV head) sample of {w.name}, at most {max_tok} tokens, "
                                   f"D={D} float64 shard partials + merge, single thread"},
        "e2e": {"value": round(value, 4), "unit": "GB/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
        "wall_s": round(wall, 1),
    }
    return line


def main(argv=None):
    args = parse(argv)
    rank, world, local = dist_env()
    if args.impl == "reference":
        line = run_reference(args, rank, world)
    else:
        line = run_ours(args, rank, world, local)
    if rank == 0 and line is not None:
        print(json.dumps(line), flush=True)
    if world > 1:
        import torch.distributed as dist
        if dist.is_initialized():
            dist.destroy_process_group()


if __name__ == "__main__":
    main()
