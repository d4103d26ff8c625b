#!/usr/bin/env python
"""Benchmark of the sharded paged decode-attention hot path on B200.

One step = the whole hot path for one decode token of every request of the
workload: all D shard partials (one ``dcp_decode_partial_all`` launch)
followed by the LSE merge (``dcp_lse_merge``), through the C ABI.  Inputs are
seeded synthetic tensors resident in HBM; before every timed step L2 is
flushed by READING a buffer twice its size (outside the timed events), so the
previous step's dirty lines are written back before the timer starts.

Default: the largest single-GPU workload, the MLA agentic mix (256 requests,
17.8 M context tokens, 20.5 GB of latent cache) at D = 8; its other D values
are measured in the same run (``other_D``), and the GQA 70B-class layer at
D = 4 is measured as a nested line (``extra``).

``e2e`` times the same step through ``dcp_decode_step_host`` -- the C-ABI
call that takes HOST buffers: every step copies its query, lengths and block
tables up from pinned host memory and its merged O and LSE back, inside the
timed region, one step after another on one stream.

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
DEFAULT_WORKLOAD = "mla_mix"
DEFAULT_EXTRA = "gqa_70b:4"


def parse(argv=None):
    ap = argparse.ArgumentParser(description=__doc__, formatter_class=argparse.RawDescriptionHelpFormatter)
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=200)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", default=DEFAULT_WORKLOAD)
    ap.add_argument("--shards", type=int, default=None, help="D (default: the largest of the workload's list)")
    ap.add_argument("--other-d-steps", type=int, default=50, help="steps for the workload's other D values (0: skip)")
    ap.add_argument("--extra", default=DEFAULT_EXTRA,
                    help="comma-separated workload:D lines measured after the headline ('' for none)")
    ap.add_argument("--extra-steps", type=int, default=300)
    ap.add_argument("--e2e-steps", type=int, default=30)
    ap.add_argument("--cpu-seconds", type=float, default=10.0, help="CPU baseline budget per leg")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--q-len", type=int, default=1,
                    help="query tokens per request (multi-token decode, causal within the draft; 1..4)")
    ap.add_argument("--kv-dtype", choices=["bf16", "fp8"], default="bf16",
                    help="cache element type (fp8: E4M3 codes, per-tensor scales 2^-7; GQA and MLA)")
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


def load_workload(name, batch_limit=None, q_len=1, kv_dtype="bf16"):
    import synth
    w = synth.workload(name)
    if batch_limit is not None and batch_limit < w.batch:
        w.seq_lens = w.seq_lens[:batch_limit]
        w.batch = batch_limit
        w.name = f"{w.name}[:{batch_limit}]"
    if q_len != 1:
        w.q_len = q_len
        w.name = f"{w.name} q_len={q_len}"
    w.extra["kv_dtype"] = kv_dtype
    if kv_dtype == "fp8":
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


MLA_SAMPLE_HEADS = 4


def _sample_at(w, i: int, max_tokens: int = None):
    """(request, q, KV source, heads, KV bytes the sample stands for).

    GQA: one (request, KV head) pair -- its G query heads are the whole work on those KV bytes.
    MLA: 4 of the 64 query heads of a request; every head reads the whole latent row, so the
    sample stands for 4/64 of the request's KV bytes."""
    import synth
    order = sorted(range(w.batch), key=lambda b: (b * 7919) % w.batch)
    b = order[i % w.batch]
    if w.layout == synth.GQA:
        h = (i // w.batch + b) % w.num_kv_heads
        G = w.num_q_heads // w.num_kv_heads
        src = w.kv_source_head(b, h, max_tokens)
        return (b, w.query(b)[h * G:(h + 1) * G], src, G, src.shape[0] * 2 * w.head_dim_qk * 2)
    src = w.kv_source(b, max_tokens)
    hq = MLA_SAMPLE_HEADS
    return (b, w.query(b)[:hq], src, hq, src.shape[0] * w.head_dim_qk * 2 * hq // w.num_q_heads)


def cpu_single_thread(w, D: int, budget_s: float):
    """Time the oracle on samples in this process until ``budget_s`` seconds of oracle work."""
    spent, kv_bytes, n, i = 0.0, 0, 0, 0
    while spent < budget_s and i < 4 * w.batch:
        s = _sample_at(w, i)
        spent += run_oracle_sample(w, D, s)
        kv_bytes += s[4]
        n += 1
        i += 1
    return kv_bytes / spent / 1e9, spent, n


def _oracle_worker(wname, batch_limit, D, indices, reps, max_tokens, start, out):
    """One process of the all-core leg: build its few samples, wait for the others, then time the
    oracle over them `reps` times (the oracle's time does not depend on the values)."""
    sys.path.insert(0, ROOT)
    w = load_workload(wname, batch_limit)
    samples = [_sample_at(w, i, max_tokens) for i in indices]
    start.wait()
    t0 = time.perf_counter()
    kv = 0
    for r in range(reps):
        s = samples[r % len(samples)]
        run_oracle_sample(w, D, s)
        kv += s[4]
    out.put((kv, time.perf_counter() - t0))


def cpu_all_cores(w, D: int, rate_1t_gbs: float, budget_s: float, batch_limit=None):
    """The oracle in one process per host core (spawned: no fork after CUDA initialisation),
    each on its own samples of at most 4,096 tokens, sized so every process has about
    ``budget_s`` seconds of oracle work.  Returns (GB/s, cores, samples, seconds)."""
    import multiprocessing as mp
    cores = len(os.sched_getaffinity(0)) if hasattr(os, "sched_getaffinity") else (os.cpu_count() or 1)
    max_tokens = 4096
    s0 = _sample_at(w, 0, max_tokens)
    per_sample_s = max(1e-3, s0[4] / (rate_1t_gbs * 1e9))
    per_worker = max(1, int(budget_s / per_sample_s))
    ctx = mp.get_context("spawn")
    start = ctx.Barrier(cores + 1)
    out = ctx.Queue()
    distinct = min(per_worker, 3)
    procs = [ctx.Process(target=_oracle_worker,
                         args=(w.name.split("[")[0].split(" ")[0], batch_limit, D,
                               [c * distinct + k for k in range(distinct)], per_worker, max_tokens, start, out))
             for c in range(cores)]
    for p in procs:
        p.start()
    try:
        start.wait(timeout=600)
        res = [out.get(timeout=600) for _ in procs]
    finally:
        for p in procs:
            p.join(timeout=60)
            if p.is_alive():
                p.terminate()
    kv = sum(r[0] for r in res)
    secs = max(r[1] for r in res)
    return kv / secs / 1e9, cores, cores * per_worker, secs, max_tokens


def cpu_baseline(w, D: int, budget_s: float, batch_limit=None):
    what = "(request, KV head) pairs" if w.layout == 0 else f"(request, {MLA_SAMPLE_HEADS} of 64 heads) pairs"
    gbs1, secs1, n1 = cpu_single_thread(w, D, budget_s)
    line = {"unit": "GB/s", "kind": "oracle",
            "single_thread": {"value": round(gbs1, 4), "cores": 1, "seconds": round(secs1, 2),
                              "sample": f"{n1} {what} of {w.name}, D={D}, whole requests"}}
    try:
        gbs, cores, n, secs, mt = cpu_all_cores(w, D, gbs1, budget_s, batch_limit)
        line.update({"value": round(gbs, 4), "cores": cores, "seconds": round(secs, 2),
                     "sample": f"{n} {what} of {w.name} (first {mt} tokens each), D={D}: float64 shard "
                               f"partials + merge, one process per host core ({cores})"})
    except Exception as e:  # the all-core leg is a report; a host that cannot spawn falls back to 1 core
        line.update({"value": round(gbs1, 4), "cores": 1, "sample": line["single_thread"]["sample"],
                     "all_cores_error": f"{type(e).__name__}: {e}"})
    line["host_cores"] = os.cpu_count()
    return line


# ----------------------------------------------------------------------------- our arm
class Bench:
    """Device-side plumbing shared by every measured line."""

    def __init__(self, local: int, world: int):
        import torch
        torch.cuda.set_device(local)
        self.dev = torch.device("cuda", local)
        self.world = world
        l2 = torch.cuda.get_device_properties(local).L2_cache_size
        # never written after this: reading it evicts L2 without adding dirty lines of its own
        self.flush_buf = torch.ones(2 * l2 // 4, dtype=torch.int32, device=self.dev)
        self.flush_out = torch.empty((), dtype=torch.int32, device=self.dev)
        self.peaks, self.peaks_kind = measured_peaks()

    def flush(self):
        import torch
        torch.amax(self.flush_buf, dim=0, out=self.flush_out)

    def build(self, w, D):
        import torch
        import synth.device as sdev
        from sequence_sharded_decode_paged_b200.cache import ShardedPagedCache
        cache = ShardedPagedCache(w.layout, w.num_q_heads, w.num_kv_heads, w.head_dim_qk, w.head_dim_v,
                                  w.block_size, D, w.seq_lens, w.softmax_scale, device=self.dev, q_len=w.q_len,
                                  kv_dtype=1 if cache_elem_bytes(w) == 1 else 0, k_scale=FP8_SCALE,
                                  v_scale=FP8_SCALE)
        kv = sdev.kv_source(w, self.dev, cache.cu_seqlens)
        cache.place(kv)
        del kv
        q = sdev.query(w, self.dev)
        torch.cuda.synchronize()
        return cache, q

    def timed(self, cache, q, steps, warmup):
        """(mean step ms, mean partials ms, mean merge ms, median step ms) over `steps` steps."""
        import torch
        for _ in range(warmup):
            self.flush()
            cache.step(q)
        torch.cuda.synchronize()
        ev = [[torch.cuda.Event(enable_timing=True) for _ in range(3)] for _ in range(steps)]
        barrier(self.world)
        torch.cuda.synchronize()
        for i in range(steps):
            self.flush()
            ev[i][0].record()
            cache.partials(q)
            ev[i][1].record()
            cache.merge()
            ev[i][2].record()
        torch.cuda.synchronize()
        barrier(self.world)
        part = [e[0].elapsed_time(e[1]) for e in ev]
        merge = [e[1].elapsed_time(e[2]) for e in ev]
        step = [e[0].elapsed_time(e[2]) for e in ev]
        return sum(step) / steps, sum(part) / steps, sum(merge) / steps, statistics.median(step)

    def merge_floor_us(self, D: int, d_v: int, steps: int = 200) -> float:
        """Event time of a merge of a single row: the launch-and-latency floor that every merge
        pays on this GPU (measured here, the same way the timed merges are)."""
        import torch
        from sequence_sharded_decode_paged_b200 import dcp
        Op = [torch.zeros(d_v, dtype=torch.float32, device=self.dev) for _ in range(D)]
        Lp = [torch.zeros(1, dtype=torch.float32, device=self.dev) for _ in range(D)]
        O = torch.empty(d_v, dtype=torch.float32, device=self.dev)
        L = torch.empty(1, dtype=torch.float32, device=self.dev)
        for _ in range(5):
            dcp.dcp_lse_merge(Op, Lp, D, 1, d_v, O, L)
        ev = [[torch.cuda.Event(enable_timing=True) for _ in range(2)] for _ in range(steps)]
        torch.cuda.synchronize()
        for i in range(steps):
            self.flush()
            ev[i][0].record()
            dcp.dcp_lse_merge(Op, Lp, D, 1, d_v, O, L)
            ev[i][1].record()
        torch.cuda.synchronize()
        return statistics.median(e[0].elapsed_time(e[1]) for e in ev) * 1e3

    def figures(self, w, D, step_ms, part_ms, merge_ms):
        """Roofline and throughput figures of one measured line (times already max over ranks)."""
        kv_b, dec_b, mrg_b = algorithmic_bytes(w, D)
        peak = self.peaks["hbm_gbs"]
        achieved = dec_b / part_ms / 1e6
        merge_ideal_us = mrg_b / (peak * 1e3)
        floor_us = self.merge_floor_us(D, w.head_dim_v)
        return {
            "kv_gbs": round(job_value(self.world, kv_b, step_ms), 1),
            "us_per_step_per_layer": round(step_ms * 1e3, 2),
            "roofline": {"bound": "hbm", "achieved": round(achieved, 1), "peak": peak, "unit": "GB/s",
                         "frac": round(achieved / peak, 4), "traffic": recorded_traffic(w.name, D, w.layout),
                         "kernel": "gqa_decode_kernel" if w.layout == 0 else "mla_decode_kernel",
                         "peak_kind": f"{self.peaks_kind} HBM copy (burst)",
                         "algorithmic_bytes_per_launch": dec_b},
            "decode_kernel_us": round(part_ms * 1e3, 2),
            "merge_kernel_us": round(merge_ms * 1e3, 2),
            "merge_gbs": round(mrg_b / merge_ms / 1e6, 1),
            "merge_frac": round(mrg_b / merge_ms / 1e6 / peak, 4),
            "merge_bytes": mrg_b,
            "merge_floor_us": round(floor_us, 2),
            "merge_bound": ("hbm" if merge_ideal_us >= floor_us else
                            f"latency: ideal {merge_ideal_us:.2f} us at the copy peak is under the "
                            f"{floor_us:.2f} us measured floor of a one-row merge"),
            "context_tokens_per_s": round(self.world * w.total_tokens / step_ms * 1e3, 1),
            "query_tokens_per_s": round(self.world * w.batch * w.q_len / step_ms * 1e3, 1),
            "frac_of_8tbs_spec": round(achieved / 8000.0, 4),
            "tensor": tensor_figures(w, part_ms, self.peaks, self.peaks_kind),
        }

    def e2e_host_calls(self, cache, q, steps):
        """Steps through dcp_decode_step_host (host inputs and outputs), one after another on one
        stream; returns (ms per step, h2d bytes, d2h bytes)."""
        import numpy as np
        import torch
        from sequence_sharded_decode_paged_b200 import dcp
        d = cache.desc
        rows = cache.batch * cache.q_len * d.num_q_heads
        h_q = torch.empty(q.numel(), dtype=torch.int16).pin_memory()
        h_q.copy_(q.reshape(-1).view(torch.int16).cpu())
        h_lens = torch.tensor(cache.seq_lens, dtype=torch.int32).pin_memory()
        h_tab = torch.from_numpy(np.ascontiguousarray(cache.tables_host, dtype=np.int32)).pin_memory()
        h_O = [torch.empty(rows * d.head_dim_v, dtype=torch.float32).pin_memory() for _ in range(2)]
        h_L = [torch.empty(rows, dtype=torch.float32).pin_memory() for _ in range(2)]
        nb = dcp.dcp_host_step_staging_bytes(d, cache.D)
        staging = torch.empty(nb, dtype=torch.uint8, device=self.dev)
        stream = torch.cuda.current_stream()

        def step(i):
            dcp.dcp_decode_step_host(d, cache.D, h_q, h_lens, h_tab, cache.pools, cache.pool_pages, staging,
                                     cache.workspace, h_O[i & 1], h_L[i & 1], stream=stream)

        for i in range(2):
            self.flush()
            step(i)
        torch.cuda.synchronize()
        barrier(self.world)
        ev = [[torch.cuda.Event(enable_timing=True) for _ in range(2)] for _ in range(steps)]
        for i in range(steps):
            self.flush()
            ev[i][0].record(stream)
            step(i)
            ev[i][1].record(stream)
        torch.cuda.synchronize()
        barrier(self.world)
        ms = sum(e[0].elapsed_time(e[1]) for e in ev) / steps
        assert np.isfinite(h_O[0].numpy()).all(), "e2e: non-finite output"
        h2d = h_q.numel() * 2 + h_lens.numel() * 4 + h_tab.numel() * 4
        d2h = h_O[0].numel() * 4 + h_L[0].numel() * 4
        return ms, h2d, d2h

    def e2e_pipelined(self, cache, q, steps):
        """The overlapped host pipeline (uploads and downloads of neighbouring steps hidden behind
        the current step's compute): a throughput figure, reported beside the per-step e2e."""
        import numpy as np
        import torch
        from sequence_sharded_decode_paged_b200.cache import HostStepPipeline
        pipe = HostStepPipeline(cache)
        host_in = pipe.pack_inputs(q.view(torch.int16).cpu().numpy(), cache.seq_lens, cache.tables_host)
        host_out = [pipe.host_output(), pipe.host_output()]
        for i in range(2):
            pipe.step(i, host_in, host_out[i & 1])
        pipe.synchronize()
        barrier(self.world)
        torch.cuda.synchronize()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(pipe.s_in)
        for i in range(steps):
            pipe.step(i, host_in, host_out[i & 1])
        e1.record(pipe.s_out)
        pipe.synchronize()
        torch.cuda.synchronize()
        barrier(self.world)
        assert np.isfinite(pipe.unpack_output(host_out[0])[0].numpy()).all()
        return e0.elapsed_time(e1) / max(1, steps)

    def append_us(self, w, cache, D):
        """Cache write of one new token per request (the append that precedes each decode step),
        20 calls captured in one CUDA graph; it rewrites each request's last slot."""
        import torch
        from sequence_sharded_decode_paged_b200 import dcp
        row_elems = w.kv_bytes_per_token // 2
        kv_row = torch.zeros((w.batch, row_elems), dtype=torch.int16, device=self.dev)
        cu_rows = torch.arange(w.batch + 1, dtype=torch.int64, device=self.dev)
        last_pos = (cache.seq_lens_dev - 1).clamp_min(0).contiguous()
        side = torch.cuda.Stream(self.dev)
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
        ms = a0.elapsed_time(a1) / 100
        del graph
        return ms


def run_ours(args, rank, world, local):
    import torch

    dist_init(world, "nccl")
    bench = Bench(local, world)
    dev = bench.dev
    w = load_workload(args.workload, args.batch_limit, args.q_len, args.kv_dtype)
    D = args.shards or max(w.shards)
    launches = 0

    cache, q = bench.build(w, D)
    sampler = ClockSampler(local)
    time.sleep(0.3)
    step_ms, part_ms, merge_ms, step_med = bench.timed(cache, q, args.steps, args.warmup)
    clocks = sampler.stop()
    launches += 2 * args.steps
    err = cache.device_error()
    if err != 0:
        raise RuntimeError(f"device status {err} during the timed run")

    e2e_ms, h2d, d2h = bench.e2e_host_calls(cache, q, args.e2e_steps)
    launches_e2e = 2 * args.e2e_steps
    pipe_ms = bench.e2e_pipelined(cache, q, args.e2e_steps)
    if cache.device_error() != 0:
        raise RuntimeError("device status set during the e2e runs")
    append_ms = bench.append_us(w, cache, D)

    step_ms, part_ms, merge_ms, e2e_ms, pipe_ms, append_ms = (
        reduce_max(x, world, dev) for x in (step_ms, part_ms, merge_ms, e2e_ms, pipe_ms, append_ms))
    fig = bench.figures(w, D, step_ms, part_ms, merge_ms)
    kv_b, _, _ = algorithmic_bytes(w, D)

    other = {}
    if args.other_d_steps > 0:
        for Dx in w.shards:
            if Dx == D:
                continue
            del cache, q
            torch.cuda.empty_cache()
            cache, q = bench.build(w, Dx)
            s_ms, p_ms, m_ms, _ = bench.timed(cache, q, args.other_d_steps, max(3, args.warmup))
            s_ms, p_ms, m_ms = (reduce_max(x, world, dev) for x in (s_ms, p_ms, m_ms))
            f = bench.figures(w, Dx, s_ms, p_ms, m_ms)
            other[str(Dx)] = {k: f[k] for k in ("kv_gbs", "us_per_step_per_layer", "decode_kernel_us",
                                                 "merge_kernel_us", "merge_gbs", "merge_bound")}
            other[str(Dx)]["roofline_frac"] = f["roofline"]["frac"]
            other[str(Dx)]["steps"] = args.other_d_steps
    del cache, q
    torch.cuda.empty_cache()

    extra = {}
    for spec in [s for s in args.extra.split(",") if s.strip()]:
        name, _, dspec = spec.partition(":")
        wx = load_workload(name.strip())
        Dx = int(dspec) if dspec else max(wx.shards)
        cx, qx = bench.build(wx, Dx)
        s_ms, p_ms, m_ms, _ = bench.timed(cx, qx, args.extra_steps, max(3, args.warmup))
        if cx.device_error() != 0:
            raise RuntimeError(f"device status set during the {name} run")
        s_ms, p_ms, m_ms = (reduce_max(x, world, dev) for x in (s_ms, p_ms, m_ms))
        f = bench.figures(wx, Dx, s_ms, p_ms, m_ms)
        f.update({"workload": f"{wx.name}: {wx.note}", "D": Dx, "steps": args.extra_steps,
                  "ms_per_step": round(s_ms, 4), "context_tokens": wx.total_tokens})
        extra[f"{wx.name}/D{Dx}"] = f
        del cx, qx
        torch.cuda.empty_cache()

    if rank != 0:
        return None
    line = {
        "metric": METRIC,
        "value": fig["kv_gbs"],
        "unit": "GB/s",
        "n_gpus": world,
        "steps": args.steps,
        "warmup": args.warmup,
        "ms_per_step": round(step_ms, 4),
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": "bf16" if cache_elem_bytes(w) == 2 else "fp8-e4m3 cache, f16 products, f32 accumulate",
        "data": "synthetic",
        "config": {"workload": f"{w.name}: {w.note}", "D": D, "batch": w.batch, "q_len": w.q_len,
                   "context_tokens": w.total_tokens, "kv_bytes_per_step": kv_b,
                   "l2": "flushed before every step by reading a buffer of 2x L2 (no writes), outside the "
                         "timed events; the KV read per step is also far larger than L2",
                   "parallelism": "replicas" if world > 1 else "single GPU (D shard pools in one HBM)"},
        "roofline": fig["roofline"],
        "us_per_step_per_layer": fig["us_per_step_per_layer"],
        "decode_kernel_us": fig["decode_kernel_us"],
        "merge_kernel_us": fig["merge_kernel_us"],
        "merge_gbs": fig["merge_gbs"],
        "merge_frac": fig["merge_frac"],
        "merge_bound": fig["merge_bound"],
        "merge_floor_us": fig["merge_floor_us"],
        "append_kernel_us": round(append_ms * 1e3, 2),
        "append_bytes_per_step": w.batch * w.kv_bytes_per_token * (2 + cache_elem_bytes(w)) // 2,
        "context_tokens_per_s": fig["context_tokens_per_s"],
        "query_tokens_per_s": fig["query_tokens_per_s"],
        "frac_of_8tbs_spec": fig["frac_of_8tbs_spec"],
        "tensor": fig["tensor"],
        "median_step_ms": round(step_med, 4),
        "gpu_launches": launches,
        "clocks": clocks,
        "e2e": {"value": round(job_value(world, kv_b, e2e_ms), 1), "unit": "GB/s",
                "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h, "ms_per_step": round(e2e_ms, 4),
                "steps": args.e2e_steps, "gpu_launches": launches_e2e,
                "api": "dcp_decode_step_host (C ABI, host buffers): per step the H2D copies of query, "
                       "lengths and tables, decode, merge and the D2H copies of O and LSE, steps serialised "
                       "on one stream",
                "pipelined": {"value": round(job_value(world, kv_b, pipe_ms), 1), "unit": "GB/s",
                              "ms_per_step": round(pipe_ms, 4),
                              "api": "HostStepPipeline: the same copies, overlapped with neighbouring steps"}},
        "other_D": other,
        "extra": extra,
    }
    if world == 1 and not args.no_cpu_baseline and w.q_len == 1 and cache_elem_bytes(w) == 2:
        line["cpu_baseline"] = cpu_baseline(w, D, args.cpu_seconds, args.batch_limit)
    return line


# ----------------------------------------------------------------------------- reference arm (the oracle)
def run_reference(args, rank, world):
    if rank != 0:  # the oracle runs once, on rank 0; other ranks have no work
        return None
    w = load_workload(args.workload, args.batch_limit, args.q_len, args.kv_dtype)
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
    what = "(request, KV head)" if w.layout == 0 else f"(request, {MLA_SAMPLE_HEADS} of 64 heads)"
    line = {
        "impl": "reference", "metric": METRIC, "value": round(value, 4), "unit": "GB/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(secs_total / args.steps * 1e3, 3),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": {"workload": f"{w.name}: {w.note}", "D": D, "batch": w.batch, "context_tokens": w.total_tokens},
        "cpu_baseline": {"value": round(value, 4), "unit": "GB/s", "cores": 1, "kind": "oracle",
                         "sample": f"each step: one {what} sample of {w.name}, at most {max_tok} tokens, "
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
