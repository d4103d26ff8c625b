"""Seeded synthetic inputs for decode-context-parallel attention.

This module is shared by the float64 oracle (``oracle/``) and by the CUDA
library's tests and benchmark.  It only *draws numbers*: it contains none of
the attention, sharding or merge arithmetic.  Two implementations of the same
generator exist: the numpy one below (host) and ``synth_fill.cu`` (device, used
to fill multi-GB caches quickly).  They produce bit-identical bf16 values; a
CPU test checks the numpy side against fixed values and a GPU test checks the
device side against the numpy side.

Generator definition (counter based, no libm, integer exact up to one IEEE
double multiply that both sides perform identically):

* ``mix64`` is the SplitMix64 output function (Steele, Lea & Flood, "Fast
  splittable pseudorandom number generators", OOPSLA 2014; constants as
  published by Vigna).  The n-th output of a SplitMix64 stream whose state
  starts at ``s`` is ``mix64(s + n * GAMMA)`` (n = 1, 2, ...).
* Stream key of (seed, tensor id, request b):
  ``k = mix64(mix64(seed + GAMMA*(1+tensor)) + GAMMA*(1+b))``.
* Element ``e`` of that stream: ``x = mix64(k + GAMMA*(1+e))``; the four
  16-bit fields of ``x`` are summed (Irwin-Hall of 4), centred and scaled to
  unit variance: ``z = (S - 131070) * INV_SD`` (double), multiplied by the
  tensor's amplitude (a power of two), rounded to float32 (RNE) and then to
  bf16 (RNE).  Values are approximately N(0, amp^2), bounded by 3.46*amp.

Element indices (logical, unsharded tensors; the caller never sees shards):

* GQA key  ``K[b][t][h][k]``: tensor ``T_K``, ``e = (t*Hkv + h)*d + k``.
* GQA value``V[b][t][h][k]``: tensor ``T_V``, same ``e``.
* MLA latent row ``C[b][t][k]`` (k < 576): tensor ``T_LATENT``, ``e = t*576 + k``.
* query ``q[b][h][k]``: tensor ``T_Q``, ``e = h*d_qk + k``; with ``q_len`` query tokens,
  ``q[b][j][h][k]`` has ``e = (j*Hq + h)*d_qk + k`` (token 0 is the single-token query).

The unsharded KV source layout consumed by the cache-placement call is
``[token][2][Hkv][d]`` for GQA and ``[token][d_qk]`` for MLA, with requests
concatenated in order.
"""
from __future__ import annotations

import math
from dataclasses import dataclass, field
from typing import List, Optional

import numpy as np

GAMMA = 0x9E3779B97F4A7C15
M1 = 0xBF58476D1CE4E5B9
M2 = 0x94D049BB133111EB
MASK64 = (1 << 64) - 1
# 1 / sqrt(4 * (65536^2 - 1) / 12): unit variance for a sum of four uniform 16-bit integers.
INV_SD = 2.6428997921303014e-05
CENTRE = 131070  # 4 * 65535 / 2

T_Q, T_K, T_V, T_LATENT = 1, 2, 3, 4

GQA, MLA = 0, 1


# ---------------------------------------------------------------------------
# scalar (python int) SplitMix64, used for keys, seq_len recipes and tests
# ---------------------------------------------------------------------------
def mix64(z: int) -> int:
    z &= MASK64
    z = ((z ^ (z >> 30)) * M1) & MASK64
    z = ((z ^ (z >> 27)) * M2) & MASK64
    return z ^ (z >> 31)


def stream_key(seed: int, tensor: int, request: int) -> int:
    k0 = mix64(seed + GAMMA * (1 + tensor))
    return mix64(k0 + GAMMA * (1 + request))


class SplitMix64:
    """Sequential SplitMix64 stream (state starts at ``seed``)."""

    def __init__(self, seed: int):
        self.state = seed & MASK64

    def next(self) -> int:
        self.state = (self.state + GAMMA) & MASK64
        return mix64(self.state)

    def uniform(self) -> float:
        """Double in (0, 1): top 53 bits, offset by half an ulp so 0 never occurs."""
        return ((self.next() >> 11) + 0.5) * (1.0 / 9007199254740992.0)


# ---------------------------------------------------------------------------
# vectorised numpy generator (bit-identical to the device generator)
# ---------------------------------------------------------------------------
def _mix64_np(z: np.ndarray) -> np.ndarray:
    z = (z ^ (z >> np.uint64(30))) * np.uint64(M1)
    z = (z ^ (z >> np.uint64(27))) * np.uint64(M2)
    return z ^ (z >> np.uint64(31))


def f32_to_bf16_bits(f: np.ndarray) -> np.ndarray:
    """Round float32 to bf16 (round to nearest, ties to even); no NaN inputs expected."""
    u = np.ascontiguousarray(f, dtype=np.float32).view(np.uint32).astype(np.uint64)
    lsb = (u >> np.uint64(16)) & np.uint64(1)
    r = (u + np.uint64(0x7FFF) + lsb) >> np.uint64(16)
    return r.astype(np.uint16)


def bf16_bits_to_f64(b: np.ndarray) -> np.ndarray:
    u = b.astype(np.uint32) << np.uint32(16)
    return u.view(np.float32).astype(np.float64)


def values_bf16(seed: int, tensor: int, request: int, e0: int, n: int, amp: float) -> np.ndarray:
    """bf16 bit patterns of elements ``e0 .. e0+n-1`` of one stream (generated in chunks)."""
    chunk = 1 << 23
    if n > chunk:
        out = np.empty(n, dtype=np.uint16)
        for c0 in range(0, n, chunk):
            out[c0:c0 + chunk] = values_bf16(seed, tensor, request, e0 + c0, min(chunk, n - c0), amp)
        return out
    with np.errstate(over="ignore"):
        key = np.uint64(stream_key(seed, tensor, request))
        e = np.arange(e0, e0 + n, dtype=np.uint64)
        x = _mix64_np(key + np.uint64(GAMMA) * (e + np.uint64(1)))
        s = ((x & np.uint64(0xFFFF)) + ((x >> np.uint64(16)) & np.uint64(0xFFFF))
             + ((x >> np.uint64(32)) & np.uint64(0xFFFF)) + (x >> np.uint64(48)))
    z = (s.astype(np.int64) - CENTRE).astype(np.float64) * INV_SD
    v = (z * amp).astype(np.float32)
    return f32_to_bf16_bits(v)


def values_bf16_at(seed: int, tensor: int, request: int, e: np.ndarray, amp: float) -> np.ndarray:
    """bf16 bit patterns of the stream elements with indices ``e`` (any shape)."""
    with np.errstate(over="ignore"):
        key = np.uint64(stream_key(seed, tensor, request))
        ee = np.asarray(e, dtype=np.uint64)
        x = _mix64_np(key + np.uint64(GAMMA) * (ee + np.uint64(1)))
        s = ((x & np.uint64(0xFFFF)) + ((x >> np.uint64(16)) & np.uint64(0xFFFF))
             + ((x >> np.uint64(32)) & np.uint64(0xFFFF)) + (x >> np.uint64(48)))
    z = (s.astype(np.int64) - CENTRE).astype(np.float64) * INV_SD
    return f32_to_bf16_bits((z * amp).astype(np.float32))


# ---------------------------------------------------------------------------
# workloads
# ---------------------------------------------------------------------------
@dataclass
class Workload:
    """One synthetic decode step: shapes, seq_lens, seeds and amplitudes."""

    name: str
    layout: int
    batch: int
    num_q_heads: int
    num_kv_heads: int
    head_dim_qk: int
    head_dim_v: int
    block_size: int
    shards: List[int]
    seq_lens: List[int]
    softmax_scale: float
    seed: int
    q_amp: float = 1.0
    kv_amp: float = 1.0
    perm_seed: int = 0
    note: str = ""
    extra: dict = field(default_factory=dict)
    q_len: int = 1  # query tokens per request (multi-token decode when > 1)

    @property
    def kv_bytes_per_token(self) -> int:
        if self.layout == GQA:
            return 2 * self.num_kv_heads * self.head_dim_qk * 2
        return self.head_dim_qk * 2

    @property
    def total_tokens(self) -> int:
        return int(sum(self.seq_lens))

    # host-side generation of one request's inputs (small / sampled cases)
    def query(self, b: int) -> np.ndarray:
        n = self.num_q_heads * self.head_dim_qk
        return values_bf16(self.seed, T_Q, b, 0, n, self.q_amp).reshape(self.num_q_heads, self.head_dim_qk)

    def queries(self, b: int) -> np.ndarray:
        """All ``q_len`` query tokens of request ``b``: ``[q_len][Hq][d_qk]``; token 0 is ``query(b)``."""
        n = self.q_len * self.num_q_heads * self.head_dim_qk
        return values_bf16(self.seed, T_Q, b, 0, n, self.q_amp).reshape(self.q_len, self.num_q_heads,
                                                                        self.head_dim_qk)

    def kv_source_head(self, b: int, h: int, n_tok: Optional[int] = None) -> np.ndarray:
        """GQA: request ``b``'s rows of KV head ``h`` only, as a one-head source ``[n][2][1][d]``
        (the first ``n_tok`` tokens if given)."""
        n_tok = self.seq_lens[b] if n_tok is None else min(n_tok, self.seq_lens[b])
        d, H = self.head_dim_qk, self.num_kv_heads
        e = (np.arange(n_tok, dtype=np.uint64)[:, None] * np.uint64(H) + np.uint64(h)) * np.uint64(d) \
            + np.arange(d, dtype=np.uint64)[None, :]
        k = values_bf16_at(self.seed, T_K, b, e, self.kv_amp)
        v = values_bf16_at(self.seed, T_V, b, e, self.kv_amp)
        return np.stack([k, v], axis=1).reshape(n_tok, 2, 1, d)

    def kv_source(self, b: int, n_tok: Optional[int] = None) -> np.ndarray:
        """Unsharded KV rows of request ``b`` (bf16 bits), the first ``n_tok`` tokens if given.

        GQA: ``[seq_len][2][Hkv][d]``; MLA: ``[seq_len][d_qk]``.
        """
        n_tok = self.seq_lens[b] if n_tok is None else min(n_tok, self.seq_lens[b])
        if self.layout == GQA:
            per = self.num_kv_heads * self.head_dim_qk
            k = values_bf16(self.seed, T_K, b, 0, n_tok * per, self.kv_amp).reshape(n_tok, 1, per)
            v = values_bf16(self.seed, T_V, b, 0, n_tok * per, self.kv_amp).reshape(n_tok, 1, per)
            return np.concatenate([k, v], axis=1).reshape(n_tok, 2, self.num_kv_heads, self.head_dim_qk)
        return values_bf16(self.seed, T_LATENT, b, 0, n_tok * self.head_dim_qk, self.kv_amp).reshape(
            n_tok, self.head_dim_qk)


def _uniform_lens(seed: int, n: int, lo: int, hi: int) -> List[int]:
    g = SplitMix64(seed)
    return [lo + g.next() % (hi - lo + 1) for _ in range(n)]


def _lognormal_lens(seed: int, n: int, median: float, sigma: float, lo: int, hi: int) -> List[int]:
    g = SplitMix64(seed)
    out = []
    for _ in range(n):
        u1, u2 = g.uniform(), g.uniform()
        z = math.sqrt(-2.0 * math.log(u1)) * math.cos(2.0 * math.pi * u2)
        out.append(int(min(hi, max(lo, round(median * math.exp(sigma * z))))))
    return out


# Piecewise log-linear inverse CDF of the agentic trace statistics
# (median ~67K, 53% > 64K, ~8% > 128K, 3-4% > 256K, 18% < 8K; capped at 320K).
AGENTIC_KNOTS = [(1024, 0.0), (8192, 0.18), (65536, 0.47), (67000, 0.50),
                 (131072, 0.92), (262144, 0.965), (327680, 1.0)]


def agentic_len(u: float) -> int:
    for (l0, c0), (l1, c1) in zip(AGENTIC_KNOTS, AGENTIC_KNOTS[1:]):
        if u <= c1:
            f = (u - c0) / (c1 - c0)
            return int(round(math.exp(math.log(l0) + f * (math.log(l1) - math.log(l0)))))
    return AGENTIC_KNOTS[-1][0]


def _agentic_lens(seed: int, n: int) -> List[int]:
    lens = [agentic_len((i + 0.5) / n) for i in range(n)]
    g = SplitMix64(seed)
    for i in range(n - 1, 0, -1):  # Fisher-Yates shuffle of the stratified quantiles
        j = g.next() % (i + 1)
        lens[i], lens[j] = lens[j], lens[i]
    return lens


def workload(name: str) -> Workload:
    """The five decode workloads (index i: seeds i*1000 + {1: q, 2: K, 3: V, 4: latent, 5: lens})."""
    if name == "gqa_tiny":
        return Workload(name, GQA, 2, 8, 2, 64, 64, 16, [2], [100, 257], 1.0 / math.sqrt(64), seed=1000,
                        note="GQA tiny: batch 2, 8 q heads, 2 KV heads, head_dim 64, block 16, D=2")
    if name == "gqa_70b":
        return Workload(name, GQA, 64, 64, 8, 128, 128, 16, [1, 2, 4],
                        _uniform_lens(2005, 64, 8192, 32768), 1.0 / math.sqrt(128), seed=2000, kv_amp=0.5,
                        note="GQA 70B-class layer: 64 q / 8 KV heads, d 128, block 16, batch 64, 8K-32K")
    if name == "mla_b32":
        return Workload(name, MLA, 32, 64, 1, 576, 512, 64, [4],
                        _lognormal_lens(3005, 32, 67000.0, 0.6, 1024, 327680), 1.0 / math.sqrt(192), seed=3000,
                        note="MLA decode: 64 heads, 576 latent, batch 32, lognormal median 67K, block 64, D=4")
    if name == "mla_long":
        return Workload(name, MLA, 4, 64, 1, 576, 512, 64, [8],
                        _uniform_lens(4005, 4, 204800, 262144), 1.0 / math.sqrt(192), seed=4000,
                        note="MLA long context: batch 4, 200K-256K, block 64, D=8")
    if name == "mla_mix":
        return Workload(name, MLA, 256, 64, 1, 576, 512, 64, [1, 2, 4, 8], _agentic_lens(5005, 256),
                        1.0 / math.sqrt(192), seed=5000,
                        note="MLA agentic mix: 256 requests, bimodal lengths median ~67K, max 320K, block 64")
    raise KeyError(name)


WORKLOADS = ["gqa_tiny", "gqa_70b", "mla_b32", "mla_long", "mla_mix"]


def custom(layout: int, seq_lens, num_q_heads: int, num_kv_heads: int, head_dim_qk: int, head_dim_v: int,
           block_size: int, seed: int, softmax_scale: Optional[float] = None, q_amp: float = 1.0,
           kv_amp: float = 1.0, name: str = "custom", q_len: int = 1) -> Workload:
    """Ad-hoc workload for edge-case tests (same generator, any shape)."""
    if softmax_scale is None:
        softmax_scale = 1.0 / math.sqrt(head_dim_qk if layout == GQA else 192)
    return Workload(name, layout, len(seq_lens), num_q_heads, num_kv_heads, head_dim_qk, head_dim_v,
                    block_size, [1], list(int(s) for s in seq_lens), softmax_scale, seed, q_amp, kv_amp,
                    q_len=q_len)
