"""Shared set-up for the GPU parity tests: build a sharded cache for a
workload through the C ABI and compute the oracle's answers for it."""
import numpy as np
import torch

import oracle
import synth
from sequence_sharded_decode_paged_b200.cache import ShardedPagedCache

# Tolerances for bf16 KV with fp32 accumulation (checked against the float64 oracle).
O_TOL = 2e-2
LSE_TOL = 1e-3
D_INVARIANCE_TOL = 1e-3
# What the arithmetic allows: the softmax weights enter the PV product rounded to
# bf16 against an integral reference maximum, so each weight carries a relative
# error of at most 2^-8, and O (a weighted mean of bf16 values bounded by 3.46 *
# amplitude) is off by at most 2^-8 * 3.46 = 0.0135 at unit amplitude.
O_BOUND_UNIT_AMP = 3.47 * 2.0 ** -8


def host_kv(w: synth.Workload, requests=None) -> np.ndarray:
    reqs = range(w.batch) if requests is None else requests
    return np.concatenate([w.kv_source(b) for b in reqs]) if w.total_tokens else np.zeros((0,), np.uint16)


def host_q(w: synth.Workload) -> np.ndarray:
    """[B][Hq][d] queries, or [B][q_len][Hq][d] for multi-token decode."""
    return np.stack([w.query(b) if w.q_len == 1 else w.queries(b) for b in range(w.batch)])


def build_cache(w: synth.Workload, D: int, perm_seed: int = 0, pool_fill=0xFFFF, device_kv: bool = False):
    """Cache with the workload's KV placed in D shard pools; returns (cache, q on device)."""
    import synth.device as sdev
    cache = ShardedPagedCache(w.layout, w.num_q_heads, w.num_kv_heads, w.head_dim_qk, w.head_dim_v, w.block_size, D,
                              w.seq_lens, w.softmax_scale, perm_seed, "cuda", pool_fill, q_len=w.q_len)
    if w.total_tokens > 0:
        if device_kv:
            kv = sdev.kv_source(w, "cuda", cache.cu_seqlens)
        else:
            kv = torch.from_numpy(host_kv(w).view(np.int16)).cuda()
        cache.place(kv)
        del kv
    if device_kv:
        q = sdev.query(w, "cuda")
    else:
        q = torch.from_numpy(host_q(w).view(np.int16)).cuda()
    return cache, q


def oracle_request(w: synth.Workload, b: int, D: int):
    """(O, LSE, O_parts[D], LSE_parts[D]) of request b in float64."""
    return oracle.sharded(w.layout, w.num_q_heads, w.num_kv_heads, w.head_dim_qk, w.head_dim_v, w.query(b),
                          w.kv_source(b), w.softmax_scale, w.block_size, D)


def assert_lse_close(got: np.ndarray, want: np.ndarray, tol: float, what: str):
    inf_w = np.isneginf(want)
    assert (np.isneginf(got) == inf_w).all(), f"{what}: -inf pattern differs"
    if (~inf_w).any():
        err = np.abs(got[~inf_w] - want[~inf_w]).max()
        assert err <= tol, f"{what}: LSE max abs error {err}"


def assert_o_close(got: np.ndarray, want: np.ndarray, tol: float, what: str):
    assert np.isfinite(got).all(), f"{what}: non-finite output"
    err = np.abs(got - want).max() if got.size else 0.0
    assert err <= tol, f"{what}: O max abs error {err}"
    return err
