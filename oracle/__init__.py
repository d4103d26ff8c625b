"""Float64 CPU oracle for decode context parallelism (test infrastructure).

Only ``tests/``, ``__graft_entry__.smoke()`` and ``bench.py`` (its CPU
baseline and reference arm) may import this package.  It shares no code with
the CUDA library; its only common dependency is the seeded input generator in
``synth``, which draws numbers and holds none of the method's arithmetic.

The C source ``oracle.c`` holds every computation; this module compiles it
with gcc on first use (or through ``build()``) and marshals numpy arrays.
Function-level citations are in ``oracle.c``.
"""
from __future__ import annotations

import ctypes as C
import os
import subprocess
import threading
from typing import List, Optional, Sequence, Tuple

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "oracle.c")
_LIB_PATH = os.path.join(_HERE, "liboracle.so")
_lib = None
_lock = threading.Lock()

GQA, MLA = 0, 1


def build(force: bool = False) -> str:
    """Compile ``oracle.c`` into ``liboracle.so`` (plain gcc, -O2, no fast-math)."""
    if force or not os.path.exists(_LIB_PATH) or os.path.getmtime(_LIB_PATH) < os.path.getmtime(_SRC):
        tmp = _LIB_PATH + f".tmp{os.getpid()}"
        subprocess.check_call(["gcc", "-O2", "-std=c11", "-fPIC", "-shared", "-fno-fast-math", "-o", tmp,
                               _SRC, "-lm"])
        os.replace(tmp, _LIB_PATH)
    return _LIB_PATH


def _load():
    global _lib
    with _lock:
        if _lib is None:
            lib = C.CDLL(build())
            p = C.c_void_p
            lib.oracle_token_shard.restype = C.c_int
            lib.oracle_token_shard.argtypes = [C.c_int64, C.c_int, C.c_int]
            lib.oracle_token_local_block.restype = C.c_int64
            lib.oracle_token_local_block.argtypes = [C.c_int64, C.c_int, C.c_int]
            lib.oracle_block_tables.restype = C.c_int
            lib.oracle_block_tables.argtypes = [p, C.c_int, C.c_int, C.c_int, C.c_uint64, C.c_int, p, p, p]
            lib.oracle_token_shard_rule.restype = C.c_int
            lib.oracle_token_shard_rule.argtypes = [C.c_int64, C.c_int, C.c_int, C.c_int, C.c_int64]
            lib.oracle_token_local_block_rule.restype = C.c_int64
            lib.oracle_token_local_block_rule.argtypes = [C.c_int64, C.c_int, C.c_int, C.c_int, C.c_int64]
            lib.oracle_block_tables_rule.restype = C.c_int
            lib.oracle_block_tables_rule.argtypes = [p, C.c_int, C.c_int, C.c_int, C.c_int, C.c_uint64, C.c_int, p, p,
                                                     p]
            lib.oracle_place_request_rule.restype = None
            lib.oracle_place_request_rule.argtypes = [C.c_int, C.c_int, C.c_int, C.c_int, C.c_int, C.c_int, C.c_int,
                                                      C.c_int, C.c_int, p, C.c_int64, p, p]
            lib.oracle_attend_rule_f64.restype = None
            lib.oracle_attend_rule_f64.argtypes = [C.c_int, C.c_int, C.c_int, C.c_int, C.c_int, p, C.c_int64, p,
                                                   C.c_double, C.c_int, C.c_int, C.c_int, C.c_int, C.c_int64, C.c_int,
                                                   C.c_int, p, p]
            lib.oracle_grow_tables.restype = C.c_int
            lib.oracle_grow_tables.argtypes = [p, p, C.c_int, C.c_int, C.c_int, C.c_int, p, p, p, p]
            lib.oracle_place_request.restype = None
            lib.oracle_place_request.argtypes = [C.c_int, C.c_int, C.c_int, C.c_int, C.c_int, C.c_int, C.c_int,
                                                 C.c_int, p, C.c_int64, p, p]
            lib.oracle_attend.restype = None
            lib.oracle_attend.argtypes = [C.c_int, C.c_int, C.c_int, C.c_int, C.c_int, p, C.c_int64, p,
                                          C.c_double, C.c_int, C.c_int, C.c_int, C.c_int, C.c_int, p, p]
            lib.oracle_attend_f64.restype = None
            lib.oracle_attend_f64.argtypes = [C.c_int, C.c_int, C.c_int, C.c_int, C.c_int, p, C.c_int64, p,
                                              C.c_double, C.c_int, C.c_int, C.c_int, C.c_int, C.c_int, p, p]
            lib.oracle_e4m3_decode.restype = C.c_double
            lib.oracle_e4m3_decode.argtypes = [C.c_uint8]
            lib.oracle_e4m3_encode.restype = C.c_uint8
            lib.oracle_e4m3_encode.argtypes = [C.c_double]
            lib.oracle_quantize_e4m3.restype = None
            lib.oracle_quantize_e4m3.argtypes = [p, C.c_int64, C.c_float, p]
            lib.oracle_dequantize_e4m3.restype = None
            lib.oracle_dequantize_e4m3.argtypes = [p, C.c_int64, C.c_double, p]
            lib.oracle_place_request_u8.restype = None
            lib.oracle_place_request_u8.argtypes = [C.c_int, C.c_int, C.c_int, C.c_int, C.c_int, C.c_int, C.c_int,
                                                    C.c_int, p, C.c_int64, p, p]
            lib.oracle_place_request_mla_u8.restype = None
            lib.oracle_place_request_mla_u8.argtypes = [C.c_int, C.c_int, C.c_int, C.c_int, C.c_int, C.c_int,
                                                        C.c_int, p, C.c_int64, p, p]
            lib.oracle_merge.restype = None
            lib.oracle_merge.argtypes = [p, p, C.c_int, C.c_int64, C.c_int, p, p]
            lib.oracle_merge_ml.restype = None
            lib.oracle_merge_ml.argtypes = [p, p, p, C.c_int, C.c_int64, C.c_int, p]
            lib.oracle_kv_bytes_per_token.restype = C.c_int64
            lib.oracle_kv_bytes_per_token.argtypes = [C.c_int, C.c_int, C.c_int]
            lib.oracle_validate_config.restype = C.c_int
            lib.oracle_validate_config.argtypes = [C.c_int, C.c_int, C.c_int, C.c_int]
            _lib = lib
    return _lib


def _ptr(a: np.ndarray):
    return a.ctypes.data_as(C.c_void_p)


# ---------------------------------------------------------------------------
# sharding
# ---------------------------------------------------------------------------
def token_shard(t: int, block_size: int, D: int) -> int:
    return _load().oracle_token_shard(t, block_size, D)


def token_local_block(t: int, block_size: int, D: int) -> int:
    return _load().oracle_token_local_block(t, block_size, D)


INTERLEAVED, CONTIGUOUS = 0, 1  # shard rules


def token_shard_rule(t: int, block_size: int, D: int, rule: int, seq_len: int) -> int:
    return _load().oracle_token_shard_rule(t, block_size, D, rule, seq_len)


def token_local_block_rule(t: int, block_size: int, D: int, rule: int, seq_len: int) -> int:
    return _load().oracle_token_local_block_rule(t, block_size, D, rule, seq_len)


def block_tables(seq_lens: Sequence[int], block_size: int, D: int, perm_seed: int = 0,
                 max_local_blocks: Optional[int] = None, rule: int = INTERLEAVED
                 ) -> Tuple[np.ndarray, np.ndarray, np.ndarray]:
    """Returns ``(tables[D][B][max_local_blocks], local_len[D][B], num_pages[D])`` (int32)."""
    sl = np.ascontiguousarray(seq_lens, dtype=np.int32)
    B = sl.shape[0]
    if max_local_blocks is None:
        nblk = (int(sl.max()) + block_size - 1) // block_size if B else 0
        max_local_blocks = (nblk + D - 1) // D
    tables = np.empty((D, B, max_local_blocks), dtype=np.int32)
    local_len = np.empty((D, B), dtype=np.int32)
    num_pages = np.empty((D,), dtype=np.int32)
    rc = _load().oracle_block_tables_rule(_ptr(sl), B, block_size, D, rule, perm_seed, max_local_blocks,
                                          _ptr(tables), _ptr(local_len), _ptr(num_pages))
    if rc != 0:
        raise ValueError(f"oracle_block_tables failed ({rc})")
    return tables, local_len, num_pages


def grow_tables(old_lens: Sequence[int], new_lens: Sequence[int], block_size: int, D: int, tables: np.ndarray,
                local_len: np.ndarray, next_page: np.ndarray, pool_pages: Sequence[int]) -> int:
    """Grow ``tables[D][B][mlb]`` / ``local_len[D][B]`` / ``next_page[D]`` in place; returns the C status."""
    o = np.ascontiguousarray(old_lens, dtype=np.int32)
    n = np.ascontiguousarray(new_lens, dtype=np.int32)
    pp = np.ascontiguousarray(pool_pages, dtype=np.int32)
    for a in (tables, local_len, next_page):
        assert a.dtype == np.int32 and a.flags.c_contiguous
    return _load().oracle_grow_tables(_ptr(o), _ptr(n), o.shape[0], block_size, D, tables.shape[2], _ptr(tables),
                                      _ptr(local_len), _ptr(next_page), _ptr(pp))


def place(layout: int, Hkv: int, d: int, block_size: int, D: int, tables: np.ndarray,
          sources: List[np.ndarray], num_pages: np.ndarray, fill: int = 0xFFFF, rule: int = INTERLEAVED
          ) -> List[np.ndarray]:
    """Reference cache placement: returns D pools (uint16 bf16 bits), unused slots set to ``fill``."""
    B = len(sources)
    mlb = tables.shape[2]
    page_elems = (2 * Hkv * block_size * d) if layout == GQA else (block_size * d)
    pools = [np.full(int(num_pages[s]) * page_elems, fill, dtype=np.uint16) for s in range(D)]
    arr = (C.c_void_p * D)(*[p.ctypes.data for p in pools])
    t = np.ascontiguousarray(tables, dtype=np.int32)
    for b, src in enumerate(sources):
        src = np.ascontiguousarray(src, dtype=np.uint16)
        _load().oracle_place_request_rule(layout, Hkv, d, block_size, D, rule, B, b, mlb, _ptr(t), src.shape[0],
                                          _ptr(src), C.cast(arr, C.c_void_p))
    return pools


# ---------------------------------------------------------------------------
# attention and merge
# ---------------------------------------------------------------------------
def attend(layout: int, Hq: int, Hkv: int, d_qk: int, d_v: int, q: np.ndarray, src: np.ndarray, scale: float,
           block_size: int = 1, D: int = 1, shard: int = -1, heads: Optional[Tuple[int, int]] = None,
           rule: int = INTERLEAVED, rule_len: Optional[int] = None) -> Tuple[np.ndarray, np.ndarray]:
    """Attention of one request (q bf16 bits [Hq][d_qk], src unsharded rows) -> (O[Hq][d_v], LSE[Hq]) f64.

    ``shard < 0``: all tokens; otherwise only the tokens shard ``shard`` stores: under the interleaved
    rule those whose logical block ``t // block_size`` is congruent to ``shard`` modulo ``D``, under the
    contiguous rule those in its chunk of a request of ``rule_len`` tokens (default: ``len(src)``).
    Heads outside ``heads = (begin, end)`` are left as NaN.
    """
    if rule != INTERLEAVED:
        bits = np.ascontiguousarray(src, dtype=np.uint16)
        wide = (bits.astype(np.uint32) << 16).view(np.float32).astype(np.float64)  # exact
        return attend_values(layout, Hq, Hkv, d_qk, d_v, q, wide, scale, block_size, D, shard, heads, rule, rule_len)
    q = np.ascontiguousarray(q, dtype=np.uint16)
    src = np.ascontiguousarray(src, dtype=np.uint16)
    hb, he = heads if heads is not None else (0, Hq)
    O = np.full((Hq, d_v), np.nan)
    LSE = np.full((Hq,), np.nan)
    _load().oracle_attend(layout, Hq, Hkv, d_qk, d_v, _ptr(q), src.shape[0], _ptr(src), scale, block_size, D,
                          shard, hb, he, _ptr(O), _ptr(LSE))
    return O, LSE


def attend_values(layout: int, Hq: int, Hkv: int, d_qk: int, d_v: int, q: np.ndarray, src: np.ndarray,
                  scale: float, block_size: int = 1, D: int = 1, shard: int = -1,
                  heads: Optional[Tuple[int, int]] = None, rule: int = INTERLEAVED,
                  rule_len: Optional[int] = None) -> Tuple[np.ndarray, np.ndarray]:
    """``attend`` with the key/value source given as float64 values (same row layout)."""
    q = np.ascontiguousarray(q, dtype=np.uint16)
    src = np.ascontiguousarray(src, dtype=np.float64)
    hb, he = heads if heads is not None else (0, Hq)
    O = np.full((Hq, d_v), np.nan)
    LSE = np.full((Hq,), np.nan)
    n = src.shape[0]
    _load().oracle_attend_rule_f64(layout, Hq, Hkv, d_qk, d_v, _ptr(q), n, _ptr(src), scale, block_size, D, shard,
                                   rule, n if rule_len is None else rule_len, hb, he, _ptr(O), _ptr(LSE))
    return O, LSE


# ---------------------------------------------------------------------------
# FP8 (E4M3) KV cache
# ---------------------------------------------------------------------------
def e4m3_decode(codes) -> np.ndarray:
    c = np.ascontiguousarray(codes, dtype=np.uint8)
    return np.array([_load().oracle_e4m3_decode(int(x)) for x in c.ravel()]).reshape(c.shape)


def e4m3_encode(x) -> np.ndarray:
    a = np.asarray(x, dtype=np.float64)
    return np.array([_load().oracle_e4m3_encode(float(v)) for v in a.ravel()], dtype=np.uint8).reshape(a.shape)


def inv_scale(scale: float) -> np.float32:
    """float32 of 1 / scale (how the cache write turns a scale into a multiplier)."""
    return np.float32(1.0) / np.float32(scale)


def quantize_e4m3(bits: np.ndarray, scale: float) -> np.ndarray:
    """bf16 bit patterns -> E4M3 codes of float32(x) * float32(1 / scale)."""
    b = np.ascontiguousarray(bits, dtype=np.uint16)
    out = np.empty(b.shape, dtype=np.uint8)
    _load().oracle_quantize_e4m3(_ptr(b), b.size, float(inv_scale(scale)), _ptr(out))
    return out


def dequantize_e4m3(codes: np.ndarray, scale: float) -> np.ndarray:
    c = np.ascontiguousarray(codes, dtype=np.uint8)
    out = np.empty(c.shape, dtype=np.float64)
    _load().oracle_dequantize_e4m3(_ptr(c), c.size, float(np.float32(scale)), _ptr(out))
    return out


def quantize_kv_gqa(src: np.ndarray, k_scale: float, v_scale: float) -> np.ndarray:
    """GQA source rows [n][2][Hkv][d] (bf16 bits) -> E4M3 codes, K with k_scale and V with v_scale."""
    codes = np.empty(src.shape, dtype=np.uint8)
    codes[:, 0] = quantize_e4m3(src[:, 0], k_scale)
    codes[:, 1] = quantize_e4m3(src[:, 1], v_scale)
    return codes


def dequantize_kv_gqa(codes: np.ndarray, k_scale: float, v_scale: float) -> np.ndarray:
    """The float64 values an FP8 GQA cache stands for: [n][2][Hkv][d]."""
    out = np.empty(codes.shape, dtype=np.float64)
    out[:, 0] = dequantize_e4m3(codes[:, 0], k_scale)
    out[:, 1] = dequantize_e4m3(codes[:, 1], v_scale)
    return out


def place_u8(Hkv: int, d: int, block_size: int, D: int, tables: np.ndarray, codes: List[np.ndarray],
             num_pages: np.ndarray, fill: int = 0xFF, rule: int = INTERLEAVED) -> List[np.ndarray]:
    """Reference placement of quantised GQA rows: D byte pools, unused bytes set to ``fill``."""
    B = len(codes)
    mlb = tables.shape[2]
    page = 2 * Hkv * block_size * d
    pools = [np.full(int(num_pages[s]) * page, fill, dtype=np.uint8) for s in range(D)]
    arr = (C.c_void_p * D)(*[p.ctypes.data for p in pools])
    t = np.ascontiguousarray(tables, dtype=np.int32)
    for b, c in enumerate(codes):
        c = np.ascontiguousarray(c, dtype=np.uint8)
        _load().oracle_place_request_u8(Hkv, d, block_size, D, rule, B, b, mlb, _ptr(t), c.shape[0], _ptr(c),
                                        C.cast(arr, C.c_void_p))
    return pools


def quantize_kv_mla(src: np.ndarray, scale: float) -> np.ndarray:
    """MLA latent rows [n][576] (bf16 bits) -> E4M3 codes.  The latent is one tensor read as both key
    (all 576 entries) and value (the first 512), so one per-tensor scale covers the whole row."""
    return quantize_e4m3(src, scale)


def dequantize_kv_mla(codes: np.ndarray, scale: float) -> np.ndarray:
    """The float64 values an FP8 MLA latent cache stands for: [n][576]."""
    return dequantize_e4m3(codes, scale)


def place_mla_u8(block_size: int, D: int, tables: np.ndarray, codes: List[np.ndarray], num_pages: np.ndarray,
                 fill: int = 0xFF, rule: int = INTERLEAVED, d: int = 576) -> List[np.ndarray]:
    """Reference placement of quantised MLA latent rows: D byte pools of [bs][d] pages, unused bytes ``fill``."""
    B = len(codes)
    mlb = tables.shape[2]
    page = block_size * d
    pools = [np.full(int(num_pages[s]) * page, fill, dtype=np.uint8) for s in range(D)]
    arr = (C.c_void_p * D)(*[p.ctypes.data for p in pools])
    t = np.ascontiguousarray(tables, dtype=np.int32)
    for b, c in enumerate(codes):
        c = np.ascontiguousarray(c, dtype=np.uint8)
        _load().oracle_place_request_mla_u8(d, block_size, D, rule, B, b, mlb, _ptr(t), c.shape[0], _ptr(c),
                                            C.cast(arr, C.c_void_p))
    return pools


def sharded_values(layout: int, Hq: int, Hkv: int, d_qk: int, d_v: int, q: np.ndarray, src: np.ndarray,
                   scale: float, block_size: int, D: int, rule: int = INTERLEAVED):
    """``sharded`` over a float64-valued source (e.g. a dequantised FP8 cache)."""
    parts = [attend_values(layout, Hq, Hkv, d_qk, d_v, q, src, scale, block_size, D, s, None, rule)
             for s in range(D)]
    Op = np.stack([p[0] for p in parts])
    Lp = np.stack([p[1] for p in parts])
    O, LSE = merge(Op, Lp)
    return O, LSE, Op, Lp


def merge(O_parts: np.ndarray, LSE_parts: np.ndarray) -> Tuple[np.ndarray, np.ndarray]:
    """LSE-weighted merge. ``O_parts[D][rows][d_v]``, ``LSE_parts[D][rows]`` -> (O[rows][d_v], LSE[rows])."""
    Op = np.ascontiguousarray(O_parts, dtype=np.float64)
    Lp = np.ascontiguousarray(LSE_parts, dtype=np.float64)
    D, rows, d_v = Op.shape
    O = np.empty((rows, d_v))
    LSE = np.empty((rows,))
    _load().oracle_merge(_ptr(Op), _ptr(Lp), D, rows, d_v, _ptr(O), _ptr(LSE))
    return O, LSE


def merge_ml(U_parts: np.ndarray, m_parts: np.ndarray, l_parts: np.ndarray) -> np.ndarray:
    """Merge in the local-max / local-sum form (unnormalised partial outputs)."""
    U = np.ascontiguousarray(U_parts, dtype=np.float64)
    m = np.ascontiguousarray(m_parts, dtype=np.float64)
    l = np.ascontiguousarray(l_parts, dtype=np.float64)
    D, rows, d_v = U.shape
    O = np.empty((rows, d_v))
    _load().oracle_merge_ml(_ptr(U), _ptr(m), _ptr(l), D, rows, d_v, _ptr(O))
    return O


def sharded(layout: int, Hq: int, Hkv: int, d_qk: int, d_v: int, q: np.ndarray, src: np.ndarray, scale: float,
            block_size: int, D: int, heads: Optional[Tuple[int, int]] = None, rule: int = INTERLEAVED):
    """Per-shard partials followed by the merge: returns (O, LSE, O_parts[D], LSE_parts[D])."""
    parts = [attend(layout, Hq, Hkv, d_qk, d_v, q, src, scale, block_size, D, s, heads, rule) for s in range(D)]
    Op = np.stack([p[0] for p in parts])
    Lp = np.stack([p[1] for p in parts])
    hb, he = heads if heads is not None else (0, Hq)
    O, LSE = merge(Op[:, hb:he], Lp[:, hb:he])
    Of = np.full((Hq, d_v), np.nan)
    Lf = np.full((Hq,), np.nan)
    Of[hb:he], Lf[hb:he] = O, LSE
    return Of, Lf, Op, Lp


# ---------------------------------------------------------------------------
# multi-token decode (q_len query tokens per request, causal within the draft)
# ---------------------------------------------------------------------------
def visible_tokens(seq_len: int, q_len: int, j: int) -> int:
    """Tokens that query token ``j`` of a ``q_len``-token draft sees: the draft tokens are the last
    ``q_len`` of the ``seq_len`` cached ones, and token j sees itself and everything before it."""
    return max(0, seq_len - (q_len - 1 - j))


def attend_mtp(layout: int, Hq: int, Hkv: int, d_qk: int, d_v: int, q: np.ndarray, src: np.ndarray, scale: float,
               q_len: int, block_size: int = 1, D: int = 1, shard: int = -1,
               heads: Optional[Tuple[int, int]] = None, rule: int = INTERLEAVED) -> Tuple[np.ndarray, np.ndarray]:
    """Attention of the ``q_len`` query tokens of one request: ``q`` bf16 bits [q_len][Hq][d_qk] ->
    (O[q_len][Hq][d_v], LSE[q_len][Hq]).  Token j is ``attend`` over the first
    ``visible_tokens(len(src), q_len, j)`` source rows (restricted to ``shard`` as in ``attend``)."""
    q = np.ascontiguousarray(q, dtype=np.uint16).reshape(q_len, Hq, d_qk)
    L = src.shape[0]
    O = np.empty((q_len, Hq, d_v))
    LSE = np.empty((q_len, Hq))
    for j in range(q_len):
        # the shard of a token follows from the whole request (L tokens), not from the visible prefix
        O[j], LSE[j] = attend(layout, Hq, Hkv, d_qk, d_v, q[j], src[:visible_tokens(L, q_len, j)], scale,
                              block_size, D, shard, heads, rule, L)
    return O, LSE


def sharded_mtp(layout: int, Hq: int, Hkv: int, d_qk: int, d_v: int, q: np.ndarray, src: np.ndarray, scale: float,
                q_len: int, block_size: int, D: int, rule: int = INTERLEAVED):
    """Per-shard multi-token partials and their merge: (O[q_len][Hq][d_v], LSE[q_len][Hq], O_parts[D], LSE_parts[D])."""
    parts = [attend_mtp(layout, Hq, Hkv, d_qk, d_v, q, src, scale, q_len, block_size, D, s, None, rule)
             for s in range(D)]
    Op = np.stack([p[0] for p in parts])
    Lp = np.stack([p[1] for p in parts])
    O, LSE = merge(Op.reshape(D, q_len * Hq, d_v), Lp.reshape(D, q_len * Hq))
    return O.reshape(q_len, Hq, d_v), LSE.reshape(q_len, Hq), Op, Lp


def kv_bytes_per_token(num_kv_heads: int, head_dim: int, elem_bytes: int) -> int:
    return _load().oracle_kv_bytes_per_token(num_kv_heads, head_dim, elem_bytes)


def validate_config(tp: int, dcp: int, num_kv_heads: int, layout: int) -> int:
    return _load().oracle_validate_config(tp, dcp, num_kv_heads, layout)
