"""Pins of the float64 oracle against what the pages and the mathematics fix.

Every check here is independent of the oracle's own code: page-printed worked
examples (tests/golden), closed forms, a library routine (torch's float64
scaled_dot_product_attention, torch.logsumexp), brute force in extended
precision without the max shift, and algebraic invariants of the merge.
"""
import math

import numpy as np
import pytest
import torch

import oracle
import synth
from helpers import golden, golden_kv

GQA, MLA = oracle.GQA, oracle.MLA


# ---------------------------------------------------------------------------
# sharding rule and tables
# ---------------------------------------------------------------------------
def test_interleave_example_from_page():
    g = golden_kv("interleave_example.txt")
    D = int(g["D"][0])
    bs = 16
    for blk in map(int, g["rank0_blocks"]):
        assert oracle.token_shard(blk * bs, bs, D) == 0
        assert oracle.token_shard(blk * bs + bs - 1, bs, D) == 0
    for blk in map(int, g["rank1_blocks"]):
        assert oracle.token_shard(blk * bs, bs, D) == 1
    t = int(g["remap_global"][0]) * bs
    assert oracle.token_shard(t, bs, D) == int(g["remap_rank"][0])
    assert oracle.token_local_block(t, bs, D) == int(g["remap_local"][0])
    total = int(g["even_split_total_blocks"][0])
    _, _, num_pages = oracle.block_tables([total * bs], bs, D)
    assert list(num_pages) == [int(g["even_split_per_rank"][0])] * D


def test_tiny_tables_worked_by_hand():
    tables, local_len, num_pages = oracle.block_tables([100, 257], 16, 2)
    for row in golden("tiny_tables.txt"):
        bar = row.index("|")
        s, b, ntok = int(row[0]), int(row[1]), int(row[2])
        gblocks = list(map(int, row[3:bar]))
        pages = list(map(int, row[bar + 1:]))
        assert local_len[s, b] == ntok
        assert list(tables[s, b, :len(pages)]) == pages
        assert all(x == -1 for x in tables[s, b, len(pages):])
        for j, gb in enumerate(gblocks):  # local block j holds global block j*D + s
            assert gb == j * 2 + s
    assert list(num_pages) == [13, 11]


@pytest.mark.parametrize("D", [1, 2, 3, 4, 8])
@pytest.mark.parametrize("bs", [1, 16, 64])
@pytest.mark.parametrize("perm", [0, 77])
def test_tables_are_a_bijection(D, bs, perm):
    rng = np.random.default_rng(D * 100 + bs + perm)
    seq_lens = list(rng.integers(0, 700, size=7)) + [1, bs, bs + 1]
    tables, local_len, num_pages = oracle.block_tables(seq_lens, bs, D, perm_seed=perm)
    seen = [set() for _ in range(D)]
    for b, n in enumerate(seq_lens):
        assert int(local_len[:, b].sum()) == n
        for t in range(n):
            s = (t // bs) % D
            page = tables[s, b, (t // bs) // D]
            assert 0 <= page < num_pages[s]
            key = (int(page), t % bs)
            assert key not in seen[s]  # no slot holds two tokens
            seen[s].add(key)
    for s in range(D):  # every page of a shard is used, ids are 0..n-1
        used = {p for p, _ in seen[s]}
        assert used == set(range(int(num_pages[s])))


def test_tables_capacity_error():
    with pytest.raises(ValueError):
        oracle.block_tables([100], 16, 2, max_local_blocks=3)


def test_permutation_relabels_only():
    seq_lens = [300, 5, 1000]
    t0, l0, n0 = oracle.block_tables(seq_lens, 16, 4)
    t1, l1, n1 = oracle.block_tables(seq_lens, 16, 4, perm_seed=12345)
    assert (l0 == l1).all() and (n0 == n1).all()
    assert ((t0 < 0) == (t1 < 0)).all()
    assert not (t0 == t1).all()
    for s in range(4):
        a, b = t0[s][t0[s] >= 0], t1[s][t1[s] >= 0]
        assert sorted(a) == sorted(b)


def test_placement_roundtrip():
    w = synth.custom(GQA, [37, 16, 1], 4, 2, 64, 64, 16, seed=9)
    D = 3
    tables, _, num_pages = oracle.block_tables(w.seq_lens, 16, D, perm_seed=5)
    srcs = [w.kv_source(b) for b in range(w.batch)]
    pools = oracle.place(GQA, 2, 64, 16, D, tables, srcs, num_pages, fill=0xFFFF)
    used = [np.zeros(p.shape, bool) for p in pools]
    for b, src in enumerate(srcs):
        for t in range(src.shape[0]):
            s = (t // 16) % D
            page = tables[s, b, (t // 16) // D]
            view = pools[s].reshape(-1, 2, 2, 16, 64)
            assert (view[page, :, :, t % 16, :] == src[t]).all()
            used[s].reshape(-1, 2, 2, 16, 64)[page, :, :, t % 16, :] = True
    for s in range(D):
        assert (pools[s][~used[s]] == 0xFFFF).all()


# ---------------------------------------------------------------------------
# arithmetic and configuration rules printed on the pages
# ---------------------------------------------------------------------------
def test_kv_size_13b_example():
    g = golden_kv("kv_size_13b.txt")
    per = oracle.kv_bytes_per_token(int(g["num_kv_heads"][0]), int(g["head_dim"][0]), int(g["elem_bytes"][0]))
    assert per == int(g["bytes_per_token_per_layer"][0])
    assert per * int(g["layers"][0]) == int(g["bytes_per_token"][0])
    assert oracle.kv_bytes_per_token(8, 128, 2) == 4096  # the 70B-class GQA layer


def test_validate_config_examples():
    for row in golden("validate_config.txt"):
        layout, tp, dcp, kvh, want = map(int, row)
        assert oracle.validate_config(tp, dcp, kvh, layout) == want, row


# ---------------------------------------------------------------------------
# direct attention
# ---------------------------------------------------------------------------
def _f64(bits):
    return synth.bf16_bits_to_f64(bits)


def _torch_reference(layout, Hq, Hkv, d_qk, d_v, q, src, scale):
    """torch float64 SDPA + logsumexp as an independent library reference."""
    qd = torch.from_numpy(_f64(q))  # [Hq, d_qk]
    if layout == GQA:
        kv = torch.from_numpy(_f64(src))  # [n, 2, Hkv, d]
        K = kv[:, 0].permute(1, 0, 2).repeat_interleave(Hq // Hkv, dim=0)  # [Hq, n, d]
        V = kv[:, 1].permute(1, 0, 2).repeat_interleave(Hq // Hkv, dim=0)
    else:
        c = torch.from_numpy(_f64(src))  # [n, d_qk]
        K = c.unsqueeze(0).expand(Hq, -1, -1)
        V = c[:, :d_v].unsqueeze(0).expand(Hq, -1, -1)
    O = torch.nn.functional.scaled_dot_product_attention(qd.unsqueeze(1), K, V, scale=scale).squeeze(1)
    S = torch.einsum("hd,hnd->hn", qd, K) * scale
    return O.numpy(), torch.logsumexp(S, dim=1).numpy()


@pytest.mark.parametrize("case", [
    (GQA, 8, 2, 64, 64, 100), (GQA, 8, 8, 128, 128, 33), (GQA, 16, 2, 64, 64, 5), (GQA, 6, 3, 64, 64, 70),
    (MLA, 4, 1, 576, 512, 90), (MLA, 64, 1, 576, 512, 17)])
def test_attend_matches_torch_sdpa(case):
    layout, Hq, Hkv, d_qk, d_v, n = case
    w = synth.custom(layout, [n], Hq, Hkv, d_qk, d_v, 16, seed=n + Hq)
    q, src = w.query(0), w.kv_source(0)
    O, LSE = oracle.attend(layout, Hq, Hkv, d_qk, d_v, q, src, w.softmax_scale)
    Ot, Lt = _torch_reference(layout, Hq, Hkv, d_qk, d_v, q, src, w.softmax_scale)
    np.testing.assert_allclose(O, Ot, rtol=0, atol=1e-12)
    np.testing.assert_allclose(LSE, Lt, rtol=1e-13, atol=1e-12)


def test_attend_bruteforce_extended_precision():
    # Naive softmax without the max shift, in x87 extended precision, on small scores.
    w = synth.custom(GQA, [23], 4, 2, 64, 64, 16, seed=3, q_amp=0.25, kv_amp=0.25)
    q, src = w.query(0), w.kv_source(0)
    O, LSE = oracle.attend(GQA, 4, 2, 64, 64, q, src, 0.125)
    qd = _f64(q).astype(np.longdouble)
    kv = _f64(src).astype(np.longdouble)
    for h in range(4):
        kvh = h // 2
        e = np.array([np.exp(np.longdouble(0.125) * np.dot(qd[h], kv[t, 0, kvh])) for t in range(23)])
        o = (e[:, None] * kv[:, 1, kvh]).sum(0) / e.sum()
        np.testing.assert_allclose(O[h], o.astype(np.float64), rtol=0, atol=1e-13)
        assert abs(LSE[h] - float(np.log(e.sum()))) < 1e-13


def test_closed_forms():
    # seq_len 1: O = v_0, LSE = s_0.
    w = synth.custom(GQA, [1], 4, 1, 64, 64, 16, seed=11)
    q, src = w.query(0), w.kv_source(0)
    O, LSE = oracle.attend(GQA, 4, 1, 64, 64, q, src, 0.5)
    for h in range(4):
        np.testing.assert_array_equal(O[h], _f64(src[0, 1, 0]))
        assert LSE[h] == pytest.approx(0.5 * float(_f64(q[h]) @ _f64(src[0, 0, 0])), abs=1e-12)
    # q = 0: uniform weights, O = mean of V, LSE = ln n.
    w = synth.custom(MLA, [37], 2, 1, 576, 512, 64, seed=12)
    src = w.kv_source(0)
    O, LSE = oracle.attend(MLA, 2, 1, 576, 512, np.zeros((2, 576), np.uint16), src, 0.1)
    np.testing.assert_allclose(O[0], _f64(src)[:, :512].mean(0), atol=1e-13)
    assert LSE[1] == pytest.approx(math.log(37), abs=1e-14)
    # all keys equal, values distinct: uniform weights again, O = mean(V), LSE = s + ln n.
    w = synth.custom(GQA, [37], 2, 1, 64, 64, 16, seed=15)
    q, src = w.query(0), w.kv_source(0).copy()
    src[:, 0] = src[0, 0]
    O, LSE = oracle.attend(GQA, 2, 1, 64, 64, q, src, 0.1)
    s0 = 0.1 * float(_f64(q[1]) @ _f64(src[0, 0, 0]))
    np.testing.assert_allclose(O[1], _f64(src[:, 1, 0]).mean(0), atol=1e-13)
    assert LSE[1] == pytest.approx(s0 + math.log(37), abs=1e-12)
    # one dominant score: O ~= v_j.
    w = synth.custom(GQA, [50], 2, 1, 64, 64, 16, seed=13)
    q, src = w.query(0), w.kv_source(0).copy()
    j = 31
    src[j, 0, 0] = q[0]  # key j = q, so s_j = scale*|q|^2 dominates by a huge margin
    O, _ = oracle.attend(GQA, 2, 1, 64, 64, q, src, 10.0)
    np.testing.assert_allclose(O[0], _f64(src[j, 1, 0]), atol=1e-12)


def test_empty_token_set():
    w = synth.custom(GQA, [16], 2, 1, 64, 64, 16, seed=14)
    O, LSE = oracle.attend(GQA, 2, 1, 64, 64, w.query(0), w.kv_source(0), 0.1, block_size=16, D=2, shard=1)
    assert (O == 0).all() and (LSE == -np.inf).all()


# ---------------------------------------------------------------------------
# sharded partials + merge == direct attention
# ---------------------------------------------------------------------------
@pytest.mark.parametrize("D", [1, 2, 3, 4, 8])
@pytest.mark.parametrize("bs", [1, 16, 64])
def test_sharded_merge_equals_direct(D, bs):
    for layout, Hq, Hkv, dqk, dv in [(GQA, 8, 2, 64, 64), (MLA, 4, 1, 576, 512)]:
        w = synth.custom(layout, [257], Hq, Hkv, dqk, dv, bs, seed=D * 7 + bs)
        q, src = w.query(0), w.kv_source(0)
        O, LSE = oracle.attend(layout, Hq, Hkv, dqk, dv, q, src, w.softmax_scale)
        Om, Lm, Op, Lp = oracle.sharded(layout, Hq, Hkv, dqk, dv, q, src, w.softmax_scale, bs, D)
        np.testing.assert_allclose(Om, O, rtol=0, atol=1e-12)
        np.testing.assert_allclose(Lm, LSE, rtol=0, atol=1e-12)
        if D == 1:
            np.testing.assert_array_equal(Op[0], O)


def test_merge_worked_example():
    g = golden_kv("merge_worked.txt")
    Op = np.array([[list(map(float, g["O1"]))], [list(map(float, g["O2"]))]])
    Lp = np.array([[float(g["LSE1"][0])], [math.log(float(g["LSE2_log_of"][0]))]])
    O, LSE = oracle.merge(Op, Lp)
    np.testing.assert_allclose(O[0], list(map(float, g["O"])), atol=1e-15)
    assert LSE[0] == pytest.approx(math.log(float(g["LSE_log_of"][0])), abs=1e-15)
    # the same instance through the local-max / local-sum form
    U = np.array([[[1.0, 0.0]], [[0.0, 1.0]]])
    m = np.array([[0.0], [math.log(3.0)]])
    l = np.array([[1.0], [1.0]])
    np.testing.assert_allclose(oracle.merge_ml(U, m, l)[0], [0.25, 0.75], atol=1e-15)


def test_merge_invariants():
    rng = np.random.default_rng(5)
    Op = rng.standard_normal((4, 6, 16))
    Lp = rng.standard_normal((4, 6)) * 5
    O, LSE = oracle.merge(Op, Lp)
    # D = 1 is the identity
    O1, L1 = oracle.merge(Op[:1], Lp[:1])
    np.testing.assert_array_equal(O1, Op[0])
    np.testing.assert_array_equal(L1, Lp[0])
    # adding a constant to every LSE_i leaves O unchanged and shifts LSE
    O2, L2 = oracle.merge(Op, Lp + 1234.5)
    np.testing.assert_allclose(O2, O, atol=1e-12)
    np.testing.assert_allclose(L2, LSE + 1234.5, atol=1e-9)
    # a -inf part is ignored
    Lq = Lp.copy()
    Lq[2] = -np.inf
    O3, L3 = oracle.merge(Op, Lq)
    O4, L4 = oracle.merge(Op[[0, 1, 3]], Lp[[0, 1, 3]])
    np.testing.assert_allclose(O3, O4, atol=1e-14)
    np.testing.assert_allclose(L3, L4, atol=1e-14)
    # all parts empty -> zeros and -inf
    O5, L5 = oracle.merge(Op, np.full_like(Lp, -np.inf))
    assert (O5 == 0).all() and (L5 == -np.inf).all()
    # weights are a convex combination: merged O lies in the hull of the parts per element
    assert (O <= Op.max(0) + 1e-12).all() and (O >= Op.min(0) - 1e-12).all()
    # the local-max / local-sum form agrees for any choice of local maxima
    m = Lp - rng.uniform(0, 3, size=Lp.shape)
    l = np.exp(Lp - m)
    U = Op * l[..., None]
    np.testing.assert_allclose(oracle.merge_ml(U, m, l), O, atol=1e-12)


# ---------------------------------------------------------------------------
# the seeded generator (shared input module)
# ---------------------------------------------------------------------------
def test_generator_rounding_matches_torch_bf16():
    v = np.random.default_rng(0).standard_normal(100000).astype(np.float32) * 3
    mine = synth.f32_to_bf16_bits(v)
    ref = torch.from_numpy(v).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    np.testing.assert_array_equal(mine, ref)


def test_generator_statistics_and_determinism():
    a = synth.values_bf16(7, synth.T_K, 3, 0, 200000, 0.5)
    b = synth.values_bf16(7, synth.T_K, 3, 100000, 100000, 0.5)
    np.testing.assert_array_equal(a[100000:], b)
    x = synth.bf16_bits_to_f64(a)
    assert abs(x.mean()) < 0.01 and abs(x.std() - 0.5) < 0.01
    assert np.abs(x).max() <= 0.5 * 3.47
    c = synth.values_bf16(7, synth.T_V, 3, 0, 1000, 0.5)
    assert not (c == a[:1000]).all()


def test_workload_recipes():
    mix = synth.workload("mla_mix").seq_lens
    s = np.array(mix)
    assert len(s) == 256 and s.max() <= 327680
    assert 60000 < np.median(s) < 75000
    assert abs((s > 65536).mean() - 0.53) < 0.01
    assert abs((s > 131072).mean() - 0.08) < 0.01
    assert 0.03 <= (s > 262144).mean() <= 0.04
    assert abs((s < 8192).mean() - 0.18) < 0.01
    g = synth.workload("gqa_70b").seq_lens
    assert len(g) == 64 and min(g) >= 8192 and max(g) <= 32768
    m = synth.workload("mla_b32").seq_lens
    assert len(m) == 32 and 40000 < np.median(m) < 100000
    lg = synth.workload("mla_long").seq_lens
    assert len(lg) == 4 and min(lg) >= 204800 and max(lg) <= 262144
    assert synth.workload("gqa_tiny").seq_lens == [100, 257]


# ---------------------------------------------------------------------------
# incremental growth of the tables (new blocks only)
# ---------------------------------------------------------------------------
def test_grow_from_empty_equals_full_build():
    seq_lens = [100, 257, 0, 64, 1]
    for D in (1, 2, 3, 4):
        t_full, l_full, n_full = oracle.block_tables(seq_lens, 16, D)
        t = np.full(t_full.shape, -1, np.int32)
        l = np.zeros(l_full.shape, np.int32)
        nxt = np.zeros(D, np.int32)
        assert oracle.grow_tables([0] * 5, seq_lens, 16, D, t, l, nxt, [10 ** 6] * D) == 0
        np.testing.assert_array_equal(t, t_full)
        np.testing.assert_array_equal(l, l_full)
        np.testing.assert_array_equal(nxt, n_full)


def test_grow_keeps_existing_pages_and_covers_new_tokens():
    rng = np.random.default_rng(8)
    D, bs, B = 3, 16, 6
    lens = rng.integers(0, 200, size=B).astype(np.int32)
    t, l, n = oracle.block_tables(lens, bs, D, max_local_blocks=40)
    nxt = n.copy()
    for step in range(30):
        new = lens + rng.integers(0, 40, size=B).astype(np.int32)
        before = t.copy()
        assert oracle.grow_tables(lens, new, bs, D, t, l, nxt, [10 ** 6] * D) == 0
        assert ((before < 0) | (t == before)).all()            # old entries never move
        for b in range(B):
            assert int(l[:, b].sum()) == new[b]
            for tok in range(0, int(new[b]), 7):
                s = (tok // bs) % D
                assert t[s, b, (tok // bs) // D] >= 0
        used = [sorted(t[s][t[s] >= 0].tolist()) for s in range(D)]
        for s in range(D):                                       # pages stay a bijection onto 0..next-1
            assert used[s] == list(range(int(nxt[s])))
        lens = new


def test_grow_errors():
    t = np.full((2, 1, 2), -1, np.int32)
    l = np.zeros((2, 1), np.int32)
    nxt = np.zeros(2, np.int32)
    assert oracle.grow_tables([5], [3], 16, 2, t, l, nxt, [9, 9]) == -1        # shrinking
    assert oracle.grow_tables([0], [16 * 5], 16, 2, t, l, nxt, [9, 9]) == -2   # local block 2 > capacity 2
    t[:] = -1; l[:] = 0; nxt[:] = 0
    assert oracle.grow_tables([0], [16 * 3], 16, 2, t, l, nxt, [1, 9]) == -3   # shard 0 has one page only


# ---------------------------------------------------------------------------
# multi-token decode (causal within the draft)
# ---------------------------------------------------------------------------
MTP_CASES = [(GQA, 8, 2, 64, 64), (MLA, 4, 1, 576, 512)]


@pytest.mark.parametrize("case", MTP_CASES)
def test_mtp_single_token_is_plain_decode(case):
    layout, Hq, Hkv, dqk, dv = case
    w = synth.custom(layout, [77], Hq, Hkv, dqk, dv, 16, seed=21, q_len=1)
    O, L = oracle.attend_mtp(layout, Hq, Hkv, dqk, dv, w.queries(0), w.kv_source(0), w.softmax_scale, 1)
    O1, L1 = oracle.attend(layout, Hq, Hkv, dqk, dv, w.query(0), w.kv_source(0), w.softmax_scale)
    np.testing.assert_array_equal(O[0], O1)
    np.testing.assert_array_equal(L[0], L1)


@pytest.mark.parametrize("case", MTP_CASES)
@pytest.mark.parametrize("q_len", [2, 3, 4])
def test_mtp_causal_boundary_by_perturbation(case, q_len):
    # Query token j must see exactly the first L - (q_len - 1 - j) tokens: replacing every
    # token after them changes nothing, replacing the last visible one changes the result.
    layout, Hq, Hkv, dqk, dv = case
    L = 41
    w = synth.custom(layout, [L], Hq, Hkv, dqk, dv, 16, seed=30 + q_len, q_len=q_len)
    other = synth.custom(layout, [L], Hq, Hkv, dqk, dv, 16, seed=999, q_len=q_len).kv_source(0)
    q, src = w.queries(0), w.kv_source(0)
    O, LSE = oracle.attend_mtp(layout, Hq, Hkv, dqk, dv, q, src, w.softmax_scale, q_len)
    for j in range(q_len):
        n = L - (q_len - 1 - j)
        tail = src.copy()
        tail[n:] = other[n:]
        Ot, Lt = oracle.attend_mtp(layout, Hq, Hkv, dqk, dv, q, tail, w.softmax_scale, q_len)
        np.testing.assert_array_equal(Ot[j], O[j])
        np.testing.assert_array_equal(Lt[j], LSE[j])
        last = src.copy()
        last[n - 1] = other[n - 1]
        Ol, Ll = oracle.attend_mtp(layout, Hq, Hkv, dqk, dv, q, last, w.softmax_scale, q_len)
        assert np.abs(Ol[j] - O[j]).max() > 1e-6 and np.abs(Ll[j] - LSE[j]).max() > 1e-9


@pytest.mark.parametrize("case", MTP_CASES)
def test_mtp_matches_masked_torch_sdpa(case):
    # Library reference: torch float64 SDPA with a boolean mask built from token counts
    # (token j of the draft sits at position L - q_len + j and sees positions <= its own).
    layout, Hq, Hkv, dqk, dv = case
    q_len, L = 3, 29
    w = synth.custom(layout, [L], Hq, Hkv, dqk, dv, 16, seed=44, q_len=q_len)
    q, src = w.queries(0), w.kv_source(0)
    O, LSE = oracle.attend_mtp(layout, Hq, Hkv, dqk, dv, q, src, w.softmax_scale, q_len)
    pos_q = torch.arange(L - q_len, L)
    allowed = torch.arange(L)[None, :] <= pos_q[:, None]  # [q_len][L]
    qd = torch.from_numpy(_f64(q)).permute(1, 0, 2)  # [Hq][q_len][d]
    if layout == GQA:
        kv = torch.from_numpy(_f64(src))
        K = kv[:, 0].permute(1, 0, 2).repeat_interleave(Hq // Hkv, dim=0)
        V = kv[:, 1].permute(1, 0, 2).repeat_interleave(Hq // Hkv, dim=0)
    else:
        c = torch.from_numpy(_f64(src))
        K = c.unsqueeze(0).expand(Hq, -1, -1)
        V = c[:, :dv].unsqueeze(0).expand(Hq, -1, -1)
    Ot = torch.nn.functional.scaled_dot_product_attention(qd, K, V, attn_mask=allowed, scale=w.softmax_scale)
    S = torch.einsum("hjd,hnd->hjn", qd, K) * w.softmax_scale
    Lt = torch.logsumexp(S.masked_fill(~allowed, -math.inf), dim=2)
    np.testing.assert_allclose(O, Ot.permute(1, 0, 2).numpy(), rtol=0, atol=1e-12)
    np.testing.assert_allclose(LSE, Lt.permute(1, 0).numpy(), rtol=0, atol=1e-12)


@pytest.mark.parametrize("D", [2, 3, 4])
def test_mtp_sharded_merge_equals_direct(D):
    for layout, Hq, Hkv, dqk, dv in MTP_CASES:
        for L in [3, 16, 17, 50]:  # draft straddling a block boundary, and L < q_len + block
            w = synth.custom(layout, [L], Hq, Hkv, dqk, dv, 16, seed=L * D, q_len=4)
            q, src = w.queries(0), w.kv_source(0)
            O, LSE = oracle.attend_mtp(layout, Hq, Hkv, dqk, dv, q, src, w.softmax_scale, 4)
            Om, Lm, _, _ = oracle.sharded_mtp(layout, Hq, Hkv, dqk, dv, q, src, w.softmax_scale, 4, 16, D)
            np.testing.assert_allclose(Om, O, rtol=0, atol=1e-12)
            np.testing.assert_allclose(Lm, LSE, rtol=0, atol=1e-12)


def test_mtp_short_sequence_sees_nothing():
    # seq_len 2 with a 4-token draft: tokens 0 and 1 see no cached token at all.
    w = synth.custom(GQA, [2], 4, 2, 64, 64, 16, seed=5, q_len=4)
    O, LSE = oracle.attend_mtp(GQA, 4, 2, 64, 64, w.queries(0), w.kv_source(0), 0.125, 4)
    assert (O[:2] == 0).all() and (LSE[:2] == -np.inf).all()
    assert np.isfinite(LSE[2:]).all()
    np.testing.assert_array_equal(O[3], oracle.attend(GQA, 4, 2, 64, 64, w.queries(0)[3], w.kv_source(0), 0.125)[0])


def test_queries_extend_the_single_token_query():
    w = synth.custom(MLA, [5], 64, 1, 576, 512, 64, seed=8, q_len=3)
    np.testing.assert_array_equal(w.queries(0)[0], w.query(0))


# ---------------------------------------------------------------------------
# FP8 (E4M3) cache: code definition, rounding, scales, placement
# ---------------------------------------------------------------------------
def test_e4m3_values_from_the_format_definition():
    # sign | exponent (bias 7) | mantissa: hand-decoded codes
    cases = {0x38: 1.0, 0x7E: 448.0, 0x01: 2.0 ** -9, 0x07: 7 * 2.0 ** -9, 0x08: 2.0 ** -6, 0x40: 2.0,
             0x3C: 1.5, 0x30: 0.5, 0xB8: -1.0, 0x00: 0.0, 0x77: 240.0, 0x7D: 416.0}
    for c, v in cases.items():
        assert oracle.e4m3_decode(np.array([c], np.uint8))[0] == v, hex(c)
    assert np.isnan(oracle.e4m3_decode(np.array([0x7F, 0xFF], np.uint8))).all()
    z = oracle.e4m3_decode(np.array([0x80], np.uint8))[0]
    assert z == 0.0 and math.copysign(1.0, z) == -1.0


def test_e4m3_decode_matches_torch_float8():
    codes = np.arange(256, dtype=np.uint8)
    ours = oracle.e4m3_decode(codes)
    ref = torch.from_numpy(codes).view(torch.float8_e4m3fn).to(torch.float64).numpy()
    np.testing.assert_array_equal(np.isnan(ours), np.isnan(ref))
    ok = ~np.isnan(ours)
    np.testing.assert_array_equal(ours[ok], ref[ok])


def test_e4m3_encode_matches_torch_float8_in_range():
    # torch's float32 -> float8_e4m3fn cast rounds to nearest even; within +-448 it must agree
    rng = np.random.default_rng(3)
    x = np.concatenate([rng.normal(0, 1, 4000), rng.normal(0, 60, 2000), rng.uniform(-448, 448, 2000),
                        rng.normal(0, 2.0 ** -8, 2000)]).astype(np.float32)
    vals = oracle.e4m3_decode(np.arange(127, dtype=np.uint8)).astype(np.float32)
    mids = ((vals[:-1].astype(np.float64) + vals[1:]) / 2).astype(np.float32)  # exact ties
    x = np.concatenate([x, mids, -mids, vals, -vals])
    ours = oracle.e4m3_encode(x.astype(np.float64))
    ref = torch.from_numpy(x).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    np.testing.assert_array_equal(ours, ref)


def test_e4m3_saturates_and_ties_to_even():
    assert list(oracle.e4m3_encode([449.0, 1e6, -1e6, 464.0, 447.0])) == [0x7E, 0x7E, 0xFE, 0x7E, 0x7E]
    # halfway between 1.0 (0x38, even) and 1.125 (0x39): to 0x38; between 1.125 and 1.25: to 0x3A
    assert list(oracle.e4m3_encode([1.0625, 1.1875, 2.0 ** -10, 3 * 2.0 ** -10])) == [0x38, 0x3A, 0x00, 0x02]


def test_quantize_rounds_the_product_in_float32_then_to_e4m3():
    w = synth.custom(GQA, [300], 8, 2, 64, 64, 16, seed=19, kv_amp=0.5)
    src = w.kv_source(0)
    for scale in (1.0, 0.75, 1.0 / 64, 3.3):
        codes = oracle.quantize_e4m3(src, scale)
        prod = synth.bf16_bits_to_f64(src).astype(np.float32) * oracle.inv_scale(scale)
        np.testing.assert_array_equal(codes, oracle.e4m3_encode(prod.astype(np.float64)))
        # dequantised values are within half a unit of the third mantissa bit (relative 2^-4)
        back = oracle.dequantize_e4m3(codes, scale)
        x = synth.bf16_bits_to_f64(src)
        big = np.abs(x / scale) >= 2.0 ** -6
        assert (np.abs(back[big] - x[big]) <= 2.0 ** -4 * np.abs(x[big]) * (1 + 1e-6)).all()


def test_quantize_roundtrips_every_finite_code():
    codes = np.array([c for c in range(256) if c not in (0x7F, 0xFF, 0x80)], dtype=np.uint8)
    vals = oracle.e4m3_decode(codes)
    bits = synth.f32_to_bf16_bits(vals.astype(np.float32))  # E4M3 values are exact in bf16
    np.testing.assert_array_equal(oracle.quantize_e4m3(bits, 1.0), codes)


def test_attend_values_equals_attend_on_widened_bf16():
    w = synth.custom(GQA, [90], 8, 2, 64, 64, 16, seed=23)
    q, src = w.query(0), w.kv_source(0)
    for D, s in [(1, -1), (3, 1)]:
        a = oracle.attend(GQA, 8, 2, 64, 64, q, src, 0.125, 16, D, s)
        b = oracle.attend_values(GQA, 8, 2, 64, 64, q, synth.bf16_bits_to_f64(src), 0.125, 16, D, s)
        np.testing.assert_array_equal(a[0], b[0])
        np.testing.assert_array_equal(a[1], b[1])


def test_fp8_placement_roundtrip():
    w = synth.custom(GQA, [70, 5, 33], 8, 2, 128, 128, 16, seed=4)
    D = 3
    tables, _, pages = oracle.block_tables(w.seq_lens, 16, D)
    codes = [oracle.quantize_kv_gqa(w.kv_source(b), 1.0, 0.5) for b in range(w.batch)]
    pools = oracle.place_u8(2, 128, 16, D, tables, codes, pages, fill=0x7F)
    for b in range(w.batch):
        for t in range(w.seq_lens[b]):
            s, j = oracle.token_shard(t, 16, D), oracle.token_local_block(t, 16, D)
            page = tables[s, b, j]
            pg = pools[s][page * 2 * 2 * 16 * 128:(page + 1) * 2 * 2 * 16 * 128].reshape(2, 2, 16, 128)
            np.testing.assert_array_equal(pg[:, :, t % 16], codes[b][t])
    used = sum(int(w.seq_lens[b]) for b in range(w.batch)) * 2 * 2 * 128
    assert sum(int((p != 0x7F).sum()) for p in pools) <= used


# FP8 MLA latent cache: one scale for the latent row (key = all 576 entries, value = the first 512)
@pytest.mark.parametrize("rule", [oracle.INTERLEAVED, oracle.CONTIGUOUS])
def test_fp8_mla_placement_roundtrip(rule):
    w = synth.custom(MLA, [130, 1, 64, 65], 4, 1, 576, 512, 64, seed=12)
    D = 3
    tables, _, pages = oracle.block_tables(w.seq_lens, 64, D, perm_seed=7, rule=rule)
    codes = [oracle.quantize_kv_mla(w.kv_source(b), 0.75) for b in range(w.batch)]
    pools = oracle.place_mla_u8(64, D, tables, codes, pages, fill=0x7F, rule=rule)
    for b, n in enumerate(w.seq_lens):
        for t in range(n):
            s = oracle.token_shard_rule(t, 64, D, rule, n)
            j = oracle.token_local_block_rule(t, 64, D, rule, n)
            off = (int(tables[s, b, j]) * 64 + t % 64) * 576
            np.testing.assert_array_equal(pools[s][off:off + 576], codes[b][t])
    used = sum(int(n) for n in w.seq_lens) * 576
    assert sum(int((p != 0x7F).sum()) for p in pools) <= used


def _exact_latent_codes(n, seed):
    rng = np.random.default_rng(seed)
    codes = rng.integers(0, 256, size=(n, 576)).astype(np.uint8)
    codes[(codes & 0x7F) == 0x7F] = 0x01  # no NaN codes
    codes[codes == 0x80] = 0x00           # no negative zero
    return codes


def test_fp8_mla_exact_codes_give_the_bf16_attention():
    # latent values that are E4M3 values times a power-of-two scale are exact in bf16 and quantise back to
    # the same codes, so attention over the FP8 cache's values equals bf16 attention over them, bit for bit
    scale = 2.0 ** -3
    codes = _exact_latent_codes(150, 3)
    vals = oracle.e4m3_decode(codes) * scale
    bits = synth.f32_to_bf16_bits(vals.astype(np.float32))
    np.testing.assert_array_equal(synth.bf16_bits_to_f64(bits), vals)
    np.testing.assert_array_equal(oracle.quantize_kv_mla(bits, scale), codes)
    np.testing.assert_array_equal(oracle.dequantize_kv_mla(codes, scale), vals)
    w = synth.custom(MLA, [150], 4, 1, 576, 512, 64, seed=8)
    q = w.query(0)
    for D, s in [(1, -1), (3, 2)]:
        a = oracle.attend(MLA, 4, 1, 576, 512, q, bits, w.softmax_scale, 64, D, s)
        b = oracle.attend_values(MLA, 4, 1, 576, 512, q, oracle.dequantize_kv_mla(codes, scale), w.softmax_scale,
                                 64, D, s)
        np.testing.assert_array_equal(a[0], b[0])
        np.testing.assert_array_equal(a[1], b[1])


def test_fp8_mla_attention_matches_torch_sdpa():
    # scores over all 576 dequantised entries, values = the first 512 (a library routine, float64)
    w = synth.custom(MLA, [200], 4, 1, 576, 512, 64, seed=31)
    scale = 0.37
    vals = oracle.dequantize_kv_mla(oracle.quantize_kv_mla(w.kv_source(0), scale), scale)
    O, LSE = oracle.attend_values(MLA, 4, 1, 576, 512, w.query(0), vals, w.softmax_scale)
    qd = torch.from_numpy(synth.bf16_bits_to_f64(w.query(0)))
    K = torch.from_numpy(vals)
    Ot = torch.nn.functional.scaled_dot_product_attention(qd[:, None], K[None].expand(4, -1, -1),
                                                          K[None, :, :512].expand(4, -1, -1),
                                                          scale=w.softmax_scale)[:, 0]
    Lt = torch.logsumexp(qd @ K.T * w.softmax_scale, dim=1)
    np.testing.assert_allclose(O, Ot.numpy(), rtol=0, atol=1e-12)
    np.testing.assert_allclose(LSE, Lt.numpy(), rtol=0, atol=1e-12)


@pytest.mark.parametrize("rule", [oracle.INTERLEAVED, oracle.CONTIGUOUS])
@pytest.mark.parametrize("D", [2, 3, 8])
def test_fp8_mla_sharded_merge_equals_direct(D, rule):
    w = synth.custom(MLA, [333], 4, 1, 576, 512, 64, seed=D + 40)
    vals = oracle.dequantize_kv_mla(oracle.quantize_kv_mla(w.kv_source(0), 0.5), 0.5)
    O, LSE = oracle.attend_values(MLA, 4, 1, 576, 512, w.query(0), vals, w.softmax_scale)
    Om, Lm, _, _ = oracle.sharded_values(MLA, 4, 1, 576, 512, w.query(0), vals, w.softmax_scale, 64, D, rule)
    np.testing.assert_allclose(Om, O, rtol=0, atol=1e-12)
    np.testing.assert_allclose(Lm, LSE, rtol=0, atol=1e-12)


# ---------------------------------------------------------------------------
# contiguous-chunk shard rule ([P1] A2 illustration: "GPU0 holds 0-50K, GPU1 50K-100K, ...")
# ---------------------------------------------------------------------------
CONTIG = oracle.CONTIGUOUS


def test_contiguous_rule_page_example():
    # 200,000 tokens on 4 shards (block 16: 12,500 blocks): shard s holds tokens [50,000 s, 50,000 (s+1))
    L = 200_000
    for t, s, j in [(0, 0, 0), (49_999, 0, 3124), (50_000, 1, 0), (99_999, 1, 3124), (150_000, 3, 0),
                    (199_999, 3, 3124)]:
        assert oracle.token_shard_rule(t, 16, 4, CONTIG, L) == s
        assert oracle.token_local_block_rule(t, 16, 4, CONTIG, L) == j
    _, local_len, pages = oracle.block_tables([L], 16, 4, rule=CONTIG)
    assert list(local_len[:, 0]) == [50_000] * 4 and list(pages) == [3125] * 4


@pytest.mark.parametrize("D", [1, 2, 3, 4, 8])
@pytest.mark.parametrize("bs", [1, 16, 64])
def test_contiguous_tables_are_a_bijection_of_contiguous_ranges(D, bs):
    rng = np.random.default_rng(D * 31 + bs)
    seq_lens = list(rng.integers(0, 700, size=7)) + [1, bs, bs + 1, 3 * bs]
    tables, local_len, num_pages = oracle.block_tables(seq_lens, bs, D, perm_seed=9, rule=CONTIG)
    seen = [set() for _ in range(D)]
    for b, n in enumerate(seq_lens):
        assert int(local_len[:, b].sum()) == n
        nblk = -(-n // bs)
        owner = [oracle.token_shard_rule(t, bs, D, CONTIG, n) for t in range(n)]
        assert owner == sorted(owner)  # each shard holds one run of consecutive tokens, in shard order
        sizes = [sum(1 for g in range(nblk) if oracle.token_shard_rule(g * bs, bs, D, CONTIG, n) == s) for s in range(D)]
        assert max(sizes) - min(sizes) <= 1  # chunks differ by at most one block
        for t in range(n):
            s, j = owner[t], oracle.token_local_block_rule(t, bs, D, CONTIG, n)
            assert j == t // bs - sum(sizes[:s])
            page = tables[s, b, j]
            assert 0 <= page < num_pages[s]
            key = (int(page), t % bs)
            assert key not in seen[s]
            seen[s].add(key)
    for s in range(D):
        assert {p for p, _ in seen[s]} == set(range(int(num_pages[s])))


def test_contiguous_with_one_shard_is_interleaved():
    seq_lens = [300, 5, 1000]
    a = oracle.block_tables(seq_lens, 16, 1)
    b = oracle.block_tables(seq_lens, 16, 1, rule=CONTIG)
    for x, y in zip(a, b):
        np.testing.assert_array_equal(x, y)


@pytest.mark.parametrize("D", [2, 3, 4, 8])
def test_contiguous_sharded_merge_equals_direct(D):
    for layout, Hq, Hkv, dqk, dv in [(GQA, 8, 2, 64, 64), (MLA, 4, 1, 576, 512)]:
        for L in [5, 40, 257]:  # fewer blocks than shards, and several blocks per shard
            w = synth.custom(layout, [L], Hq, Hkv, dqk, dv, 16, seed=L + D)
            q, src = w.query(0), w.kv_source(0)
            O, LSE = oracle.attend(layout, Hq, Hkv, dqk, dv, q, src, w.softmax_scale)
            Om, Lm, _, Lp = oracle.sharded(layout, Hq, Hkv, dqk, dv, q, src, w.softmax_scale, 16, D, rule=CONTIG)
            np.testing.assert_allclose(Om, O, rtol=0, atol=1e-12)
            np.testing.assert_allclose(Lm, LSE, rtol=0, atol=1e-12)


def test_contiguous_multi_token_merge_equals_direct():
    w = synth.custom(GQA, [70], 8, 2, 64, 64, 16, seed=71, q_len=3)
    q, src = w.queries(0), w.kv_source(0)
    O, LSE = oracle.attend_mtp(GQA, 8, 2, 64, 64, q, src, w.softmax_scale, 3)
    Om, Lm, _, _ = oracle.sharded_mtp(GQA, 8, 2, 64, 64, q, src, w.softmax_scale, 3, 16, 3, rule=CONTIG)
    np.testing.assert_allclose(Om, O, rtol=0, atol=1e-12)
    np.testing.assert_allclose(Lm, LSE, rtol=0, atol=1e-12)
    # the drafts (the last tokens) all fall in the last shard: on the other shards every draft sees the
    # whole shard, so its partial is plain attention over that shard
    _, _, Op, Lp = oracle.sharded_mtp(GQA, 8, 2, 64, 64, q, src, w.softmax_scale, 3, 16, 3, rule=CONTIG)
    for s in range(2):
        for j in range(3):
            Os, Ls = oracle.attend(GQA, 8, 2, 64, 64, q[j], src, w.softmax_scale, 16, 3, s, rule=CONTIG)
            np.testing.assert_array_equal(Op[s][j], Os)
            np.testing.assert_array_equal(Lp[s][j], Ls)


def test_contiguous_placement_roundtrip():
    w = synth.custom(GQA, [37, 16, 1, 100], 4, 2, 64, 64, 16, seed=9)
    D = 3
    tables, _, num_pages = oracle.block_tables(w.seq_lens, 16, D, perm_seed=5, rule=CONTIG)
    srcs = [w.kv_source(b) for b in range(w.batch)]
    pools = oracle.place(GQA, 2, 64, 16, D, tables, srcs, num_pages, fill=0xFFFF, rule=CONTIG)
    for b, n in enumerate(w.seq_lens):
        for t in range(n):
            s, j = oracle.token_shard_rule(t, 16, D, CONTIG, n), oracle.token_local_block_rule(t, 16, D, CONTIG, n)
            pg = pools[s][tables[s, b, j] * 2 * 2 * 16 * 64:(tables[s, b, j] + 1) * 2 * 2 * 16 * 64].reshape(2, 2, 16, 64)
            np.testing.assert_array_equal(pg[:, :, t % 16], srcs[b][t])
