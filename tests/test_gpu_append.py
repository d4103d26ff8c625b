"""Decode steps that grow the cache: incremental table growth plus the KV append
kernel, checked against the oracle after every step and byte for byte at the end."""
import numpy as np
import pytest
import torch

import oracle
import synth
from gpu_cases import LSE_TOL, O_TOL, assert_lse_close, assert_o_close
from sequence_sharded_decode_paged_b200 import dcp

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("layout,D", [(synth.GQA, 3), (synth.MLA, 2)])
def test_growing_decode(layout, D):
    if layout == synth.GQA:
        Hq, Hkv, dqk, dv, bs = 16, 2, 128, 128, 16
    else:
        Hq, Hkv, dqk, dv, bs = 64, 1, 576, 512, 64
    L0 = np.array([40, 0, 130, 17], np.int32)
    incs = [np.array([1, 1, 1, 1], np.int32)] * 4 + [np.array([1, 70, 1, 150], np.int32)] + \
        [np.array([1, 1, 1, 1], np.int32)] * 3
    final = L0 + sum(incs)
    w = synth.custom(layout, final.tolist(), Hq, Hkv, dqk, dv, bs, seed=99)  # token values depend on (b, t) only
    B = w.batch
    mlb, pages = dcp.dcp_block_table_extent(final, bs, D)
    desc = dcp.make_desc(layout, B, Hq, Hkv, dqk, dv, bs, mlb, w.softmax_scale)
    page_bytes = dcp.dcp_kv_page_bytes(desc)
    pools = [torch.full((max(1, int(n)) * page_bytes // 2,), -1, dtype=torch.int16, device="cuda") for n in pages]
    tables = np.full((D, B, mlb), -1, np.int32)
    local_len = np.zeros((D, B), np.int32)
    next_page = np.zeros(D, np.int32)
    t_or, l_or, n_or = tables.copy(), local_len.copy(), next_page.copy()
    tables_dev = [torch.from_numpy(tables[s]).cuda() for s in range(D)]
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    ws = torch.empty(dcp.dcp_decode_workspace_bytes(desc, D), dtype=torch.uint8, device="cuda")
    dcp.dcp_workspace_init(ws)
    O_parts = torch.empty((D, B, Hq, dv), device="cuda")
    L_parts = torch.empty((D, B, Hq), device="cuda")
    O = torch.empty((B, Hq, dv), device="cuda")
    L = torch.empty((B, Hq), device="cuda")
    q = torch.from_numpy(np.stack([w.query(b) for b in range(B)]).view(np.int16)).cuda()
    full_src = [w.kv_source(b) for b in range(B)]
    lens = np.zeros(B, np.int32)
    for inc in [L0] + incs:
        new = lens + inc
        dcp.dcp_grow_block_table(lens, new, bs, D, tables, local_len, next_page, pages)
        assert oracle.grow_tables(lens, new, bs, D, t_or, l_or, n_or, pages) == 0
        np.testing.assert_array_equal(tables, t_or)
        for s in range(D):
            tables_dev[s].copy_(torch.from_numpy(tables[s]))
        rows = [full_src[b][lens[b]:new[b]] for b in range(B)]
        cu = np.zeros(B + 1, np.int64)
        cu[1:] = np.cumsum([r.shape[0] for r in rows])
        kv_new = torch.from_numpy(np.concatenate(rows).view(np.int16)).cuda()
        dcp.dcp_append_kv(desc, D, kv_new, torch.from_numpy(cu).cuda(), torch.from_numpy(lens).cuda(), tables_dev,
                          pools, pages, err)
        lens = new
        sl = torch.from_numpy(lens).cuda()
        dcp.dcp_decode_partial_all(desc, q, pools, pages, tables_dev, sl, D, list(O_parts), list(L_parts), ws)
        dcp.dcp_lse_merge(list(O_parts), list(L_parts), D, B * Hq, dv, O, L)
        torch.cuda.synchronize()
        Og, Lg = O.cpu().numpy(), L.cpu().numpy()
        for b in range(B):
            Ow, Lw, _, _ = oracle.sharded(layout, Hq, Hkv, dqk, dv, w.query(b), full_src[b][:lens[b]],
                                          w.softmax_scale, bs, D)
            assert_o_close(Og[b], Ow, O_TOL, f"O[{b}] at lengths {lens.tolist()}")
            assert_lse_close(Lg[b], Lw, LSE_TOL, f"LSE[{b}]")
    assert int(err.item()) == 0 and dcp.dcp_read_device_error(ws) == 0
    ref = oracle.place(layout, Hkv, dqk, bs, D, t_or, full_src, n_or, fill=0xFFFF)
    for s in range(D):
        got = pools[s].cpu().numpy().view(np.uint16)[:ref[s].size]
        np.testing.assert_array_equal(got, ref[s])


@pytest.mark.parametrize("layout,D,q_len,kv_dtype", [(synth.GQA, 3, 3, dcp.DCP_KV_BF16), (synth.GQA, 2, 2, dcp.DCP_KV_FP8_E4M3),
                                                     (synth.MLA, 2, 2, dcp.DCP_KV_BF16)])
def test_speculative_decode_loop(layout, D, q_len, kv_dtype):
    """Each step appends q_len draft tokens' KV, then decodes those q_len tokens causally: the
    append path and multi-token decode together, against the oracle after every step."""
    if layout == synth.GQA:
        Hq, Hkv, dqk, dv, bs = 64, 8, 128, 128, 16
    else:
        Hq, Hkv, dqk, dv, bs = 64, 1, 576, 512, 64
    L0 = np.array([37, 0, 100], np.int32)
    steps = 5
    final = L0 + steps * q_len
    w = synth.custom(layout, final.tolist(), Hq, Hkv, dqk, dv, bs, seed=123, q_len=q_len, kv_amp=0.5)
    B = w.batch
    scale = 2.0 ** -7
    mlb, pages = dcp.dcp_block_table_extent(final, bs, D)
    desc = dcp.make_desc(layout, B, Hq, Hkv, dqk, dv, bs, mlb, w.softmax_scale, q_len, kv_dtype, scale, scale)
    page_bytes = dcp.dcp_kv_page_bytes(desc)
    pools = [torch.full((max(1, int(n)) * page_bytes // 2,), -1, dtype=torch.int16, device="cuda") for n in pages]
    tables = np.full((D, B, mlb), -1, np.int32)
    local_len = np.zeros((D, B), np.int32)
    next_page = np.zeros(D, np.int32)
    tables_dev = [torch.from_numpy(tables[s]).cuda() for s in range(D)]
    ws = torch.empty(dcp.dcp_decode_workspace_bytes(desc, D), dtype=torch.uint8, device="cuda")
    dcp.dcp_workspace_init(ws)
    O_parts = torch.empty((D, B, q_len, Hq, dv), device="cuda")
    L_parts = torch.empty((D, B, q_len, Hq), device="cuda")
    O = torch.empty((B, q_len, Hq, dv), device="cuda")
    Lm = torch.empty((B, q_len, Hq), device="cuda")
    full_src = [w.kv_source(b) for b in range(B)]
    lens = np.zeros(B, np.int32)
    for step in range(steps + 1):
        new = L0.copy() if step == 0 else lens + q_len
        dcp.dcp_grow_block_table(lens, new, bs, D, tables, local_len, next_page, pages)
        for s in range(D):
            tables_dev[s].copy_(torch.from_numpy(tables[s]))
        rows = [full_src[b][lens[b]:new[b]] for b in range(B)]
        cu = np.zeros(B + 1, np.int64)
        cu[1:] = np.cumsum([r.shape[0] for r in rows])
        kv_new = torch.from_numpy(np.concatenate(rows).view(np.int16)).cuda()
        dcp.dcp_append_kv(desc, D, kv_new, torch.from_numpy(cu).cuda(), torch.from_numpy(lens).cuda(), tables_dev,
                          pools, pages)
        lens = new
        # the drafts of this step are the last q_len tokens of each request; their queries differ per step
        wq = synth.custom(layout, final.tolist(), Hq, Hkv, dqk, dv, bs, seed=500 + step, q_len=q_len)
        q = torch.from_numpy(np.stack([wq.queries(b) for b in range(B)]).view(np.int16)).cuda()
        dcp.dcp_decode_partial_all(desc, q, pools, pages, tables_dev, torch.from_numpy(lens).cuda(), D,
                                   list(O_parts), list(L_parts), ws)
        dcp.dcp_lse_merge(list(O_parts), list(L_parts), D, B * q_len * Hq, dv, O, Lm)
        torch.cuda.synchronize()
        Og, Lg = O.cpu().numpy(), Lm.cpu().numpy()
        for b in range(B):
            src = full_src[b][:lens[b]]
            if kv_dtype == dcp.DCP_KV_FP8_E4M3:
                src_vals = oracle.dequantize_kv_gqa(oracle.quantize_kv_gqa(src, scale, scale), scale, scale)
            else:
                src_vals = synth.bf16_bits_to_f64(src)
            for j in range(q_len):
                n = oracle.visible_tokens(int(lens[b]), q_len, j)
                parts = [oracle.attend_values(layout, Hq, Hkv, dqk, dv, wq.queries(b)[j], src_vals[:n],
                                              w.softmax_scale, bs, D, s) for s in range(D)]
                Ow, Lw = oracle.merge(np.stack([p[0] for p in parts]), np.stack([p[1] for p in parts]))
                assert_o_close(Og[b, j], Ow, O_TOL, f"O[{b}][{j}] step {step}")
                assert_lse_close(Lg[b, j], Lw, LSE_TOL, f"LSE[{b}][{j}] step {step}")
    assert dcp.dcp_read_device_error(ws) == 0
