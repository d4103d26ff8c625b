"""Decode calls whose device lengths outgrow the block tables.

A request's local page count comes from its device length; if that length
grew past what the tables were sized for (an append without growing the
tables, or a stale descriptor), local blocks j >= max_local_blocks have no
table entry.  The kernels must treat them like out-of-pool pages: never read
the table past its row, leave their tokens out, and record status bit 0.

The tables here get spare rows after the last request that hold a VALID page
id, so even a read past the row stays inside the allocation and would use a
real page without flagging anything: only the bound makes the status appear.
"""
import numpy as np
import pytest
import torch

import synth
from gpu_cases import O_TOL, LSE_TOL, assert_lse_close, assert_o_close, build_cache, oracle_request

pytestmark = pytest.mark.gpu


def _pad_tables(cache, spare_rows: int, fill: int):
    """Give every shard table `spare_rows` extra rows after the last request."""
    for s in range(cache.D):
        t = cache.tables[s]
        padded = torch.full((t.shape[0] + spare_rows, t.shape[1]), fill, dtype=t.dtype, device=t.device)
        padded[:t.shape[0]] = t
        cache.tables[s] = padded


@pytest.mark.parametrize("layout", ["gqa", "mla"])
def test_lengths_past_the_table_are_flagged_and_skipped(layout):
    if layout == "gqa":
        w = synth.custom(synth.GQA, [300, 40, 333], 8, 2, 64, 64, 16, seed=41)
        D, grow = 2, 5 * 16 * 2  # five more local blocks in every shard
    else:
        w = synth.custom(synth.MLA, [260, 70, 330], 64, 1, 576, 512, 64, seed=42)
        D, grow = 2, 3 * 64 * 2
    # zero-filled pools: the grown request's formerly partial last page then holds zeros
    # (finite) in the slots past its old end
    cache, q = build_cache(w, D, pool_fill=0)
    last = w.batch - 1  # the longest request sets max_local_blocks; it is also the last row
    assert cache.local_len[0][last] == max(cache.local_len[0])
    _pad_tables(cache, spare_rows=4, fill=0)
    lens = torch.tensor(w.seq_lens, dtype=torch.int32)
    lens[last] += grow
    cache.seq_lens_dev.copy_(lens.cuda())
    cache.step(q)
    torch.cuda.synchronize()
    assert cache.device_error() == 1
    O = cache.O.cpu().numpy()
    L = cache.LSE.cpu().numpy()
    assert np.isfinite(O).all() and np.isfinite(L).all()
    # the requests whose lengths still fit their rows are unaffected
    for b in range(w.batch - 1):
        Ow, Lw, _, _ = oracle_request(w, b, D)
        assert_o_close(O[b], Ow, O_TOL, f"O[{b}]")
        assert_lse_close(L[b], Lw, LSE_TOL, f"LSE[{b}]")
    # restoring the lengths restores a clean call
    cache.seq_lens_dev.copy_(torch.tensor(w.seq_lens, dtype=torch.int32).cuda())
    cache.step(q)
    torch.cuda.synchronize()
    assert cache.device_error() == 0
    Ow, Lw, _, _ = oracle_request(w, last, D)
    assert_o_close(cache.O.cpu().numpy()[last], Ow, O_TOL, f"O[{last}]")
