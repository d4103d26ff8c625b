"""LSE merge kernel vs the oracle's merge on the same fp32 partials."""
import numpy as np
import pytest
import torch

import oracle
from sequence_sharded_decode_paged_b200 import dcp

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("D", [1, 2, 3, 4, 8, 16])
@pytest.mark.parametrize("d_v", [64, 128, 512])
def test_merge_matches_oracle(D, d_v):
    rng = np.random.default_rng(D * 7 + d_v)
    rows = 333
    Op = rng.standard_normal((D, rows, d_v)).astype(np.float32)
    Lp = (rng.standard_normal((D, rows)) * 4).astype(np.float32)
    Lp[:, 5] = -np.inf                     # a row with no tokens anywhere
    if D > 1:
        Lp[1, 7:40] = -np.inf              # an empty shard for some rows
        Lp[0, 41] = 80.0                   # a dominant shard
    O_parts = [torch.from_numpy(Op[i]).cuda() for i in range(D)]
    L_parts = [torch.from_numpy(Lp[i]).cuda() for i in range(D)]
    O = torch.empty((rows, d_v), device="cuda")
    L = torch.empty((rows,), device="cuda")
    dcp.dcp_lse_merge(O_parts, L_parts, D, rows, d_v, O, L)
    Ow, Lw = oracle.merge(Op.astype(np.float64), Lp.astype(np.float64))
    got_o, got_l = O.cpu().numpy(), L.cpu().numpy()
    assert np.abs(got_o - Ow).max() < 2e-5
    fin = np.isfinite(Lw)
    assert (np.isneginf(got_l) == ~fin).all()
    assert np.abs(got_l[fin] - Lw[fin]).max() < 2e-5
    assert (got_o[5] == 0).all()


def test_merge_without_lse_output():
    O_parts = [torch.randn(10, 128, device="cuda") for _ in range(3)]
    L_parts = [torch.randn(10, device="cuda") for _ in range(3)]
    O = torch.empty(10, 128, device="cuda")
    dcp.dcp_lse_merge(O_parts, L_parts, 3, 10, 128, O, None)
    Ow, _ = oracle.merge(np.stack([o.cpu().numpy() for o in O_parts]).astype(np.float64),
                         np.stack([l.cpu().numpy() for l in L_parts]).astype(np.float64))
    assert np.abs(O.cpu().numpy() - Ow).max() < 2e-5
