"""The host-to-host step pipeline gives the same results as the plain device step."""
import numpy as np
import pytest
import torch

import synth
from gpu_cases import build_cache, host_q
from sequence_sharded_decode_paged_b200.cache import HostStepPipeline

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("layout", [synth.GQA, synth.MLA])
def test_pipeline_matches_device_step(layout):
    if layout == synth.GQA:
        w = synth.custom(synth.GQA, [3000, 17, 900, 0], 16, 2, 128, 128, 16, seed=31)
    else:
        w = synth.custom(synth.MLA, [3000, 17, 900], 64, 1, 576, 512, 64, seed=32)
    cache, q = build_cache(w, 4)
    O_ref, L_ref = [t.clone() for t in cache.step(q)]
    pipe = HostStepPipeline(cache)
    host_in = pipe.pack_inputs(host_q(w).view(np.int16), w.seq_lens, cache.tables_host)
    outs = [pipe.host_output(), pipe.host_output()]
    for i in range(5):  # several steps through both buffer sets
        pipe.step(i, host_in, outs[i & 1])
    pipe.synchronize()
    for buf in outs:
        O, L = pipe.unpack_output(buf)
        assert torch.equal(O, O_ref.cpu()) and torch.equal(L, L_ref.cpu())


@pytest.mark.parametrize("layout", [synth.GQA, synth.MLA])
@pytest.mark.parametrize("pinned", [True, False])
def test_host_step_call_matches_device_step(layout, pinned):
    """dcp_decode_step_host (host inputs and outputs through the C ABI) equals the device step bit for bit."""
    from sequence_sharded_decode_paged_b200 import dcp
    if layout == synth.GQA:
        w = synth.custom(synth.GQA, [2500, 1, 700, 0, 64], 32, 4, 128, 128, 16, seed=33, kv_amp=0.5)
    else:
        w = synth.custom(synth.MLA, [4000, 65, 0, 1500], 64, 1, 576, 512, 64, seed=34)
    cache, q = build_cache(w, 3)
    O_ref, L_ref = [t.clone().cpu() for t in cache.step(q)]
    hq = torch.from_numpy(np.ascontiguousarray(host_q(w)).view(np.int16).reshape(-1).copy())
    hl = torch.tensor(w.seq_lens, dtype=torch.int32)
    ht = torch.from_numpy(np.ascontiguousarray(cache.tables_host, dtype=np.int32))
    hO = torch.full(O_ref.shape, float("nan"), dtype=torch.float32)
    hL = torch.full(L_ref.shape, float("nan"), dtype=torch.float32)
    if pinned:
        hq, hl, ht, hO, hL = (t.pin_memory() for t in (hq, hl, ht, hO, hL))
    staging = torch.empty(dcp.dcp_host_step_staging_bytes(cache.desc, cache.D), dtype=torch.uint8, device="cuda")
    for _ in range(2):  # the second step reuses the staging buffer
        dcp.dcp_decode_step_host(cache.desc, cache.D, hq, hl, ht, cache.pools, cache.pool_pages, staging,
                                 cache.workspace, hO, hL)
        torch.cuda.synchronize()
        assert torch.equal(hO, O_ref) and torch.equal(hL, L_ref)
    assert cache.device_error() == 0


def test_host_step_call_rejects_small_staging():
    from sequence_sharded_decode_paged_b200 import dcp
    w = synth.custom(synth.GQA, [100, 50], 8, 2, 64, 64, 16, seed=35)
    cache, q = build_cache(w, 2)
    need = dcp.dcp_host_step_staging_bytes(cache.desc, cache.D)
    staging = torch.empty(need - 256, dtype=torch.uint8, device="cuda")
    hq = torch.from_numpy(np.ascontiguousarray(host_q(w)).view(np.int16).reshape(-1).copy())
    hO = torch.empty(cache.O.shape, dtype=torch.float32)
    with pytest.raises(dcp.DcpError) as e:
        dcp.dcp_decode_step_host(cache.desc, cache.D, hq, torch.tensor(w.seq_lens, dtype=torch.int32),
                                 torch.from_numpy(np.ascontiguousarray(cache.tables_host)), cache.pools,
                                 cache.pool_pages, staging, cache.workspace, hO)
    assert e.value.status == dcp.DCP_ERR_CAPACITY
