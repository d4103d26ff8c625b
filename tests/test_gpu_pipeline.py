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
