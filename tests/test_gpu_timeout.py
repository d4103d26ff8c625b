"""The decode kernels' bounded pipeline waits: a wait that never completes gives up after the
limit and reports through the workspace status word, and the CUDA context stays usable.  The
wait runs on a barrier that nothing arrives on (no copy or product is in flight), so the test
neither faults nor hangs the GPU."""
import time

import numpy as np
import pytest
import torch

import synth
from gpu_cases import LSE_TOL, O_TOL, assert_lse_close, assert_o_close, build_cache, oracle_request
from sequence_sharded_decode_paged_b200 import dcp

pytestmark = pytest.mark.gpu

TIMEOUT_BIT = 2  # bit 1 of the status word: a pipeline wait timed out


def test_wait_gives_up_reports_and_the_next_call_is_correct():
    w = synth.custom(synth.GQA, [300, 17, 1000], 8, 2, 64, 64, 16, seed=71)
    D = 2
    cache, q = build_cache(w, D)
    assert cache.device_error() == 0
    t0 = time.perf_counter()
    dcp.dcp_check_wait_timeout(cache.workspace)
    torch.cuda.synchronize()
    waited = time.perf_counter() - t0
    assert 1.0 < waited < 30.0  # the limit is about 4 s: the wait gave up, it did not spin on
    assert cache.device_error() == TIMEOUT_BIT
    assert cache.device_error() == 0  # reading clears the word
    # the context is intact: a normal decode step right after is exact
    cache.step(q)
    torch.cuda.synchronize()
    assert cache.device_error() == 0
    O, L = cache.O.cpu().numpy(), cache.LSE.cpu().numpy()
    for b in range(w.batch):
        Ob, Lb, _, _ = oracle_request(w, b, D)
        assert_o_close(O[b], Ob, O_TOL, f"O[{b}]")
        assert_lse_close(L[b], Lb, LSE_TOL, f"LSE[{b}]")
