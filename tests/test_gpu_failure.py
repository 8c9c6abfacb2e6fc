"""Failure detection on the GPU without a fault: a bounded wait that runs out.

The library's kernels wait on mbarriers with a wall-time limit; on expiry the waiting role
records a timeout in a device error word and every role leaves its loop, so nothing hangs
and the context stays usable.  This test runs that path in isolation (one CTA whose wait
nothing completes) under a host watchdog, checks that the status comes back as
FA_ERR_TIMEOUT, and that the next attention call on the same context is correct.
"""

import time

import numpy as np
import pytest
import torch

import oracle
from exact_io_aware_91_b200 import api, inputs

pytestmark = pytest.mark.gpu


def test_bounded_wait_reports_timeout_and_the_context_stays_usable():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    torch.cuda.set_device(0)
    assert api.fa_last_device_status() == api.FA_OK
    stream = torch.cuda.current_stream()
    api.fa_selftest_wait_timeout(stream)
    # host watchdog: the wait gives up after ~2 s; allow 30 s before declaring it stuck
    t0 = time.time()
    while not stream.query():
        assert time.time() - t0 < 30.0, "bounded wait did not return"
        time.sleep(0.05)
    assert time.time() - t0 > 1.0  # it did wait for its limit
    assert api.fa_last_device_status() == api.FA_ERR_TIMEOUT
    assert api.fa_last_device_status() == api.FA_OK  # cleared by the read
    # the context is still usable: a normal forward + backward matches the oracle
    inp = inputs.make_qkv(1, 2, 200, 64, seed=3, device="cuda")
    q, k, v, do = (inp[n] for n in ("q", "k", "v", "do"))
    o, lse, res = api.fa_fwd_gqa(q, k, v, causal=True, save_residual=True)
    dq, dk, dv = api.fa_bwd_gqa(q, k, v, o, do, lse, causal=True, o_resid=res)
    torch.cuda.synchronize()
    assert api.fa_last_device_status() == api.FA_OK
    O, _ = oracle.attention_forward(q, k, v, 1 / np.sqrt(64), True)
    assert np.abs(o.float().cpu().numpy() - O).max() < 2e-2
    for got, ref in zip((dq, dk, dv), oracle.attention_backward(q, k, v, do, 1 / np.sqrt(64), True)):
        assert np.abs(got.cpu().numpy() - ref).max() < 5e-2
