"""fa_bwd_noalloc: the backward pass for callers that cannot allocate device memory.

Such callers (an engine plugin whose enqueue path may not allocate, a latency-bound loop
that cannot afford cudaMalloc's implicit synchronisation) run the backward pass with the
library's built-in scratch array instead of a workspace of their own.  These tests call
that entry point through the C ABI and compare it with fa_bwd_gqa (H_kv = H), which gets a
freshly allocated workspace, on two calls in a row: the second call finds the first call's
data still in the shared scratch array and must not depend on it.  Both run the same
deterministic kernels, so the results must be the same bits; the first case is also checked
against the oracle.
"""

import numpy as np
import pytest
import torch

from exact_io_aware_91_b200 import api, inputs
from exact_io_aware_91_b200 import build as fa_build

TOL_GRAD = 5e-2  # the gradient tolerance of the parity tests


@pytest.fixture(scope="module")
def lib():
    fa_build.build()  # so that this file also runs on its own, on a fresh checkout
    return api.library()


def _problem(B, H, N, d, causal, seed):
    inp = inputs.make_qkv(B, H, N, d, seed=seed, device="cuda")
    o, lse, res = api.fa_fwd_gqa(inp["q"], inp["k"], inp["v"], causal=causal, save_residual=True)
    return inp, o, lse, res


@pytest.mark.gpu
def test_noalloc_backward_matches_fa_bwd_on_two_calls_in_a_row(lib):
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    import oracle

    torch.cuda.set_device(0)
    cases = [(1, 4, 1000, 128, True, 21), (2, 3, 777, 64, False, 22)]
    for n_case, (B, H, N, d, causal, seed) in enumerate(cases):
        assert api.fa_bwd_workspace_size(B, H, N, d) <= api.FA_BWD_NOALLOC_MAX_WORKSPACE
        inp, o, lse, res = _problem(B, H, N, d, causal, seed)
        q, k, v, do = inp["q"], inp["k"], inp["v"], inp["do"]
        ref = api.fa_bwd_gqa(q, k, v, o, do, lse, causal=causal, o_resid=res)
        outs = [torch.full((B, H, N, d), float("nan"), device="cuda") for _ in range(3)]
        got = api.fa_bwd_noalloc(q, k, v, o, do, lse, *outs, causal=causal, o_resid=res)
        torch.cuda.synchronize()
        assert api.fa_last_device_status() == api.FA_OK
        for name, g, r in zip(("dQ", "dK", "dV"), got, ref):
            assert torch.equal(g, r), f"{name} differs from fa_bwd_gqa (N={N}, d={d})"
        if n_case == 0:
            want = oracle.attention_backward(q, k, v, do, 1.0 / np.sqrt(d), causal)
            for name, g, r in zip(("dQ", "dK", "dV"), got, want):
                err = np.abs(g.double().cpu().numpy() - r).max()
                assert err <= TOL_GRAD, f"{name} max-abs {err:.3e} against the oracle"


def test_noalloc_rejects_problems_larger_than_its_scratch(lib):
    # checked on the host before anything is launched: no GPU needed
    A = 0x10000
    B, H, N, d = 1, 64, 8192, 128  # workspace ~0.54 GB > 64 MiB
    assert api.fa_bwd_workspace_size(B, H, N, d) > api.FA_BWD_NOALLOC_MAX_WORKSPACE
    st = lib.fa_bwd_noalloc(A, A, A, A, None, A, A, A, A, A, B, H, N, d, 0.088, 1, None)
    assert st == api.FA_ERR_UNSUPPORTED
    # empty and invalid problems take fa_bwd_gqa's answers
    assert lib.fa_bwd_noalloc(None, None, None, None, None, None, None, None, None, None,
                              1, 1, 0, 128, 0.088, 1, None) == api.FA_OK
    assert lib.fa_bwd_noalloc(A, A, A, A, None, A, A, A, A, A, 1, 1, 16, 96, 0.1, 0, None) == api.FA_ERR_UNSUPPORTED
    assert lib.fa_bwd_noalloc(A, A, A, A, None, A, A, A, A, A, 1, 1, 16, 64, -1.0, 0, None) == api.FA_ERR_INVALID_ARG
