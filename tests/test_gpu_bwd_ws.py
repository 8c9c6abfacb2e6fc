"""GPU checks of fa_bwd_ws, the backward that reuses the fp16 copy of V which fa_fwd_ws left
in its workspace: its gradients are bit-identical to fa_bwd_gqa's (which converts V itself)
on plain, grouped-query, ragged and d = 256 shapes and at workload 2's size, including when the
bound on the fp16 dS makes the backward choose another exponent for V than the forward did
(the backward then converts V again into the forward's copy and records the new exponent, so a
later backward on the same forward workspace is still right)."""

import pytest
import torch

from exact_io_aware_91_b200 import api, inputs

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _device():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    torch.cuda.set_device(0)
    yield
    assert api.fa_last_device_status() == api.FA_OK


def v_copy_exponent(fws, B, Hkv, N, d):
    """The exponent recorded with the forward workspace's V copy (int32 at byte 4 of the control
    block that follows the copy)."""
    off = (B * Hkv * N * d * 2 + 255) // 256 * 256 + 4
    return int(fws[off:off + 4].view(torch.int32).item())


def both_backwards(inp, causal, scale, v_scale=1.0, do_scales=(1.0,)):
    """One fa_fwd_ws, then for each dO scaling fa_bwd_gqa and fa_bwd_ws (forward workspace
    reused across the calls); returns the pairs of gradient triples and the V copy's exponent
    after each fa_bwd_ws."""
    q, k = inp["q"], inp["k"]
    v = (inp["v"].float() * v_scale).to(torch.bfloat16)
    B, H, N, d = q.shape
    Hkv = k.shape[1]
    fws = torch.empty(api.fa_fwd_workspace_size(B, Hkv, N, d), dtype=torch.uint8, device="cuda")
    o, lse, res = api.fa_fwd_ws(q, k, v, causal=causal, scale=scale, save_residual=True, workspace=fws)
    out, exps = [], []
    for s in do_scales:
        do = (inp["do"].float() * s).to(torch.bfloat16)
        ref = api.fa_bwd_gqa(q, k, v, o, do, lse, causal=causal, scale=scale, o_resid=res)
        got = api.fa_bwd_ws(q, k, v, o, do, lse, fws, causal=causal, scale=scale, o_resid=res)
        torch.cuda.synchronize()
        assert api.fa_last_device_status() == api.FA_OK
        out.append((ref, got))
        exps.append(v_copy_exponent(fws, B, Hkv, N, d))
    return out, exps


SHAPES = [  # B, H, H_kv, N, d, causal
    (1, 2, 2, 300, 128, True),
    (2, 4, 1, 1000, 64, False),
    (1, 4, 2, 777, 128, True),
    (1, 2, 2, 513, 256, True),
    (2, 3, 3, 129, 64, True),
]


@pytest.mark.parametrize("B,H,Hkv,N,d,causal", SHAPES)
def test_gradients_identical_to_the_backward_with_its_own_copy(B, H, Hkv, N, d, causal):
    inp = inputs.make_qkv(B, H, N, d, seed=31 + N, device="cuda", kv_heads=None if Hkv == H else Hkv,
                          spiky_frac=0.01)
    pairs, exps = both_backwards(inp, causal, d ** -0.5)
    assert exps == [0]  # max |V| in [2^-4, 2^15]: both keep exponent 0
    for ref, got in pairs:
        for name, a, b in zip(("dq", "dk", "dv"), ref, got):
            assert torch.equal(a, b), f"{name} differs"


def test_workload2_size():
    w = inputs.workload(2)
    inp = inputs.make_qkv(w.B, w.H, w.N, w.d, seed=w.seed, device="cuda")
    pairs, _ = both_backwards(inp, w.causal, w.scale)
    for ref, got in pairs:
        for name, a, b in zip(("dq", "dk", "dv"), ref, got):
            assert torch.equal(a, b), f"{name} differs"


def test_backward_rescales_the_forward_copy_when_needed():
    # max |V| ~ 1.1e3: the forward keeps the V copy at exponent 0 (inside [2^-4, 2^15]).  With
    # dO ~ N(0, 1) the dS bound 2 d max|dO| max|V| exceeds 2^15, so the backward picks the
    # exponent that brings max |V| into [4, 8) (-8) and converts V again into the forward's
    # copy; a dO with max |dO| ~ 0.09 (still exponent 0 for its copy) keeps the bound within
    # 2^15, so the next backward wants exponent 0 and converts the copy back; then -8 again
    inp = inputs.make_qkv(1, 2, 640, 128, seed=5, device="cuda")
    vmax = 250.0 * float(inp["v"].float().abs().max())
    assert 1024.0 <= vmax < 2048.0
    small = 0.09 / float(inp["do"].float().abs().max())
    pairs, exps = both_backwards(inp, True, 128 ** -0.5, v_scale=250.0, do_scales=(1.0, small, 1.0))
    assert exps == [-8, 0, -8]
    for ref, got in pairs:
        for name, a, b in zip(("dq", "dk", "dv"), ref, got):
            assert torch.equal(a, b), f"{name} differs"


def test_forward_and_backward_allocate_nothing():
    # with caller workspaces the training path (fa_fwd_ws + fa_bwd_ws) allocates no device memory
    B, H, N, d = 1, 4, 4096, 128
    inp = inputs.make_qkv(B, H, N, d, seed=3, device="cuda")
    q, k, v, do = inp["q"], inp["k"], inp["v"], inp["do"]
    fws = torch.empty(api.fa_fwd_workspace_size(B, H, N, d), dtype=torch.uint8, device="cuda")
    ws = torch.empty(api.fa_bwd_ws_workspace_size(B, H, H, N, d), dtype=torch.uint8, device="cuda")
    o, lse, res = torch.empty_like(q), torch.empty((B, H, N), device="cuda"), torch.empty_like(q)
    dq = torch.empty(q.shape, dtype=torch.float32, device="cuda")
    dk, dv = torch.empty_like(dq), torch.empty_like(dq)
    torch.cuda.synchronize()
    free0 = torch.cuda.mem_get_info()[0]
    api.fa_fwd_ws(q, k, v, causal=True, o=o, lse=lse, o_resid=res, workspace=fws)
    api.fa_bwd_ws(q, k, v, o, do, lse, fws, causal=True, workspace=ws, dq=dq, dk=dk, dv=dv, o_resid=res)
    torch.cuda.synchronize()
    assert api.fa_last_device_status() == api.FA_OK
    assert torch.cuda.mem_get_info()[0] >= free0 - (2 << 20)  # no N x N (or any) device buffer
