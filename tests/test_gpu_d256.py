"""GPU parity of head dimension 256 against the fp64 oracle: the forward (fa_fwd_ws /
fa_attn_fwd; its own persistent kernel, one 128-row query tile per work unit, S double-
buffered in TMEM) with the bf16 tolerances O max-abs 2e-2, mean-abs 2e-3, LSE 1e-3, and the
backward (fa_attn_bwd / fa_bwd; dK/dV per d-half with S^T, dP^T recomputed, dQ with S single-
buffered) with dQ/dK/dV max-abs 5e-2.  The oracle takes any head dimension."""

import numpy as np
import pytest
import torch

import oracle
from exact_io_aware_91_b200 import api, inputs

pytestmark = pytest.mark.gpu

TOL_O_MAX = 2e-2
TOL_O_MEAN = 2e-3
TOL_LSE = 1e-3
TOL_GRAD = 5e-2


@pytest.fixture(scope="module", autouse=True)
def _device():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    torch.cuda.set_device(0)
    yield
    assert api.fa_last_device_status() == api.FA_OK


def f64(t):
    return t.detach().float().cpu().numpy().astype(np.float64)


CASES = [  # B, H, H_kv, N, causal, window, spiky
    (1, 2, 2, 256, True, (-1, -1), 0.0),
    (1, 2, 2, 1000, False, (-1, -1), 0.0),
    (2, 4, 2, 777, True, (-1, -1), 0.0),
    (1, 4, 1, 640, False, (-1, -1), 0.0),
    (1, 2, 2, 1500, True, (300, -1), 0.0),
    (1, 2, 2, 900, False, (100, 60), 0.0),
    (1, 2, 2, 2048, True, (-1, -1), 0.01),
    (1, 1, 1, 129, True, (-1, -1), 0.0),
    (1, 1, 1, 1, False, (-1, -1), 0.0),
]


def assert_grads(got, want, tag):
    for name, g, r in zip(("dQ", "dK", "dV"), got, want):
        err = np.abs(f64(g) - r).max()
        assert err <= TOL_GRAD, f"{tag}: {name} max-abs {err:.3e}"


@pytest.mark.parametrize("B,H,Hkv,N,causal,window,spiky", CASES)
def test_d256_forward_backward(B, H, Hkv, N, causal, window, spiky):
    inp = inputs.make_qkv(B, H, N, 256, spiky_frac=spiky, seed=21 + N, device="cuda", kv_heads=Hkv)
    q, k, v, do = inp["q"], inp["k"], inp["v"], inp["do"]
    scale = 1.0 / 16.0
    o, lse, res = api.fa_attn_fwd(q, k, v, causal=causal, scale=scale, window=window, save_residual=True)
    grads = api.fa_attn_bwd(q, k, v, o, do, lse, causal=causal, scale=scale, window=window, o_resid=res)
    torch.cuda.synchronize()
    tag = f"d=256 B={B} H={H} Hkv={Hkv} N={N} causal={causal} window={window}"
    assert_grads(grads, oracle.attention_backward_gqa(q.cpu(), k.cpu(), v.cpu(), do.cpu(), scale, causal, window),
                 tag)
    O, L = oracle.attention_forward_gqa(q.cpu(), k.cpu(), v.cpu(), scale, causal, window)
    err = np.abs(f64(o) - O)
    assert err.max() <= TOL_O_MAX, f"O max-abs {err.max():.3e}"
    assert err.mean() <= TOL_O_MEAN, f"O mean-abs {err.mean():.3e}"
    assert np.abs(f64(lse) - L).max() <= TOL_LSE
    # the residual is the rounding of the fp32 O to bf16: O + residual is closer to the oracle
    # (up to the ~1e-4 relative error of the kernel's exponentials, visible where O's bf16
    # rounding happens to be exact)
    err2 = np.abs(f64(o) + f64(res) - O)
    assert err2.mean() <= err.mean() + 1e-4


def test_d256_plain_entry_point_and_workspace_path_agree():
    inp = inputs.make_qkv(1, 4, 700, 256, backward=False, seed=3, device="cuda")
    a = api.fa_fwd_ws(inp["q"], inp["k"], inp["v"], causal=True)
    b = api.fa_attn_fwd(inp["q"], inp["k"], inp["v"], causal=True)
    torch.cuda.synchronize()
    assert torch.equal(a[0], b[0]) and torch.equal(a[1], b[1])


def test_d256_long_sampled_rows():
    B, H, N, d = 1, 8, 8192, 256
    inp = inputs.make_qkv(B, H, N, d, spiky_frac=0.01, backward=False, seed=9, device="cuda")
    scale = 1.0 / 16.0
    o, lse = api.fa_fwd_ws(inp["q"], inp["k"], inp["v"], causal=True, scale=scale)
    torch.cuda.synchronize()
    rows = sorted({0, 1, 127, 128, 255, 4095, 4096, N - 2, N - 1} |
                  set(np.random.default_rng(4).integers(0, N, 23).tolist()))
    for h in (0, 5):
        q, k, v = (inp[n][0, h].cpu() for n in ("q", "k", "v"))
        O, L = oracle.attention_forward_rows(q, k, v, scale, True, rows)
        err = np.abs(f64(o[0, h])[rows] - O)
        assert err.max() <= TOL_O_MAX and err.mean() <= TOL_O_MEAN, f"head {h}: {err.max():.3e}"
        assert np.abs(f64(lse[0, h])[rows] - L).max() <= TOL_LSE


def test_d256_plain_signatures():
    # fa_fwd has no workspace, hence no d = 256 kernel (V is converted on chip only for d <= 128);
    # fa_bwd takes d = 256 and matches the oracle on the workspace forward's O and LSE
    inp = inputs.make_qkv(1, 2, 300, 256, seed=1, device="cuda")
    q, k, v, do = inp["q"], inp["k"], inp["v"], inp["do"]
    with pytest.raises(api.FAError) as e:
        api.fa_fwd(q, k, v)
    assert e.value.status == api.FA_ERR_UNSUPPORTED
    o, lse = api.fa_fwd_ws(q, k, v, causal=True)
    grads = api.fa_bwd(q, k, v, o, do, lse, causal=True)
    torch.cuda.synchronize()
    assert_grads(grads, oracle.attention_backward(q.cpu(), k.cpu(), v.cpu(), do.cpu(), 1 / 16, True), "fa_bwd d=256")


def test_d256_backward_long_spiky():
    # many units per CTA and every key tile of a 4096-token causal head with peaked rows
    B, H, N, d = 1, 3, 4096, 256
    inp = inputs.make_qkv(B, H, N, d, spiky_frac=0.01, seed=8, device="cuda")
    q, k, v, do = inp["q"], inp["k"], inp["v"], inp["do"]
    o, lse, res = api.fa_fwd_ws(q, k, v, causal=True, scale=1 / 16, save_residual=True)
    grads = api.fa_bwd_gqa(q, k, v, o, do, lse, causal=True, scale=1 / 16, o_resid=res)
    torch.cuda.synchronize()
    for h in range(H):
        ref = oracle.attention_backward(q[0, h].cpu(), k[0, h].cpu(), v[0, h].cpu(), do[0, h].cpu(), 1 / 16, True)
        assert_grads((grads[0][0, h], grads[1][0, h], grads[2][0, h]), ref, f"d=256 N=4096 head {h}")
