"""Value range: bf16 inputs far outside fp16's range (and far below it).

The kernels' fp16 copies are each the bf16 input times a power of two 2^e chosen from the
tensor's largest magnitude, undone exactly in the products' scalars.  So multiplying an input
by a power of two 2^a must multiply each result by exactly the factor the mathematics gives,
bit for bit, as long as the copies come out the same: V 2^a scales O and dQ, dK by 2^a and
leaves dV and LSE; dO 2^a scales the three gradients by 2^a; Q 2^a, K 2^a with scale 2^-2a
leave O, LSE, dV and scale dQ, dK by 2^-a.  The base draws have their largest magnitude in
[4, 8), where the chosen exponent cancels the scaling exactly.  Inputs that are not powers
of two times a plain draw (|V| ~ 1e5, |Q|, |K| ~ 1e5 with a small scale, dO ~ 1e4 and ~1e-6)
are checked against the oracle with the parity tolerances times the inputs' scale.  Inputs
that no scaling can handle (non-finite values, scores beyond fp32) must be reported as
FA_ERR_RANGE, not pass silently.
"""

import math

import numpy as np
import pytest
import torch

import oracle
from exact_io_aware_91_b200 import api, inputs

pytestmark = pytest.mark.gpu

TOL_O_MAX, TOL_O_MEAN, TOL_LSE, TOL_GRAD = 2e-2, 2e-3, 1e-3, 5e-2


@pytest.fixture(scope="module", autouse=True)
def _device():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    torch.cuda.set_device(0)
    yield
    assert api.fa_last_device_status() == api.FA_OK


def f64(t):
    return t.detach().double().cpu().numpy()


def scaled(t: torch.Tensor, a: int) -> torch.Tensor:
    """t * 2^a, exact for bf16 / fp32 values inside the range."""
    return (t.double() * 2.0 ** a).to(t.dtype)


def base_inputs(B, H, N, d, seed, kv_heads=None):
    inp = inputs.make_qkv(B, H, N, d, seed=seed, device="cuda", kv_heads=kv_heads)
    for name in ("q", "k", "v", "do"):  # the exponent chosen for 2^a t is then exactly -a
        amax = float(inp[name].float().abs().max())
        assert 4.0 <= amax < 8.0, f"{name}: largest magnitude {amax} outside [4, 8)"
    return inp


def run_path(inp, causal, scale, d256=False):
    """fa_fwd_ws (with residual) then fa_bwd_gqa (with residual); d = 256: forward only."""
    q, k, v = inp["q"], inp["k"], inp["v"]
    o, lse, res = api.fa_fwd_ws(q, k, v, causal=causal, scale=scale, save_residual=True)
    grads = None
    if not d256:
        grads = api.fa_bwd_gqa(q, k, v, o, inp["do"], lse, causal=causal, scale=scale, o_resid=res)
    torch.cuda.synchronize()
    assert api.fa_last_device_status() == api.FA_OK
    return o, lse, res, grads


# ------------------------------------------------------------------ exact power-of-two scaling
CASES = {
    # name: (input scalings {tensor: a}, scale factor 2^s, result exponents (O, LSE, dQ, dK, dV))
    "V x 2^17": ({"v": 17}, 0, (17, 0, 17, 17, 0)),
    "V x 2^-20": ({"v": -20}, 0, (-20, 0, -20, -20, 0)),
    "dO x 2^13": ({"do": 13}, 0, (0, 0, 13, 13, 13)),
    "dO x 2^-20": ({"do": -20}, 0, (0, 0, -20, -20, -20)),
    "Q, K x 2^17, scale x 2^-34": ({"q": 17, "k": 17}, -34, (0, 0, -17, -17, 0)),
    # dS scales with dO V (2^5); dQ = scale dS K: 2^(-11+5-9), dK = scale dS^T Q: 2^(-11+5+20)
    "all at once": ({"q": 20, "k": -9, "v": 30, "do": -25}, -11, (30, 0, -15, 14, -25)),
}


@pytest.mark.parametrize("name", list(CASES))
@pytest.mark.parametrize("B,H,Hkv,N,d,causal", [(1, 3, 3, 700, 128, True), (2, 4, 2, 333, 64, False)])
def test_power_of_two_scaling_is_exact(name, B, H, Hkv, N, d, causal):
    ins, s, (eo, el, edq, edk, edv) = CASES[name]
    inp = base_inputs(B, H, N, d, seed=N + d + H, kv_heads=Hkv)
    scale = 1.0 / math.sqrt(d)
    o0, l0, r0, g0 = run_path(inp, causal, scale)
    inp_s = {n: scaled(t, ins.get(n, 0)) for n, t in inp.items()}
    o1, l1, r1, g1 = run_path(inp_s, causal, scale * 2.0 ** s)
    assert torch.equal(o1, scaled(o0, eo)), f"{name}: O"
    assert torch.equal(l1, l0 if el == 0 else scaled(l0, el)), f"{name}: LSE"
    assert torch.equal(r1, scaled(r0, eo)), f"{name}: residual"
    for g, ref, e, what in zip(g1, g0, (edq, edk, edv), ("dQ", "dK", "dV")):
        assert torch.equal(g, scaled(ref, e)), f"{name}: {what}"


def test_power_of_two_scaling_is_exact_d256_forward():
    inp = base_inputs(1, 2, 500, 256, seed=44)
    o0, l0, r0, _ = run_path(inp, True, 1 / 16, d256=True)
    o1, l1, r1, _ = run_path({**inp, "v": scaled(inp["v"], 17)}, True, 1 / 16, d256=True)
    assert torch.equal(o1, scaled(o0, 17)) and torch.equal(l1, l0) and torch.equal(r1, scaled(r0, 17))


# ------------------------------------------------------------------ large and small magnitudes against the oracle
def assert_fwd_scaled(o, lse, O, L, f, tag):
    err = np.abs(f64(o) - O)
    assert err.max() <= TOL_O_MAX * f, f"{tag}: O max-abs {err.max():.3e} > {TOL_O_MAX * f:.3e}"
    assert err.mean() <= TOL_O_MEAN * f, f"{tag}: O mean-abs {err.mean():.3e}"
    assert np.abs(f64(lse) - L).max() <= TOL_LSE, f"{tag}: LSE"


def assert_grads_scaled(got, want, fs, tag):
    for name, g, r, f in zip(("dQ", "dK", "dV"), got, want, fs):
        err = np.abs(f64(g) - r).max()
        assert err <= TOL_GRAD * f, f"{tag}: {name} max-abs {err:.3e} > {TOL_GRAD * f:.3e}"
        assert np.isfinite(f64(g)).all(), f"{tag}: {name} not finite"


# (fq, fk, fv, fdo, scale factor): inputs multiplied in fp32 before the bf16 cast
MAGNITUDES = {
    "|V| ~ 1e5": (1.0, 1.0, 1e5, 1.0, 1.0),
    "|Q|, |K| ~ 1e5, small scale": (1e5, 1e5, 1.0, 1.0, 1e-10),
    "dO ~ 1e4": (1.0, 1.0, 1.0, 1e4, 1.0),
    "dO ~ 1e-6": (1.0, 1.0, 1.0, 1e-6, 1.0),
    "V ~ 1e-7, dO ~ 3e3": (1.0, 1.0, 1e-7, 3e3, 1.0),
}


def magnitude_inputs(fq, fk, fv, fdo, B, H, N, d, seed, spiky):
    f = inputs.make_qkv(B, H, N, d, dtype=torch.float32, seed=seed, spiky_frac=spiky)
    out = {n: (t * c).to(torch.bfloat16).cuda() for (n, t), c in zip(f.items(), (fq, fk, fv, fdo))}
    return out


@pytest.mark.parametrize("name", list(MAGNITUDES))
def test_magnitudes_against_the_oracle(name):
    fq, fk, fv, fdo, fs = MAGNITUDES[name]
    B, H, N, d, causal = 1, 2, 1024, 128, True
    inp = magnitude_inputs(fq, fk, fv, fdo, B, H, N, d, seed=123, spiky=0.01)
    q, k, v, do = (inp[n] for n in ("q", "k", "v", "do"))
    scale = fs / math.sqrt(d)
    O, L = oracle.attention_forward(q, k, v, scale, causal)
    ref = oracle.attention_backward(q, k, v, do, scale, causal)
    # the exact attention scales: O with V; dV with dO; dQ and dK with dO V and with scale times
    # K (resp. Q) -- the factors the parity tolerances scale by
    fo, fdv = fv, fdo
    fdq, fdk = fdo * fv * fs * fk, fdo * fv * fs * fq
    # the benchmarked path: V pass + persistent forward, backward with the residual
    o, lse, res = api.fa_fwd_ws(q, k, v, causal=causal, scale=scale, save_residual=True)
    grads = api.fa_bwd_gqa(q, k, v, o, do, lse, causal=causal, scale=scale, o_resid=res)
    torch.cuda.synchronize()
    assert api.fa_last_device_status() == api.FA_OK
    assert_fwd_scaled(o, lse, O, L, fo, f"{name} fa_fwd_ws")
    assert_grads_scaled(grads, ref, (fdq, fdk, fdv), f"{name} fa_bwd_gqa")
    # the workspace-less forward: V tiles are scaled on chip, down only, so V elements below
    # 2^-14 keep fp16's subnormal grid (absolute error <= 2^-25 each, <= 2^-25 in O)
    o2, lse2 = api.fa_fwd(q, k, v, causal=causal, scale=scale)
    torch.cuda.synchronize()
    assert api.fa_last_device_status() == api.FA_OK
    if fo >= 1.0:
        assert_fwd_scaled(o2, lse2, O, L, fo, f"{name} fa_fwd")
    else:
        err = np.abs(f64(o2) - O).max()
        assert err <= TOL_O_MAX * fo + 2.0 ** -25, f"{name} fa_fwd: O max-abs {err:.3e}"
        assert np.abs(f64(lse2) - L).max() <= TOL_LSE


@pytest.mark.parametrize("fv", [1e8, 3e8])
def test_on_chip_forward_scales_large_v_tiles(fv):
    # largest |v| ~ 5e8 and ~1.5e9 (below the 2^31 limit): tiles scaled by 2^-14 and 2^-15, so
    # the running maximum may lag the true one by 1 and 0 only
    inp = magnitude_inputs(1.0, 1.0, fv, 1.0, 1, 2, 700, 64, seed=7, spiky=0.0)
    q, k, v = inp["q"], inp["k"], inp["v"]
    O, L = oracle.attention_forward(q, k, v, 0.125, False)
    o, lse = api.fa_fwd(q, k, v, causal=False, scale=0.125)
    torch.cuda.synchronize()
    assert api.fa_last_device_status() == api.FA_OK
    assert_fwd_scaled(o, lse, O, L, fv, f"on-chip |V| ~ {fv:g}")


# ------------------------------------------------------------------ what no scaling can handle
def test_non_finite_and_overflowing_inputs_are_reported():
    inp = inputs.make_qkv(1, 2, 300, 128, seed=5, device="cuda")
    q, k, v, do = (inp[n] for n in ("q", "k", "v", "do"))
    nan_v = v.clone()
    nan_v[0, 1, 17, 3] = float("nan")
    api.fa_fwd_ws(q, k, nan_v, causal=True)
    assert api.fa_last_device_status() == api.FA_ERR_RANGE
    assert api.fa_last_device_status() == api.FA_OK  # cleared by the read
    inf_q = q.clone()
    inf_q[0, 0, 5, 0] = float("inf")
    api.fa_fwd(inf_q, k, v, causal=True)
    assert api.fa_last_device_status() == api.FA_ERR_RANGE
    # scores beyond fp32: |Q| = |K| = 2^70, even with a scale that would make them moderate
    big = 2.0 ** 70
    api.fa_fwd((q.float() * big).bfloat16(), (k.float() * big).bfloat16(), v, causal=True, scale=2.0 ** -140)
    assert api.fa_last_device_status() == api.FA_ERR_RANGE
    # V beyond what a per-tile copy 2^-15 holds (the workspace forward scales it per tensor)
    huge_v = (v.float() * 2.0 ** 32).bfloat16()
    api.fa_fwd(q, k, huge_v, causal=True)
    assert api.fa_last_device_status() == api.FA_ERR_RANGE
    o, lse = api.fa_fwd_ws(q, k, huge_v, causal=True)
    torch.cuda.synchronize()
    assert api.fa_last_device_status() == api.FA_OK
    O, L = oracle.attention_forward(q, k, huge_v, 1 / math.sqrt(128), True)
    assert_fwd_scaled(o, lse, O, L, 2.0 ** 32, "fa_fwd_ws |V| ~ 2^32")
    # a non-finite dO in the backward
    o, lse = api.fa_fwd(q, k, v, causal=True)
    nan_do = do.clone()
    nan_do[0, 0, 0, 0] = float("nan")
    api.fa_bwd(q, k, v, o, nan_do, lse, causal=True)
    assert api.fa_last_device_status() == api.FA_ERR_RANGE
    assert api.fa_last_device_status() == api.FA_OK


# ------------------------------------------------------------------ the FMA-pipe exponential
def test_fma_pipe_exp2_error():
    # every softmax kernel evaluates part of its exponentials with this polynomial; its stated
    # relative error bound is 7.5e-5 over the arguments the kernels produce, [-125.99, 8]
    # (an fp32 emulation of its steps peaks at 7.48e-5 there)
    grid = np.concatenate([np.linspace(-125.99, 8.0, 1 << 21), np.arange(-125, 9, dtype=np.float64),
                           np.arange(-125, 8, dtype=np.float64) + 0.5,
                           np.random.default_rng(0).uniform(-125.99, 8.0, 1 << 18)]).astype(np.float32)
    x = torch.from_numpy(grid).cuda()
    y = api.fa_selftest_exp2(x)
    torch.cuda.synchronize()
    want = np.exp2(grid.astype(np.float64))
    rel = np.abs(y.double().cpu().numpy() - want) / want
    assert rel.max() <= 7.5e-5, f"max relative error {rel.max():.3e}"
    # down to the clamp at -126 the results reach fp32's denormals (1.5e-4 there), and below it
    # every argument gives 2^-126; all of these round to 0 in fp16
    edge = torch.linspace(-126.0, -125.99, 4097, device="cuda")
    ye = api.fa_selftest_exp2(edge).double().cpu().numpy()
    we = np.exp2(edge.double().cpu().numpy())
    assert (np.abs(ye - we) / we).max() <= 1.5e-4
    low = torch.tensor([-126.5, -200.0, float("-inf")], device="cuda")
    got = api.fa_selftest_exp2(low).double().cpu().numpy()
    assert np.all(np.abs(got / 2.0 ** -126 - 1.0) <= 1.5e-4)
    # NaN passes the clamp and comes out NaN or huge (>= 1e38), never as a plausible probability
    nan_out = api.fa_selftest_exp2(torch.tensor([float("nan")], device="cuda")).item()
    assert not (nan_out < 1e38)
