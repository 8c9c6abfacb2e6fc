"""GPU parity: the CUDA path (through the C ABI) against the fp64 oracle.

Tolerances (fp32 accumulation, bf16 inputs): O max-abs 2e-2 and mean-abs 2e-3,
LSE max-abs 1e-3, dQ/dK/dV max-abs 5e-2.  Inputs are the seeded synthetic
workloads of ``exact_io_aware_91_b200.inputs``; the oracle gets the very same
(bf16-rounded) values widened exactly to fp64.
"""

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


def f64(t: torch.Tensor) -> np.ndarray:
    return t.detach().float().cpu().numpy().astype(np.float64)


def assert_fwd(o, lse, O, L, tag=""):
    err = np.abs(f64(o) - O)
    assert err.max() <= TOL_O_MAX, f"{tag} O max-abs {err.max():.3e}"
    assert err.mean() <= TOL_O_MEAN, f"{tag} O mean-abs {err.mean():.3e}"
    lerr = np.abs(f64(lse) - L).max()
    assert lerr <= TOL_LSE, f"{tag} LSE max-abs {lerr:.3e}"


def assert_grads(gpu, ref, tag=""):
    for name, g, r in zip(("dQ", "dK", "dV"), gpu, ref):
        err = np.abs(f64(g) - r).max()
        assert err <= TOL_GRAD, f"{tag} {name} max-abs {err:.3e}"


@pytest.fixture(scope="module", autouse=True)
def _device():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    torch.cuda.set_device(0)
    yield
    assert api.fa_last_device_status() == api.FA_OK


def run_fwd_bwd(w: inputs.Workload | None = None, *, B=1, H=2, N=128, d=128, causal=True, seed=0,
                backward=True, spiky=0.0, check_on_chip=False):
    """The path the benchmark times: fa_fwd_ws (V pass + persistent kernel, with the
    residual) then fa_bwd_gqa with the residual.  check_on_chip: also run the workspace-less
    forward (fa_fwd_gqa, V converted on chip, one CTA per unit) and require the same bits."""
    if w is not None:
        inp = inputs.make_inputs(w, device="cuda")
        d, causal, backward, scale = w.d, w.causal, w.backward, w.scale
    else:
        inp = inputs.make_qkv(B, H, N, d, seed=seed, spiky_frac=spiky, backward=backward, device="cuda")
        scale = 1.0 / np.sqrt(d)
    o, lse, res = api.fa_fwd_ws(inp["q"], inp["k"], inp["v"], causal=causal, scale=scale, save_residual=True)
    out = {"inp": inp, "o": o, "lse": lse, "res": res, "scale": scale, "causal": causal}
    if check_on_chip:
        o2, lse2, res2 = api.fa_fwd_gqa(inp["q"], inp["k"], inp["v"], causal=causal, scale=scale, save_residual=True)
        torch.cuda.synchronize()
        assert torch.equal(o, o2) and torch.equal(lse, lse2) and torch.equal(res, res2), "fa_fwd_ws != fa_fwd_gqa"
        del o2, lse2, res2
    if backward:
        out["grads"] = api.fa_bwd_gqa(inp["q"], inp["k"], inp["v"], o, inp["do"], lse, causal=causal, scale=scale,
                                      o_resid=res)
    torch.cuda.synchronize()
    return out


# ------------------------------------------------------------------ small and ragged shapes
SMALL = [(n, d, c) for n in (1, 63, 127, 128, 129, 255, 257, 300, 1000) for d in (64, 128) for c in (False, True)]


@pytest.mark.parametrize("N,d,causal", SMALL)
def test_small_and_ragged_fwd_bwd(N, d, causal):
    r = run_fwd_bwd(B=1, H=2, N=N, d=d, causal=causal, seed=N * 7 + d + causal)
    q, k, v, do = (r["inp"][n] for n in ("q", "k", "v", "do"))
    O, L = oracle.attention_forward(q, k, v, r["scale"], causal)
    assert_fwd(r["o"], r["lse"], O, L, f"N={N} d={d} causal={causal}")
    ref = oracle.attention_backward(q, k, v, do, r["scale"], causal)
    assert_grads(r["grads"], ref, f"N={N} d={d} causal={causal}")


def test_batched_heads_are_independent():
    r = run_fwd_bwd(B=3, H=5, N=200, d=64, causal=True, seed=5)
    q, k, v, do = (r["inp"][n] for n in ("q", "k", "v", "do"))
    O, L = oracle.attention_forward(q, k, v, r["scale"], True)
    assert_fwd(r["o"], r["lse"], O, L)
    assert_grads(r["grads"], oracle.attention_backward(q, k, v, do, r["scale"], True))


# ------------------------------------------------------------------ grouped-query attention
GQA = [(B, H, Hkv, N, d, c) for (B, H, Hkv) in ((1, 4, 2), (2, 6, 1), (1, 8, 8), (1, 6, 3))
       for N, d in ((300, 128), (257, 64)) for c in (False, True)]


@pytest.mark.parametrize("B,H,Hkv,N,d,causal", GQA)
def test_gqa_fwd_bwd(B, H, Hkv, N, d, causal):
    inp = inputs.make_qkv(B, H, N, d, seed=H * 31 + Hkv * 7 + N + causal, kv_heads=Hkv, device="cuda")
    q, k, v, do = (inp[n] for n in ("q", "k", "v", "do"))
    scale = 1.0 / np.sqrt(d)
    o, lse, res = api.fa_fwd_gqa(q, k, v, causal=causal, scale=scale, save_residual=True)
    grads = api.fa_bwd_gqa(q, k, v, o, do, lse, causal=causal, scale=scale, o_resid=res)
    torch.cuda.synchronize()
    tag = f"B={B} H={H} Hkv={Hkv} N={N} d={d} causal={causal}"
    O, L = oracle.attention_forward_gqa(q, k, v, scale, causal)
    assert_fwd(o, lse, O, L, tag)
    assert_grads(grads, oracle.attention_backward_gqa(q, k, v, do, scale, causal), tag)
    if Hkv == H:  # with H_kv = H and no residual the grouped entry points are fa_fwd / fa_bwd
        o2, lse2 = api.fa_fwd(q, k, v, causal=causal, scale=scale)
        g1 = api.fa_bwd_gqa(q, k, v, o2, do, lse2, causal=causal, scale=scale)
        g2 = api.fa_bwd(q, k, v, o2, do, lse2, causal=causal, scale=scale)
        torch.cuda.synchronize()
        assert torch.equal(o, o2) and torch.equal(lse, lse2)
        for a, b in zip(g1, g2):
            assert torch.equal(a, b)


@pytest.mark.parametrize("B,H,Hkv,N,d,causal", [(1, 2, 2, 300, 128, True), (1, 2, 2, 257, 64, False),
                                                (2, 4, 1, 1000, 128, True), (1, 6, 3, 129, 64, True)])
def test_forward_with_workspace_matches_on_chip_conversion(B, H, Hkv, N, d, causal):
    # fa_fwd_ws (V converted to fp16 by a separate pass) == fa_fwd_gqa (converted on chip), bit for bit
    inp = inputs.make_qkv(B, H, N, d, seed=N + H + Hkv, kv_heads=Hkv, backward=False, device="cuda")
    q, k, v = inp["q"], inp["k"], inp["v"]
    scale = 1.0 / np.sqrt(d)
    o1, l1, r1 = api.fa_fwd_gqa(q, k, v, causal=causal, scale=scale, save_residual=True)
    o2, l2, r2 = api.fa_fwd_ws(q, k, v, causal=causal, scale=scale, save_residual=True)
    torch.cuda.synchronize()
    assert torch.equal(o1, o2) and torch.equal(l1, l2) and torch.equal(r1, r2)
    O, L = oracle.attention_forward_gqa(q, k, v, scale, causal)
    assert_fwd(o2, l2, O, L, f"fa_fwd_ws B={B} H={H} Hkv={Hkv} N={N} d={d} causal={causal}")


# the d = 64 workspace forward (the persistent kernel with the 64-byte rows of one swizzle span):
# several units per head and per CTA, ragged last units, causal, windows, grouped heads and
# 2 % spiky keys, with the residual checked where O's bf16 rounding dominates its error
@pytest.mark.parametrize("B,H,Hkv,N,causal,window", [(2, 4, 2, 2100, True, (-1, -1)),
                                                     (2, 4, 2, 2100, False, (-1, -1)),
                                                     (1, 6, 3, 1500, True, (200, -1)),
                                                     (1, 3, 3, 1300, False, (100, 300)),
                                                     (3, 2, 1, 130, True, (-1, -1)),
                                                     (1, 2, 2, 640, False, (0, 0))])
def test_workspace_forward_d64(B, H, Hkv, N, causal, window):
    d = 64
    inp = inputs.make_qkv(B, H, N, d, seed=N + 13 * H + Hkv + causal, spiky_frac=0.02, kv_heads=Hkv,
                          backward=False, device="cuda")
    q, k, v = inp["q"], inp["k"], inp["v"]
    scale = 1.0 / np.sqrt(d)
    tag = f"d=64 B={B} H={H} Hkv={Hkv} N={N} causal={causal} window={window}"
    o, lse, res = api.fa_attn_fwd(q, k, v, causal=causal, scale=scale, window=window, save_residual=True)
    torch.cuda.synchronize()
    O, L = oracle.attention_forward_gqa(q, k, v, scale, causal, window=window)
    assert_fwd(o, lse, O, L, tag)
    err_bf16 = np.abs(f64(o) - O).max()
    if err_bf16 > 1e-3:  # O's bf16 rounding dominates its error: the residual recovers most of it
        assert np.abs(f64(o) + f64(res) - O).max() < 0.25 * err_bf16, tag
    if window == (-1, -1):  # fa_fwd_ws takes the same path: the same bits
        o2, lse2, r2 = api.fa_fwd_ws(q, k, v, causal=causal, scale=scale, save_residual=True)
        torch.cuda.synchronize()
        assert torch.equal(o, o2) and torch.equal(lse, lse2) and torch.equal(res, r2), tag


WINDOWS = [(True, (0, -1)), (True, (127, -1)), (True, (128, -1)), (True, (300, -1)), (True, (5, 7)),
           (False, (64, 64)), (False, (0, 0)), (False, (-1, 200)), (False, (333, -1))]


@pytest.mark.parametrize("causal,window", WINDOWS)
@pytest.mark.parametrize("N,d,H,Hkv", [(1000, 128, 2, 2), (577, 64, 4, 2)])
def test_sliding_window_fwd_bwd(causal, window, N, d, H, Hkv):
    inp = inputs.make_qkv(1, H, N, d, seed=N + window[0] + 3 * window[1] + causal, kv_heads=Hkv, device="cuda")
    q, k, v, do = (inp[n] for n in ("q", "k", "v", "do"))
    scale = 1.0 / np.sqrt(d)
    o, lse, res = api.fa_attn_fwd(q, k, v, causal=causal, scale=scale, window=window, save_residual=True)
    grads = api.fa_attn_bwd(q, k, v, o, do, lse, causal=causal, scale=scale, window=window, o_resid=res)
    torch.cuda.synchronize()
    tag = f"window={window} causal={causal} N={N} d={d} H={H} Hkv={Hkv}"
    O, L = oracle.attention_forward_gqa(q, k, v, scale, causal, window=window)
    assert_fwd(o, lse, O, L, tag)
    assert_grads(grads, oracle.attention_backward_gqa(q, k, v, do, scale, causal, window=window), tag)


def test_unbounded_window_is_the_plain_path():
    inp = inputs.make_qkv(1, 2, 700, 128, seed=9, device="cuda")
    q, k, v, do = (inp[n] for n in ("q", "k", "v", "do"))
    o1, l1, r1 = api.fa_attn_fwd(q, k, v, causal=True, window=(-1, -1), save_residual=True)
    o2, l2, r2 = api.fa_fwd_ws(q, k, v, causal=True, save_residual=True)
    g1 = api.fa_attn_bwd(q, k, v, o1, do, l1, causal=True, window=(-1, -1), o_resid=r1)
    g2 = api.fa_bwd_gqa(q, k, v, o2, do, l2, causal=True, o_resid=r2)
    torch.cuda.synchronize()
    assert torch.equal(o1, o2) and torch.equal(l1, l2)
    for a, b in zip(g1, g2):
        assert torch.equal(a, b)


def test_gqa_long_spiky_matches_oracle_rows():
    # a long grouped problem with peaked softmax rows: all of dK/dV of one key/value head
    # against the oracle, which materialises N x N per query head
    B, H, Hkv, N, d = 1, 4, 1, 4096, 128
    inp = inputs.make_qkv(B, H, N, d, seed=77, spiky_frac=0.01, kv_heads=Hkv, device="cuda")
    q, k, v, do = (inp[n] for n in ("q", "k", "v", "do"))
    scale = 1.0 / np.sqrt(d)
    o, lse, res = api.fa_fwd_gqa(q, k, v, causal=True, scale=scale, save_residual=True)
    grads = api.fa_bwd_gqa(q, k, v, o, do, lse, causal=True, scale=scale, o_resid=res)
    torch.cuda.synchronize()
    O, L = oracle.attention_forward_gqa(q, k, v, scale, True)
    assert_fwd(o, lse, O, L, "MQA N=4096 spiky")
    assert_grads(grads, oracle.attention_backward_gqa(q, k, v, do, scale, True), "MQA N=4096 spiky")


# ------------------------------------------------------------------ the five workloads
def test_workload1_fp32_forward():
    w = inputs.workload(1)
    inp = inputs.make_inputs(w, device="cuda")
    o, lse = api.fa_fwd_f32(inp["q"], inp["k"], inp["v"], causal=w.causal, scale=w.scale)
    torch.cuda.synchronize()
    O, L = oracle.attention_forward(inp["q"], inp["k"], inp["v"], w.scale, w.causal)
    assert_fwd(o, lse, O, L, "workload 1")
    # fp32 all the way: far inside the bar
    assert np.abs(f64(o) - O).max() < 1e-4


def test_workload2_full():
    w = inputs.workload(2)
    r = run_fwd_bwd(w, check_on_chip=True)
    q, k, v, do = (r["inp"][n] for n in ("q", "k", "v", "do"))
    O, L = oracle.attention_forward(q, k, v, w.scale, w.causal)
    assert_fwd(r["o"], r["lse"], O, L, "workload 2")
    ref = oracle.attention_backward(q, k, v, do, w.scale, w.causal)
    assert_grads(r["grads"], ref, "workload 2")
    # invariants that hold at any size: sum_j dV_j = sum_i dO_i, sum_j dK_j = 0 (per head)
    dq, dk, dv = r["grads"]
    assert np.abs(f64(dv).sum(-2) - f64(do).sum(-2)).max() < 1.0
    assert np.abs(f64(dk).sum(-2)).max() < 1.0


def test_workload3_sampled_heads_and_rows():
    # the benchmark's forward at full size: 2048 work units on one CTA per SM, so every CTA
    # takes many units in turn; bit-equal to the one-CTA-per-unit forward
    w = inputs.workload(3)
    r = run_fwd_bwd(w, check_on_chip=True)
    q, k, v, do = (r["inp"][n] for n in ("q", "k", "v", "do"))
    o, lse = r["o"], r["lse"]
    dq, dk, dv = r["grads"]
    rng = np.random.default_rng(3)
    # every head: 16 sampled query rows (plus tile edges) against the row oracle
    rows = np.unique(np.concatenate([[0, 127, 128, 255, 256, w.N - 1], rng.integers(0, w.N, 10)]))
    for b in range(w.B):
        for h in range(w.H):
            Or, Lr = oracle.attention_forward_rows(q[b, h], k[b, h], v[b, h], w.scale, w.causal, rows)
            assert_fwd(o[b, h, rows], lse[b, h, rows], Or, Lr, f"workload 3 b={b} h={h}")
    # two sampled heads: full forward and backward
    for b, h in [(0, int(rng.integers(w.H))), (1, int(rng.integers(w.H)))]:
        O, L = oracle.attention_forward(q[b, h], k[b, h], v[b, h], w.scale, w.causal)
        assert_fwd(o[b, h], lse[b, h], O, L, f"workload 3 head ({b},{h})")
        ref = oracle.attention_backward(q[b, h], k[b, h], v[b, h], do[b, h], w.scale, w.causal)
        assert_grads((dq[b, h], dk[b, h], dv[b, h]), ref, f"workload 3 head ({b},{h})")


def test_workload4_full_forward():
    w = inputs.workload(4)
    r = run_fwd_bwd(w, check_on_chip=True)
    q, k, v = (r["inp"][n] for n in ("q", "k", "v"))
    O, L = oracle.attention_forward(q, k, v, w.scale, w.causal)
    assert_fwd(r["o"], r["lse"], O, L, "workload 4")


def test_workload5_sampled_rows_and_prefix():
    w = inputs.workload(5)
    r = run_fwd_bwd(w)
    q, k, v, do = (r["inp"][n] for n in ("q", "k", "v", "do"))
    o, lse = r["o"], r["lse"]
    dq_full = r["grads"][0]
    N = w.N
    rng = np.random.default_rng(5)
    fixed = [0, 1, 127, 128, 4095, 4096, 65535, 65536, N - 2, N - 1]
    rows = np.unique(np.concatenate([fixed, rng.integers(0, N, 64 - len(fixed))]))
    h = int(rng.integers(w.H))
    Or, Lr = oracle.attention_forward_rows(q[0, h], k[0, h], v[0, h], w.scale, True, rows)
    assert_fwd(o[0, h, rows], lse[0, h, rows], Or, Lr, "workload 5 rows")
    # backward: the 4096-token prefix problem run on its own ...
    P = 4096
    qp, kp, vp, dop = (t[:, :, :P].contiguous() for t in (q, k, v, do))
    op, lsep, rp = api.fa_fwd_ws(qp, kp, vp, causal=True, scale=w.scale, save_residual=True)
    gp = api.fa_bwd_gqa(qp, kp, vp, op, dop, lsep, causal=True, scale=w.scale, o_resid=rp)
    torch.cuda.synchronize()
    ref = oracle.attention_backward(qp[0], kp[0], vp[0], dop[0], w.scale, True)
    assert_grads((gp[0][0], gp[1][0], gp[2][0]), ref, "workload 5 prefix")
    # ... and dQ of the full run on those rows (causal dQ_i depends only on keys <= i)
    err = np.abs(f64(dq_full[0, :, :P]) - ref[0]).max()
    assert err <= TOL_GRAD, f"workload 5 full-run dQ prefix max-abs {err:.3e}"


# ------------------------------------------------------------------ properties
def test_deterministic():
    a = run_fwd_bwd(B=2, H=3, N=777, d=128, causal=True, seed=11)
    o2, lse2, r2 = api.fa_fwd_ws(a["inp"]["q"], a["inp"]["k"], a["inp"]["v"], causal=True, save_residual=True)
    g2 = api.fa_bwd_gqa(a["inp"]["q"], a["inp"]["k"], a["inp"]["v"], a["o"], a["inp"]["do"], a["lse"], causal=True,
                        o_resid=a["res"])
    torch.cuda.synchronize()
    assert torch.equal(a["o"], o2) and torch.equal(a["lse"], lse2) and torch.equal(a["res"], r2)
    for x, y in zip(a["grads"], g2):
        assert torch.equal(x, y)


def test_library_allocates_nothing():
    inp = inputs.make_qkv(1, 4, 4096, 128, seed=2, device="cuda")
    o = torch.empty_like(inp["q"])
    lse = torch.empty((1, 4, 4096), device="cuda")
    torch.cuda.synchronize()
    free0 = torch.cuda.mem_get_info()[0]
    api.fa_fwd(inp["q"], inp["k"], inp["v"], causal=True, o=o, lse=lse)
    torch.cuda.synchronize()
    assert torch.cuda.mem_get_info()[0] >= free0 - (2 << 20)  # no N x N (or any) device buffer


def test_residual_is_the_rounding_of_o():
    # O + residual is the forward's fp32 O: much closer to the oracle than the bf16 O alone
    inp = inputs.make_qkv(1, 2, 1000, 128, seed=9, device="cuda")
    o, lse, res = api.fa_fwd_gqa(inp["q"], inp["k"], inp["v"], causal=True, save_residual=True)
    torch.cuda.synchronize()
    O, _ = oracle.attention_forward(inp["q"], inp["k"], inp["v"], 1 / np.sqrt(128), True)
    full = f64(o) + f64(res)
    assert np.abs(full - O).max() < 0.25 * np.abs(f64(o) - O).max()
    assert np.abs(f64(res)).max() <= np.abs(f64(o)).max() * 2.0 ** -8


def test_backward_without_residual_on_a_plain_workload():
    # without the residual D uses the bf16 O: still inside the bar on N(0,1) inputs
    inp = inputs.make_qkv(1, 2, 700, 64, seed=10, device="cuda")
    o, lse = api.fa_fwd(inp["q"], inp["k"], inp["v"], causal=False)
    g = api.fa_bwd(inp["q"], inp["k"], inp["v"], o, inp["do"], lse, causal=False)
    torch.cuda.synchronize()
    ref = oracle.attention_backward(inp["q"], inp["k"], inp["v"], inp["do"], 1 / np.sqrt(64), False)
    assert_grads(g, ref, "no residual")


# ------------------------------------------------------------------ the boundary's own signatures
@pytest.mark.parametrize("N,d,causal", [(1, 64, True), (300, 128, True), (1000, 64, False), (257, 128, False)])
def test_exact_signatures_small(N, d, causal):
    # fa_fwd(q,k,v,o,lse,B,H,N,d,scale,causal,stream) and
    # fa_bwd(q,k,v,o,dout,lse,dq,dk,dv,B,H,N,d,scale,causal,workspace,stream) through ctypes
    inp = inputs.make_qkv(2, 3, N, d, seed=N + d + 5 * causal, device="cuda")
    q, k, v, do = (inp[n] for n in ("q", "k", "v", "do"))
    scale = 1.0 / np.sqrt(d)
    o, lse = api.fa_fwd(q, k, v, causal=causal, scale=scale)
    grads = api.fa_bwd(q, k, v, o, do, lse, causal=causal, scale=scale)
    torch.cuda.synchronize()
    tag = f"fa_fwd/fa_bwd N={N} d={d} causal={causal}"
    O, L = oracle.attention_forward(q, k, v, scale, causal)
    assert_fwd(o, lse, O, L, tag)
    assert_grads(grads, oracle.attention_backward(q, k, v, do, scale, causal), tag)


def test_exact_signatures_workload2():
    # the boundary's plain pair (no residual: D from the bf16 O) on workload 2 in full
    w = inputs.workload(2)
    inp = inputs.make_inputs(w, device="cuda")
    q, k, v, do = (inp[n] for n in ("q", "k", "v", "do"))
    o, lse = api.fa_fwd(q, k, v, causal=w.causal, scale=w.scale)
    grads = api.fa_bwd(q, k, v, o, do, lse, causal=w.causal, scale=w.scale)
    torch.cuda.synchronize()
    O, L = oracle.attention_forward(q, k, v, w.scale, w.causal)
    assert_fwd(o, lse, O, L, "fa_fwd workload 2")
    assert_grads(grads, oracle.attention_backward(q, k, v, do, w.scale, w.causal), "fa_bwd workload 2")
