"""GPU parity of the 8-bit forward (``fa_attn_fwd_fp8``) against the fp64 oracle.

The oracle is the exact attention of the dequantized E4M3 inputs (``oracle/fp8.py``).
The kernel rounds the probabilities P to E4M3 before the P V product and divides by the
row sum of P before that rounding, so its output differs from the oracle by at most

    |dO_ic| <= (2^-4 + 4e-4) * sum_j P_ij |V_jc|                     (E4M3, normal range)
               + 2^-10 * max_j P_ij * sum_{j: 0 < P_ij < 2^-6 max_j P_ij} |V_jc|   (subnormal range)
               + 2^-8 |O_ic| + 1e-6                                   (bf16 output, fp32)

with P the exact probabilities: E4M3 keeps 3 mantissa bits (rounding error at most 2^-4
of the value from 2^-6 up, at most 2^-10 absolute below, on the kernel's unnormalised
scale where the largest probability of a row is >= 1; masked keys have P = 0 exactly and no
rounding error); 4e-4 covers the exponential's polynomial / approximate evaluation and the
fp32 sums.  tests/test_fp8_bound.py checks on the CPU that the bound covers an emulation of
that arithmetic (up to 0.8 of it) and that a rounding one bit coarser breaks it.  That bound is checked element by
element.  LSE uses the unrounded probabilities and is held to the bf16 forward's 1e-3.
A case with every probability an exact power of two (representable in E4M3) checks O
to fp32 / bf16 rounding only.
"""

import math

import numpy as np
import pytest
import torch

import oracle
from exact_io_aware_91_b200 import api, inputs

pytestmark = pytest.mark.gpu

TOL_LSE = 1e-3


@pytest.fixture(scope="module", autouse=True)
def _device():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    torch.cuda.set_device(0)
    yield
    assert api.fa_last_device_status() == api.FA_OK


def codes(t: torch.Tensor) -> np.ndarray:
    return t.view(torch.uint8).cpu().numpy()


def probs_rows(q, k, scale, causal, window, rows):
    """Probabilities of the given query rows of one head (fp64), for the error bound only."""
    s = scale * (q[rows] @ k.T)
    n = k.shape[0]
    j = np.arange(n)[None, :]
    i = np.asarray(rows)[:, None]
    vis = np.ones(s.shape, bool)
    if causal:
        vis &= j <= i
    left, right = window
    if left >= 0:
        vis &= j >= i - left
    if right >= 0:
        vis &= j <= i + right
    s = np.where(vis, s, -np.inf)
    p = np.exp(s - s.max(axis=1, keepdims=True))
    return p / p.sum(axis=1, keepdims=True)


def o_bound(p, v, o_ref):
    """Per-element bound of |O_gpu - O_ref| for probability rows p (rows x keys)."""
    av = np.abs(v)
    pmax = p.max(axis=1, keepdims=True)
    small = (p < 2.0**-6 * pmax) & (p > 0)  # visible keys in E4M3's subnormal range
    return ((2.0**-4 + 4e-4) * (p @ av) + 2.0**-10 * pmax * (small.astype(np.float64) @ av)
            + 2.0**-8 * np.abs(o_ref) + 1e-6)


def check_heads(x, o, lse, scale, causal, window, heads, rows=None, tag=""):
    """O and LSE of the given heads (and rows) against the oracle's 8-bit forward; the
    probabilities computed here serve only the per-element bound."""
    H, Hkv = x["q"].shape[1], x["k"].shape[1]
    qc, kc, vc = codes(x["q"]), codes(x["k"]), codes(x["v"])
    ds = (x["q_descale"], x["k_descale"], x["v_descale"])
    o = o.float().cpu().numpy()
    lse = lse.cpu().numpy()
    worst = 0.0
    for b, h in heads:
        g = h // (H // Hkv)
        r = np.arange(qc.shape[2]) if rows is None else np.asarray(rows)
        o_ref, lse_ref = oracle.attention_forward_fp8_rows(qc[b, h], kc[b, g], vc[b, g], *ds, scale, causal, r,
                                                           window)
        qh = x["q_descale"] * oracle.e4m3_decode(qc[b, h])  # dequantized, one head at a time (bound only)
        kh = x["k_descale"] * oracle.e4m3_decode(kc[b, g])
        vh = x["v_descale"] * oracle.e4m3_decode(vc[b, g])
        p = probs_rows(qh, kh, scale, causal, window, r)
        err = np.abs(o[b, h][r] - o_ref)
        bound = o_bound(p, vh, o_ref)
        assert np.all(err <= bound), f"{tag} (b={b}, h={h}) O error {err.max():.3e} above its bound"
        lerr = np.abs(lse[b, h][r] - lse_ref).max()
        assert lerr <= TOL_LSE, f"{tag} (b={b}, h={h}) LSE max-abs {lerr:.3e}"
        worst = max(worst, float((err / bound).max()))
    return worst


CASES = [  # B, H, H_kv, N, causal, window, spiky
    (1, 2, 2, 256, True, (-1, -1), 0.0),
    (2, 4, 4, 1000, False, (-1, -1), 0.0),
    (1, 4, 2, 1536, True, (-1, -1), 0.0),
    (1, 4, 1, 777, True, (-1, -1), 0.0),
    (1, 2, 2, 1200, True, (200, -1), 0.0),
    (1, 2, 2, 900, False, (100, 50), 0.0),
    (1, 2, 2, 4096, True, (-1, -1), 0.01),
    (1, 2, 2, 129, False, (-1, -1), 0.0),
]


# head dim 64: rows of 64 bytes (the 64-byte swizzle), O of 64 TMEM columns per tile
CASES_D64 = [
    (1, 2, 2, 256, True, (-1, -1), 0.0),
    (2, 4, 4, 1000, False, (-1, -1), 0.0),
    (1, 4, 1, 777, True, (-1, -1), 0.0),
    (1, 2, 2, 900, False, (100, 50), 0.0),
    (1, 2, 2, 2048, True, (-1, -1), 0.01),
    (1, 2, 2, 1, False, (-1, -1), 0.0),
]


@pytest.mark.parametrize("d,B,H,Hkv,N,causal,window,spiky",
                         [(128,) + c for c in CASES] + [(64,) + c for c in CASES_D64])
def test_fp8_forward_within_its_rounding_bound(d, B, H, Hkv, N, causal, window, spiky):
    x = inputs.make_qkv_fp8(B, H, N, d, kv_heads=Hkv, spiky_frac=spiky, seed=11 + N + d, device="cuda")
    scale = 1.0 / math.sqrt(d)
    o, lse = api.fa_attn_fwd_fp8(x["q"], x["k"], x["v"], x["q_descale"], x["k_descale"], x["v_descale"],
                                 causal=causal, scale=scale, window=window)
    torch.cuda.synchronize()
    heads = [(b, h) for b in range(B) for h in range(H)]
    check_heads(x, o, lse, scale, causal, window, heads, tag=f"N={N}")


@pytest.mark.parametrize("d", [128, 64])
def test_fp8_exact_probabilities(d):
    # scale = ln 2 and integer scores in [-4, 4]: every probability the kernel forms is a
    # power of two in [2^-8, 2^8], exact in E4M3, so only fp32 sums and the bf16 output round
    B, H, N = 1, 2, 2048
    g = torch.Generator().manual_seed(5)
    q = torch.zeros(B, H, N, d)
    q[..., 0] = 1.0
    k = torch.randn(B, H, N, d, generator=g)
    k[..., 0] = torch.randint(-4, 5, (B, H, N), generator=g).float()
    v = torch.randn(B, H, N, d, generator=g)
    x = {"q": q.to(torch.float8_e4m3fn).cuda(), "k": k.to(torch.float8_e4m3fn).cuda(),
         "v": v.to(torch.float8_e4m3fn).cuda()}
    scale = float(np.float32(math.log(2.0)))
    for causal in (True, False):
        o, lse = api.fa_attn_fwd_fp8(x["q"], x["k"], x["v"], 1.0, 1.0, 0.5, causal=causal, scale=scale)
        torch.cuda.synchronize()
        O, L = oracle.attention_forward_fp8(codes(x["q"]), codes(x["k"]), codes(x["v"]), 1.0, 1.0, 0.5, scale,
                                            causal)
        got = o.float().cpu().numpy()
        err = np.abs(got - O)
        vmax = 0.5 * np.abs(oracle.e4m3_decode(codes(x["v"]))).max()
        assert np.all(err <= 2.0**-8 * np.abs(O) + 2e-4 * vmax), f"causal={causal} max err {err.max():.3e}"
        assert np.abs(lse.cpu().numpy() - L).max() <= TOL_LSE


def test_fp8_workload3_shape_sampled_rows():
    # the bf16 bench shape (B=2, H=32, N=8192, d=128, causal, 1 % of keys x8) in E4M3
    w = inputs.workload(3)
    x = inputs.make_qkv_fp8(w.B, w.H, w.N, w.d, spiky_frac=w.spiky_frac, seed=w.seed, device="cuda")
    o, lse = api.fa_attn_fwd_fp8(x["q"], x["k"], x["v"], x["q_descale"], x["k_descale"], x["v_descale"],
                                 causal=True, scale=w.scale)
    torch.cuda.synchronize()
    rows = sorted({0, 1, 127, 128, 255, 256, 4095, 4096, w.N - 2, w.N - 1} |
                  set(np.random.default_rng(3).integers(0, w.N, 22).tolist()))
    check_heads(x, o, lse, w.scale, True, (-1, -1), [(0, 0), (1, 31), (0, 17)], rows=rows, tag="workload 3")


def test_fp8_workload4_shape_sampled_heads():
    # workload 4's shape (B=64, H=16, N=512, d=64, no mask, U(-1, 1)) in E4M3: 512 work units,
    # several per CTA; every row of a sample of heads
    w = inputs.workload(4)
    x = inputs.make_qkv_fp8(w.B, w.H, w.N, w.d, dist=w.dist, seed=w.seed, device="cuda")
    o, lse = api.fa_attn_fwd_fp8(x["q"], x["k"], x["v"], x["q_descale"], x["k_descale"], x["v_descale"],
                                 causal=False, scale=w.scale)
    torch.cuda.synchronize()
    heads = [(0, 0), (17, 5), (40, 9), (63, 15)]
    check_heads(x, o, lse, w.scale, False, (-1, -1), heads, tag="workload 4")


def test_fp8_argument_checks():
    x = inputs.make_qkv_fp8(1, 2, 64, 128, seed=1, device="cuda")
    with pytest.raises(api.FAError) as e:
        api.fa_attn_fwd_fp8(x["q"], x["k"], x["v"], 0.0, 1.0, 1.0)
    assert e.value.status == api.FA_ERR_INVALID_ARG
    with pytest.raises(api.FAError) as e:
        api.fa_attn_fwd_fp8(x["q"], x["k"], x["v"], 1.0, float("nan"), 1.0)
    assert e.value.status == api.FA_ERR_INVALID_ARG
    y = inputs.make_qkv_fp8(1, 2, 64, 256, seed=1, device="cuda")
    with pytest.raises(api.FAError) as e:
        api.fa_attn_fwd_fp8(y["q"], y["k"], y["v"], 1.0, 1.0, 1.0)
    assert e.value.status == api.FA_ERR_UNSUPPORTED
    z = inputs.make_qkv_fp8(1, 2, 0, 128, seed=1, device="cuda")
    api.fa_attn_fwd_fp8(z["q"], z["k"], z["v"], 1.0, 1.0, 1.0)  # empty problem: nothing to do


def test_fp8_deterministic():
    x = inputs.make_qkv_fp8(1, 4, 1000, 128, seed=2, device="cuda")
    a = api.fa_attn_fwd_fp8(x["q"], x["k"], x["v"], x["q_descale"], x["k_descale"], x["v_descale"], causal=True)
    b = api.fa_attn_fwd_fp8(x["q"], x["k"], x["v"], x["q_descale"], x["k_descale"], x["v_descale"], causal=True)
    torch.cuda.synchronize()
    assert torch.equal(a[0], b[0]) and torch.equal(a[1], b[1])
