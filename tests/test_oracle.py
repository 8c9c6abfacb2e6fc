"""Pins of the fp64 oracle against what the pages and the mathematics fix.

None of these checks retypes the oracle's own formula: they use closed forms,
invariants, a hand-derived worked example, finite differences, an independent
loop restatement, a library special case and the blockwise online-softmax
recurrence the pages describe.  A final test plants mistakes in the oracle (on
the CPU) and checks that the pins catch each one.
"""

import json
import math
import os

import numpy as np
import pytest

import oracle
import oracle.attention as oa
from oracle import (
    attention_backward,
    attention_backward_gqa,
    attention_forward_gqa,
    attention_forward,
    attention_forward_rows,
    attention_probs,
    loop_attention_backward,
    loop_attention_forward,
    online_softmax_forward,
)

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "worked_examples.json")


def randn(shape, seed):
    return np.random.default_rng(seed).standard_normal(shape)


# ---------------------------------------------------------------- softmax normalisation
@pytest.mark.parametrize("causal", [False, True])
def test_probability_rows_sum_to_one(causal):
    q, k = randn((2, 3, 37, 16), 1), randn((2, 3, 37, 16), 2)
    P, _ = attention_probs(q, k, 0.25, causal)
    np.testing.assert_allclose(P.sum(-1), 1.0, atol=1e-12)
    assert np.all(P >= 0)
    if causal:
        upper = np.triu(np.ones((37, 37), dtype=bool), 1)
        assert np.all(P[..., upper] == 0.0)


# ---------------------------------------------------------------- O formula
@pytest.mark.parametrize("causal", [False, True])
def test_uniform_values_return_that_value(causal):
    q, k = randn((1, 2, 29, 8), 3), randn((1, 2, 29, 8), 4)
    row = randn((8,), 5)
    v = np.broadcast_to(row, (1, 2, 29, 8)).copy()
    O, _ = attention_forward(q, k, v, 1 / math.sqrt(8), causal)
    np.testing.assert_allclose(O, v, atol=1e-13)


@pytest.mark.parametrize("causal", [False, True])
def test_single_dominant_logit_returns_its_value_row(causal):
    n, d = 24, 6
    jstar = 0 if causal else 17  # under causal every row must see the dominant key
    q = np.zeros((n, d))
    q[:, 0] = 1.0
    k = 0.01 * randn((n, d), 6)
    k[:, 0] = 0.0
    k[jstar, 0] = 50.0
    v = randn((n, d), 7)
    O, L = attention_forward(q, k, v, 1.0, causal)
    np.testing.assert_allclose(O, np.broadcast_to(v[jstar], O.shape), atol=n * math.exp(-49))
    np.testing.assert_allclose(L, 50.0, atol=n * math.exp(-49))


def test_noncausal_output_invariant_under_key_permutation():
    q, k, v = randn((3, 41, 16), 8), randn((3, 41, 16), 9), randn((3, 41, 16), 10)
    perm = np.random.default_rng(11).permutation(41)
    O1, L1 = attention_forward(q, k, v, 0.3, False)
    O2, L2 = attention_forward(q, k[:, perm], v[:, perm], 0.3, False)
    np.testing.assert_allclose(O1, O2, atol=1e-12)
    np.testing.assert_allclose(L1, L2, atol=1e-12)


# ---------------------------------------------------------------- closed forms
@pytest.mark.parametrize("causal", [False, True])
def test_single_token(causal):
    q, k, v = randn((1, 5), 12), randn((1, 5), 13), randn((1, 5), 14)
    O, L = attention_forward(q, k, v, 0.7, causal)
    np.testing.assert_allclose(O, v, atol=1e-15)
    np.testing.assert_allclose(L, [0.7 * float(np.dot(q[0], k[0]))], atol=1e-14)


def test_causal_first_row_is_first_value():
    q, k, v = randn((19, 4), 15), randn((19, 4), 16), randn((19, 4), 17)
    O, L = attention_forward(q, k, v, 0.5, True)
    np.testing.assert_allclose(O[0], v[0], atol=1e-15)
    np.testing.assert_allclose(L[0], 0.5 * float(np.dot(q[0], k[0])), atol=1e-14)


@pytest.mark.parametrize("causal", [False, True])
def test_zero_queries_average_the_visible_values(causal):
    n, d = 33, 7
    q = np.zeros((n, d))
    k, v = randn((n, d), 18), randn((n, d), 19)
    O, L = attention_forward(q, k, v, 1.0, causal)
    if causal:
        expect = np.cumsum(v, axis=0) / np.arange(1, n + 1)[:, None]
        lse = np.log(np.arange(1, n + 1))
    else:
        expect = np.broadcast_to(v.mean(0), (n, d))
        lse = np.full(n, math.log(n))
    np.testing.assert_allclose(O, expect, atol=1e-13)
    np.testing.assert_allclose(L, lse, atol=1e-13)


def test_golden_worked_examples():
    cases = json.load(open(GOLDEN))["cases"]
    for c in cases:
        q, k, v = (np.array(c[n], dtype=np.float64) for n in ("q", "k", "v"))
        O, L = attention_forward(q, k, v, c["scale"], c["causal"])
        np.testing.assert_allclose(O, c["o"], atol=1e-14, err_msg=c["name"])
        np.testing.assert_allclose(L, c["lse"], atol=1e-14, err_msg=c["name"])
        if "do" in c:
            do = np.array(c["do"])
            dq, dk, dv, D = attention_backward(q, k, v, do, c["scale"], c["causal"], return_delta=True)
            np.testing.assert_allclose(D, c["delta"], atol=1e-14, err_msg=c["name"])
            np.testing.assert_allclose(dq, c["dq"], atol=1e-14, err_msg=c["name"])
            np.testing.assert_allclose(dk, c["dk"], atol=1e-14, err_msg=c["name"])
            np.testing.assert_allclose(dv, c["dv"], atol=1e-14, err_msg=c["name"])


# ---------------------------------------------------------------- online recurrence
@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("bq,bk", [(1, 1), (5, 3), (16, 16), (7, 40), (64, 13)])
def test_online_softmax_recurrence_equals_definition(causal, bq, bk):
    n, d = 37, 12
    q, k, v = 2 * randn((n, d), 20), 2 * randn((n, d), 21), randn((n, d), 22)
    O1, L1 = attention_forward(q, k, v, 0.4, causal)
    O2, L2 = online_softmax_forward(q, k, v, 0.4, causal, bq, bk)
    np.testing.assert_allclose(O2, O1, atol=1e-12)
    np.testing.assert_allclose(L2, L1, atol=1e-12)


# ---------------------------------------------------------------- loop restatement
@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("n,d", [(1, 3), (5, 4), (16, 8)])
def test_loop_restatement_matches_numpy_oracle(causal, n, d):
    q, k, v, do = (randn((n, d), s) for s in (23, 24, 25, 26))
    O1, L1 = attention_forward(q, k, v, 0.6, causal)
    O2, L2 = loop_attention_forward(q, k, v, 0.6, causal)
    np.testing.assert_allclose(O1, O2, atol=1e-13)
    np.testing.assert_allclose(L1, L2, atol=1e-13)
    g1 = attention_backward(q, k, v, do, 0.6, causal)
    g2 = loop_attention_backward(q, k, v, do, 0.6, causal)
    for a, b in zip(g1, g2):
        np.testing.assert_allclose(a, b, atol=1e-12)


def test_row_sampler_matches_full_forward():
    # the full forward with a window is pinned by its own tests (SDPA with the explicit mask,
    # closed forms); the row sampler must agree with it row by row
    q, k, v = randn((50, 8), 27), randn((50, 8), 28), randn((50, 8), 29)
    rows = [0, 1, 17, 48, 49]
    for causal in (False, True):
        for window in ((-1, -1), (5, -1), (3, 4), (0, 0), (-1, 2)):
            O, L = attention_forward(q, k, v, 0.35, causal, window=window)
            Or, Lr = attention_forward_rows(q, k, v, 0.35, causal, rows, window=window)
            np.testing.assert_allclose(Or, O[rows], atol=1e-14)
            np.testing.assert_allclose(Lr, L[rows], atol=1e-14)


def test_row_dq_matches_full_backward_and_finite_differences():
    # against the full backward (itself pinned by finite differences below) and, for one row,
    # directly against central finite differences of sum(O * dO) in that row's query
    q, k, v, do = randn((40, 8), 31), randn((40, 8), 32), randn((40, 8), 33), randn((40, 8), 34)
    rows = [0, 1, 13, 38, 39]
    for causal in (False, True):
        dq, _, _ = attention_backward(q, k, v, do, 0.4, causal)
        np.testing.assert_allclose(oracle.attention_backward_dq_rows(q, k, v, do, 0.4, causal, rows), dq[rows],
                                   atol=1e-13)
        i, h = 13, 1e-6
        g = oracle.attention_backward_dq_rows(q, k, v, do, 0.4, causal, [i])[0]
        num = np.empty(8)
        for c in range(8):
            qp, qm = q.copy(), q.copy()
            qp[i, c] += h
            qm[i, c] -= h
            num[c] = (_loss(qp, k, v, do, 0.4, causal) - _loss(qm, k, v, do, 0.4, causal)) / (2 * h)
        assert np.max(np.abs(num - g)) <= 1e-6 * max(1.0, np.max(np.abs(g)))


# ---------------------------------------------------------------- backward
def _loss(q, k, v, do, scale, causal):
    O, _ = attention_forward(q, k, v, scale, causal)
    return float(np.sum(O * do))


@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("n,d", [(1, 2), (5, 3), (8, 4)])
def test_backward_matches_central_finite_differences(causal, n, d):
    q, k, v, do = (randn((n, d), s) for s in (30, 31, 32, 33))
    scale = 0.8
    grads = attention_backward(q, k, v, do, scale, causal)
    h = 1e-6
    for which, g in zip(range(3), grads):
        args = [q, k, v]
        num = np.zeros_like(args[which])
        for idx in np.ndindex(args[which].shape):
            plus = [a.copy() for a in args]
            minus = [a.copy() for a in args]
            plus[which][idx] += h
            minus[which][idx] -= h
            num[idx] = (_loss(*plus, do, scale, causal) - _loss(*minus, do, scale, causal)) / (2 * h)
        err = np.max(np.abs(num - g)) / max(1.0, np.max(np.abs(g)))
        assert err <= 1e-6, (which, err)


@pytest.mark.parametrize("causal", [False, True])
def test_backward_invariants(causal):
    q, k, v, do = (randn((2, 45, 10), s) for s in (34, 35, 36, 37))
    dq, dk, dv, D = attention_backward(q, k, v, do, 0.3, causal, return_delta=True)
    # sum_j dV_j = sum_i dO_i  (rows of P sum to one)
    np.testing.assert_allclose(dv.sum(-2), do.sum(-2), atol=1e-11)
    # sum_j dK_j = 0  (rows of dS sum to zero)
    np.testing.assert_allclose(dk.sum(-2), 0.0, atol=1e-11)
    # D_i = sum_j P_ij dP_ij equals rowsum(dO * O)
    O, _ = attention_forward(q, k, v, 0.3, causal)
    np.testing.assert_allclose(D, np.sum(do * O, axis=-1), atol=1e-12)


# ---------------------------------------------------------------- library special case
@pytest.mark.parametrize("causal", [False, True])
def test_agrees_with_torch_sdpa_math_path_fp64(causal):
    torch = pytest.importorskip("torch")
    import torch.nn.functional as F

    q, k, v, do = (randn((2, 3, 31, 16), s) for s in (38, 39, 40, 41))
    tq, tk, tv = (torch.tensor(x, requires_grad=True) for x in (q, k, v))
    out = F.scaled_dot_product_attention(tq, tk, tv, is_causal=causal, scale=0.25)
    out.backward(torch.tensor(do))
    O, _ = attention_forward(q, k, v, 0.25, causal)
    np.testing.assert_allclose(O, out.detach().numpy(), atol=1e-10)
    dq, dk, dv = attention_backward(q, k, v, do, 0.25, causal)
    np.testing.assert_allclose(dq, tq.grad.numpy(), atol=1e-10)
    np.testing.assert_allclose(dk, tk.grad.numpy(), atol=1e-10)
    np.testing.assert_allclose(dv, tv.grad.numpy(), atol=1e-10)


# ---------------------------------------------------------------- planted mistakes
def _pins_pass() -> bool:
    """A compact run of the pins above; False as soon as one fails."""
    checks = [
        test_golden_worked_examples,
        lambda: test_causal_first_row_is_first_value(),
        lambda: test_zero_queries_average_the_visible_values(True),
        lambda: test_zero_queries_average_the_visible_values(False),
        lambda: test_single_token(False),
        lambda: test_online_softmax_recurrence_equals_definition(True, 5, 3),
        lambda: test_probability_rows_sum_to_one(True),
    ]
    for c in checks:
        try:
            with np.errstate(all="ignore"):
                c()
        except AssertionError:
            return False
    return True


def _bad_scores_no_scale(q2, k2, scale, causal):
    return _orig_scores(q2, k2, 1.0, causal)


def _bad_scores_strict_mask(q2, k2, scale, causal):
    s = scale * (q2 @ k2.T)
    if causal:
        i = np.arange(s.shape[0])[:, None]
        j = np.arange(s.shape[1])[None, :]
        s = np.where(j >= i, -np.inf, s)  # hides the diagonal too
    return s


def _bad_scores_mask_transposed(q2, k2, scale, causal):
    s = scale * (q2 @ k2.T)
    if causal:
        i = np.arange(s.shape[0])[:, None]
        j = np.arange(s.shape[1])[None, :]
        s = np.where(j < i, -np.inf, s)
    return s


def _bad_scores_transposed_operands(q2, k2, scale, causal):
    return _orig_scores(k2, q2, scale, causal)


def _bad_lse_log2(s):
    m = np.max(s, axis=-1, keepdims=True)
    return (m + np.log2(np.sum(np.exp(s - m), axis=-1, keepdims=True)))[..., 0]


def _bad_lse_max_only(s):
    return np.max(s, axis=-1)


_orig_scores = oa._scores


@pytest.mark.parametrize("name,attr,bad", [
    ("dropped scale", "_scores", _bad_scores_no_scale),
    ("diagonal masked", "_scores", _bad_scores_strict_mask),
    ("mask transposed", "_scores", _bad_scores_mask_transposed),
    ("Q and K swapped", "_scores", _bad_scores_transposed_operands),
    ("log2 in LSE", "_lse_rows", _bad_lse_log2),
    ("LSE without the sum", "_lse_rows", _bad_lse_max_only),
])
def test_pins_catch_planted_mistakes(monkeypatch, name, attr, bad):
    assert _pins_pass(), "pins must pass on the unmodified oracle"
    monkeypatch.setattr(oa, attr, bad)
    assert not _pins_pass(), f"planted mistake not caught: {name}"


# ---------------------------------------------------------------- grouped-query attention
def _cumulative_mean(v):
    """Row i: mean of rows 0..i (the closed form of causal attention with zero queries)."""
    return np.cumsum(v, axis=-2) / np.arange(1, v.shape[-2] + 1)[:, None]


@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("H,Hkv", [(4, 2), (6, 1), (6, 3)])
def test_gqa_zero_queries_average_their_group_values(causal, H, Hkv):
    # Q = 0: every score is 0, so query head h averages the visible rows of V[h // (H / Hkv)]
    B, N, d = 2, 13, 5
    q = np.zeros((B, H, N, d))
    k, v = randn((B, Hkv, N, d), 60), randn((B, Hkv, N, d), 61)
    O, L = attention_forward_gqa(q, k, v, 0.5, causal)
    for h in range(H):
        g = h // (H // Hkv)
        want = _cumulative_mean(v[:, g]) if causal else np.broadcast_to(v[:, g].mean(-2, keepdims=True), (B, N, d))
        np.testing.assert_allclose(O[:, h], want, atol=1e-13)
        want_l = np.log(np.arange(1, N + 1)) if causal else np.full(N, math.log(N))
        np.testing.assert_allclose(L[:, h], np.broadcast_to(want_l, (B, N)), atol=1e-13)


@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("H,Hkv", [(4, 1), (4, 2), (6, 3), (3, 3)])
def test_gqa_agrees_with_torch_sdpa_enable_gqa_fp64(causal, H, Hkv):
    torch = pytest.importorskip("torch")
    import torch.nn.functional as F

    q, do = randn((2, H, 23, 8), 62), randn((2, H, 23, 8), 63)
    k, v = randn((2, Hkv, 23, 8), 64), randn((2, Hkv, 23, 8), 65)
    tq, tk, tv = (torch.tensor(x, requires_grad=True) for x in (q, k, v))
    out = F.scaled_dot_product_attention(tq, tk, tv, is_causal=causal, scale=0.3, enable_gqa=True)
    out.backward(torch.tensor(do))
    O, _ = attention_forward_gqa(q, k, v, 0.3, causal)
    np.testing.assert_allclose(O, out.detach().numpy(), atol=1e-10)
    dq, dk, dv = attention_backward_gqa(q, k, v, do, 0.3, causal)
    np.testing.assert_allclose(dq, tq.grad.numpy(), atol=1e-10)
    np.testing.assert_allclose(dk, tk.grad.numpy(), atol=1e-10)
    np.testing.assert_allclose(dv, tv.grad.numpy(), atol=1e-10)


def _gqa_loss(q, k, v, do, scale, causal):
    O, _ = attention_forward_gqa(q, k, v, scale, causal)
    return float(np.sum(O * do))


@pytest.mark.parametrize("causal", [False, True])
def test_gqa_backward_matches_central_finite_differences(causal):
    q, do = randn((1, 4, 5, 3), 66), randn((1, 4, 5, 3), 67)
    k, v = randn((1, 2, 5, 3), 68), randn((1, 2, 5, 3), 69)
    scale = 0.7
    grads = attention_backward_gqa(q, k, v, do, scale, causal)
    h = 1e-6
    for which, g in zip(range(3), grads):
        args = [q, k, v]
        num = np.zeros_like(args[which])
        for idx in np.ndindex(args[which].shape):
            plus = [a.copy() for a in args]
            minus = [a.copy() for a in args]
            plus[which][idx] += h
            minus[which][idx] -= h
            num[idx] = (_gqa_loss(*plus, do, scale, causal) - _gqa_loss(*minus, do, scale, causal)) / (2 * h)
        err = np.max(np.abs(num - g)) / max(1.0, np.max(np.abs(g)))
        assert err <= 1e-6, (which, err)


@pytest.mark.parametrize("causal", [False, True])
def test_gqa_backward_invariants(causal):
    H, Hkv = 6, 2
    q, do = randn((2, H, 19, 7), 70), randn((2, H, 19, 7), 71)
    k, v = randn((2, Hkv, 19, 7), 72), randn((2, Hkv, 19, 7), 73)
    dq, dk, dv = attention_backward_gqa(q, k, v, do, 0.4, causal)
    # rows of each head's dS sum to zero; rows of its P sum to one
    np.testing.assert_allclose(dk.sum(-2), 0.0, atol=1e-11)
    group_do = do.reshape(2, Hkv, H // Hkv, 19, 7).sum(axis=(2, 3))
    np.testing.assert_allclose(dv.sum(-2), group_do, atol=1e-11)


def test_gqa_pin_catches_a_wrong_group_mapping(monkeypatch):
    # interleaved groups (h % H_kv) instead of consecutive ones
    monkeypatch.setattr(oa, "kv_head_of", lambda h, n_heads, n_kv_heads: h % n_kv_heads)
    with pytest.raises(AssertionError):
        test_gqa_zero_queries_average_their_group_values(True, 4, 2)


# ---------------------------------------------------------------- sliding window
@pytest.mark.parametrize("causal", [False, True])
def test_window_covering_everything_is_no_window(causal):
    q, k, v = randn((2, 23, 6), 80), randn((2, 23, 6), 81), randn((2, 23, 6), 82)
    O1, L1 = attention_forward(q, k, v, 0.4, causal)
    O2, L2 = attention_forward(q, k, v, 0.4, causal, window=(23, 23))
    np.testing.assert_allclose(O2, O1, atol=1e-14)
    np.testing.assert_allclose(L2, L1, atol=1e-14)


@pytest.mark.parametrize("causal,window", [(True, (0, -1)), (False, (0, 0)), (True, (0, 5))])
def test_window_of_one_key_returns_its_own_value(causal, window):
    # each query sees only its own key: O_i = V_i, LSE_i = scale * q_i . k_i
    q, k, v = randn((19, 7), 83), randn((19, 7), 84), randn((19, 7), 85)
    O, L = attention_forward(q, k, v, 0.3, causal, window=window)
    np.testing.assert_allclose(O, v, atol=1e-13)
    np.testing.assert_allclose(L, 0.3 * np.sum(q * k, axis=-1), atol=1e-13)


@pytest.mark.parametrize("left", [1, 3, 7])
def test_zero_queries_average_the_window(left):
    # Q = 0, causal, window (left, -1): query i averages V rows max(0, i - left) .. i
    n, d = 17, 4
    v = randn((n, d), 86)
    O, L = attention_forward(np.zeros((n, d)), randn((n, d), 87), v, 1.0, True, window=(left, -1))
    for i in range(n):
        lo = max(0, i - left)
        np.testing.assert_allclose(O[i], v[lo:i + 1].mean(0), atol=1e-13)
        np.testing.assert_allclose(L[i], math.log(i - lo + 1), atol=1e-13)


@pytest.mark.parametrize("causal,window", [(True, (4, -1)), (False, (3, 2)), (False, (-1, 1))])
def test_window_agrees_with_torch_sdpa_explicit_mask_fp64(causal, window):
    torch = pytest.importorskip("torch")
    import torch.nn.functional as F

    n = 29
    q, k, v, do = (randn((2, 3, n, 8), s) for s in (88, 89, 90, 91))
    i = np.arange(n)[:, None]
    j = np.arange(n)[None, :]
    allow = np.ones((n, n), dtype=bool)
    if causal:
        allow &= j <= i
    if window[0] >= 0:
        allow &= j >= i - window[0]
    if window[1] >= 0:
        allow &= j <= i + window[1]
    tq, tk, tv = (torch.tensor(x, requires_grad=True) for x in (q, k, v))
    out = F.scaled_dot_product_attention(tq, tk, tv, attn_mask=torch.tensor(allow), scale=0.35)
    out.backward(torch.tensor(do))
    O, _ = attention_forward(q, k, v, 0.35, causal, window=window)
    np.testing.assert_allclose(O, out.detach().numpy(), atol=1e-10)
    dq, dk, dv = attention_backward(q, k, v, do, 0.35, causal, window=window)
    np.testing.assert_allclose(dq, tq.grad.numpy(), atol=1e-10)
    np.testing.assert_allclose(dk, tk.grad.numpy(), atol=1e-10)
    np.testing.assert_allclose(dv, tv.grad.numpy(), atol=1e-10)


@pytest.mark.parametrize("causal,window", [(True, (2, -1)), (False, (1, 2))])
def test_window_backward_matches_central_finite_differences(causal, window):
    q, k, v, do = (randn((6, 3), s) for s in (92, 93, 94, 95))
    grads = attention_backward(q, k, v, do, 0.9, causal, window=window)
    loss = lambda a, b, c: float(np.sum(attention_forward(a, b, c, 0.9, causal, window=window)[0] * do))  # noqa: E731
    h = 1e-6
    for which, g in zip(range(3), grads):
        args = [q, k, v]
        num = np.zeros_like(args[which])
        for idx in np.ndindex(args[which].shape):
            plus = [a.copy() for a in args]
            minus = [a.copy() for a in args]
            plus[which][idx] += h
            minus[which][idx] -= h
            num[idx] = (loss(*plus) - loss(*minus)) / (2 * h)
        assert np.max(np.abs(num - g)) / max(1.0, np.max(np.abs(g))) <= 1e-6


def test_window_pin_catches_an_off_by_one(monkeypatch):
    def wider(s, window=(-1, -1)):  # one key too many on the left
        left, right = window
        return _orig_window(s, (left + 1 if left >= 0 else left, right))
    monkeypatch.setattr(oa, "apply_window", wider)
    with pytest.raises(AssertionError):
        test_zero_queries_average_the_window(3)


_orig_window = oa.apply_window
