"""Plain, slow, obviously-correct fp64 oracle of exact attention.

TEST INFRASTRUCTURE ONLY -- see the package docstring.  Nothing here is tiled,
fused or reordered beyond what the cited definition states; numpy matrix
products and ``exp``/``log`` are the only library primitives used.

Sources (titles of the web pages this method is described on):

* "FlashAttention (EL)", section "Problem of standard attention"
  (Problematiki tou typikou attention): the attention formula
  Attention(Q,K,V) = softmax(Q K^T / sqrt(d_k)) V.  The scale is passed in
  explicitly; callers use 1/sqrt(d).
* "Flash Attention: Ako transformery zvladaju miliony tokenov", section
  "5. Limity a co dalej" (causal vs. bidirectional masking) and section
  "6. Ako ho zapnut" (the ``is_causal=True`` call): the causal mask.  Reading
  taken: square problem, query i attends to keys j <= i (diagonal included).
* The same page, section "2. Riesenie: IO-aware algoritmus", and "FlashAttention
  (EL)", section "Online computation of Softmax": the online softmax keeps a
  running maximum and a running sum of exponentials, updated per block, and
  reaches the exact result.  ``online_softmax_forward`` restates that
  recurrence; it exists only to pin the plain definition against the pages'
  claim of exactness.
* "Flash Attention uitgelegd: een uitgebreide gids", section "Recomputation":
  the backward pass recomputes the attention probabilities instead of storing
  them.  The gradient formulas themselves are not printed on the pages; the
  ones below are the softmax Jacobian applied to the definition (derived):
  dV = P^T dO, dP = dO V^T, D_i = sum_j P_ij dP_ij, dS = P * (dP - D),
  dQ = scale * dS K, dK = scale * dS^T Q.  D is formed from P and dP, not
  from O, so the oracle does not share the kernels' rowsum(dO * O) identity.

LSE (the per-row log-sum-exp that the forward saves for the backward) is the
natural log of the row sum of exp of the scaled, masked scores.

Grouped-query and multi-query attention ("Flash Attention: Ako transformery
zvladaju miliony tokenov", section "5. Limity a co dalej", and "FlashAttention
(EL)", the closing list of extensions, name GQA/MQA support without defining
it).  Reading taken: H query heads share H_kv key/value heads (H a multiple of
H_kv; H_kv = 1 is MQA), query head h reads key/value head h // (H / H_kv) --
consecutive query heads form a group -- and each head's attention is the
definition above.  The gradients of a shared K or V are the sums of the
per-query-head gradients over its group (the chain rule through the sharing).

Sliding-window (local) attention ("Flash Attention uitgelegd: een uitgebreide
gids", section on open problems, names sliding window attention for very long
contexts without defining it).  Reading taken: a window (left, right) hides key j
from query i unless i - left <= j <= i + right, a bound of -1 being unbounded; it
combines with the causal mask, and every row keeps at least its own key.

Parity pins: every function here is pinned by ``tests/test_oracle.py``
(closed forms, invariants, finite differences, a hand-computed worked example,
a library special case and a brute-force loop restatement).
"""

from __future__ import annotations

import math

import numpy as np

__all__ = [
    "attention_probs",
    "attention_forward",
    "attention_forward_rows",
    "attention_backward",
    "online_softmax_forward",
    "loop_attention_forward",
    "loop_attention_backward",
    "kv_head_of",
    "attention_forward_gqa",
    "attention_backward_gqa",
    "apply_window",
]


def _as_f64(x) -> np.ndarray:
    """Exact widening to float64 (bf16 and fp32 values are representable)."""
    if hasattr(x, "detach"):  # torch tensor: go through fp32, which holds bf16 exactly
        x = x.detach().to("cpu").float().numpy()
    return np.asarray(x, dtype=np.float64)


def _heads(x: np.ndarray) -> tuple[np.ndarray, tuple]:
    """View a (..., N, d) array as (heads, N, d)."""
    lead = x.shape[:-2]
    return x.reshape((-1,) + x.shape[-2:]), lead


def _scores(q2: np.ndarray, k2: np.ndarray, scale: float, causal: bool) -> np.ndarray:
    """S = scale * Q K^T for one head, with -inf where the causal mask hides key j > i."""
    s = scale * (q2 @ k2.T)
    if causal:
        n_q, n_k = s.shape
        i = np.arange(n_q)[:, None]
        j = np.arange(n_k)[None, :]
        s = np.where(j > i, -np.inf, s)
    return s


def apply_window(s: np.ndarray, window=(-1, -1)) -> np.ndarray:
    """S_ij = -inf outside the sliding window: query i sees key j only if
    i - left <= j <= i + right (a bound of -1 is unbounded)."""
    left, right = window
    if left < 0 and right < 0:
        return s
    i = np.arange(s.shape[-2])[:, None]
    j = np.arange(s.shape[-1])[None, :]
    hide = np.zeros(s.shape[-2:], dtype=bool)
    if left >= 0:
        hide |= j < i - left
    if right >= 0:
        hide |= j > i + right
    return np.where(hide, -np.inf, s)


def _lse_rows(s: np.ndarray) -> np.ndarray:
    """ln sum_j exp(S_ij), computed stably as M_i + ln sum_j exp(S_ij - M_i)."""
    m = np.max(s, axis=-1, keepdims=True)
    return (m + np.log(np.sum(np.exp(s - m), axis=-1, keepdims=True)))[..., 0]


def attention_probs(q, k, scale: float, causal: bool):
    """Materialised probabilities P = softmax(scale * Q K^T + mask) and LSE.

    Returns (P of shape (..., N, N), LSE of shape (..., N)), both float64.
    """
    q = _as_f64(q)
    k = _as_f64(k)
    q3, lead = _heads(q)
    k3, _ = _heads(k)
    n = q3.shape[1]
    P = np.empty((q3.shape[0], n, k3.shape[1]))
    L = np.empty((q3.shape[0], n))
    for h in range(q3.shape[0]):
        s = _scores(q3[h], k3[h], scale, causal)
        lse = _lse_rows(s)
        P[h] = np.exp(s - lse[:, None])
        L[h] = lse
    return P.reshape(lead + P.shape[1:]), L.reshape(lead + (n,))


def attention_forward(q, k, v, scale: float, causal: bool, window=(-1, -1)):
    """O = P V and LSE, one head at a time (the N x N matrix is materialised per head).

    Inputs (..., N, d); returns O (..., N, d) and LSE (..., N) in float64.  ``window``:
    optional sliding window (left, right), see ``apply_window``.
    """
    q = _as_f64(q)
    k = _as_f64(k)
    v = _as_f64(v)
    q3, lead = _heads(q)
    k3, _ = _heads(k)
    v3, _ = _heads(v)
    O = np.empty_like(q3, shape=q3.shape[:2] + (v3.shape[2],))
    L = np.empty(q3.shape[:2])
    for h in range(q3.shape[0]):
        s = apply_window(_scores(q3[h], k3[h], scale, causal), window)
        lse = _lse_rows(s)
        p = np.exp(s - lse[:, None])
        O[h] = p @ v3[h]
        L[h] = lse
    return O.reshape(lead + O.shape[1:]), L.reshape(lead + (q3.shape[1],))


def attention_forward_rows(q, k, v, scale: float, causal: bool, rows, window=(-1, -1)):
    """The same definition evaluated only for the query rows ``rows`` of one head.

    q, k, v: (N, d) for a single head.  Returns O[rows] (len(rows), d) and LSE[rows].
    Row i sees keys 0..i when causal, all keys otherwise, and with a sliding window
    (left, right) only keys i - left .. i + right (as ``apply_window``).  Used where the
    full N x N matrix would not fit in host memory.
    """
    q = _as_f64(q)
    k = _as_f64(k)
    v = _as_f64(v)
    rows = np.asarray(rows, dtype=np.int64)
    s = scale * (q[rows] @ k.T)
    j = np.arange(k.shape[0])[None, :]
    i = rows[:, None]
    if causal:
        s = np.where(j > i, -np.inf, s)
    left, right = window
    if left >= 0:
        s = np.where(j < i - left, -np.inf, s)
    if right >= 0:
        s = np.where(j > i + right, -np.inf, s)
    lse = _lse_rows(s)
    p = np.exp(s - lse[:, None])
    return p @ v, lse


def attention_backward_dq_rows(q, k, v, do, scale: float, causal: bool, rows):
    """dQ of the given query rows of one head, from the definition row by row.

    q, k, v, do: (N, d) for a single head.  A row's dQ depends only on its own probabilities:
    with P_i = softmax of the row's scaled, masked scores, dP_ij = dO_i . V_j,
    D_i = sum_j P_ij dP_ij and dS_ij = P_ij (dP_ij - D_i), dQ_i = scale * sum_j dS_ij K_j.
    Used where the full N x N matrices would not fit in host memory.
    """
    q, k, v, do = _as_f64(q), _as_f64(k), _as_f64(v), _as_f64(do)
    rows = np.asarray(rows, dtype=np.int64)
    s = scale * (q[rows] @ k.T)
    if causal:
        j = np.arange(k.shape[0])[None, :]
        s = np.where(j > rows[:, None], -np.inf, s)
    p = np.exp(s - _lse_rows(s)[:, None])
    dp = do[rows] @ v.T
    delta = (p * dp).sum(axis=1, keepdims=True)
    return scale * ((p * (dp - delta)) @ k)


def attention_backward(q, k, v, do, scale: float, causal: bool, return_delta: bool = False, window=(-1, -1)):
    """Gradients of L = sum(O * dO) with respect to Q, K and V, from the definition.

    P is recomputed from Q and K (the backward never reuses a stored P).
    Returns (dQ, dK, dV) in float64, each shaped like its input; with
    ``return_delta`` also D (..., N) = sum_j P_ij dP_ij.
    """
    q = _as_f64(q)
    k = _as_f64(k)
    v = _as_f64(v)
    do = _as_f64(do)
    q3, lead = _heads(q)
    k3, _ = _heads(k)
    v3, _ = _heads(v)
    do3, _ = _heads(do)
    dq = np.empty_like(q3)
    dk = np.empty_like(k3)
    dv = np.empty_like(v3)
    D = np.empty(q3.shape[:2])
    for h in range(q3.shape[0]):
        s = apply_window(_scores(q3[h], k3[h], scale, causal), window)
        p = np.exp(s - _lse_rows(s)[:, None])
        dv[h] = p.T @ do3[h]
        dp = do3[h] @ v3[h].T
        delta = np.sum(p * dp, axis=-1)
        ds = p * (dp - delta[:, None])
        dq[h] = scale * (ds @ k3[h])
        dk[h] = scale * (ds.T @ q3[h])
        D[h] = delta
    out = (dq.reshape(q.shape), dk.reshape(k.shape), dv.reshape(v.shape))
    if return_delta:
        return out + (D.reshape(lead + (q3.shape[1],)),)
    return out


def online_softmax_forward(q, k, v, scale: float, causal: bool, block_q: int, block_k: int):
    """Blockwise restatement of the online softmax the pages describe in words.

    For each block of queries, key/value blocks arrive one at a time; the
    running row maximum m and running exp-sum l are updated and the partial
    output is rescaled by exp(m_old - m_new) each time (derived from the
    pages' description; no blocking beyond what the recurrence states).
    Returns O and LSE = m + ln l, float64.  Single head: q, k, v are (N, d).
    """
    q = _as_f64(q)
    k = _as_f64(k)
    v = _as_f64(v)
    n_q, n_k = q.shape[0], k.shape[0]
    O = np.zeros((n_q, v.shape[1]))
    L = np.zeros(n_q)
    for qs in range(0, n_q, block_q):
        qe = min(qs + block_q, n_q)
        m = np.full(qe - qs, -np.inf)
        l = np.zeros(qe - qs)
        acc = np.zeros((qe - qs, v.shape[1]))
        for ks in range(0, n_k, block_k):
            ke = min(ks + block_k, n_k)
            s = scale * (q[qs:qe] @ k[ks:ke].T)
            if causal:
                i = np.arange(qs, qe)[:, None]
                j = np.arange(ks, ke)[None, :]
                s = np.where(j > i, -np.inf, s)
            m_new = np.maximum(m, np.max(s, axis=1))
            # rows whose every key so far is masked keep m = -inf; guard exp(-inf - -inf)
            corr = np.where(np.isneginf(m_new), 1.0, np.exp(m - m_new))
            p = np.where(np.isneginf(m_new)[:, None], 0.0, np.exp(s - m_new[:, None]))
            l = l * corr + np.sum(p, axis=1)
            acc = acc * corr[:, None] + p @ v[ks:ke]
            m = m_new
        O[qs:qe] = acc / l[:, None]
        L[qs:qe] = m + np.log(l)
    return O, L


def loop_attention_forward(q, k, v, scale: float, causal: bool):
    """Pure-Python triple loop over the definition, for tiny single-head inputs.

    No numpy products: every dot product, max, exp and sum is an explicit loop,
    so it pins the numpy oracle's use of BLAS and broadcasting.
    """
    q = [[float(x) for x in row] for row in _as_f64(q)]
    k = [[float(x) for x in row] for row in _as_f64(k)]
    v = [[float(x) for x in row] for row in _as_f64(v)]
    n, d, dv = len(q), len(q[0]), len(v[0])
    O, L = [], []
    for i in range(n):
        s = []
        for j in range(len(k)):
            if causal and j > i:
                continue
            dot = 0.0
            for c in range(d):
                dot += q[i][c] * k[j][c]
            s.append((j, scale * dot))
        mx = max(x for _, x in s)
        tot = 0.0
        for _, x in s:
            tot += math.exp(x - mx)
        lse = mx + math.log(tot)
        o = [0.0] * dv
        for j, x in s:
            pij = math.exp(x - lse)
            for c in range(dv):
                o[c] += pij * v[j][c]
        O.append(o)
        L.append(lse)
    return np.array(O), np.array(L)


def loop_attention_backward(q, k, v, do, scale: float, causal: bool):
    """Pure-Python loop restatement of the derived gradient formulas (tiny inputs)."""
    qf = [[float(x) for x in row] for row in _as_f64(q)]
    kf = [[float(x) for x in row] for row in _as_f64(k)]
    vf = [[float(x) for x in row] for row in _as_f64(v)]
    dof = [[float(x) for x in row] for row in _as_f64(do)]
    n, d = len(qf), len(qf[0])
    nk = len(kf)
    P = [[0.0] * nk for _ in range(n)]
    for i in range(n):
        s = {}
        for j in range(nk):
            if causal and j > i:
                continue
            s[j] = scale * sum(qf[i][c] * kf[j][c] for c in range(d))
        mx = max(s.values())
        tot = sum(math.exp(x - mx) for x in s.values())
        for j, x in s.items():
            P[i][j] = math.exp(x - mx) / tot
    dQ = [[0.0] * d for _ in range(n)]
    dK = [[0.0] * d for _ in range(nk)]
    dV = [[0.0] * len(vf[0]) for _ in range(nk)]
    for i in range(n):
        dp = [sum(dof[i][c] * vf[j][c] for c in range(len(vf[0]))) for j in range(nk)]
        delta = sum(P[i][j] * dp[j] for j in range(nk))
        for j in range(nk):
            ds = P[i][j] * (dp[j] - delta)
            for c in range(len(vf[0])):
                dV[j][c] += P[i][j] * dof[i][c]
            for c in range(d):
                dQ[i][c] += scale * ds * kf[j][c]
                dK[j][c] += scale * ds * qf[i][c]
    return np.array(dQ), np.array(dK), np.array(dV)


# ---------------------------------------------------------------- grouped-query attention
def kv_head_of(h: int, n_heads: int, n_kv_heads: int) -> int:
    """Key/value head read by query head h: consecutive groups of H / H_kv query heads."""
    return h // (n_heads // n_kv_heads)


def _check_gqa_shapes(q, k, v):
    if q.ndim != 4 or k.ndim != 4 or v.ndim != 4:
        raise ValueError("grouped-query attention takes (B, H, N, d) arrays")
    B, H, N, _ = q.shape
    if k.shape[:3] != (B, k.shape[1], N) or v.shape[:3] != k.shape[:3] or k.shape[1] == 0 or H % k.shape[1]:
        raise ValueError("K and V need (B, H_kv, N, .) with H a multiple of H_kv")


def attention_forward_gqa(q, k, v, scale: float, causal: bool, window=(-1, -1)):
    """O and LSE of grouped-query attention, one query head at a time.

    q: (B, H, N, d); k, v: (B, H_kv, N, d).  Returns O (B, H, N, d_v), LSE (B, H, N).
    """
    q, k, v = _as_f64(q), _as_f64(k), _as_f64(v)
    _check_gqa_shapes(q, k, v)
    B, H, N, _ = q.shape
    Hkv = k.shape[1]
    O = np.empty((B, H, N, v.shape[3]))
    L = np.empty((B, H, N))
    for b in range(B):
        for h in range(H):
            g = kv_head_of(h, H, Hkv)
            s = apply_window(_scores(q[b, h], k[b, g], scale, causal), window)
            lse = _lse_rows(s)
            O[b, h] = np.exp(s - lse[:, None]) @ v[b, g]
            L[b, h] = lse
    return O, L


def attention_backward_gqa(q, k, v, do, scale: float, causal: bool, window=(-1, -1)):
    """dQ (B, H, N, d), dK and dV (B, H_kv, N, d) of L = sum(O * dO) for grouped-query attention.

    Per query head the gradients are those of the plain definition (see
    ``attention_backward``); a shared key/value head accumulates the dK and dV of
    every query head of its group.
    """
    q, k, v, do = _as_f64(q), _as_f64(k), _as_f64(v), _as_f64(do)
    _check_gqa_shapes(q, k, v)
    B, H, N, _ = q.shape
    Hkv = k.shape[1]
    dq = np.empty_like(q)
    dk = np.zeros_like(k)
    dv = np.zeros_like(v)
    for b in range(B):
        for h in range(H):
            g = kv_head_of(h, H, Hkv)
            s = apply_window(_scores(q[b, h], k[b, g], scale, causal), window)
            p = np.exp(s - _lse_rows(s)[:, None])
            dp = do[b, h] @ v[b, g].T
            ds = p * (dp - np.sum(p * dp, axis=-1)[:, None])
            dq[b, h] = scale * (ds @ k[b, g])
            dk[b, g] += scale * (ds.T @ q[b, h])
            dv[b, g] += p.T @ do[b, h]
    return dq, dk, dv
