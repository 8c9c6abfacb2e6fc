"""The 8-bit forward's tolerance, checked on the CPU against an fp64 emulation of the
arithmetic the kernel performs (not of its code): P is formed on a row scale whose largest
value lies in [1, 2^8) (the running maximum may lag the true one by less than 8 in base-2
exponent), rounded to E4M3 (torch's round-to-nearest-even conversion), multiplied with the
dequantized V and divided by the row sum of the unrounded P; the result is rounded to bf16.
The bound used by the GPU test must cover that arithmetic, and must not be vacuous: a
rounding one bit coarser than E4M3's breaks it.
"""

import importlib.util
import math
import os

import numpy as np
import torch

import oracle
from exact_io_aware_91_b200 import inputs

_spec = importlib.util.spec_from_file_location(
    "gpu_fp8_bound", os.path.join(os.path.dirname(os.path.abspath(__file__)), "test_gpu_fp8.py"))
_mod = importlib.util.module_from_spec(_spec)
_spec.loader.exec_module(_mod)
o_bound, probs_rows = _mod.o_bound, _mod.probs_rows


def _round_mantissa(x: np.ndarray, bits: int) -> np.ndarray:
    """Round to `bits` explicit mantissa bits (no exponent limits): a rounding coarser than E4M3."""
    m, e = np.frexp(x)
    return np.ldexp(np.round(m * 2.0 ** (bits + 1)) / 2.0 ** (bits + 1), e)


def _emulate(p: np.ndarray, v: np.ndarray, lag: np.ndarray, rounding) -> np.ndarray:
    pu = p / p.max(axis=1, keepdims=True) * lag  # the kernel's unnormalised P
    pq = rounding(pu)
    o = (pq @ v) / pu.sum(axis=1, keepdims=True)
    return torch.from_numpy(o).to(torch.bfloat16).to(torch.float64).numpy()


def _e4m3(x: np.ndarray) -> np.ndarray:
    return torch.from_numpy(x).to(torch.float8_e4m3fn).to(torch.float64).numpy()


def _case(N, spiky, causal, seed):
    x = inputs.make_qkv_fp8(1, 1, N, 128, spiky_frac=spiky, seed=seed)
    q, k, v = (x[n + "_descale"] * oracle.e4m3_decode(x[n].view(torch.uint8).numpy()[0, 0]) for n in "qkv")
    p = probs_rows(q, k, 1.0 / math.sqrt(128), causal, (-1, -1), np.arange(N))
    return p, v, p @ v


def test_fp8_bound_covers_the_kernel_arithmetic():
    rng = np.random.default_rng(0)
    for N, spiky, causal in ((700, 0.0, True), (1024, 0.01, True), (513, 0.0, False), (2048, 0.01, True)):
        p, v, o_ref = _case(N, spiky, causal, seed=N)
        bound = o_bound(p, v, o_ref)
        for top in (0.0, 4.0, 7.99):
            lag = 2.0 ** rng.uniform(0.0, top, size=(N, 1))
            err = np.abs(_emulate(p, v, lag, _e4m3) - o_ref)
            assert np.all(err <= bound), f"N={N} lag<2^{top}: {(err / bound).max():.3f} of the bound"


def test_fp8_bound_is_not_vacuous():
    # two mantissa bits instead of E4M3's three: errors twice as large must exceed the bound
    rng = np.random.default_rng(1)
    p, v, o_ref = _case(1024, 0.01, True, seed=3)
    bound = o_bound(p, v, o_ref)
    lag = 2.0 ** rng.uniform(0.0, 7.99, size=(1024, 1))
    err = np.abs(_emulate(p, v, lag, lambda x: _round_mantissa(x, 1)) - o_ref)
    assert np.any(err > bound)
