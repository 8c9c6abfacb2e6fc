"""Seeded synthetic inputs shared by the tests, the bench and the oracle checks.

This module holds no attention arithmetic: it only draws random tensors.  Both
the CUDA path and the fp64 oracle are fed the same tensors from here.

The five workloads stand in for "long-context LLM attention heads"; none of the
pages' own benchmarks (model training runs) is reproduced.  Every tensor is laid
out (B, H, N, d), d innermost, the convention of the ``scaled_dot_product_attention``
call shown on "Flash Attention: Ako transformery zvladaju miliony tokenov",
section "6. Ako ho zapnut".
"""

from __future__ import annotations

import dataclasses
import math

import torch

__all__ = ["Workload", "WORKLOADS", "workload", "make_inputs", "make_qkv", "make_qkv_fp8"]


@dataclasses.dataclass(frozen=True)
class Workload:
    name: str
    B: int
    H: int
    N: int
    d: int
    causal: bool
    dtype: torch.dtype
    dist: str           # "normal" -> N(0,1), "uniform" -> U(-1,1)
    backward: bool      # whether dO is drawn and the backward is part of the workload
    spiky_frac: float   # fraction of key rows per (b,h) multiplied by 8 before the cast
    seed: int

    @property
    def scale(self) -> float:
        return 1.0 / math.sqrt(self.d)

    @property
    def fwd_flops(self) -> float:
        """4*B*H*N^2*d, halved under the causal mask (the metric's convention)."""
        f = 4.0 * self.B * self.H * self.N * self.N * self.d
        return f / 2 if self.causal else f

    @property
    def bwd_flops(self) -> float:
        """2.5x the forward figure."""
        return 2.5 * self.fwd_flops


WORKLOADS = {
    1: Workload("fwd_f32_n128_d64", 1, 1, 128, 64, False, torch.float32, "normal", False, 0.0, 1001),
    2: Workload("causal_b4_h16_n2048_d128", 4, 16, 2048, 128, True, torch.bfloat16, "normal", True, 0.0, 1002),
    3: Workload("causal_b2_h32_n8192_d128_spiky", 2, 32, 8192, 128, True, torch.bfloat16, "normal", True, 0.01, 1003),
    4: Workload("noncausal_b64_h16_n512_d64", 64, 16, 512, 64, False, torch.bfloat16, "uniform", False, 0.0, 1004),
    5: Workload("causal_b1_h8_n131072_d128", 1, 8, 131072, 128, True, torch.bfloat16, "normal", True, 0.0, 1005),
}


def workload(idx: int) -> Workload:
    return WORKLOADS[idx]


def _draw(shape, dist: str, g: torch.Generator) -> torch.Tensor:
    if dist == "normal":
        return torch.randn(shape, generator=g, dtype=torch.float32)
    if dist == "uniform":
        return torch.rand(shape, generator=g, dtype=torch.float32) * 2.0 - 1.0
    raise ValueError(f"unknown distribution {dist!r}")


def make_qkv(B: int, H: int, N: int, d: int, *, dtype=torch.bfloat16, dist: str = "normal",
             spiky_frac: float = 0.0, backward: bool = True, seed: int = 0,
             device: str | torch.device = "cpu", kv_heads: int | None = None) -> dict:
    """Draw q, k, v (and do when ``backward``) on the host from one seeded generator.

    Values are drawn in fp32 and then cast to ``dtype`` (round to nearest even).
    With ``spiky_frac`` > 0, for each (b, h) a seeded set of ceil(spiky_frac * N)
    key rows is multiplied by 8 in fp32 before the cast (x8 is exact in bf16),
    which makes many softmax rows nearly one-hot.  ``kv_heads`` (grouped-query
    attention) gives k and v that many heads instead of H.
    """
    g = torch.Generator(device="cpu")
    g.manual_seed(seed)
    shape = (B, H, N, d)
    kv_shape = (B, H if kv_heads is None else kv_heads, N, d)
    q = _draw(shape, dist, g)
    k = _draw(kv_shape, dist, g)
    v = _draw(kv_shape, dist, g)
    if spiky_frac > 0.0:
        n_spiky = int(math.ceil(spiky_frac * N))
        for b in range(B):
            for h in range(kv_shape[1]):
                idx = torch.randperm(N, generator=g)[:n_spiky]
                k[b, h, idx, :] *= 8.0
    out = {"q": q, "k": k, "v": v}
    if backward:
        out["do"] = torch.randn(shape, generator=g, dtype=torch.float32)
    return {name: t.to(dtype).to(device) for name, t in out.items()}


def make_inputs(idx_or_workload, device: str | torch.device = "cpu") -> dict:
    """Inputs of one of the five named workloads."""
    w = idx_or_workload if isinstance(idx_or_workload, Workload) else WORKLOADS[idx_or_workload]
    return make_qkv(w.B, w.H, w.N, w.d, dtype=w.dtype, dist=w.dist, spiky_frac=w.spiky_frac,
                    backward=w.backward, seed=w.seed, device=device)


E4M3_MAX = 448.0  # largest finite E4M3 value


def make_qkv_fp8(B: int, H: int, N: int, d: int, *, dist: str = "normal", spiky_frac: float = 0.0,
                 seed: int = 0, device: str | torch.device = "cpu", kv_heads: int | None = None) -> dict:
    """8-bit inputs: the fp32 draws of ``make_qkv`` (same seed, same spiky keys), each tensor
    divided by its own descale amax / 448 and rounded to E4M3 (torch's round to nearest even).

    Returns {"q", "k", "v": torch.float8_e4m3fn tensors, "q_descale", "k_descale",
    "v_descale": floats}; the real-valued inputs are descale * tensor."""
    f = make_qkv(B, H, N, d, dtype=torch.float32, dist=dist, spiky_frac=spiky_frac, backward=False, seed=seed,
                 kv_heads=kv_heads)
    out = {}
    for name in ("q", "k", "v"):
        x = f[name]
        amax = float(x.abs().max()) if x.numel() else 1.0
        # a float32 value, as the C interface receives it
        descale = float(torch.tensor(amax / E4M3_MAX if amax > 0 else 1.0, dtype=torch.float32))
        out[name] = (x / descale).clamp(-E4M3_MAX, E4M3_MAX).to(torch.float8_e4m3fn).to(device)
        out[name + "_descale"] = descale
    return out

