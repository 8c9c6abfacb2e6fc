"""Pins of the 8-bit part of the oracle (``oracle/fp8.py``).

The E4M3 decoder is pinned by values that follow from the format's definition
(bias 7, subnormals, NaN codes, largest finite value), by an independent library
routine (torch's float8_e4m3fn conversion) on all 256 codes, and by monotonicity.
The dequantized attention is pinned by a hand-computed worked example, by the
closed form of zero queries, and by how each descale must act (V's descale scales O
and leaves LSE alone; Q's and K's act only through the product with the scale).
The last tests plant mistakes in the oracle and check that these pins catch them.
"""

import math

import numpy as np
import pytest
import torch

import oracle
import oracle.fp8 as of8
from exact_io_aware_91_b200 import inputs


# ---------------------------------------------------------------- decoder
CLOSED_FORMS = {
    0x00: 0.0,
    0x01: 2.0**-9,              # smallest subnormal: 2^-6 * 1/8
    0x07: 7.0 * 2.0**-9,        # largest subnormal
    0x08: 2.0**-6,              # smallest normal
    0x38: 1.0,                  # e = 7 (the bias), m = 0
    0x3F: 1.875,                # 1 + 7/8
    0x40: 2.0,
    0x7E: 448.0,                # largest finite: 2^8 * 1.75
    0xB8: -1.0,
    0xFE: -448.0,
}


def test_e4m3_closed_forms():
    for code, val in CLOSED_FORMS.items():
        assert oracle.e4m3_decode(np.array([code], dtype=np.uint8))[0] == val, hex(code)
    neg_zero = oracle.e4m3_decode(np.array([0x80], dtype=np.uint8))[0]
    assert neg_zero == 0.0 and math.copysign(1.0, neg_zero) < 0
    assert np.isnan(oracle.e4m3_decode(np.array([0x7F, 0xFF], dtype=np.uint8))).all()


def test_e4m3_matches_torch_on_every_code():
    codes = np.arange(256, dtype=np.uint8)
    ref = torch.from_numpy(codes).view(torch.float8_e4m3fn).to(torch.float64).numpy()
    got = oracle.e4m3_decode(codes)
    assert np.array_equal(got, ref, equal_nan=True)


def test_e4m3_positive_codes_increase_and_negative_codes_mirror():
    pos = oracle.e4m3_decode(np.arange(0x00, 0x7F, dtype=np.uint8))
    assert np.all(np.diff(pos) > 0)
    neg = oracle.e4m3_decode(np.arange(0x80, 0xFF, dtype=np.uint8))
    assert np.array_equal(neg[1:], -pos[1:])


# ---------------------------------------------------------------- dequantized attention
def _codes(x: torch.Tensor) -> np.ndarray:
    return x.view(torch.uint8).numpy()


def test_worked_example_two_queries_two_keys():
    # q0 = (1, 0, ..), q1 = 0; k0 = (2, 0, ..), k1 = 0; v0 = (1, 0, ..), v1 = (0, 1, 0, ..);
    # descales 0.5 (q), 3 (k), 2 (v), scale 0.25: row 0 scores (0.25 * 0.5 * 3 * 2, 0) =
    # (0.75, 0); row 1 scores (0, 0), so its output is the mean of the two values
    d = 4
    q = np.zeros((1, 1, 2, d), np.uint8); q[0, 0, 0, 0] = 0x38
    k = np.zeros((1, 1, 2, d), np.uint8); k[0, 0, 0, 0] = 0x40
    v = np.zeros((1, 1, 2, d), np.uint8); v[0, 0, 0, 0] = 0x38; v[0, 0, 1, 1] = 0x38
    o, lse = oracle.attention_forward_fp8(q, k, v, 0.5, 3.0, 2.0, 0.25, False)
    p0 = math.exp(0.75) / (math.exp(0.75) + 1.0)
    assert abs(o[0, 0, 0, 0] - 2.0 * p0) < 1e-14
    assert abs(o[0, 0, 0, 1] - 2.0 * (1.0 - p0)) < 1e-14
    assert abs(lse[0, 0, 0] - math.log(math.exp(0.75) + 1.0)) < 1e-14
    assert np.allclose(o[0, 0, 1], [1.0, 1.0, 0.0, 0.0], atol=1e-15, rtol=0)
    assert abs(lse[0, 0, 1] - math.log(2.0)) < 1e-15


@pytest.mark.parametrize("causal", [False, True])
def test_zero_queries_average_the_dequantized_values(causal):
    x = inputs.make_qkv_fp8(1, 2, 40, 16, seed=5)
    q = np.zeros(_codes(x["q"]).shape, np.uint8)
    v = _codes(x["v"])
    o, lse = oracle.attention_forward_fp8(q, _codes(x["k"]), v, 1.0, x["k_descale"], 0.25, 0.3, causal)
    vals = torch.from_numpy(v).view(torch.float8_e4m3fn).to(torch.float64).numpy() * 0.25
    if causal:
        counts = np.arange(1, 41, dtype=np.float64)
        expect = np.cumsum(vals, axis=2) / counts[None, None, :, None]
        assert np.allclose(lse, np.log(counts)[None, None, :], atol=1e-13, rtol=0)
    else:
        expect = np.broadcast_to(vals.mean(axis=2, keepdims=True), vals.shape)
        assert np.allclose(lse, math.log(40), atol=1e-13, rtol=0)
    assert np.allclose(o, expect, atol=1e-13, rtol=0)


def test_value_descale_scales_the_output_only():
    x = inputs.make_qkv_fp8(1, 2, 33, 16, seed=6)
    args = (_codes(x["q"]), _codes(x["k"]), _codes(x["v"]))
    o1, l1 = oracle.attention_forward_fp8(*args, 0.1, 0.2, 1.0, 0.5, True)
    o3, l3 = oracle.attention_forward_fp8(*args, 0.1, 0.2, 3.0, 0.5, True)
    assert np.allclose(o3, 3.0 * o1, atol=1e-13, rtol=1e-13)
    assert np.array_equal(l1, l3)


def test_query_and_key_descales_act_through_the_scale():
    x = inputs.make_qkv_fp8(1, 2, 33, 16, seed=7)
    args = (_codes(x["q"]), _codes(x["k"]), _codes(x["v"]))
    base = oracle.attention_forward_fp8(*args, 1.0, 1.0, 0.7, 0.2, True)
    for qd, kd, sc in ((2.0, 1.0, 0.1), (1.0, 4.0, 0.05), (0.5, 0.5, 0.8)):
        o, lse = oracle.attention_forward_fp8(*args, qd, kd, 0.7, sc, True)
        assert np.allclose(o, base[0], atol=1e-12, rtol=0)
        assert np.allclose(lse, base[1], atol=1e-12, rtol=0)


# ---------------------------------------------------------------- planted mistakes
def _decode_no_subnormals(bits):
    b = np.asarray(bits, dtype=np.uint8)
    val = _orig_decode(b)
    return np.where((b & 0x78) == 0, 0.0, val)


_orig_decode = of8.e4m3_decode


def _bias8(bits):  # exponent bias 8 instead of 7: every value one binade low
    return _orig_decode(bits) / 2.0


@pytest.mark.parametrize("bad", [_bias8, _decode_no_subnormals])
def test_decoder_pins_catch_planted_mistakes(monkeypatch, bad):
    monkeypatch.setattr(oracle, "e4m3_decode", bad)
    with pytest.raises(AssertionError):
        test_e4m3_closed_forms()


def test_descale_pins_catch_a_descale_on_the_wrong_operand(monkeypatch):
    def swapped(q_bits, k_bits, v_bits, q_descale, k_descale, v_descale, scale, causal, window=(-1, -1)):
        q = q_descale * _orig_decode(q_bits)
        k = v_descale * _orig_decode(k_bits)  # V's descale applied to K
        v = k_descale * _orig_decode(v_bits)
        return oracle.attention_forward_gqa(q, k, v, scale, causal, window)
    monkeypatch.setattr(oracle, "attention_forward_fp8", swapped)
    with pytest.raises(AssertionError):
        test_value_descale_scales_the_output_only()


@pytest.mark.parametrize("causal,window", [(False, (-1, -1)), (True, (-1, -1)), (True, (7, -1)), (False, (5, 3))])
def test_row_sampler_matches_the_full_8bit_forward(causal, window):
    # the per-head row sampler used for long sequences must agree with the pinned full forward
    x = inputs.make_qkv_fp8(1, 2, 60, 16, seed=9, spiky_frac=0.05)
    bits = {n: x[n].view(torch.uint8).numpy() for n in ("q", "k", "v")}
    ds = (x["q_descale"], x["k_descale"], x["v_descale"])
    O, L = oracle.attention_forward_fp8(bits["q"], bits["k"], bits["v"], *ds, 0.25, causal, window)
    rows = [0, 1, 29, 58, 59]
    for h in range(2):
        Or, Lr = oracle.attention_forward_fp8_rows(bits["q"][0, h], bits["k"][0, h], bits["v"][0, h], *ds, 0.25,
                                                   causal, rows, window)
        np.testing.assert_allclose(Or, O[0, h, rows], atol=1e-13)
        np.testing.assert_allclose(Lr, L[0, h, rows], atol=1e-13)
