"""8-bit (E4M3) inputs of the attention forward: decoding, and the exact attention of the
dequantized values.

TEST INFRASTRUCTURE ONLY -- see the package docstring.

Sources: "Flash Attention uitgelegd: een uitgebreide gids", section "Native FP8-precisie",
and "FlashAttention (EL)", section "FlashAttention-3 (2024)": FlashAttention-3 runs the
attention products in FP8 on the tensor cores.  The pages name no format and no scaling
scheme.  Reading taken:

* the format is the 8-bit floating point format E4M3: one sign bit s, four exponent bits e
  (bias 7) and three mantissa bits m.  e = 0 encodes the subnormals (-1)^s * 2^-6 * m / 8;
  otherwise the value is (-1)^s * 2^(e - 7) * (1 + m / 8).  The two codes with e = 15 and
  m = 7 are NaN; there are no infinities, so the largest finite value is 2^8 * 1.75 = 448;
* each input tensor carries one positive descale factor: the real-valued operand is the
  descale times the decoded value.

What the 8-bit forward computes is then the attention definition (``attention.py``) of the
dequantized Q, K and V; the rounding the kernels apply on the way (the probabilities are
rounded to E4M3 before the P V product) is a property of the kernels, bounded in the tests.
"""

import numpy as np

from .attention import attention_forward_gqa, attention_forward_rows


def e4m3_decode(bits) -> np.ndarray:
    """float64 values of E4M3 codes (an array of uint8, any shape)."""
    b = np.asarray(bits, dtype=np.uint8).astype(np.int64)
    sign = (b >> 7) & 1
    e = (b >> 3) & 15
    m = (b & 7).astype(np.float64)
    subnormal = m / 8.0 * 2.0**-6
    normal = (1.0 + m / 8.0) * np.power(2.0, (e - 7).astype(np.float64))
    val = np.where(e == 0, subnormal, normal)
    val = np.where((e == 15) & (b & 7 == 7), np.nan, val)
    return np.where(sign == 1, -val, val)


def attention_forward_fp8(q_bits, k_bits, v_bits, q_descale: float, k_descale: float, v_descale: float,
                          scale: float, causal: bool, window=(-1, -1)):
    """(O, LSE) of the attention of q_descale * Q, k_descale * K, v_descale * V.

    q_bits (B, H, N, d), k_bits and v_bits (B, H_kv, N, d): E4M3 codes as uint8.  Grouped
    heads, the causal mask and the sliding window as in ``attention_forward_gqa``."""
    q = q_descale * e4m3_decode(q_bits)
    k = k_descale * e4m3_decode(k_bits)
    v = v_descale * e4m3_decode(v_bits)
    return attention_forward_gqa(q, k, v, scale, causal, window)


def attention_forward_fp8_rows(q_bits, k_bits, v_bits, q_descale: float, k_descale: float, v_descale: float,
                               scale: float, causal: bool, rows, window=(-1, -1)):
    """(O[rows], LSE[rows]) of one head of the same attention, for long sequences.

    q_bits, k_bits, v_bits: (N, d) E4M3 codes of one query head and its key/value head."""
    q = q_descale * e4m3_decode(q_bits)
    k = k_descale * e4m3_decode(k_bits)
    v = v_descale * e4m3_decode(v_bits)
    return attention_forward_rows(q, k, v, scale, causal, rows, window)
