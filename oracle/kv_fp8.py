"""fp8 (e4m3) KV pages with one scale per token row, and attention over them, in fp64.

Test infrastructure (the oracle): only tests, the smoke check and bench.py's CPU baseline use
it; the product path never imports it.

The review of the method published 2026-09-20 ("on-demand attention recall-head paper",
section 六, on putting the method to use) suggests combining the access policy with KV
quantisation, without evaluating it or fixing a format.  The format here is a reading, chosen
so that the scales stay out of a decode kernel's inner loops:
  * element format: OCP FP8 E4M3FN — 1 sign bit, 4 exponent bits (bias 7), 3 mantissa bits; no
    infinities; exponent 1111 with mantissa 111 is NaN; the largest finite magnitude is 448 and
    the smallest subnormal 2^-9;
  * one fp32 scale per (token, KV head) row of 128 values: s = max|x| / 448 (s = 1 for an
    all-zero row), codes = round-to-nearest-even(x / s), saturating at +-448;
  * decode: x~ = s * value(code).  In attention the K scale multiplies the score q . k~ of its
    token and the V scale multiplies that token's softmax weight, so both fold out of the
    per-element products.
Attention over a quantised cache is the plain definition (oracle.attention) applied to the
decoded K~, V~.
"""
import numpy as np

E4M3_MAX = 448.0
_BIAS = 7


def e4m3_value(code: int) -> float:
    """The value of one e4m3 code, from the format's definition."""
    code = int(code) & 0xFF
    sign = -1.0 if code & 0x80 else 1.0
    e = (code >> 3) & 0xF
    m = code & 0x7
    if e == 0xF and m == 0x7:
        return float("nan")
    if e == 0:
        return sign * (m / 8.0) * 2.0 ** (1 - _BIAS)
    return sign * (1.0 + m / 8.0) * 2.0 ** (e - _BIAS)


E4M3_TABLE = np.array([e4m3_value(c) for c in range(256)], dtype=np.float64)


def e4m3_decode(codes) -> np.ndarray:
    return E4M3_TABLE[np.asarray(codes, dtype=np.uint8)]


def e4m3_encode(x) -> np.ndarray:
    """Round to nearest, ties to even mantissa, saturating at +-448; NaN -> 0x7F."""
    x = np.asarray(x, dtype=np.float64)
    out = np.zeros(x.shape, dtype=np.uint8)
    finite_pos = np.array([c for c in range(0x7F)], dtype=np.uint8)      # 0x00..0x7E, ascending
    vals = E4M3_TABLE[finite_pos]
    flat = x.reshape(-1)
    res = out.reshape(-1)
    for i, v in enumerate(flat):
        if np.isnan(v):
            res[i] = 0x7F
            continue
        a = min(abs(v), E4M3_MAX)
        j = int(np.searchsorted(vals, a))          # vals[j-1] < a <= vals[j]
        if j == 0:
            c = 0
        elif j >= len(vals):
            c = len(vals) - 1
        else:
            lo, hi = vals[j - 1], vals[j]
            if a - lo < hi - a:
                c = j - 1
            elif hi - a < a - lo:
                c = j
            else:                                   # tie: the code with an even mantissa
                c = j - 1 if ((j - 1) & 1) == 0 else j
        res[i] = c | (0x80 if (v < 0 or (v == 0 and np.signbit(v))) else 0)
    return out


def quantize_rows(x):
    """Per-row scales and codes of x [..., 128]: s = max|x| / 448 (1 for a zero row)."""
    x = np.asarray(x, dtype=np.float64)
    amax = np.max(np.abs(x), axis=-1, keepdims=True)
    s = np.where(amax > 0, amax / E4M3_MAX, 1.0)
    return e4m3_encode(x / s), s[..., 0]


def dequantize_rows(codes, scales) -> np.ndarray:
    return e4m3_decode(codes) * np.asarray(scales, np.float64)[..., None]
