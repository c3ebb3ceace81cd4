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
    all-zero row; NaN entries do not count toward the maximum), codes =
    round-to-nearest-even(x / s), saturating at +-448.  Where floating point decides these
    integer codes it is fp32, the precision the quantising kernel computes in: max|x| of bf16
    values is exact, then s = fl32(max|x| / 448) and x / s = fl32(x / s), each one IEEE
    correctly rounded division, then the one rounding to e4m3;
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
    """Round to nearest, ties to even mantissa, saturating at +-448; NaN -> 0x7F.

    For each |x| (clipped to 448): find the two neighbouring finite codes lo < |x| <= hi in the
    ascending table of non-negative values, take the nearer one, and on a tie the one with the
    even mantissa (even code); then set the sign bit (also for -0.0)."""
    x = np.asarray(x, dtype=np.float64)
    vals = E4M3_TABLE[:0x7F]                         # codes 0x00..0x7E, ascending values
    with np.errstate(invalid="ignore"):
        a = np.minimum(np.abs(x), E4M3_MAX)
        j = np.clip(np.searchsorted(vals, a), 1, len(vals) - 1)   # vals[j-1] < a <= vals[j]
        lo, hi = vals[j - 1], vals[j]
        d_lo, d_hi = a - lo, hi - a
        even_lo = ((j - 1) & 1) == 0
        c = np.where(d_lo < d_hi, j - 1, np.where(d_hi < d_lo, j, np.where(even_lo, j - 1, j)))
        neg = (x < 0) | ((x == 0) & np.signbit(x))
    out = (c.astype(np.uint8) | np.where(neg, 0x80, 0x00).astype(np.uint8)).astype(np.uint8)
    out = np.where(np.isnan(x), np.uint8(0x7F), out).astype(np.uint8)
    return out


def quantize_rows(x):
    """Per-row scales and codes of x [..., 128]: s = fl32(max|x| / 448) (1 for a zero row),
    codes = e4m3(fl32(x / s)).  x is taken as fp32 (bf16 values are exact in it)."""
    x32 = np.asarray(x, dtype=np.float32)
    amax = np.fmax.reduce(np.abs(x32), axis=-1, keepdims=True)        # NaN entries skipped
    s = np.where(amax > 0, amax / np.float32(E4M3_MAX), np.float32(1.0)).astype(np.float32)
    with np.errstate(invalid="ignore", divide="ignore"):
        y = (x32 / s).astype(np.float64)
    return e4m3_encode(y), s[..., 0].astype(np.float64)


def dequantize_rows(codes, scales) -> np.ndarray:
    return e4m3_decode(codes) * np.asarray(scales, np.float64)[..., None]


def attend_quantized(q_bits, cache_k_bits, cache_v_bits, k_new_bits, v_new_bits, S):
    """Attention of one decode query over a cache held in this format.

    [notes §2.1, eq. o_t] with K~, V~ = the cached positions 1..t-1 as stored (every (token,
    KV head) row quantised, then decoded: s * value(code)) followed by the current token's own
    key and value at position t, exactly as the branch computed them (bf16; a row is
    quantised only when it is committed).  Inputs are bf16 bit patterns: q [Hq, d], cache
    [t-1, Hkv, d], current k/v [Hkv, d]; the plain definition (oracle.attention.attend) does
    the rest in fp64.
    """
    from .attention import append_current, attend, bf16_to_f64
    kc, ks = quantize_rows(bf16_to_f64(cache_k_bits))
    vc, vs = quantize_rows(bf16_to_f64(cache_v_bits))
    K = append_current(dequantize_rows(kc, ks), bf16_to_f64(k_new_bits))
    V = append_current(dequantize_rows(vc, vs), bf16_to_f64(v_new_bits))
    return attend(bf16_to_f64(q_bits), K, V, S)
