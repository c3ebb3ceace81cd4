"""Pins of the fp8 KV oracle (oracle.kv_fp8): the e4m3 code table against independent
constructions and the format's fixed points, round-to-nearest-even with saturation, the
per-row scale, and attention over a quantised cache against the plain definition."""
import math

import numpy as np
import pytest

from oracle import kv_fp8
from oracle.attention import attend


def test_code_table_fixed_points():
    T = kv_fp8.E4M3_TABLE
    assert T[0x00] == 0.0 and T[0x80] == 0.0 and math.copysign(1, T[0x80]) == -1
    assert T[0x38] == 1.0 and T[0xB8] == -1.0          # exponent field 7 = bias
    assert T[0x7E] == 448.0 and T[0xFE] == -448.0      # largest finite magnitude
    assert T[0x08] == 2.0 ** -6                        # smallest normal
    assert T[0x01] == 2.0 ** -9                        # smallest subnormal
    assert T[0x07] == 7 * 2.0 ** -9                    # largest subnormal
    assert np.isnan(T[0x7F]) and np.isnan(T[0xFF])     # the only NaNs; no infinities
    assert np.sum(np.isnan(T)) == 2 and np.all(np.isfinite(T[~np.isnan(T)]))


def test_code_table_matches_an_independent_construction():
    # positive finite values in increasing order: subnormals k/8 * 2^-6, then for each binade
    # e = -6..8 the eight values (1 + k/8) 2^e, the last binade stopping before NaN
    want = [k / 8 * 2.0 ** -6 for k in range(8)]
    for e in range(-6, 9):
        want += [(1 + k / 8) * 2.0 ** e for k in range(8)]
    want = want[:0x7F]
    assert np.array_equal(kv_fp8.E4M3_TABLE[:0x7F], np.array(want))
    assert np.array_equal(kv_fp8.E4M3_TABLE[0x80:0xFF], -np.array(want))


def test_encode_inverts_decode_on_every_finite_code():
    codes = np.array([c for c in range(256) if c not in (0x7F, 0xFF)], dtype=np.uint8)
    assert np.array_equal(kv_fp8.e4m3_encode(kv_fp8.e4m3_decode(codes)), codes)


def test_round_to_nearest_even_and_saturation():
    enc = kv_fp8.e4m3_encode
    # between 1.0 (0x38) and 1.125 (0x39): below, above and exactly at the midpoint
    assert enc(1.06)[()] == 0x38 and enc(1.07)[()] == 0x39
    assert enc(1.0625)[()] == 0x38          # tie -> even mantissa (0x38)
    assert enc(1.1875)[()] == 0x3A          # tie between 0x39 and 0x3A -> 0x3A
    assert enc(460.0)[()] == 0x7E and enc(1e9)[()] == 0x7E and enc(-1e9)[()] == 0xFE
    assert enc(2.0 ** -11)[()] == 0x00      # below half the smallest subnormal
    assert enc(float("nan"))[()] == 0x7F
    rng = np.random.default_rng(0)
    x = rng.normal(0, 50, 4000)
    y = kv_fp8.e4m3_decode(kv_fp8.e4m3_encode(x))
    # nearest representable: no table value is strictly closer
    T = np.sort(np.unique(kv_fp8.E4M3_TABLE[np.isfinite(kv_fp8.E4M3_TABLE)]))
    for xi, yi in zip(x[:500], y[:500]):
        c = np.clip(xi, -448, 448)
        assert abs(c - yi) <= np.min(np.abs(T - c)) + 1e-15


def test_row_scales_and_error_bound():
    rng = np.random.default_rng(1)
    x = rng.normal(0, 1, (64, 128))
    x[3] = 0.0
    codes, s = kv_fp8.quantize_rows(x)
    assert s[3] == 1.0 and not np.any(codes[3] & 0x7F)
    assert np.allclose(s[[0, 1]], np.max(np.abs(x[[0, 1]]), axis=1) / 448.0)
    xd = kv_fp8.dequantize_rows(codes, s)
    # the row maximum maps to 448 exactly; every element is within half a step of its binade
    assert np.allclose(np.max(np.abs(xd[[0, 1]]), axis=1), np.max(np.abs(x[[0, 1]]), axis=1))
    rel = np.abs(xd - x) / np.maximum(np.abs(x), s[:, None] * 2.0 ** -6)
    assert np.max(rel) <= 2.0 ** -4 + 1e-6      # + the fp32 rounding of x and of x / s


def test_scale_and_scaled_values_are_fp32():
    """The decisions are taken in fp32: the scale is an fp32 number, and a value whose fp64
    quotient x / s lies just past a rounding midpoint but whose fp32 quotient lands on it rounds
    as the fp32 quotient says."""
    rng = np.random.default_rng(3)
    x = rng.normal(0, 1, (16, 128)).astype(np.float32)
    _, s = kv_fp8.quantize_rows(x)
    assert np.array_equal(s, s.astype(np.float32).astype(np.float64))
    # a row with max 448 (s = 1): x / s = x exactly, so the codes are the plain encoding
    row = np.zeros(128, np.float32)
    row[0], row[1], row[2] = 448.0, 1.0625, 1.1875
    c, s1 = kv_fp8.quantize_rows(row)
    assert s1 == 1.0 and c[1] == 0x38 and c[2] == 0x3A and c[0] == 0x7E
    # fp32 division: 1 / fl32(1/3) rounded in fp32 is exactly 3 (the fp64 quotient is not)
    amax = np.float32(448.0) * np.float32(3.0)
    r2 = np.zeros(128, np.float32)
    r2[0] = amax
    r2[1] = np.float32(1.0)
    c2, s2 = kv_fp8.quantize_rows(r2)
    assert s2 == np.float32(amax / np.float32(448.0))
    assert kv_fp8.e4m3_decode(c2[1]) == kv_fp8.e4m3_decode(kv_fp8.e4m3_encode(
        float(np.float32(1.0) / np.float32(s2))))


def test_nan_entries_do_not_set_the_scale():
    x = np.ones((1, 128))
    x[0, 5] = np.nan
    x[0, 7] = 2.0
    c, s = kv_fp8.quantize_rows(x)
    assert s[0] == np.float32(2.0 / 448.0)
    assert c[0, 5] == 0x7F and kv_fp8.e4m3_decode(c[0, 7]) * s[0] == pytest.approx(2.0)


def test_attention_over_a_quantised_cache_is_the_plain_definition():
    rng = np.random.default_rng(2)
    n = 40
    K, V = rng.normal(0, 1, (n, 128)), rng.normal(0, 1, (n, 128))
    q = rng.normal(0, 1, 128)
    kc, ks = kv_fp8.quantize_rows(K)
    vc, vs = kv_fp8.quantize_rows(V)
    Kd, Vd = kv_fp8.dequantize_rows(kc, ks), kv_fp8.dequantize_rows(vc, vs)
    S = set(range(1, n + 1))
    o = attend(q[None, :], Kd[:, None, :], Vd[:, None, :], S)[0]
    # the scales fold out: scores s_j = ks_j (q . value(kc_j)), weights scaled by vs_j
    sc = ks * (kv_fp8.e4m3_decode(kc) @ q) / math.sqrt(128)
    w = np.exp(sc - sc.max())
    w /= w.sum()
    o2 = (w * vs) @ kv_fp8.e4m3_decode(vc)
    assert np.allclose(o, o2, rtol=1e-12, atol=1e-12)
    # and it stays close to attention over the unquantised cache (e4m3 keeps 3 mantissa bits)
    o_ref = attend(q[None, :], K[:, None, :], V[:, None, :], S)[0]
    assert np.linalg.norm(o - o_ref) / np.linalg.norm(o_ref) < 0.08


def test_attend_quantized_is_attention_over_the_decoded_cache_plus_the_exact_current_token():
    from oracle.attention import append_current, bf16_to_f64
    from oracle.sets import full_set, local_set
    from workload import gen
    t = 70
    bits = lambda tag, n: gen.normal_bf16(gen.key(5, tag), n)  # noqa: E731
    q = bits(1, 4 * 128).reshape(4, 128)
    kc = bits(2, (t - 1) * 2 * 128).reshape(t - 1, 2, 128)
    vc = bits(3, (t - 1) * 2 * 128).reshape(t - 1, 2, 128)
    kn, vn = bits(4, 256).reshape(2, 128), bits(5, 256).reshape(2, 128)
    for S in (full_set(t), local_set(t, 4, 32)):
        got = kv_fp8.attend_quantized(q, kc, vc, kn, vn, S)
        Kc, Ks = kv_fp8.quantize_rows(bf16_to_f64(kc))
        Vc, Vs = kv_fp8.quantize_rows(bf16_to_f64(vc))
        K = append_current(kv_fp8.dequantize_rows(Kc, Ks), bf16_to_f64(kn))
        V = append_current(kv_fp8.dequantize_rows(Vc, Vs), bf16_to_f64(vn))
        # written out directly: per head, scores over the set's rows, softmax, weighted values
        rows = np.array(sorted(S)) - 1
        for h in range(4):
            kh = h // 2
            sc = K[rows, kh] @ bf16_to_f64(q[h]) / math.sqrt(128)
            w = np.exp(sc - sc.max())
            w /= w.sum()
            assert np.allclose(got[h], w @ V[rows, kh], rtol=1e-12, atol=1e-12)
        # the current token is not quantised: changing its value moves the output exactly as
        # the exact value says (position t always belongs to both sets)
        assert t in S