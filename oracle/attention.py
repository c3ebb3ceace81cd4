"""Softmax attention of one decode query over an explicit index set.

[notes §2.1, eq. o_t]: o_t = softmax(q_t K~_t[S_t]^T / sqrt(d_k)) V~_t[S_t], where
K~_t, V~_t are the cached keys/values with the current token's key/value appended, and S_t
selects the positions taking part.  The page omits layer and head indices; grouped-query
attention maps query head h to KV head floor(h / g), g = Hq / Hkv (consecutive grouping).

Everything here is fp64: bf16 inputs are decoded exactly, scores, weights and outputs are
formed directly from the definition (no online softmax, no blocking).
"""
import math

import numpy as np


def bf16_to_f64(bits: np.ndarray) -> np.ndarray:
    """Exact value of bf16 bit patterns (the upper half of an fp32 word)."""
    b = np.asarray(bits, dtype=np.uint16).astype(np.uint32) << np.uint32(16)
    return b.view(np.float32).astype(np.float64)


def append_current(cache: np.ndarray, current: np.ndarray) -> np.ndarray:
    """K~_t = cache (positions 1..t-1) with the current token's row (position t) appended."""
    return np.concatenate([cache, current[None]], axis=0)


def softmax_weights(scores: np.ndarray) -> np.ndarray:
    e = np.exp(scores - scores.max())
    return e / e.sum()


def attend(q: np.ndarray, K_tilde: np.ndarray, V_tilde: np.ndarray, S) -> np.ndarray:
    """o [Hq, d] for query q [Hq, d] over rows S (1-based positions) of K~, V~ [t, Hkv, d].

    All arrays fp64.  Query head h reads KV head h // (Hq // Hkv).
    """
    Hq, d = q.shape
    Hkv = K_tilde.shape[1]
    g = Hq // Hkv
    rows = np.array(sorted(S), dtype=np.int64) - 1
    out = np.empty((Hq, d), dtype=np.float64)
    for h in range(Hq):
        kh = h // g
        K = K_tilde[rows, kh, :]
        V = V_tilde[rows, kh, :]
        w = softmax_weights(K @ q[h] / math.sqrt(d))
        out[h] = w @ V
    return out


def attend_bits(q_bits, cache_k_bits, cache_v_bits, k_new_bits, v_new_bits, S) -> np.ndarray:
    """attend() on bf16 bit-pattern inputs: cache [t-1, Hkv, d], current k/v [Hkv, d]."""
    K = append_current(bf16_to_f64(cache_k_bits), bf16_to_f64(k_new_bits))
    V = append_current(bf16_to_f64(cache_v_bits), bf16_to_f64(v_new_bits))
    return attend(bf16_to_f64(q_bits), K, V, S)
