"""Synthetic frozen backbone around the restricted attention layers, in fp64.  TEST
INFRASTRUCTURE ONLY (the oracle): only tests, the smoke check and bench.py's CPU baseline use it.

The method keeps the pretrained backbone frozen and only changes which positions each attention
layer reads [notes §2.1]; its throughput figures time the whole decode step - every layer, the
recall head, the conditional full pass, the commit and the LM head [notes §3.3; §2.3, eq. h_t,
p_t].  No weights exist here, so this stand-in has the shape of a Qwen3 decoder layer with
random bf16 weights (a reading: the pages name the models but give no layer internals):

  n = RMSNorm(x) * g_attn            (eps 1e-6; x is the fp32 residual stream)
  [q | k | v] = W_qkv bf16(n)        q: Hq heads, k, v: Hkv heads of 128, stored as bf16
  x = x + W_o bf16(o)                o: the attention output of the layer (all heads)
  m = RMSNorm(x) * g_mlp
  x = x + W_down bf16(SiLU(W_gate bf16(m)) * (W_up bf16(m)))
and after the last layer h = RMSNorm(x) * g_final (the "last-layer normalised hidden" the recall
head reads [notes §2.2]).  The step ends with the LM head on the committed hidden h_t: logits
= E bf16(h_t) with the embedding table E (tied), the next token = argmax (greedy; the smallest
index among equal maxima), and E(x_{t+1}) = its embedding row.  No positional rotation and no
per-head q/k normalisation are applied (random weights give them nothing to preserve).

Everything is fp64 except the bf16 roundings written above, which are part of the stand-in's
definition (the inputs of every projection, q/k/v and the MLP activation are bf16 in a bf16
model); bf16() rounds an fp64 value to the nearest bf16, ties to even.
"""
from __future__ import annotations

import numpy as np

from .attention import bf16_to_f64

EPS = 1e-6


def bf16(x) -> np.ndarray:
    """Nearest bf16 value (ties to even) of fp64 values, as fp64."""
    x = np.asarray(x, dtype=np.float64)
    m, e = np.frexp(x)                       # x = m 2^e, 0.5 <= |m| < 1
    e = np.maximum(e, -125)                  # bf16 subnormals: fixed spacing 2^-133
    return np.ldexp(np.rint(np.ldexp(x, 8 - e)), e - 8)


def bf16_bits(x) -> np.ndarray:
    """bf16 bit patterns (uint16) of bf16-representable fp64 values."""
    v = np.asarray(x, dtype=np.float64).astype(np.float32)
    return (v.view(np.uint32) >> np.uint32(16)).astype(np.uint16)


def rmsnorm(x, g) -> np.ndarray:
    """x / sqrt(mean(x^2) + eps) * g over the last axis."""
    x = np.asarray(x, dtype=np.float64)
    return x / np.sqrt(np.mean(x * x, axis=-1, keepdims=True) + EPS) * np.asarray(g, np.float64)


def silu(z) -> np.ndarray:
    return z / (1.0 + np.exp(-z))


def project(W_bits, a) -> np.ndarray:
    """W a for bf16 weights W [out, in] (bit patterns) and inputs a [..., in] (fp64)."""
    return np.asarray(a, np.float64) @ bf16_to_f64(W_bits).T


def attn_in(x, g_attn, W_qkv, Hq: int, Hkv: int):
    """q [B, Hq, 128], k, v [B, Hkv, 128] as bf16 bit patterns, from the residual x [B, D]."""
    y = bf16(project(W_qkv, bf16(rmsnorm(x, g_attn))))
    B = y.shape[0]
    q = y[:, :Hq * 128].reshape(B, Hq, 128)
    k = y[:, Hq * 128:(Hq + Hkv) * 128].reshape(B, Hkv, 128)
    v = y[:, (Hq + Hkv) * 128:].reshape(B, Hkv, 128)
    return bf16_bits(q), bf16_bits(k), bf16_bits(v)


def attn_out(x, o, W_o) -> np.ndarray:
    """x + W_o bf16(o): o [B, Hq * 128] the layer's attention output."""
    return np.asarray(x, np.float64) + project(W_o, bf16(o))


def mlp(x, g_mlp, W_gate, W_up, W_down) -> np.ndarray:
    """x + W_down bf16(SiLU(W_gate m) * W_up m), m = bf16(RMSNorm(x) * g_mlp)."""
    m = bf16(rmsnorm(x, g_mlp))
    a = bf16(silu(project(W_gate, m)) * project(W_up, m))
    return np.asarray(x, np.float64) + project(W_down, a)


def lm_head(h, E_bits):
    """(logits [B, V], token [B]) for the committed hidden h [B, D]: logits = E bf16(h),
    token = the smallest index of the largest logit."""
    logits = project(E_bits, bf16(h))
    return logits, np.argmax(logits, axis=-1).astype(np.int32)
