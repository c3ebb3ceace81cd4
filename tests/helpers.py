"""Shared helpers of the GPU parity tests: tolerances, buffer setup, comparisons."""
from __future__ import annotations

import numpy as np

# Tolerances: attention outputs within max-abs 1e-2 and relative L2 2e-3, recall scores within
# relative 1e-4 (a floor of 1e-3 on |q|), routing compared outside the |q| < 1e-5 tie band:
ATTN_MAX_ABS = 1e-2     # per (sequence, layer) output
ATTN_REL_L2 = 2e-3
SCORE_REL = 1e-4        # |dq| <= 1e-4 * max(|q_ref|, 1e-3)
SCORE_FLOOR = 1e-3
TIE_BAND = 1e-5         # routing decisions with |q| < 1e-5 are not compared


def attn_close(got: np.ndarray, ref: np.ndarray):
    """(ok, max_abs, rel_l2) of one output block."""
    got = np.asarray(got, np.float64)
    ref = np.asarray(ref, np.float64)
    d = got - ref
    max_abs = float(np.max(np.abs(d))) if d.size else 0.0
    rel = float(np.linalg.norm(d) / max(np.linalg.norm(ref), 1e-30))
    return (max_abs <= ATTN_MAX_ABS and rel <= ATTN_REL_L2), max_abs, rel


def score_close(got: float, ref: float) -> bool:
    return abs(got - ref) <= SCORE_REL * max(abs(ref), SCORE_FLOOR)


def build_all():
    from conditional_sparse_attention_b200 import build
    from workload import device
    build.build()
    device.build()


def logical_cache(pool_u16: np.ndarray, page_table: np.ndarray, b: int, n_tokens: int) -> np.ndarray:
    """Gather tokens 0..n-1 of sequence b from a paged pool [n_pages, Hkv, 16, 128] (host)."""
    pages = page_table[b, :(n_tokens + 15) // 16]
    toks = pool_u16[pages].transpose(0, 2, 1, 3).reshape(-1, pool_u16.shape[1], 128)
    return toks[:n_tokens]
