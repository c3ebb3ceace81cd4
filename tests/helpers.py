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


def v8_slot_token(s: int) -> int:
    """Token held by slot s of a V row of an fp8 page block (layout stated in include/oda.h)."""
    return 2 * (s // 4) + (s % 2) + 8 * ((s // 2) % 2)


def decode_kv8_block(blk: np.ndarray):
    """(K codes [16,128], V codes [16,128], K scales [16], V scales [16]) of one fp8 page block,
    read by the layout stated in include/oda.h."""
    blk = np.ascontiguousarray(blk, dtype=np.uint8)
    K = np.empty((16, 128), np.uint8)
    for j in range(16):
        row = blk[128 * j:128 * (j + 1)].reshape(8, 16)
        K[j] = row[[k ^ (j & 7) for k in range(8)]].reshape(128)
    Vt = blk[2048:4096].reshape(128, 16)
    V = np.empty((16, 128), np.uint8)
    for s in range(16):
        V[v8_slot_token(s)] = Vt[:, s]
    sk = blk[4096:4160].view(np.float32).astype(np.float64)
    sv = blk[4160:4224].view(np.float32).astype(np.float64)
    return K, V, sk, sv


def logical_cache8(pool: np.ndarray, page_table: np.ndarray, b: int, n_tokens: int, table):
    """Decoded values (fp64 [n, Hkv, 128]) of tokens 0..n-1 of sequence b from an fp8 pool
    [n_pages, Hkv, 4224]; `table` maps codes to values."""
    Hkv = pool.shape[1]
    K = np.empty((n_tokens, Hkv, 128))
    V = np.empty((n_tokens, Hkv, 128))
    for tok in range(n_tokens):
        phys = page_table[b, tok // 16]
        for h in range(Hkv):
            kc, vc, sk, sv = decode_kv8_block(pool[phys, h])
            j = tok % 16
            K[tok, h] = table[kc[j]] * sk[j]
            V[tok, h] = table[vc[j]] * sv[j]
    return K, V


def packed_index(rows, cols):
    """Element offset of W[n][k] in the projections' packed layout, written out from the formula
    in include/oda_backbone.h (16 x 512 blocks, tile-major; 16-byte chunk j of row r at slot
    j ^ (r mod 8))."""
    n = np.arange(rows)[:, None]
    k = np.arange(cols)[None, :]
    return (((n // 16) * (cols // 512) + k // 512) * 8192 + (n % 16) * 512
            + (((k % 512) // 8) ^ (n % 8)) * 8 + k % 8)
