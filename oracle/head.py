"""Recall head R_psi(h_{t-1}, E(x_t), h_t^L) -> scalar score q_t, in fp64.

[notes §2.2, eq. q_t and the paragraph after it] fix the topology and size for
Qwen3-1.7B: three 2048-d inputs (previous chosen final hidden, frozen input embedding,
local pass's last-layer normalised hidden), each independently normalised, projected and
activated to 1024-d; an interaction vector keeping the three vectors, their pairwise
element-wise products and pairwise absolute differences (9216-d); a projection with a
residual fusion; two residual gated feed-forward blocks; a scalar output; fp32, exactly
28,325,889 parameters.  The page does not give the layer details.  Reading used here
(it reproduces the exact count):

  n_i   = RMSNorm(x_i) * gamma_i                      (eps 1e-6, weight [D])
  u_i   = SiLU(W_i n_i + b_i)                         (W_i [1024, D], b_i [1024])
  z     = [u1, u2, u3, u1*u2, u1*u3, u2*u3, |u1-u2|, |u1-u3|, |u2-u3|]
  f     = W_f z + b_f + (u1 + u2 + u3) / 3            (W_f [1024, 9216]; residual fusion
                                                       = the parameter-free tower mean)
  block j = 0, 1:  m = RMSNorm(f) * gamma_j ;  f = f + W_d,j (SiLU(W_g,j m) * (W_u,j m))
                                                      (W_g, W_u [2048, 1024], W_d [1024, 2048])
  q     = w_o . (RMSNorm(f) * gamma_o) + b_o          (w_o [1024], b_o scalar)

Inputs ordered (h_{t-1}, E(x_t), h_t^L).  Parity against the paper's trained head is
unpinned (no weights exist); the parameter count is pinned by the page.
"""
import numpy as np
from scipy.special import expit

EPS = 1e-6


def rmsnorm(x: np.ndarray, weight=None, eps: float = EPS) -> np.ndarray:
    y = x / np.sqrt(np.mean(x * x) + eps)
    return y if weight is None else y * weight


def silu(x: np.ndarray) -> np.ndarray:
    return x * expit(x)


def tower(x, norm_w, W, b):
    """u_i = SiLU(W_i (RMSNorm(x_i) * gamma_i) + b_i)."""
    return silu(W @ rmsnorm(x, norm_w) + b)


def interaction(u1, u2, u3) -> np.ndarray:
    """The 9216-d interaction vector: 3 vectors, 3 pairwise products, 3 pairwise |diffs|."""
    return np.concatenate([u1, u2, u3, u1 * u2, u1 * u3, u2 * u3,
                           np.abs(u1 - u2), np.abs(u1 - u3), np.abs(u2 - u3)])


def gated_ffn_block(f, norm_w, Wg, Wu, Wd):
    """f + W_d (SiLU(W_g m) * (W_u m)), m = RMSNorm(f) * gamma."""
    m = rmsnorm(f, norm_w)
    return f + Wd @ (silu(Wg @ m) * (Wu @ m))


def _p(P, name):
    return np.asarray(P[name], dtype=np.float64)


def recall_head(P: dict, h_prev: np.ndarray, emb: np.ndarray, h_loc: np.ndarray) -> float:
    """Score q_t of one sequence (inputs are 1-d vectors of width D)."""
    xs = (np.asarray(h_prev, np.float64), np.asarray(emb, np.float64),
          np.asarray(h_loc, np.float64))
    u = [tower(xs[i], _p(P, f"tower_norm{i}"), _p(P, f"tower_w{i}"), _p(P, f"tower_b{i}"))
         for i in range(3)]
    f = _p(P, "fuse_w") @ interaction(*u) + _p(P, "fuse_b") + (u[0] + u[1] + u[2]) / 3.0
    for j in range(2):
        f = gated_ffn_block(f, _p(P, f"ffn_norm{j}"), _p(P, f"ffn_gate{j}"),
                            _p(P, f"ffn_up{j}"), _p(P, f"ffn_down{j}"))
    return float(_p(P, "out_w") @ rmsnorm(f, _p(P, "out_norm")) + _p(P, "out_b")[0])


def recall_head_batch(P: dict, h_prev, emb, h_loc) -> np.ndarray:
    return np.array([recall_head(P, h_prev[b], emb[b], h_loc[b]) for b in range(len(h_prev))])


def param_count(P: dict) -> int:
    return int(sum(np.asarray(v).size for v in P.values()))
