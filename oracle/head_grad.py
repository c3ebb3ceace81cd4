"""Gradient of the recall head's training loss with respect to every head parameter, in fp64.

Test infrastructure (the oracle): only tests, the smoke check and bench.py's CPU baseline use
it; the product path never imports it.

[notes §2.2, eq. L(psi) and the text after it]: the loss is the mean, over the valid positions E
(reference label valid and the two access sets different), of the Huber error with threshold 1
between the head's score q_t and the label y_t.  Only the recall head receives gradients; the
backbone, the embedding and the vocabulary projection only produce the supervision and the
features.  Labels follow [notes §2.1, eq. g_t; §2.2, eqs. d_t and y_t] (oracle.labels).

The forward is the reading of the head in oracle.head, with its intermediate values kept; the
backward is the chain rule through it, written out by hand (one sequence at a time; weight
gradients are summed over the batch):

  output   q = w_o . n_o + b_o,  n_o = RMSNorm(f2) * gamma_o
  block j  f_{j+1} = f_j + W_d a,  a = SiLU(g) * v,  g = W_g m,  v = W_u m,  m = RMSNorm(f_j) * gamma_j
  fusion   f0 = W_f z + b_f + (u0 + u1 + u2) / 3,  z = interaction(u0, u1, u2)
  towers   u_i = SiLU(p_i),  p_i = W_i n_i + b_i,  n_i = RMSNorm(x_i) * gamma_i

RMSNorm backward (y = x s gamma, s = (mean(x^2) + eps)^-1/2): with h = dy * gamma,
dx = s h - s^3 x (h . x) / N and dgamma = dy * x s.  SiLU'(x) = sigma(x) (1 + x (1 - sigma(x))).
The absolute differences of the interaction take sign(0) = 0 (a subgradient).
"""
import numpy as np
from scipy.special import expit

from oracle import labels
from oracle.head import EPS, interaction

HUBER_DELTA = 1.0


def _p(P, name):
    return np.asarray(P[name], dtype=np.float64)


def _rms_scale(x: np.ndarray) -> float:
    return 1.0 / np.sqrt(np.mean(x * x) + EPS)


def _rmsnorm_backward(dy: np.ndarray, x: np.ndarray, gamma: np.ndarray):
    """(dx, dgamma) of y = RMSNorm(x) * gamma."""
    s = _rms_scale(x)
    h = dy * gamma
    dx = s * h - s ** 3 * x * float(h @ x) / x.size
    return dx, dy * x * s


def _silu_grad(x: np.ndarray) -> np.ndarray:
    sg = expit(x)
    return sg * (1.0 + x * (1.0 - sg))


def forward_saved(P: dict, h_prev, emb, h_loc) -> dict:
    """The head's forward for one sequence with every intermediate needed by the backward."""
    xs = [np.asarray(v, np.float64) for v in (h_prev, emb, h_loc)]
    A = {"x": xs, "n": [], "p": [], "u": []}
    for i in range(3):
        n = xs[i] * _rms_scale(xs[i]) * _p(P, f"tower_norm{i}")
        p = _p(P, f"tower_w{i}") @ n + _p(P, f"tower_b{i}")
        A["n"].append(n)
        A["p"].append(p)
        A["u"].append(p * expit(p))
    u = A["u"]
    A["z"] = interaction(*u)
    f = _p(P, "fuse_w") @ A["z"] + _p(P, "fuse_b") + (u[0] + u[1] + u[2]) / 3.0
    A["f"], A["m"], A["g"], A["v"], A["a"] = [f], [], [], [], []
    for j in range(2):
        m = f * _rms_scale(f) * _p(P, f"ffn_norm{j}")
        g = _p(P, f"ffn_gate{j}") @ m
        v = _p(P, f"ffn_up{j}") @ m
        a = g * expit(g) * v
        f = f + _p(P, f"ffn_down{j}") @ a
        A["m"].append(m)
        A["g"].append(g)
        A["v"].append(v)
        A["a"].append(a)
        A["f"].append(f)
    A["n_o"] = f * _rms_scale(f) * _p(P, "out_norm")
    A["q"] = float(_p(P, "out_w") @ A["n_o"] + _p(P, "out_b")[0])
    return A


def backward(P: dict, A: dict, dq: float) -> dict:
    """Gradients of dq * q with respect to every parameter, for one sequence."""
    G = {}
    G["out_b"] = np.array([dq])
    G["out_w"] = dq * A["n_o"]
    dn_o = dq * _p(P, "out_w")
    df, G["out_norm"] = _rmsnorm_backward(dn_o, A["f"][2], _p(P, "out_norm"))
    for j in (1, 0):
        a, g, v, m = A["a"][j], A["g"][j], A["v"][j], A["m"][j]
        Wd, Wg, Wu = _p(P, f"ffn_down{j}"), _p(P, f"ffn_gate{j}"), _p(P, f"ffn_up{j}")
        G[f"ffn_down{j}"] = np.outer(df, a)
        da = Wd.T @ df
        dg = da * v * _silu_grad(g)
        dv = da * g * expit(g)
        G[f"ffn_gate{j}"] = np.outer(dg, m)
        G[f"ffn_up{j}"] = np.outer(dv, m)
        dm = Wg.T @ dg + Wu.T @ dv
        dfj, G[f"ffn_norm{j}"] = _rmsnorm_backward(dm, A["f"][j], _p(P, f"ffn_norm{j}"))
        df = df + dfj
    # fusion: f0 = W_f z + b_f + mean(u)
    G["fuse_w"] = np.outer(df, A["z"])
    G["fuse_b"] = df.copy()
    dz = (_p(P, "fuse_w").T @ df).reshape(9, -1)
    u0, u1, u2 = A["u"]
    s01, s02, s12 = np.sign(u0 - u1), np.sign(u0 - u2), np.sign(u1 - u2)
    du = [df / 3.0 + dz[0] + dz[3] * u1 + dz[4] * u2 + dz[6] * s01 + dz[7] * s02,
          df / 3.0 + dz[1] + dz[3] * u0 + dz[5] * u2 - dz[6] * s01 + dz[8] * s12,
          df / 3.0 + dz[2] + dz[4] * u0 + dz[5] * u1 - dz[7] * s02 - dz[8] * s12]
    for i in range(3):
        dp = du[i] * _silu_grad(A["p"][i])
        G[f"tower_w{i}"] = np.outer(dp, A["n"][i])
        G[f"tower_b{i}"] = dp
        dn = _p(P, f"tower_w{i}").T @ dp
        _, G[f"tower_norm{i}"] = _rmsnorm_backward(dn, A["x"][i], _p(P, f"tower_norm{i}"))
    return G


def labels_and_dq(q, p_full, p_local, valid, lam: float):
    """Per sequence: label y = label(gain - lambda), residual r = q - y, the loss (mean Huber
    over the valid sequences, 0 if none) and dL/dq (the Huber derivative over |E|; 0 where not
    valid)."""
    B = len(q)
    y = np.zeros(B)
    dq = np.zeros(B)
    n_valid = int(np.sum(np.asarray(valid, bool)))
    loss = 0.0
    for b in range(B):
        if not valid[b]:
            continue
        y[b] = labels.label(labels.penalised(labels.gain(float(p_full[b]), float(p_local[b])), lam))
        r = float(q[b]) - y[b]
        loss += labels.huber(r, HUBER_DELTA) / n_valid
        dq[b] = float(np.clip(r, -HUBER_DELTA, HUBER_DELTA)) / n_valid
    return loss, y, dq


def loss_and_grad(P: dict, h_prev, emb, h_loc, p_full, p_local, valid, lam: float):
    """(loss, q [B], y [B], gradients summed over the batch) of the head's training loss."""
    B = len(h_prev)
    acts = [forward_saved(P, h_prev[b], emb[b], h_loc[b]) for b in range(B)]
    q = np.array([A["q"] for A in acts])
    loss, y, dq = labels_and_dq(q, p_full, p_local, valid, lam)
    grads = {k: np.zeros(np.shape(v), np.float64) for k, v in P.items()}
    for b in range(B):
        if dq[b] == 0.0:
            continue
        for k, v in backward(P, acts[b], dq[b]).items():
            grads[k] += np.reshape(v, grads[k].shape)
    return loss, q, y, grads
