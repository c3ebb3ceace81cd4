"""Training-signal arithmetic of the paired supervision, and the compute-saving formula.

  gain       [notes §2.1, eq. g_t]: g_t = NLL_L(x_{t+1}) - NLL_F(x_{t+1})
                                        = log p^F_t(x_{t+1}) - log p^L_t(x_{t+1})  (nats)
  penalised  [notes §2.2, eq. d_t]: d_t = g_t - lambda, lambda >= 0
  label      [notes §2.2, eq. y_t]: y_t = sign(d_t) log(1 + |d_t|)   (sign(0) = 0)
  loss       [notes §2.2, eq. L(psi)]: mean over valid positions E (reference label valid
             and the two access sets differ) of Huber_1(q_t - y_t)
  Delta F    [notes §2.3, eq. Delta F]: (1 - rho) F_F - (F_L + F_R)
  routings   [notes §2.3, after eq. h_t/C_t]: the full prefill gives the first output, so
             N generated tokens take N - 1 routing decisions.
"""
import math

import numpy as np


def nll(p: float) -> float:
    return -math.log(p)


def gain(p_full: float, p_local: float) -> float:
    """g_t = NLL_L - NLL_F."""
    return nll(p_local) - nll(p_full)


def penalised(g: float, lam: float) -> float:
    if lam < 0:
        raise ValueError("lambda must be >= 0")
    return g - lam


def label(d: float) -> float:
    s = 0.0 if d == 0 else math.copysign(1.0, d)
    return s * math.log1p(abs(d))


def huber(r: float, delta: float = 1.0) -> float:
    """Huber loss with threshold delta: quadratic for |r| <= delta, linear beyond."""
    a = abs(r)
    return 0.5 * r * r if a <= delta else delta * (a - 0.5 * delta)


def huber_loss(q, y, valid) -> float:
    q = np.asarray(q, np.float64)
    y = np.asarray(y, np.float64)
    m = np.asarray(valid, bool)
    if not m.any():
        return 0.0
    return float(np.mean([huber(a - b) for a, b in zip(q[m], y[m])]))


def delta_F(rho: float, F_F: float, F_L: float, F_R: float) -> float:
    return (1.0 - rho) * F_F - (F_L + F_R)


def routed_steps(n_generated: int) -> int:
    return max(0, n_generated - 1)
