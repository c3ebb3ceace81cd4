"""Gated-delta recurrent layer: the stand-in for the hybrid backbone's linear-recurrent layers.

[notes §3.1] names the hybrid Qwen3.5-2B backbone: 6 softmax-attention layers are
restricted by the method and 18 Gated DeltaNet layers keep their native computation.
[notes §2.3, third paragraph]: for hybrid models the conv and recurrent states must be
saved, and the pre-step state restored before the full retry, so the state is never
advanced twice.

The synthetic layer (weights are not available) per sequence and step:
  conv state  : the last 4 conv inputs (a 4 x 2048 shift register including the current one)
  u           = sum_i taps[i] * conv_state[i]                      (depthwise causal conv)
  per head h  : k_h = u_h / ||u_h||,  q_h = k_h
                S_h <- alpha_h S_h (I - beta_h k_h k_h^T) + beta_h v_h k_h^T   (gated delta rule)
                o_h = S_h q_h
S_h is [dv=128, dk=128]; o is the 16 heads' outputs concatenated (2048).
"""
import numpy as np

HEADS = 16
DIM = 128


def conv_step(conv_state: np.ndarray, c: np.ndarray, taps: np.ndarray):
    """Shift the new input into the 4-row state and apply the taps: (new_state, u)."""
    new_state = np.concatenate([conv_state[1:], c[None]], axis=0)
    u = np.sum(taps * new_state, axis=0)
    return new_state, u


def gdn_update(S: np.ndarray, k: np.ndarray, v: np.ndarray, alpha: float, beta: float):
    """S' = alpha S (I - beta k k^T) + beta v k^T, written with explicit matrices."""
    eye = np.eye(k.shape[0])
    return alpha * (S @ (eye - beta * np.outer(k, k))) + beta * np.outer(v, k)


def gdn_layer(S_heads, conv_state, c, v, alpha, beta, taps):
    """One layer for one sequence: returns (S_heads', conv_state', o [2048])."""
    conv_new, u = conv_step(conv_state, c, taps)
    S_new = np.empty_like(S_heads)
    outs = []
    for h in range(HEADS):
        uh = u[h * DIM:(h + 1) * DIM]
        k = uh / np.linalg.norm(uh)
        S_new[h] = gdn_update(S_heads[h], k, v[h], alpha[h], beta[h])
        outs.append(S_new[h] @ k)
    return S_new, conv_new, np.concatenate(outs)
