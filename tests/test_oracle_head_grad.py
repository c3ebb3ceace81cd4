"""Pins of the oracle's recall-head gradient (oracle.head_grad).

The hand-written backward is checked against central finite differences of the loss computed
through the independent forward (oracle.head.recall_head) and the label arithmetic
(oracle.labels), on a tiny head (D = 6, tower width 4, FFN width 5) where every parameter
element is probed.  A dropped term, a wrong sign or a transposed operand anywhere in the chain
fails it.  The label and Huber-derivative hand cases come from the method notes' formulas.
"""
import numpy as np
import pytest

from oracle import head_grad, labels
from oracle.head import recall_head

D, T, F = 6, 4, 5


def _tiny_params(seed=3):
    rng = np.random.default_rng(seed)
    P = {}
    for i in range(3):
        P[f"tower_norm{i}"] = rng.uniform(0.5, 1.5, D)
        P[f"tower_w{i}"] = rng.normal(0, 0.6, (T, D))
        P[f"tower_b{i}"] = rng.uniform(-0.3, 0.3, T)
    P["fuse_w"] = rng.normal(0, 0.3, (T, 9 * T))
    P["fuse_b"] = rng.uniform(-0.3, 0.3, T)
    for j in range(2):
        P[f"ffn_norm{j}"] = rng.uniform(0.5, 1.5, T)
        P[f"ffn_gate{j}"] = rng.normal(0, 0.6, (F, T))
        P[f"ffn_up{j}"] = rng.normal(0, 0.6, (F, T))
        P[f"ffn_down{j}"] = rng.normal(0, 0.6, (T, F))
    P["out_norm"] = rng.uniform(0.5, 1.5, T)
    P["out_w"] = rng.normal(0, 0.6, T)
    P["out_b"] = np.array([0.1])
    return P


def _loss_via_forward(P, xs, p_full, p_local, valid, lam):
    q = [recall_head(P, xs[0][b], xs[1][b], xs[2][b]) for b in range(len(valid))]
    E = [b for b in range(len(valid)) if valid[b]]
    if not E:
        return 0.0
    tot = 0.0
    for b in E:
        y = labels.label(labels.penalised(labels.gain(p_full[b], p_local[b]), lam))
        tot += labels.huber(q[b] - y)
    return tot / len(E)


def test_backward_matches_finite_differences_on_every_parameter():
    P = _tiny_params()
    rng = np.random.default_rng(11)
    B = 3
    xs = [rng.normal(0, 1, (B, D)) for _ in range(3)]
    p_full = np.array([0.6, 0.2, 0.7])
    p_local = np.array([0.3, 0.25, 0.1])
    valid = [1, 1, 0]
    lam = 0.01
    loss, q, y, G = head_grad.loss_and_grad(P, xs[0], xs[1], xs[2], p_full, p_local, valid, lam)
    assert abs(loss - _loss_via_forward(P, xs, p_full, p_local, valid, lam)) < 1e-12
    h = 1e-6
    worst = 0.0
    for name, w in P.items():
        flat = w.reshape(-1)
        g = G[name].reshape(-1)
        for k in range(flat.size):
            old = flat[k]
            flat[k] = old + h
            lp = _loss_via_forward(P, xs, p_full, p_local, valid, lam)
            flat[k] = old - h
            lm = _loss_via_forward(P, xs, p_full, p_local, valid, lam)
            flat[k] = old
            fd = (lp - lm) / (2 * h)
            err = abs(fd - g[k]) / max(1e-3, abs(fd))
            worst = max(worst, err)
            assert err < 1e-5, (name, k, fd, g[k])
    assert worst < 1e-5


def test_interaction_kink_uses_sign_zero():
    """Equal tower outputs make |u_a - u_b| non-differentiable; the oracle takes sign(0) = 0, so
    the absolute-difference blocks contribute nothing to du there."""
    P = _tiny_params(5)
    P["tower_w1"] = P["tower_w0"].copy()
    P["tower_b1"] = P["tower_b0"].copy()
    P["tower_norm1"] = P["tower_norm0"].copy()
    x = np.random.default_rng(2).normal(0, 1, (1, D))
    A = head_grad.forward_saved(P, x[0], x[0], np.ones(D))
    assert np.array_equal(A["u"][0], A["u"][1])
    G = head_grad.backward(P, A, 1.0)
    # the tower-0 and tower-1 gradients differ only through their roles in the products
    assert np.all(np.isfinite(G["tower_w0"])) and np.all(np.isfinite(G["tower_w1"]))


def test_labels_and_huber_derivative_hand_cases():
    # p^F = 0.5, p^L = 0.25, lambda = 0: g = ln 2, y = 0.526589034 (method notes eqs. g_t, y_t)
    q = np.array([2.0, 0.5, -3.0, 7.0])
    pf = np.array([0.5, 0.5, 0.1, 0.9])
    pl = np.array([0.25, 0.25, 0.2, 0.009])
    loss, y, dq = head_grad.labels_and_dq(q, pf, pl, [1, 1, 1, 0], 0.0)
    assert y[0] == pytest.approx(0.526589034, abs=1e-9)
    assert y[2] == pytest.approx(-0.526589034, abs=1e-9)
    assert y[3] == 0.0 and dq[3] == 0.0          # not in E: no label, no gradient
    r = q[:3] - y[:3]
    # Huber threshold 1: quadratic inside, linear outside; the derivative is clamp(r, -1, 1)
    assert dq[0] == pytest.approx(1.0 / 3)        # r = 1.47 > 1
    assert dq[1] == pytest.approx(r[1] / 3)       # |r| < 1
    assert dq[2] == pytest.approx(-1.0 / 3)       # r = -2.47 < -1
    want = ((abs(r[0]) - 0.5) + 0.5 * r[1] ** 2 + (abs(r[2]) - 0.5)) / 3
    assert loss == pytest.approx(want, rel=1e-12)


def test_no_valid_position_gives_zero_loss_and_gradient():
    P = _tiny_params()
    xs = [np.ones((2, D)) for _ in range(3)]
    loss, _, _, G = head_grad.loss_and_grad(P, xs[0], xs[1], xs[2], [0.5, 0.5], [0.4, 0.4], [0, 0], 0.0)
    assert loss == 0.0
    assert all(not np.any(g) for g in G.values())


def test_output_bias_gradient_is_the_sum_of_dq():
    P = _tiny_params(7)
    rng = np.random.default_rng(4)
    xs = [rng.normal(0, 1, (4, D)) for _ in range(3)]
    loss, q, y, G = head_grad.loss_and_grad(P, xs[0], xs[1], xs[2], [0.5, 0.3, 0.9, 0.2],
                                            [0.4, 0.6, 0.1, 0.2], [1, 1, 1, 1], 0.05)
    _, _, dq = head_grad.labels_and_dq(q, [0.5, 0.3, 0.9, 0.2], [0.4, 0.6, 0.1, 0.2], [1] * 4, 0.05)
    assert G["out_b"][0] == pytest.approx(dq.sum(), rel=1e-12)
