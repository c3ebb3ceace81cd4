"""Pins of oracle.head: the page's parameter count, closed forms, invariances, hand cases,
and a composition of torch.nn library modules on small widths."""
import json
import math
import os

import numpy as np
import pytest
import torch

from oracle import head as H
from workload import configs, inputs

FACTS = json.load(open(os.path.join(os.path.dirname(__file__), "golden", "page_facts.json")))


def _small_params(rng, D=8, T=4, F=6, scale=0.5):
    P = {}
    for i in range(3):
        P[f"tower_norm{i}"] = rng.uniform(0.5, 1.5, D)
        P[f"tower_w{i}"] = rng.standard_normal((T, D)) * scale
        P[f"tower_b{i}"] = rng.standard_normal(T) * 0.1
    P["fuse_w"] = rng.standard_normal((T, 9 * T)) * scale
    P["fuse_b"] = rng.standard_normal(T) * 0.1
    for j in range(2):
        P[f"ffn_norm{j}"] = rng.uniform(0.5, 1.5, T)
        P[f"ffn_gate{j}"] = rng.standard_normal((F, T)) * scale
        P[f"ffn_up{j}"] = rng.standard_normal((F, T)) * scale
        P[f"ffn_down{j}"] = rng.standard_normal((T, F)) * scale
    P["out_norm"] = rng.uniform(0.5, 1.5, T)
    P["out_w"] = rng.standard_normal(T)
    P["out_b"] = rng.standard_normal(1)
    return P


def test_parameter_count_is_page_value():
    P = inputs.head_weights(configs.cfg0())
    assert H.param_count(P) == FACTS["head_param_count_qwen3_1p7b"]["value"] == 28_325_889
    assert P["tower_w0"].shape == (FACTS["head_tower_width"]["value"],
                                   FACTS["head_input_width"]["value"])
    assert P["fuse_w"].shape[1] == FACTS["head_interaction_width"]["value"]
    assert inputs.head_param_count(4096) == 34_623_489


def test_zero_weights_give_output_bias():
    P = {k: np.zeros_like(v) for k, v in _small_params(np.random.default_rng(0)).items()}
    P["out_b"] = np.array([0.375])
    rng = np.random.default_rng(1)
    assert H.recall_head(P, *(rng.standard_normal(8) for _ in range(3))) == 0.375


def test_interaction_hand_case():
    u1, u2, u3 = np.array([1.0, -2.0]), np.array([3.0, 5.0]), np.array([-4.0, 0.5])
    z = H.interaction(u1, u2, u3)
    assert z.tolist() == [1, -2, 3, 5, -4, 0.5, 3, -10, -4, -1, -12, 2.5, 2, 7, 5, 2.5, 7, 4.5]


def test_tower_hand_case():
    # x = [2,-2,2,-2]: mean square 4 -> RMSNorm = [1,-1,1,-1]; W n = ln 3; SiLU(ln 3) = 0.75 ln 3
    x = np.array([2.0, -2.0, 2.0, -2.0])
    W = np.array([[math.log(3) / 2, -math.log(3) / 2, 0.0, 0.0]])
    u = H.tower(x, np.ones(4), W, np.zeros(1))
    assert abs(u[0] - 0.75 * math.log(3)) < 1e-6
    # bias and norm weight act: gamma = 2 doubles W n, bias shifts it
    u2 = H.tower(x, np.full(4, 2.0), W / 2, np.array([0.0]))
    assert abs(u2[0] - 0.75 * math.log(3)) < 1e-6
    u3 = H.tower(x, np.ones(4), np.zeros((1, 4)), np.array([math.log(3)]))
    assert abs(u3[0] - 0.75 * math.log(3)) < 1e-12


def test_gated_ffn_hand_case():
    f = np.array([1.0, -1.0])
    Wg = np.array([[math.log(3), 0.0]])
    Wu = np.array([[2.0, 0.0]])
    Wd = np.array([[1.0], [0.0]])
    out = H.gated_ffn_block(f, np.ones(2), Wg, Wu, Wd)
    assert abs(out[0] - (1.0 + 1.5 * math.log(3))) < 1e-5 and out[1] == -1.0


def test_silu_and_rmsnorm_closed_forms():
    assert H.silu(np.array([0.0]))[0] == 0.0
    assert abs(H.silu(np.array([math.log(3)]))[0] - 0.75 * math.log(3)) < 1e-15
    y = H.rmsnorm(np.array([3.0, 4.0]), eps=0.0)
    assert np.allclose(y, [3 / math.sqrt(12.5), 4 / math.sqrt(12.5)], atol=1e-15)


def test_input_scale_invariance():
    rng = np.random.default_rng(3)
    P = _small_params(rng)
    xs = [rng.standard_normal(8) for _ in range(3)]
    q0 = H.recall_head(P, *xs)
    for i in range(3):
        ys = list(xs)
        ys[i] = xs[i] * 3.0
        assert abs(H.recall_head(P, *ys) - q0) < 1e-5 * max(1.0, abs(q0))


def test_every_parameter_matters():
    rng = np.random.default_rng(4)
    P = _small_params(rng)
    xs = [rng.standard_normal(8) for _ in range(3)]
    q0 = H.recall_head(P, *xs)
    for name in P:
        Q = dict(P)
        Q[name] = P[name] + 0.3 * np.sign(rng.standard_normal(P[name].shape)) + 0.05
        assert abs(H.recall_head(Q, *xs) - q0) > 1e-9, name


def test_input_order_matters():
    rng = np.random.default_rng(5)
    P = _small_params(rng)
    a, b, c = (rng.standard_normal(8) for _ in range(3))
    assert abs(H.recall_head(P, a, b, c) - H.recall_head(P, c, b, a)) > 1e-9


def test_matches_torch_module_composition():
    """The same reading built from torch.nn.RMSNorm / nn.Linear / F.silu in fp64."""
    rng = np.random.default_rng(6)
    D, T, F = 8, 4, 6
    P = _small_params(rng, D, T, F)
    tt = lambda a: torch.tensor(a, dtype=torch.float64)  # noqa: E731

    def norm(w):
        m = torch.nn.RMSNorm(len(w), eps=1e-6, dtype=torch.float64)
        m.weight.data = tt(w)
        return m

    def lin(W, b=None):
        m = torch.nn.Linear(W.shape[1], W.shape[0], bias=b is not None, dtype=torch.float64)
        m.weight.data = tt(W)
        if b is not None:
            m.bias.data = tt(b)
        return m

    silu = torch.nn.functional.silu
    for trial in range(5):
        xs = [rng.standard_normal(D) * (trial + 1) for _ in range(3)]
        with torch.no_grad():
            u = [silu(lin(P[f"tower_w{i}"], P[f"tower_b{i}"])(norm(P[f"tower_norm{i}"])(tt(xs[i]))))
                 for i in range(3)]
            pairs = [(0, 1), (0, 2), (1, 2)]
            z = torch.cat(u + [u[a] * u[b] for a, b in pairs] + [(u[a] - u[b]).abs() for a, b in pairs])
            f = lin(P["fuse_w"], P["fuse_b"])(z) + (u[0] + u[1] + u[2]) / 3
            for j in range(2):
                m = norm(P[f"ffn_norm{j}"])(f)
                f = f + lin(P[f"ffn_down{j}"])(silu(lin(P[f"ffn_gate{j}"])(m)) * lin(P[f"ffn_up{j}"])(m))
            q = lin(P["out_w"][None], P["out_b"])(norm(P["out_norm"])(f))
        assert abs(float(q) - H.recall_head(P, *xs)) < 1e-12


def test_workload_weight_init_is_xavier():
    P = inputs.head_weights(configs.cfg0())
    a = math.sqrt(6.0 / (2048 + 1024))
    w = P["tower_w0"]
    assert w.min() >= -a and w.max() <= a and abs(w.std() - a / math.sqrt(3)) < 0.01 * a
    assert (P["fuse_b"] == 0).all() and (P["ffn_norm1"] == 1).all()
