"""Pins of oracle.gate and oracle.labels: the page's rules and hand-worked closed forms."""
import json
import math
import os

import numpy as np
import pytest

from oracle import labels
from oracle.gate import route_full

G = os.path.join(os.path.dirname(__file__), "golden")
LAB = json.load(open(os.path.join(G, "labels.json")))
FACTS = json.load(open(os.path.join(G, "page_facts.json")))


def test_gate_rule():
    th = FACTS["theta_default"]["value"]
    assert route_full(1e-30, th) and not route_full(0.0, th) and not route_full(-0.0, th)
    assert not route_full(-1e-30, th)
    for bad in (float("nan"), float("inf"), float("-inf")):
        assert route_full(bad, th)
    assert not route_full(0.5, 0.5) and route_full(0.5000001, 0.5)
    assert route_full(np.float32("nan"))


@pytest.mark.parametrize("case", LAB["gain_cases"])
def test_gain_and_label_hand_cases(case):
    g = labels.gain(case["p_full"], case["p_local"])
    d = labels.penalised(g, case["lambda"])
    y = labels.label(d)
    assert abs(g - case["g"]) < 1e-15 and abs(d - case["d"]) < 1e-15 and abs(y - case["y"]) < 1e-15


def test_gain_sign_convention():
    # positive gain favours the full branch: it assigns the reference token more probability
    assert labels.gain(0.8, 0.2) > 0 > labels.gain(0.2, 0.8)
    assert labels.nll(0.25) - labels.nll(0.5) == pytest.approx(math.log(2), abs=1e-15)
    with pytest.raises(ValueError):
        labels.penalised(0.1, -0.5)


@pytest.mark.parametrize("case", LAB["huber_cases"])
def test_huber_hand_cases(case):
    assert labels.huber(case["r"]) == case["loss"]


def test_huber_loss_mean_over_valid_positions():
    q = [0.5, 2.0, -3.0, 100.0]
    y = [0.0, 0.0, 0.0, 0.0]
    valid = [True, True, True, False]   # the last position is excluded (e.g. sets coincide)
    assert labels.huber_loss(q, y, valid) == pytest.approx((0.125 + 1.5 + 2.5) / 3, abs=1e-15)
    assert labels.huber_loss(q, y, [False] * 4) == 0.0


def test_delta_F_reproduces_page_flops_fraction():
    rho = 0.125
    frac = FACTS["flops_fraction_at_rho_0p125"]["value"]
    overhead = frac - rho   # (F_L + F_R) / F_F implied by the page's 24.26%
    saving = labels.delta_F(rho, 1.0, overhead, 0.0)
    assert saving == pytest.approx(FACTS["flops_saving_at_rho_0p125"]["value"], abs=1e-12)
    assert labels.delta_F(1.0, 1.0, 0.1, 0.02) < 0   # all-full calls cost more than always-full


def test_routings_for_generated_tokens():
    assert labels.routed_steps(1024) == FACTS["generated_1024_routings"]["value"]
    assert labels.routed_steps(1) == 0
