"""Routing gate.  [notes §2.3, first paragraph]: after the local pass the score is computed;
by default the full pass is re-run only when the score exceeds zero (theta = 0), and a
non-finite score falls back to the full pass.  The rule is strict (q = theta routes local).
"""
import math


def route_full(q: float, theta: float = 0.0) -> bool:
    q = float(q)
    if math.isnan(q) or math.isinf(q):
        return True
    return q > theta
