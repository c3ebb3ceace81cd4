"""Pins of oracle.sets against the page's set definition and the facts it prints."""
import json
import os

import pytest

from oracle.sets import full_set, local_set

FACTS = json.load(open(os.path.join(os.path.dirname(__file__), "golden", "page_facts.json")))


def test_page_constants():
    assert FACTS["sinks"]["value"] == 4 and FACTS["window"]["value"] == 2048


@pytest.mark.parametrize("t", [1, 2, 3, 4, 5, 16, 17, 2047, 2048, 2049, 2051, 2052])
def test_sets_coincide_up_to_2052(t):
    assert local_set(t) == full_set(t)


def test_first_differing_position_is_page_value():
    first = next(t for t in range(1, 4000) if local_set(t) != full_set(t))
    assert first == FACTS["first_position_where_sets_differ"]["value"] == 2053
    assert full_set(2053) - local_set(2053) == {5}


@pytest.mark.parametrize("t", [1, 3, 4, 5, 2052, 2053, 2054, 2060, 4100, 131073])
def test_local_size_and_subset(t):
    L, F = local_set(t), full_set(t)
    assert L <= F
    assert len(L) == min(t, 2052)
    assert t in L  # the window includes the current position


def test_hand_listed_sets():
    assert local_set(3) == {1, 2, 3}
    assert local_set(2060) == {1, 2, 3, 4} | set(range(13, 2061))
    assert local_set(5000) == {1, 2, 3, 4} | set(range(2953, 5001))
    assert local_set(2055) == {1, 2, 3, 4} | set(range(8, 2056))
    assert full_set(1) == {1}
