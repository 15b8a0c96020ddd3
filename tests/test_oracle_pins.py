"""The CPU oracle against closed forms, invariants, textbook routines and
brute force (see oracle_pins.py); plus the spec constants printed on the pages."""
import json
import os

import pytest

import oracle
from oracle_pins import ALL_PINS

HERE = os.path.dirname(os.path.abspath(__file__))


@pytest.fixture(scope="module")
def O():
    return oracle.Oracle()


@pytest.mark.parametrize("pin", ALL_PINS, ids=[p.__name__ for p in ALL_PINS])
def test_pin(O, pin):
    pin(O)


def test_spec_constants_match_pages():
    spec = json.load(open(os.path.join(HERE, "golden", "qsa_spec.json")))
    P = oracle.params()
    assert P.n_q_heads == spec["n_q_heads"]["value"]
    assert P.n_kv_heads == spec["n_kv_heads"]["value"]
    assert P.head_dim == spec["head_dim"]["value"]
    assert P.rope_dim == spec["rope_dim"]["value"]
    assert P.rope_dim == spec["partial_rotary_factor"]["value"] * spec["head_dim"]["value"]
    assert P.rope_theta == spec["rope_theta"]["value"]
    assert P.idx_heads == spec["idx_heads"]["value"]
    assert P.idx_dim == spec["idx_dim"]["value"]
    assert P.block == spec["block_size"]["value"]
    assert P.budget == spec["budget_blocks"]["value"]
    assert P.budget * P.block == spec["budget_tokens"]["value"]
