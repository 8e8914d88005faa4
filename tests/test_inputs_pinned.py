"""The seeded synthetic inputs are the ones recorded in
tests/golden/input_sha256.txt (written by tests/golden/make_input_sha256.py):
the draw order and distributions of every workload are fixed, so every
recorded measurement and parity result refers to the same bytes."""

import os
import sys

import pytest

HERE = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, os.path.join(HERE, "golden"))

import make_input_sha256 as M  # noqa: E402

from ternary_weight_selective_b200 import synthetic as S  # noqa: E402


def _recorded():
    rows = {}
    with open(os.path.join(HERE, "golden", "input_sha256.txt")) as f:
        for line in f:
            if line.startswith("#") or not line.strip():
                continue
            name, hx, hw = line.split()
            rows[name] = (hx, hw)
    return rows


@pytest.mark.parametrize("name", ["tiny", "trissm", "trissm_decode", "trissm_block", "stack12"])
def test_inputs_match_recorded_digests(name):
    assert M.digests(S.WORKLOADS[name]) == _recorded()[name]


def test_every_workload_is_recorded():
    assert set(_recorded()) == set(S.WORKLOADS)
