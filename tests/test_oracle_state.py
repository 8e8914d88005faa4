"""Pins of the oracle's carried-state form (the decode step), CPU only.

Every stage of the mixer except the recurrence is token-local, and the
recurrence's only link between steps is the state h.  So running a sequence
in pieces, or one token at a time, with the state handed from piece to
piece must give exactly what one call over the whole sequence gives.  The
whole-sequence layer is pinned in test_oracle_scan.py; these tests tie the
new entry points to it."""

import numpy as np
import pytest

from oracle import bitssm_oracle as O
from ternary_weight_selective_b200 import synthetic as S


def _layer(act):
    if act == "A8":
        wl = S.Workload("st_a8", 2, 20, 64, 128, 16, 4, "f32", "A8")
    else:
        wl = S.Workload("st_a16", 2, 20, 128, 256, 16, 16, "bf16", "A16")
    x, layers = S.make_inputs(wl, seed=7)
    return x, O.TernaryLayer(layers[0], act)


@pytest.mark.parametrize("act", ["A8", "A16"])
def test_pieces_with_carried_state_equal_one_call(act):
    x, P = _layer(act)
    out_full, st_full = O.bitssm_layer(x, P)
    out_a, st_a = O.bitssm_layer(x[:, :7], P)
    out_b, st_b = O.bitssm_layer(x[:, 7:], P, st_a["h_last"])
    out_pieces = np.concatenate([out_a, out_b], axis=1)
    assert np.allclose(out_pieces, out_full, rtol=1e-12, atol=1e-14)
    assert np.allclose(st_b["h_last"], st_full["h_last"], rtol=1e-12, atol=1e-14)
    # a zero start state is the default
    out_z, _ = O.bitssm_layer(x, P, np.zeros_like(st_full["h_last"]))
    assert np.array_equal(out_z, out_full)


@pytest.mark.parametrize("act", ["A8", "A16"])
def test_decode_steps_equal_the_sequence(act):
    x, P = _layer(act)
    out_full, st_full = O.bitssm_layer(x, P)
    h = np.zeros_like(st_full["h_last"])
    for t in range(x.shape[1]):
        o_t, h = O.bitssm_step(x[:, t], P, h)
        assert np.allclose(o_t, out_full[:, t], rtol=1e-12, atol=1e-14)
    assert np.allclose(h, st_full["h_last"], rtol=1e-12, atol=1e-14)


def test_state_is_what_carries_history():
    # the same token after different histories gives different outputs,
    # and equal states give equal outputs
    x, P = _layer("A8")
    _, st = O.bitssm_layer(x[:, :5], P)
    o1, _ = O.bitssm_step(x[:, 5], P, st["h_last"])
    o0, _ = O.bitssm_step(x[:, 5], P, np.zeros_like(st["h_last"]))
    assert not np.allclose(o1, o0)
    o1b, _ = O.bitssm_step(x[:, 5], P, st["h_last"].copy())
    assert np.array_equal(o1, o1b)
