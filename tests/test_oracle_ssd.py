"""Pins of the SSD scan oracle (Mamba-2's scalar-decay-per-head selective
recurrence), CPU only.

The three evaluations (step by step, attention form, chunked) are different
algorithms and are held to one another; the recurrence itself is held to
the mixer's already-pinned selective scan (with the per-head decay and step
broadcast over the head's channels and states), to a cumulative sum when the
decay is zero, and to the geometric series for constant inputs.  A wrong
decay index (cum[t] - cum[s] off by one step), a missing dt on the input, a
head mapped to the wrong B/C group or a dropped carried state fails here."""

import numpy as np
import pytest

from oracle import bitssm_oracle as O
from oracle import ssd_oracle as SSD


def _inputs(seed, Bsz=2, L=37, H=4, P=3, G=2, N=5):
    rng = np.random.default_rng(seed)
    x = rng.normal(size=(Bsz, L, H, P))
    dt = np.log1p(np.exp(rng.normal(-1.0, 1.0, size=(Bsz, L, H))))   # softplus > 0
    A = -np.exp(rng.uniform(0.0, np.log(8.0), size=(H,)))
    Bm = rng.normal(size=(Bsz, L, G, N))
    Cm = rng.normal(size=(Bsz, L, G, N))
    D = rng.normal(size=(H,))
    return x, dt, A, Bm, Cm, D


@pytest.mark.parametrize("Q", [1, 3, 16, 64])
def test_chunked_equals_sequential(Q):
    args = _inputs(1)
    y_s, S_s = SSD.ssd_sequential(*args)
    y_c, S_c = SSD.ssd_chunked(*args, Q=Q)
    np.testing.assert_allclose(y_c, y_s, rtol=1e-11, atol=1e-12)
    np.testing.assert_allclose(S_c, S_s, rtol=1e-11, atol=1e-12)


def test_quadratic_equals_sequential():
    args = _inputs(2, L=23)
    y_s, _ = SSD.ssd_sequential(*args)
    y_q = SSD.ssd_quadratic(*args)
    np.testing.assert_allclose(y_q, y_s, rtol=1e-11, atol=1e-12)


def test_zero_decay_is_a_cumulative_sum():
    x, dt, A, Bm, Cm, D = _inputs(3, G=1)
    A = np.zeros_like(A)
    y, _ = SSD.ssd_sequential(x, dt, A, Bm, Cm, D)
    # S_t = sum_{s <= t} dt_s x_s (outer) B_s
    terms = (dt[..., None] * x)[..., None] * Bm[:, :, 0, None, None, :]   # [B, L, H, P, N]
    S = np.cumsum(terms, axis=1)
    ref = np.einsum("blhpn,bln->blhp", S, Cm[:, :, 0, :]) + D[None, None, :, None] * x
    np.testing.assert_allclose(y, ref, rtol=1e-12, atol=1e-12)


@pytest.mark.parametrize("G", [1, 2])
def test_equals_mixer_scan_with_broadcast_decay(G):
    """Head h, channel p is channel e = h*P + p of the mixer's scan with
    A[e, n] = A[h] and delta[e] = dt[h]; heads of group g read group g's B, C."""
    Bsz, L, H, P, N = 2, 19, 4, 3, 16
    x, dt, A, Bm, Cm, D = _inputs(4, Bsz, L, H, P, G, N)
    y, S = SSD.ssd_sequential(x, dt, A, Bm, Cm, D)
    per = H // G
    for g in range(G):
        hs = slice(g * per, (g + 1) * per)
        E = per * P
        u = x[:, :, hs, :].reshape(Bsz, L, E)
        delta = np.repeat(dt[:, :, hs], P, axis=2)
        A_e = np.repeat(A[hs], P)[:, None] * np.ones((1, N))
        D_e = np.repeat(D[hs], P)
        y_ref, h_ref = O.selective_scan(u, delta, A_e, Bm[:, :, g, :], Cm[:, :, g, :], D_e)
        np.testing.assert_allclose(y[:, :, hs, :].reshape(Bsz, L, E), y_ref, rtol=1e-12, atol=1e-12)
        np.testing.assert_allclose(S[:, hs].reshape(Bsz, E, N), h_ref, rtol=1e-12, atol=1e-12)


def test_geometric_series_for_constant_inputs():
    L = 30
    xv, dtv, Av, Bv, Cv, Dv = 0.7, 0.3, -0.9, 1.3, -0.4, 0.25
    x = np.full((1, L, 1, 1), xv)
    dt = np.full((1, L, 1), dtv)
    y, _ = SSD.ssd_chunked(x, dt, np.array([Av]), np.full((1, L, 1, 1), Bv),
                           np.full((1, L, 1, 1), Cv), np.array([Dv]), Q=8)
    a = np.exp(dtv * Av)
    t = np.arange(1, L + 1)
    S = dtv * xv * Bv * (1 - a ** t) / (1 - a)
    np.testing.assert_allclose(y[0, :, 0, 0], Cv * S + Dv * xv, rtol=1e-13)


@pytest.mark.parametrize("cut", [1, 16, 20])
def test_carried_state_splits_the_sequence(cut):
    x, dt, A, Bm, Cm, D = _inputs(5)
    y_all, S_all = SSD.ssd_chunked(x, dt, A, Bm, Cm, D, Q=8)
    y1, S1 = SSD.ssd_chunked(x[:, :cut], dt[:, :cut], A, Bm[:, :cut], Cm[:, :cut], D, Q=8)
    y2, S2 = SSD.ssd_chunked(x[:, cut:], dt[:, cut:], A, Bm[:, cut:], Cm[:, cut:], D, Q=8, S0=S1)
    np.testing.assert_allclose(np.concatenate([y1, y2], axis=1), y_all, rtol=1e-11, atol=1e-12)
    np.testing.assert_allclose(S2, S_all, rtol=1e-11, atol=1e-12)
    y3, _ = SSD.ssd_sequential(x[:, cut:], dt[:, cut:], A, Bm[:, cut:], Cm[:, cut:], D, S0=S1)
    np.testing.assert_allclose(y3, y_all[:, cut:], rtol=1e-11, atol=1e-12)


def test_causal():
    x, dt, A, Bm, Cm, D = _inputs(6)
    y0, _ = SSD.ssd_chunked(x, dt, A, Bm, Cm, D, Q=4)
    x2 = x.copy()
    x2[1, 10] += 3.0
    y1, _ = SSD.ssd_chunked(x2, dt, A, Bm, Cm, D, Q=4)
    assert np.array_equal(y0[0], y1[0])
    assert np.array_equal(y0[1, :10], y1[1, :10])
    assert not np.allclose(y0[1, 10:], y1[1, 10:])
