"""Pins of the oracle's selective scan and mixer (CPU only): closed forms,
special cases, brute force, associativity, causality and segmenting."""

import math

import numpy as np

from oracle import bitssm_oracle as O
from ternary_weight_selective_b200 import synthetic as S


def test_softplus_special_values():
    assert abs(O.softplus(0.0) - math.log(2.0)) < 1e-16
    assert O.softplus(800.0) == 800.0
    z = -40.0
    assert abs(O.softplus(z) - math.exp(z)) / math.exp(z) < 1e-12
    zs = np.linspace(-30, 30, 2001)
    assert np.allclose(O.softplus(zs), np.logaddexp(0.0, zs), rtol=1e-14, atol=0)


def test_scan_geometric_closed_form():
    # constant a = exp(dt A), b = dt B u, h_0 = 0:  h_t = b (1 - a^t) / (1 - a)
    Bsz, L, E, N = 2, 50, 3, 4
    dt, u0, Bv, Cv = 0.05, 1.5, 0.7, -1.3
    A = -np.array([[1.0, 2.0, 4.0, 8.0]] * E)
    u = np.full((Bsz, L, E), u0)
    delta = np.full((Bsz, L, E), dt)
    Bm = np.full((Bsz, L, N), Bv)
    Cm = np.full((Bsz, L, N), Cv)
    D = np.full(E, 0.25)
    y, hL = O.selective_scan(u, delta, A, Bm, Cm, D)
    a = np.exp(dt * A[0])
    b = dt * Bv * u0
    for t in range(1, L + 1):
        h = b * (1 - a ** t) / (1 - a)
        ref = Cv * h.sum() + 0.25 * u0
        assert abs(y[0, t - 1, 0] - ref) < 1e-12 * max(1.0, abs(ref))
    assert np.allclose(hL[1, 2], b * (1 - a ** L) / (1 - a), rtol=1e-12)


def test_scan_A_zero_is_prefix_sum_and_C_zero_is_skip():
    u, dr, bias, A, Bm, Cm, D = S.random_scan_inputs(1, 2, 40, 6, 5)
    delta = O.softplus(dr + bias)
    y, h = O.selective_scan(u, delta, np.zeros_like(A), Bm, Cm, D)
    pref = np.cumsum(delta[..., None] * Bm[:, :, None, :] * u[..., None], axis=1)  # [B,L,E,N]
    ref = (pref * Cm[:, :, None, :]).sum(-1) + D * u
    assert np.allclose(y, ref, rtol=1e-12, atol=1e-12)
    y0, _ = O.selective_scan(u, delta, A, Bm, np.zeros_like(Cm), D)
    assert np.array_equal(y0, D * u.astype(np.float64))


def test_scan_brute_force_tiny():
    # pure-Python loops with math.exp, one state at a time
    u, dr, bias, A, Bm, Cm, D = S.random_scan_inputs(2, 1, 3, 2, 2)
    delta = O.softplus(dr + bias)
    y, _ = O.selective_scan(u, delta, A, Bm, Cm, D)
    for e in range(2):
        h = [0.0, 0.0]
        for t in range(3):
            dt = float(delta[0, t, e])
            acc = 0.0
            for n in range(2):
                h[n] = math.exp(dt * float(A[e, n])) * h[n] + dt * float(Bm[0, t, n]) * float(u[0, t, e])
                acc += float(Cm[0, t, n]) * h[n]
            ref = acc + float(D[e]) * float(u[0, t, e])
            assert abs(y[0, t, e] - ref) < 1e-14 * (1 + abs(ref))


def test_associative_scan_equals_sequential():
    for (Bsz, L, E, N, chunk, seed) in [(2, 64, 8, 16, 16, 3), (1, 37, 5, 3, 8, 4), (3, 5, 4, 16, 16, 5)]:
        u, dr, bias, A, Bm, Cm, D = S.random_scan_inputs(seed, Bsz, L, E, N)
        delta = O.softplus(dr + bias)
        h0 = np.random.default_rng(seed).normal(size=(Bsz, E, N))
        for init in (None, h0):
            y1, h1 = O.selective_scan(u, delta, A, Bm, Cm, D, init)
            y2, h2 = O.selective_scan_associative(u, delta, A, Bm, Cm, D, init, chunk=chunk)
            scale = np.abs(y1).max()
            assert np.abs(y1 - y2).max() <= 1e-12 * scale
            assert np.abs(h1 - h2).max() <= 1e-12 * np.abs(h1).max()


def test_scan_causality_and_segmenting():
    u, dr, bias, A, Bm, Cm, D = S.random_scan_inputs(6, 2, 60, 4, 16)
    delta = O.softplus(dr + bias)
    y, hL = O.selective_scan(u, delta, A, Bm, Cm, D)
    t0 = 33
    u2, Bm2 = u.copy(), Bm.copy()
    u2[:, t0] += 5.0
    Bm2[:, t0] -= 2.0
    y2, _ = O.selective_scan(u2, delta, A, Bm2, Cm, D)
    assert np.array_equal(y[:, :t0], y2[:, :t0])
    assert not np.allclose(y[:, t0:], y2[:, t0:])
    ya, ha = O.selective_scan(u[:, :25], delta[:, :25], A, Bm[:, :25], Cm[:, :25], D)
    yb, hb = O.selective_scan(u[:, 25:], delta[:, 25:], A, Bm[:, 25:], Cm[:, 25:], D, ha)
    assert np.allclose(np.concatenate([ya, yb], 1), y, rtol=1e-13, atol=1e-13)
    assert np.allclose(hb, hL, rtol=1e-13, atol=1e-13)


def _tiny_layer(act="A8"):
    wl = S.WORKLOADS["tiny"]
    x, layers = S.make_inputs(wl, seed=0)
    return x, O.TernaryLayer(layers[0], act)


def test_layer_shapes_and_integer_stages():
    x, P = _tiny_layer()
    out, st = O.bitssm_layer(x, P)
    assert out.shape == x.shape
    for k in ("q_x", "q_u", "q_dt", "q_y"):
        assert st[k].min() >= -128 and st[k].max() <= 127
    assert st["q_u"].shape == (64, 128) and st["q_dt"].shape == (64, 4)
    assert (st["delta"] > 0).all()


def test_layer_causality_and_batch_independence():
    wl = S.WORKLOADS["tiny"]
    x, layers = S.make_inputs(wl, seed=1, batch=3, seqlen=40)
    for act in ("A8", "A16"):
        P = O.TernaryLayer(layers[0], act)
        out, _ = O.bitssm_layer(x, P)
        x2 = x.copy()
        x2[1, 20] += 3.0
        out2, _ = O.bitssm_layer(x2, P)
        assert np.array_equal(out[:, :20], out2[:, :20])
        assert np.array_equal(out[0], out2[0]) and np.array_equal(out[2], out2[2])
        assert not np.allclose(out[1, 20:], out2[1, 20:])


def test_stack_one_layer_is_residual_layer():
    x, P = _tiny_layer()
    out, _ = O.bitssm_layer(x, P)
    h, ins = O.bitssm_stack(x, [P], io_bf16=False)
    assert np.array_equal(h, x + out) and len(ins) == 1


def test_layer_wiring_special_cases():
    """Structural pins of the mixer's wiring: the x_proj slices equal the
    separate projections, equal weights give equal B and C, a zero Delta-up
    leaves Delta = softplus(bias), and zero C with D = 0 silences the output."""
    import copy
    wl = S.WORKLOADS["tiny"]
    x, layers = S.make_inputs(wl, seed=2)
    lw = copy.deepcopy(layers[0])
    lw.W_C = lw.W_B.copy()
    lw.W_dt_up = np.zeros_like(lw.W_dt_up)
    P = O.TernaryLayer(lw)
    out, st = O.bitssm_layer(x, P)
    assert np.array_equal(st["Bm"], st["Cm"])
    assert np.allclose(st["delta"], O.softplus(P.dt_bias)[None].repeat(64, 0), rtol=0, atol=0)
    c_u = float(P.s["W_in"]) * st["deq_x"]
    for name, sl in (("W_dt_down", slice(0, 4)), ("W_B", slice(4, 20)), ("W_C", slice(20, 36))):
        sep, _ = O.bitlinear_a8_int_input(st["acc_in"], c_u, P.Wq[name], P.s[name])
        full = st["dt_low"] if name == "W_dt_down" else st["Bm" if name == "W_B" else "Cm"]
        assert np.allclose(sep, full, rtol=1e-14, atol=0)
        assert np.array_equal(st["acc_x"][:, sl], O.int_gemm(st["q_u"], P.Wq[name]))
    lw2 = copy.deepcopy(layers[0])
    lw2.W_C = np.zeros_like(lw2.W_C)
    lw2.D = np.zeros_like(lw2.D)
    out2, st2 = O.bitssm_layer(x, O.TernaryLayer(lw2))
    assert not st2["y"].any() and not out2.any()
