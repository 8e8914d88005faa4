"""Pins of the oracle's Mamba-1 block form (conv1d, SiLU, z gate), CPU only.

The conv is pinned to numpy's own convolution, the SiLU to scipy's logistic
function, and the whole block to a second, loop-by-loop restatement on a tiny
input (every index written out, nothing vectorised), so that a shifted or
reversed conv tap, a gate taken from the wrong branch, a dropped bias or a
transposed projection fails here.  Degenerate cases: a one-hot conv is a pure
delay, an all-zero gate branch zeroes the output, and the block is causal."""

import math

import numpy as np
import pytest
from scipy.special import expit

from oracle import bitssm_oracle as O
from ternary_weight_selective_b200 import synthetic as S


@pytest.mark.parametrize("K", [1, 2, 3, 4])
@pytest.mark.parametrize("L", [1, 3, 17])
def test_conv_matches_numpy_convolve(K, L):
    rng = np.random.default_rng(10 * K + L)
    E = 5
    v = rng.normal(size=(2, L, E))
    w = rng.normal(size=(E, K))
    b = rng.normal(size=(E,))
    out = O.causal_conv1d(v, w, b)
    for bi in range(2):
        for e in range(E):
            # np.convolve(a, k)[n] = sum_m a[m] k[n - m]: the causal filter
            # with the current step on tap K-1 is the reversed tap vector
            ref = np.convolve(v[bi, :, e], w[e, ::-1])[:L] + b[e]
            np.testing.assert_allclose(out[bi, :, e], ref, rtol=1e-13, atol=1e-13)


@pytest.mark.parametrize("tap", [0, 1, 2, 3])
def test_one_hot_conv_is_a_delay(tap):
    rng = np.random.default_rng(3)
    K, L, E = 4, 9, 6
    v = rng.normal(size=(1, L, E))
    w = np.zeros((E, K))
    w[:, tap] = 1.0
    out = O.causal_conv1d(v, w, None)
    shift = K - 1 - tap
    ref = np.zeros_like(v)
    ref[:, shift:] = v[:, :L - shift]
    assert np.array_equal(out, ref)


def test_conv_is_causal():
    rng = np.random.default_rng(4)
    v = rng.normal(size=(1, 12, 3))
    w = rng.normal(size=(3, 4))
    base = O.causal_conv1d(v, w, None)
    v2 = v.copy()
    v2[0, 7] += 5.0
    moved = O.causal_conv1d(v2, w, None)
    assert np.array_equal(base[0, :7], moved[0, :7])
    assert not np.array_equal(base[0, 7:11], moved[0, 7:11])   # taps reach 3 steps ahead
    assert np.array_equal(base[0, 11:], moved[0, 11:])


def test_silu_against_scipy_and_limits():
    v = np.concatenate([np.linspace(-40, 40, 801), [-1e4, -745.0, 0.0, 745.0, 1e4]])
    with np.errstate(over="raise", invalid="raise", divide="raise"):
        got = O.silu(v)
    np.testing.assert_allclose(got, v * expit(v), rtol=1e-14, atol=1e-300)
    assert O.silu(np.array(0.0)) == 0.0
    assert O.silu(np.array(1e4)) == 1e4
    assert O.silu(np.array(-1e4)) == 0.0


# ---------------------------------------------------------------- the block

def _tiny_block(seed=21, K=3):
    wl = S.Workload("blk_tiny", 2, 6, 8, 12, 4, 2, "f32", "A8", block=True, d_conv=K)
    x, layers = S.make_inputs(wl, seed=seed)
    return x, O.TernaryLayer(layers[0], "A8")


def _codes(row):
    """int8 absmax codes of a row decided in float32, its max and the
    dequantisation factor of the unit-gain-normalised row."""
    r32 = [np.float32(v) for v in row]
    m = max(abs(v) for v in r32)
    if m == 0:
        q = [0] * len(row)
    else:
        sig = np.float32(127.0) / np.float32(m)
        q = [int(np.rint(np.float32(v * sig))) for v in r32]
    ms = sum(float(v) * float(v) for v in row) / len(row)
    return q, float(m), float(m) / math.sqrt(ms + 1e-5) / 127.0


def _silu(v):
    return v / (1.0 + math.exp(-v)) if v >= 0 else v * math.exp(v) / (1.0 + math.exp(v))


def _softplus(v):
    return max(v, 0.0) + math.log1p(math.exp(-abs(v)))


def _brute_block(x, P):
    """The block written out loop by loop (B, L, channels, taps, states)."""
    Bsz, L, d = x.shape
    Win, Wz, Wdt, WB, WC, Wup, Wout = (P.Wq[n].astype(int) for n in
                                       ("W_in", "W_z", "W_dt_down", "W_B", "W_C", "W_dt_up", "W_out"))
    s = {n: float(P.s[n]) for n in P.s}
    E, K = P.conv_w.shape
    R, N = P.R, P.N
    out = np.zeros((Bsz, L, d))
    for b in range(Bsz):
        u_pre = [[0.0] * E for _ in range(L)]
        z = [[0.0] * E for _ in range(L)]
        for t in range(L):
            q, _, deq = _codes(list(x[b, t]))
            for e in range(E):
                u_pre[t][e] = sum(q[k] * Win[e][k] for k in range(d)) * s["W_in"] * deq
                z[t][e] = sum(q[k] * Wz[e][k] for k in range(d)) * s["W_z"] * deq
        u = [[0.0] * E for _ in range(L)]
        for t in range(L):
            for e in range(E):
                acc = float(P.conv_b[e])
                for back in range(K):            # back = steps into the past
                    if t - back >= 0:
                        acc += float(P.conv_w[e][K - 1 - back]) * u_pre[t - back][e]
                u[t][e] = _silu(acc)
        h = [[0.0] * N for _ in range(E)]
        for t in range(L):
            qu, _, deq_u = _codes(u[t])
            acc_dt = [sum(qu[k] * Wdt[j][k] for k in range(E)) for j in range(R)]
            Bt = [sum(qu[k] * WB[n][k] for k in range(E)) * s["W_B"] * deq_u for n in range(N)]
            Ct = [sum(qu[k] * WC[n][k] for k in range(E)) * s["W_C"] * deq_u for n in range(N)]
            # Delta-up on the integer Delta-down row: codes of the integer row,
            # dequantisation of the real row c * acc_dt
            c = s["W_dt_down"] * deq_u
            qd, md, _ = _codes([float(a) for a in acc_dt])
            ms = sum((c * a) ** 2 for a in acc_dt) / R
            deq_dt = c * md / math.sqrt(ms + 1e-5) / 127.0
            yg = [0.0] * E
            for e in range(E):
                draw = sum(qd[j] * Wup[e][j] for j in range(R)) * s["W_dt_up"] * deq_dt
                dl = _softplus(draw + float(P.dt_bias[e]))
                y = float(P.D[e]) * u[t][e]
                for n in range(N):
                    h[e][n] = math.exp(dl * float(P.A[e][n])) * h[e][n] + dl * Bt[n] * u[t][e]
                    y += Ct[n] * h[e][n]
                yg[e] = y * _silu(z[t][e])
            qy, _, deq_y = _codes(yg)
            for j in range(d):
                out[b, t, j] = sum(qy[k] * Wout[j][k] for k in range(E)) * s["W_out"] * deq_y
    return out


@pytest.mark.parametrize("K", [2, 4])
def test_block_matches_loop_restatement(K):
    x, P = _tiny_block(seed=20 + K, K=K)
    got, st = O.bitssm_block_a8(x, P)
    ref = _brute_block(x, P)
    np.testing.assert_allclose(got, ref, rtol=1e-11, atol=1e-13)
    assert np.abs(got).max() > 0


def test_block_zero_gate_branch_gives_zero_output():
    x, P = _tiny_block()
    P.Wq["W_z"] = np.zeros_like(P.Wq["W_z"])
    out, st = O.bitssm_block_a8(x, P)
    assert np.all(st["z"] == 0) and np.all(st["yg"] == 0)
    assert np.all(out == 0)


def test_block_is_causal_and_sequences_independent():
    x, P = _tiny_block(seed=5, K=4)
    base, _ = O.bitssm_block_a8(x, P)
    x2 = x.copy()
    x2[1, 3] += 1.0
    moved, _ = O.bitssm_block_a8(x2, P)
    assert np.array_equal(base[0], moved[0])           # the other sequence
    assert np.array_equal(base[1, :3], moved[1, :3])   # earlier steps
    assert not np.array_equal(base[1, 3:], moved[1, 3:])


def test_block_refuses_carried_state_and_a16():
    x, P = _tiny_block()
    with pytest.raises(NotImplementedError):
        O.bitssm_layer(x, P, np.zeros((2, 12, 4)))
    out, _ = O.bitssm_layer(x, P)                      # dispatches to the block
    assert np.array_equal(out, O.bitssm_block_a8(x, P)[0])
