"""The C host oracle (oracle/c/, entry points prefixed `oracle_`) held to
the numpy oracle and to closed forms, CPU only.

The two oracles are written separately (plain C loops against numpy array
code); every integer result (ternary codes, scales, packed bytes, activation
codes) must agree bit for bit and every float64 result to 1e-12, on the
mixer's shapes in both activation modes, with and without a carried state.
The scan is also pinned directly to the geometric series and to a cumulative
sum."""

import numpy as np
import pytest

from oracle import bitssm_oracle as O
from oracle import c_oracle as C
from oracle import ssd_oracle as SSD
from ternary_weight_selective_b200 import synthetic as S
from tests._helpers import rel_err


@pytest.mark.parametrize("n,k,group", [(16, 64, 0), (33, 200, 128), (8, 512, 128), (5, 7, 0)])
def test_ternarisation_and_packing_bit_exact(n, k, group):
    W = np.random.default_rng(n * k).normal(0, 0.02, size=(n, k)).astype(np.float32)
    Wq_c, s_c = C.absmean_ternary(W, group)
    Wq_n, s_n = O.absmean_ternary(W, group)
    assert np.array_equal(Wq_c, Wq_n)
    assert np.array_equal(np.asarray(s_c, np.float32), np.asarray(s_n, np.float32))
    assert np.array_equal(C.pack_ternary(Wq_c), O.pack_ternary(Wq_n))


def test_pack_hand_example():
    # codes w + 1 = [0, 1, 2, 2] -> 0 | 1 << 2 | 2 << 4 | 2 << 6 = 164; a lone
    # element pads with code 1: 2 | 1 << 2 | 1 << 4 | 1 << 6 = 86
    assert C.pack_ternary(np.array([[-1, 0, 1, 1, 1]], np.int8)).tolist() == [[164, 86]]


def test_activation_codes_bit_exact():
    v = S.random_rows(3, 40, 96, scale=3.0, zero_rows=(5,))
    v[7, :4] = [0.5, -1.5, 2.5, 127.0]       # ties at .5 after the scale 127/127
    q_c, m_c = C.absmax_codes(v)
    q_n, m_n = O.absmax_codes(v)
    assert np.array_equal(q_c, q_n) and np.array_equal(m_c, m_n)
    assert not q_c[5].any() and q_c[7, :4].tolist() == [0, -2, 2, 127]


@pytest.mark.parametrize("act", ["A8", "A16"])
def test_bitlinear_matches_numpy(act):
    rng = np.random.default_rng(11)
    x = S.round_to_bf16(rng.normal(size=(37, 256)).astype(np.float32))
    W = rng.normal(0, 0.02, size=(48, 256)).astype(np.float32)
    group = 0 if act == "A8" else 128
    Wq, s = O.absmean_ternary(W, group)
    y_c = C.bitlinear(x, Wq, s, group, 0 if act == "A8" else 1)
    y_n = (O.bitlinear_a8(x, Wq, s)[0] if act == "A8"
           else O.bitlinear_a16(x, Wq, s, group))
    assert rel_err(y_c, y_n) <= 1e-12


def test_scan_matches_numpy_and_closed_forms():
    u, draw, bias, A, Bm, Cm, D = S.random_scan_inputs(4, 2, 30, 24, 16)
    delta = O.softplus(draw + bias[None, None, :])
    h0 = np.random.default_rng(5).normal(size=(2, 24, 16))
    y_c, h_c = C.selective_scan(u, delta, A, Bm, Cm, D, h0)
    y_n, h_n = O.selective_scan(u, delta, A, Bm, Cm, D, h0)
    assert rel_err(y_c, y_n) <= 1e-12 and rel_err(h_c, h_n) <= 1e-12
    # constant inputs: h_t = b (1 - a^t) / (1 - a)
    L = 25
    dv, av, bv, cv, uv = 0.2, -0.7, 1.1, 0.9, -0.6
    ones = np.ones((1, L, 1))
    y, _ = C.selective_scan(uv * ones, dv * ones, np.array([[av]]), bv * ones, cv * ones,
                            np.array([0.5]))
    a = np.exp(dv * av)
    t = np.arange(1, L + 1)
    h = dv * bv * uv * (1 - a ** t) / (1 - a)
    np.testing.assert_allclose(y[0, :, 0], cv * h + 0.5 * uv, rtol=1e-13)
    # zero decay: a prefix sum
    y0, _ = C.selective_scan(u, delta, np.zeros_like(A), Bm, Cm, np.zeros_like(D))
    hs = np.cumsum(delta[..., None] * Bm[:, :, None, :] * u[..., None], axis=1)
    np.testing.assert_allclose(y0, (hs * Cm[:, :, None, :]).sum(-1), rtol=1e-11, atol=1e-12)


@pytest.mark.parametrize("name,act,B,L", [("tiny", "A8", 1, 64), ("trissm", "A8", 2, 40),
                                          ("a16", "A16", 2, 24)])
def test_mixer_matches_numpy(name, act, B, L):
    if name == "a16":
        wl = S.Workload("a16_small", 2, 24, 256, 512, 16, 16, "bf16", "A16")
    else:
        wl = S.WORKLOADS[name]
    x, layers = S.make_inputs(wl, seed=9, batch=B, seqlen=L)
    Pn = O.TernaryLayer(layers[0], act)
    Pc = C.Layer(layers[0], act)
    h0 = np.random.default_rng(6).normal(size=(B, wl.d_inner, wl.d_state)) * 0.1
    out_c, h_c = C.bitssm_forward(x, Pc, h0)
    out_n, st = O.bitssm_layer(x, Pn, h0)
    assert rel_err(out_c, out_n) <= 1e-12
    assert rel_err(h_c, st["h_last"]) <= 1e-12
    out_c0, _ = C.bitssm_forward(x, Pc)
    out_n0, _ = O.bitssm_layer(x, Pn)
    assert rel_err(out_c0, out_n0) <= 1e-12


def test_invalid_arguments_are_refused():
    with pytest.raises(ValueError):
        C.bitlinear(np.zeros((2, 8), np.float32), np.zeros((4, 8), np.int8), np.ones(1), 128, 0)
    with pytest.raises(ValueError):
        C.absmean_ternary(np.zeros((0, 4), np.float32))


@pytest.mark.parametrize("K,B,L", [(4, 2, 30), (2, 1, 3), (3, 2, 1)])
def test_block_form_matches_numpy(K, B, L):
    wl = S.Workload("blk_c", B, L, 64, 128, 16, 4, "f32", "A8", block=True, d_conv=K)
    x, layers = S.make_inputs(wl, seed=K * 10 + L)
    out_c, h_c = C.bitssm_forward(x, C.Layer(layers[0], "A8"))
    out_n, st = O.bitssm_block_a8(x, O.TernaryLayer(layers[0], "A8"))
    assert rel_err(out_c, out_n) <= 1e-12
    assert rel_err(h_c, st["h_last"]) <= 1e-12
    # the block form has no carried-state form
    with pytest.raises(ValueError):
        C.bitssm_forward(x, C.Layer(layers[0], "A8"), np.zeros((B, 128, 16)))


@pytest.mark.parametrize("G", [1, 2])
def test_ssd_scan_matches_numpy(G):
    args = S.random_ssd_inputs(G, 2, 21, 4, 8, G, 16)
    S0 = np.random.default_rng(2).normal(size=(2, 4, 8, 16))
    y_c, s_c = C.ssd_scan(*args, S0=S0)
    y_n, s_n = SSD.ssd_sequential(*args, S0=S0)
    assert rel_err(y_c, y_n) <= 1e-12 and rel_err(s_c, s_n) <= 1e-12

