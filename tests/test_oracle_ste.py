"""Pins of the straight-through-estimator backward oracle (oracle/ste_oracle.py),
CPU only.

* With the quantisers off the layer is smooth, and every gradient autograd
  gives must match central finite differences of the forward (a different
  computation: no autograd).
* One BitLinear with the quantisers on: the gradients match their closed
  forms, dW = g^T a (a = the dequantised activations) and
  dv = RMSNorm'(v)^T (g W_q) (the straight-through quantisers pass the
  gradient unchanged), written out in numpy.
* With the quantisers on, the forward equals the pinned inference oracle's.
"""

import numpy as np
import pytest
import torch

from oracle import bitssm_oracle as O
from oracle import ste_oracle as T
from ternary_weight_selective_b200 import synthetic as S


def _layer(seed=3, B=1, L=6):
    wl = S.Workload("ste", B, L, 16, 32, 4, 2, "f32", "A8")
    x, layers = S.make_inputs(wl, seed=seed)
    lw = layers[0]
    # weights large enough that the float layer has sizeable gradients
    for n in ("W_in", "W_dt_down", "W_B", "W_C", "W_dt_up", "W_out"):
        setattr(lw, n, getattr(lw, n) * 10.0)
    return x.astype(np.float64), lw


def test_float_layer_gradients_match_finite_differences():
    x, lw = _layer()
    p = T.params_from(lw)
    g = np.random.default_rng(1).normal(size=x.shape)
    _, grads = T.mixer_backward(x, p, g, quant=False)

    def loss(xv, pv):
        with torch.no_grad():
            out = T.mixer_forward(torch.tensor(xv), pv, quant=False)
        return float((out.numpy() * g).sum())

    base = {n: p[n].detach().clone() for n in T.PARAMS}
    rng = np.random.default_rng(2)
    h = 1e-6
    # x
    for _ in range(6):
        idx = tuple(rng.integers(0, s) for s in x.shape)
        xp, xm = x.copy(), x.copy()
        xp[idx] += h
        xm[idx] -= h
        fd = (loss(xp, base) - loss(xm, base)) / (2 * h)
        assert abs(fd - float(grads["x"][idx])) <= 1e-6 * max(1.0, abs(fd)), ("x", idx)
    # every parameter
    for n in T.PARAMS:
        for _ in range(3):
            idx = tuple(int(rng.integers(0, s)) for s in base[n].shape)
            pp = dict(base)
            pm = dict(base)
            pp[n] = base[n].clone()
            pm[n] = base[n].clone()
            pp[n][idx] += h
            pm[n][idx] -= h
            fd = (loss(x, pp) - loss(x, pm)) / (2 * h)
            assert abs(fd - float(grads[n][idx])) <= 1e-6 * max(1.0, abs(fd)), (n, idx)


def test_one_bitlinear_ste_gradients_closed_form():
    rng = np.random.default_rng(5)
    M, K, n = 7, 24, 5
    v = rng.normal(size=(M, K))
    W = rng.normal(0, 0.05, size=(n, K))
    g = rng.normal(size=(M, n))
    vt = torch.tensor(v, requires_grad=True)
    Wt = torch.tensor(W, requires_grad=True)
    out = T.bitlinear(vt, Wt)
    dv, dW = torch.autograd.grad((out * torch.tensor(g)).sum(), [vt, Wt])
    # closed forms in numpy
    r = 1.0 / np.sqrt((v * v).mean(axis=1, keepdims=True) + 1e-5)
    vn = v * r
    m = np.abs(vn).max(axis=1, keepdims=True)
    a = np.clip(np.rint(vn * (127.0 / m)), -128, 127) / (127.0 / m)   # dequantised activations
    s = np.abs(W).mean()
    Wq = np.clip(np.rint(W / (s + 1e-5)), -1, 1) * s
    np.testing.assert_allclose(out.detach().numpy(), a @ Wq.T, rtol=1e-12, atol=1e-12)
    np.testing.assert_allclose(dW.numpy(), g.T @ a, rtol=1e-12, atol=1e-12)
    dvn = g @ Wq
    dv_ref = r * dvn - v * r ** 3 * (v * dvn).sum(axis=1, keepdims=True) / K
    np.testing.assert_allclose(dv.numpy(), dv_ref, rtol=1e-10, atol=1e-12)


def test_quantised_forward_equals_inference_oracle():
    wl = S.WORKLOADS["tiny"]
    x, layers = S.make_inputs(wl, seed=0, seqlen=24)
    ref, _ = O.bitssm_layer_a8(x, O.TernaryLayer(layers[0], "A8"))
    with torch.no_grad():
        out = T.mixer_forward(torch.tensor(x, dtype=torch.float64), T.params_from(layers[0]))
    out = out.numpy()
    # the same numbers in real arithmetic.  The inference oracle stores the
    # weight scales and row maxima in float32, this form keeps float64, so
    # they differ at the 1e-7 level; on this input no code decision falls at
    # a near-tie (a flipped code would show as ~1e-3)
    assert np.abs(out - ref).max() <= 1e-6 * np.abs(ref).max()


def test_ste_gradient_ignores_quantiser_steps():
    """A straight-through quantiser passes the gradient unchanged: for one
    BitLinear, dv with the quantisers on equals the float layer's dv taken at
    the same weights' dequantised values."""
    rng = np.random.default_rng(8)
    v = torch.tensor(rng.normal(size=(4, 16)), requires_grad=True)
    W = torch.tensor(rng.normal(0, 0.05, size=(3, 16)))
    g = torch.tensor(rng.normal(size=(4, 3)))
    dv_q, = torch.autograd.grad((T.bitlinear(v, W) * g).sum(), [v])
    Wq = T.quant_weight(W).detach()
    dv_f, = torch.autograd.grad((T.bitlinear(v, Wq, act_quant=False, weight_quant=False) * g).sum(), [v])
    assert torch.allclose(dv_q, dv_f, rtol=1e-12, atol=1e-14)
