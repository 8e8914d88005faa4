"""CPU oracle of the BitSSM mixer's backward pass under the straight-through
estimator (the QAT form of the layer).

TEST INFRASTRUCTURE ONLY.  Only ``tests/``, ``__graft_entry__.smoke()`` and
the CPU-baseline leg of ``bench.py`` may import this module.  Plain PyTorch
CPU ops in float64; the derivative is taken by autograd over the forward
written out below, and the pins check it against finite differences and
closed forms that do not use autograd.

Sources (page title, then the part of the page):

* "Associative Recall Under Ternary Quantization ..." (TriSSM README): the
  Delta, B, C projections are BitNet b1.58 BitLinear layers trained with
  ternary weights and int8 activations (opening paragraph; "Repository
  structure": bitlinear.py holds the BitLinear with its straight-through
  estimator).
* "Ternary Mamba: Grouped Quantization-Aware Training of W1.58A16 State Space
  Models", abstract: quantisation-aware training of a ternary SSM.

Readings (the pages name the straight-through estimator but write no
formula): in the forward, every quantiser replaces its input by the
dequantised value (weights: s * clip(rint(W / (s + eps)), -1, 1) with
s = mean|W|; activations: per-row absmax codes times max / 127 after a
unit-gain RMSNorm); in the backward, every quantiser passes the gradient
through unchanged (the scales s and max|v| are not differentiated).  The
RMSNorm, softplus and the recurrence are differentiated exactly.  The forward
values equal those of the inference forward in real arithmetic.
"""

from __future__ import annotations

import torch

EPS_NORM = 1e-5
EPS_W = 1e-5
Q_ACT = 127.0


def rmsnorm(v: torch.Tensor) -> torch.Tensor:
    """Unit-gain RMSNorm over the last axis (differentiated exactly)."""
    return v / torch.sqrt((v * v).mean(dim=-1, keepdim=True) + EPS_NORM)


def ste(value: torch.Tensor, through: torch.Tensor) -> torch.Tensor:
    """Forward: ``value``; backward: the gradient of ``through``."""
    return through + (value - through).detach()


def quant_weight(W: torch.Tensor, group: int = 0, enabled: bool = True) -> torch.Tensor:
    """Dequantised absmean ternary weights with a straight-through gradient.
    group 0: one scale for the matrix; group g: one per run of g K-elements."""
    if not enabled:
        return W
    with torch.no_grad():
        if group == 0:
            s = W.abs().mean()
            Wq = torch.clamp(torch.round(W / (s + EPS_W)), -1, 1) * s
        else:
            n, k = W.shape
            Wq = torch.empty_like(W)
            for j0 in range(0, k, group):
                blk = W[:, j0:j0 + group]
                s = blk.abs().mean(dim=1, keepdim=True)
                Wq[:, j0:j0 + group] = torch.clamp(torch.round(blk / (s + EPS_W)), -1, 1) * s
    return ste(Wq, W)


def quant_act(v: torch.Tensor, enabled: bool = True) -> torch.Tensor:
    """Per-row absmax int8 quantise-dequantise with a straight-through
    gradient (round half to even; a zero row stays zero)."""
    if not enabled:
        return v
    with torch.no_grad():
        m = v.abs().amax(dim=-1, keepdim=True)
        sigma = torch.where(m > 0, Q_ACT / torch.where(m > 0, m, torch.ones_like(m)),
                            torch.zeros_like(m))
        q = torch.clamp(torch.round(v * sigma), -128, 127)
        deq = torch.where(m > 0, q / torch.where(sigma > 0, sigma, torch.ones_like(sigma)),
                          torch.zeros_like(q))
    return ste(deq, v)


def bitlinear(v, W, act_quant=True, weight_quant=True, group=0):
    """RMSNorm -> quantise (A8) -> ternary projection, straight-through."""
    vn = rmsnorm(v)
    return quant_act(vn, act_quant) @ quant_weight(W, group, weight_quant).T


def scan(u, delta, A, Bm, Cm, D):
    """The selective recurrence, step by step (u, delta [B, L, E]; A [E, N];
    Bm, Cm [B, L, N]; D [E]), differentiable."""
    Bsz, L, E = u.shape
    N = A.shape[1]
    h = torch.zeros((Bsz, E, N), dtype=u.dtype)
    ys = []
    for t in range(L):
        dt = delta[:, t, :, None]
        h = torch.exp(dt * A[None]) * h + dt * Bm[:, t, None, :] * u[:, t, :, None]
        ys.append((h * Cm[:, t, None, :]).sum(-1) + D[None] * u[:, t])
    return torch.stack(ys, dim=1)


def mixer_forward(x, p, quant=True):
    """The A8 mixer in its training form.  x [B, L, d]; p a dict of float64
    tensors W_in, W_dt_down, W_B, W_C, W_dt_up, W_out, A, D, dt_bias.
    ``quant=False`` drops every quantiser (the float layer the STE follows)."""
    Bsz, L, d = x.shape
    xt = x.reshape(Bsz * L, d)
    kw = dict(act_quant=quant, weight_quant=quant)
    u = bitlinear(xt, p["W_in"], **kw)
    B = bitlinear(u, p["W_B"], **kw)
    C = bitlinear(u, p["W_C"], **kw)
    dt_low = bitlinear(u, p["W_dt_down"], **kw)
    delta = torch.nn.functional.softplus(bitlinear(dt_low, p["W_dt_up"], **kw) + p["dt_bias"])
    E, N = u.shape[1], B.shape[1]
    y = scan(u.reshape(Bsz, L, E), delta.reshape(Bsz, L, E), p["A"],
             B.reshape(Bsz, L, N), C.reshape(Bsz, L, N), p["D"])
    return bitlinear(y.reshape(Bsz * L, E), p["W_out"], **kw).reshape(Bsz, L, d)


PARAMS = ("W_in", "W_dt_down", "W_B", "W_C", "W_dt_up", "W_out", "A", "D", "dt_bias")


def params_from(lw) -> dict:
    """float64 leaf tensors (requires_grad) from synthetic LayerWeights."""
    return {n: torch.tensor(getattr(lw, n), dtype=torch.float64, requires_grad=True)
            for n in PARAMS}


def mixer_backward(x, p, grad_out, quant=True):
    """Gradients of sum(grad_out * mixer_forward(x, p)) with respect to x and
    every parameter.  Returns (out, {"x": dx, name: dW ...})."""
    xt = torch.as_tensor(x, dtype=torch.float64).clone().requires_grad_(True)
    out = mixer_forward(xt, p, quant)
    g = torch.as_tensor(grad_out, dtype=torch.float64)
    leaves = [xt] + [p[n] for n in PARAMS]
    grads = torch.autograd.grad((out * g).sum(), leaves)
    return out.detach(), dict(zip(["x", *PARAMS], [gr.detach() for gr in grads]))
