"""Plain CPU oracle of the SSD (state space duality) scan of Mamba-2.

TEST INFRASTRUCTURE ONLY.  Only ``tests/``, ``__graft_entry__.smoke()`` and
the CPU-baseline leg of ``bench.py`` may import this module.  It shares no
code with the CUDA library and imports only numpy.

Sources (page title, then the part of the page):

* [TernaryMamba] "Ternary Mamba: Grouped Quantization-Aware Training of
  W1.58A16 State Space Models", abstract: the W1.58A16 model is Mamba-2 1.3B.
* [SSDi8] "SSDi8: Accurate and Efficient 8-bit Quantization for State Space
  Duality", abstract: Mamba-2's SSD joins a recurrent mode and an attention
  mode of one operator; its index page lists "Transformers are SSMs:
  Generalized Models and Efficient Algorithms Through Structured State Space
  Duality", the paper that defines it.

The pages print no formula.  What the oracle computes is the SSD operator as
that title names it: the selective recurrence of the mixer with the decay a
scalar per head instead of a value per (channel, state), which makes the
recurrence equal to a masked, decayed attention (the "duality"), and the
chunked algorithm that uses it.  Per sequence, head h of H (head dimension P)
and group g = h // (H / G) of the B, C projections (state size N):

    S_t = exp(dt_t[h] A[h]) S_{t-1} + dt_t[h] x_t[h] (outer) B_t[g]    S: [P, N]
    y_t[h] = S_t C_t[g] + D[h] x_t[h]

dt is the step size after its softplus (given, > 0), A[h] < 0.

Three evaluations, each a different algorithm for the same numbers:

* ``ssd_sequential``: the recurrence, one step at a time (the definition);
* ``ssd_quadratic``: the attention form, the [L, L] lower-triangular matrix
  M[t, s] = (C_t . B_s) exp(sum_{k=s+1..t} dt_k A) dt_s applied to x;
* ``ssd_chunked``: chunks of Q steps; inside a chunk the attention form, the
  state at each chunk's end formed from the chunk's inputs, carried across
  chunks by the recurrence, and read out at every step of the next chunk.

All in float64.  Pins: ``tests/test_oracle_ssd.py``.
"""

from __future__ import annotations

import numpy as np


def _group_of(H: int, G: int) -> np.ndarray:
    assert H % G == 0, "heads must split evenly over the B/C groups"
    return np.arange(H) // (H // G)


def ssd_sequential(x, dt, A, Bm, Cm, D, S0=None):
    """The SSD recurrence step by step.

    x [Bsz, L, H, P], dt [Bsz, L, H] (> 0), A [H] (< 0), Bm, Cm [Bsz, L, G, N],
    D [H], S0 [Bsz, H, P, N] or None (zero).  Returns (y [Bsz, L, H, P],
    S_L [Bsz, H, P, N])."""
    x = np.asarray(x, np.float64)
    dt = np.asarray(dt, np.float64)
    A = np.asarray(A, np.float64)
    Bm = np.asarray(Bm, np.float64)
    Cm = np.asarray(Cm, np.float64)
    D = np.asarray(D, np.float64)
    Bsz, L, H, P = x.shape
    G, N = Bm.shape[2], Bm.shape[3]
    g = _group_of(H, G)
    S = np.zeros((Bsz, H, P, N)) if S0 is None else np.array(S0, np.float64)
    y = np.zeros((Bsz, L, H, P))
    for t in range(L):
        decay = np.exp(dt[:, t, :] * A[None, :])                      # [Bsz, H]
        Bt = Bm[:, t, g, :]                                           # [Bsz, H, N]
        Ct = Cm[:, t, g, :]
        S = decay[:, :, None, None] * S + \
            (dt[:, t, :, None] * x[:, t])[:, :, :, None] * Bt[:, :, None, :]
        y[:, t] = np.einsum("bhpn,bhn->bhp", S, Ct) + D[None, :, None] * x[:, t]
    return y, S


def ssd_quadratic(x, dt, A, Bm, Cm, D):
    """The attention form from a zero state: for each head,
    y = (M (*) (C B^T)) (dt x) + D x with the decay mask
    M[t, s] = exp(cum[t] - cum[s]) for s <= t (else 0), cum[t] = sum_{k<=t} dt_k A."""
    x = np.asarray(x, np.float64)
    dt = np.asarray(dt, np.float64)
    A = np.asarray(A, np.float64)
    Bm = np.asarray(Bm, np.float64)
    Cm = np.asarray(Cm, np.float64)
    D = np.asarray(D, np.float64)
    Bsz, L, H, P = x.shape
    G = Bm.shape[2]
    g = _group_of(H, G)
    y = np.zeros_like(x)
    tri = np.tril(np.ones((L, L), dtype=bool))
    for b in range(Bsz):
        for h in range(H):
            cum = np.cumsum(dt[b, :, h] * A[h])                       # [L]
            diff = cum[:, None] - cum[None, :]
            M = np.where(tri, np.exp(np.where(tri, diff, 0.0)), 0.0)  # [L, L]
            CB = Cm[b, :, g[h], :] @ Bm[b, :, g[h], :].T              # [L, L]
            W = M * CB * dt[b, None, :, h]
            y[b, :, h, :] = W @ x[b, :, h, :] + D[h] * x[b, :, h, :]
    return y


def ssd_chunked(x, dt, A, Bm, Cm, D, Q: int = 16, S0=None):
    """The chunked SSD algorithm with chunk length Q (the last chunk may be
    shorter).  For a chunk [c0, c1) with local cumulative log-decay
    cum[t] = sum_{k=c0..t} dt_k A and entering state S_in:

      1. y_intra[t] = sum_{s=c0..t} exp(cum[t] - cum[s]) (C_t . B_s) dt_s x_s
      2. y_inter[t] = exp(cum[t]) S_in C_t
      3. S_out = exp(cum[c1-1]) S_in + sum_s exp(cum[c1-1] - cum[s]) dt_s x_s (outer) B_s
      y = y_intra + y_inter + D x,  S_in of the next chunk = S_out.

    Returns (y, S_L)."""
    x = np.asarray(x, np.float64)
    dt = np.asarray(dt, np.float64)
    A = np.asarray(A, np.float64)
    Bm = np.asarray(Bm, np.float64)
    Cm = np.asarray(Cm, np.float64)
    D = np.asarray(D, np.float64)
    Bsz, L, H, P = x.shape
    G, N = Bm.shape[2], Bm.shape[3]
    g = _group_of(H, G)
    S = np.zeros((Bsz, H, P, N)) if S0 is None else np.array(S0, np.float64)
    y = np.zeros_like(x)
    for c0 in range(0, L, Q):
        c1 = min(c0 + Q, L)
        n = c1 - c0
        tri = np.tril(np.ones((n, n), dtype=bool))
        for b in range(Bsz):
            for h in range(H):
                cum = np.cumsum(dt[b, c0:c1, h] * A[h])               # [n]
                Bc = Bm[b, c0:c1, g[h], :]                            # [n, N]
                Cc = Cm[b, c0:c1, g[h], :]
                xs = dt[b, c0:c1, h, None] * x[b, c0:c1, h, :]        # [n, P]
                diff = cum[:, None] - cum[None, :]
                M = np.where(tri, np.exp(np.where(tri, diff, 0.0)), 0.0)
                y_intra = (M * (Cc @ Bc.T)) @ xs                      # [n, P]
                y_inter = np.exp(cum)[:, None] * (Cc @ S[b, h].T)     # [n, P]
                y[b, c0:c1, h, :] = y_intra + y_inter + D[h] * x[b, c0:c1, h, :]
                w_end = np.exp(cum[-1] - cum)                         # [n]
                S[b, h] = np.exp(cum[-1]) * S[b, h] + (w_end[:, None] * xs).T @ Bc
    return y, S
