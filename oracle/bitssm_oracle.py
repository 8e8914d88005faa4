"""Plain, slow, obviously-correct CPU oracle of the BitSSM forward pass.

TEST INFRASTRUCTURE ONLY.  Only ``tests/``, ``__graft_entry__.smoke()`` and
the CPU-baseline leg of ``bench.py`` may import this module.  It shares no
code with the CUDA library (no kernels, headers, helpers, tables or constant
generators) and imports only numpy.

Arithmetic: float64 throughout, except where a floating-point value decides an
integer (the int8 activation code and the ternary weight code): there the
decision is taken in IEEE float32 with round-to-nearest, exactly as the
quantiser definitions below state, so that the CUDA path, which takes the same
decisions in float32, can be held bit-exact.

Sources (page title, then the part of the page):

* [TriSSM] "Associative Recall Under Ternary Quantization: A Controlled
  Comparison of State Space Models and Transformers at 5M Parameters"
  (TriSSM repository README): the opening paragraph (the Delta, B, C
  projections are BitNet b1.58 BitLinear layers with ternary {-1, 0, +1}
  weights and int8 activations), the caption "The BitSSM sequence mixer"
  (an RMSNorm precedes each ternary projection; the recurrence is evaluated
  with a parallel associative scan), the Overview table (TriSSM: selective
  SSM, 12 layers, d=256, ternary Delta, B, C) and "Repository structure"
  (bitlinear.py: BitLinear; ssm.py: BitSSM block and parallel associative
  scan).
* [TernaryMamba] "Ternary Mamba: Grouped Quantization-Aware Training of
  W1.58A16 State Space Models", abstract: W1.58A16 (ternary weights, 16-bit
  activations) with grouped weight quantisation.
* [TernarySSM] "Ternary State-Space Models: Hardware-Efficient Language
  Modeling with -1, 0, +1 Weights", abstract: multiply-free inference through
  add / subtract / skip; SSM parallel scan.
* [SSDi8] "SSDi8: Accurate and Efficient 8-bit Quantization for State Space
  Duality", abstract: reuse of quantised activations across modules.

The Mamba-1 block form (``bitssm_block_a8``: a depthwise causal conv1d and a
SiLU on the in_proj branch, a SiLU gate from a second in_proj branch z on the
scan output) is named by none of the pages; it is the block that the pages'
Mamba checkpoints carry around the same selective scan (the [TernaryMamba]
abstract quantises Mamba models), with every projection a ternary BitLinear
as in the mixer.

The pages name these operations but print no formula.  The formulas used here
are the BitNet b1.58 definitions the pages refer to by name (absmean ternary
weights, absmax int8 activations with Q = 127, int32 accumulation, rescale by
absmean x absmax / 127) and the Mamba-style selective recurrence
h_t = exp(Delta_t A) * h_{t-1} + Delta_t B_t x_t, y_t = C_t . h_t + D x_t with
Delta = softplus(Delta_raw + bias).  Every point the pages leave open is
listed, with the reading taken, in the constants and docstrings below.

Pins: every function here is checked by ``tests/test_oracle_*.py`` against
brute force, closed forms, special cases and invariants (no page prints a
worked example, so nothing is pinned to a printed value).
"""

from __future__ import annotations

import numpy as np

# Readings of points the pages leave open.
EPS_NORM = 1e-5   # RMSNorm epsilon; the RMSNorm has unit gain
EPS_W = 1e-5      # absmean epsilon, added only inside the weight-code division
Q_ACT = 127       # absmax activation range
GROUP = 128       # W1.58A16 weight-group size along K

F32 = np.float32


# ---------------------------------------------------------------------------
# Weights: absmean ternary quantisation and the 2-bit encoding
# ---------------------------------------------------------------------------

def absmean_ternary(W: np.ndarray, group: int = 0):
    """BitNet b1.58 absmean weight quantisation ([TriSSM] opening paragraph;
    grouped form: [TernaryMamba] abstract).

    s = mean |W| (summed in float64, stored as float32);
    W_q = clip(rint(W / (s + eps)), -1, 1), the division in float32.
    ``group`` = 0: one scale per matrix.  ``group`` = g: one scale per run of
    g consecutive K-elements of an output row, s[n, j] over W[n, j*g:(j+1)*g]
    (the last run may be shorter).

    Returns (W_q int8 [n_out, k_in], s) with s a float32 scalar array of
    shape () for group 0, else float32 [n_out, ceil(k_in / g)].
    """
    W = np.asarray(W, dtype=F32)
    n_out, k_in = W.shape
    if group == 0:
        s = F32(np.abs(W.astype(np.float64)).sum() / W.size)
        denom = F32(s + F32(EPS_W))
        Wq = np.clip(np.rint(W / denom), -1, 1).astype(np.int8)
        return Wq, np.array(s, dtype=F32)
    n_groups = -(-k_in // group)
    s = np.zeros((n_out, n_groups), dtype=F32)
    Wq = np.zeros((n_out, k_in), dtype=np.int8)
    for j in range(n_groups):
        blk = W[:, j * group:(j + 1) * group]
        sj = (np.abs(blk.astype(np.float64)).sum(axis=1) / blk.shape[1]).astype(F32)
        s[:, j] = sj
        denom = (sj + F32(EPS_W)).astype(F32)
        Wq[:, j * group:(j + 1) * group] = np.clip(np.rint(blk / denom[:, None]), -1, 1)
    return Wq, s


def pack_ternary(Wq: np.ndarray) -> np.ndarray:
    """2-bit encoding of ternary codes: code c = w + 1 in {0, 1, 2} stored at
    bits 2*(k mod 4) of byte k // 4 of its row; rows padded with w = 0.
    Returns uint8 [n_out, ceil(k_in / 4)]."""
    Wq = np.asarray(Wq, dtype=np.int64)
    n_out, k_in = Wq.shape
    kb = -(-k_in // 4)
    codes = np.ones((n_out, kb * 4), dtype=np.int64)
    codes[:, :k_in] = Wq + 1
    packed = np.zeros((n_out, kb), dtype=np.int64)
    for i in range(4):
        packed |= codes[:, i::4] << (2 * i)
    return packed.astype(np.uint8)


# ---------------------------------------------------------------------------
# Activations: absmax int8 quantisation with the RMSNorm folded in
# ---------------------------------------------------------------------------

def absmax_codes(v32: np.ndarray):
    """Per-row absmax int8 codes ([TriSSM] opening paragraph: int8 activations).

    For each row: m = max_k |v_k| (float32, exact); sigma = fl32(127 / m);
    q_k = clamp(rint(fl32(v_k * sigma)), -128, 127), rint = round half to
    even.  A row with m = 0 gets all-zero codes.
    Returns (q int32 [..., K], m float32 [...]).
    """
    v32 = np.asarray(v32, dtype=F32)
    m = np.abs(v32).max(axis=-1).astype(F32)
    safe = np.where(m > 0, m, F32(1.0)).astype(F32)
    sigma = (F32(Q_ACT) / safe).astype(F32)
    prod = (v32 * sigma[..., None]).astype(F32)
    q = np.clip(np.rint(prod), -128, 127).astype(np.int32)
    q[m == 0] = 0
    return q, m


def rms_factor(v: np.ndarray) -> np.ndarray:
    """Unit-gain RMSNorm factor r = 1 / sqrt(mean_k v_k^2 + eps) per row
    ([TriSSM] caption: an RMSNorm precedes each ternary projection)."""
    v = np.asarray(v, dtype=np.float64)
    return 1.0 / np.sqrt((v * v).mean(axis=-1) + EPS_NORM)


def int_gemm(q: np.ndarray, Wq: np.ndarray) -> np.ndarray:
    """acc[m, j] = sum_k q[m, k] * W_q[j, k], exact.

    Computed as a float64 matmul of integer-valued matrices: every product and
    every partial sum is an integer of magnitude <= 128 * K < 2^53, so float64
    represents each exactly and the result is the exact integer sum.  Asserted
    to fit int32 (the accumulator width of the method)."""
    q = np.asarray(q)
    Wq = np.asarray(Wq)
    K = q.shape[-1]
    assert 128 * K < 2 ** 53
    acc = q.astype(np.float64) @ Wq.astype(np.float64).T
    acc = acc.astype(np.int64)
    assert np.abs(acc).max(initial=0) < 2 ** 31
    return acc


def bitlinear_a8(v: np.ndarray, Wq: np.ndarray, s) -> tuple[np.ndarray, dict]:
    """BitLinear with int8 activations on input rows v ([TriSSM] opening
    paragraph and caption; multiply-free ternary GEMM: [TernarySSM] abstract).

    RMSNorm (unit gain) -> absmax int8 -> ternary GEMM (int32) -> rescale by
    absmean x absmax / 127.  The RMSNorm scales a row by r > 0, and
    max|v r| = m r, so the codes of the normalised row equal the codes of v
    (computed from v's float32 value); the rescale is
    out_j = acc_j * s * (m * r) / 127, in float64.
    Returns (out float64 [..., n_out], stages dict).
    """
    v = np.asarray(v)
    q, m = absmax_codes(v.astype(F32))
    acc = int_gemm(q, Wq)
    r = rms_factor(v)
    deq = m.astype(np.float64) * r / Q_ACT
    out = acc.astype(np.float64) * np.float64(s) * deq[..., None]
    return out, dict(q=q, m=m, r=r, deq=deq, acc=acc)


def bitlinear_a8_int_input(acc_in: np.ndarray, c: np.ndarray, Wq: np.ndarray, s):
    """BitLinear whose input row is c_t * acc_in[t, :] with c_t > 0 and acc_in
    an integer row (the output of an earlier BitLinear before its rescale).

    Reading (the pages do not say in which precision the chained quantiser
    runs): the absmax codes are decided on the integer row itself, converted to
    float32 (exact: |acc_in| < 2^24).  In real arithmetic this equals the codes
    of the rescaled row, since absmax codes do not change under a positive row
    scale.  The dequantisation uses the real row v = c * acc_in:
    m = max|v|, r = RMSNorm factor of v, out = acc * s * m * r / 127.
    Returns (out float64, stages dict with v, q, acc, deq).
    """
    acc_in = np.asarray(acc_in, dtype=np.int64)
    c = np.asarray(c, dtype=np.float64)
    assert np.abs(acc_in).max(initial=0) < 2 ** 24
    q, m_int = absmax_codes(acc_in.astype(F32))
    v = c[..., None] * acc_in.astype(np.float64)
    m = c * m_int.astype(np.float64)
    r = rms_factor(v)
    deq = m * r / Q_ACT
    acc = int_gemm(q, Wq)
    out = acc.astype(np.float64) * np.float64(s) * deq[..., None]
    return out, dict(v=v, q=q, acc=acc, deq=deq, r=r)


def bitlinear_a16(v: np.ndarray, Wq: np.ndarray, s_groups: np.ndarray,
                  group: int = GROUP) -> np.ndarray:
    """W1.58A16 BitLinear ([TernaryMamba] abstract): 16-bit activations with
    no activation quantisation, ternary weights with one absmean scale per
    group of ``group`` K-elements.  Reading: the RMSNorm before the projection
    (unit gain) is kept.

    out_n = r * sum_j s[n, j] * sum_{k in group j} W_q[n, k] * v_k  (float64).
    """
    v = np.asarray(v, dtype=np.float64)
    Wq = np.asarray(Wq, dtype=np.float64)
    K = v.shape[-1]
    r = rms_factor(v)
    out = np.zeros(v.shape[:-1] + (Wq.shape[0],), dtype=np.float64)
    for j in range(s_groups.shape[1]):
        sl = slice(j * group, min((j + 1) * group, K))
        part = v[..., sl] @ Wq[:, sl].T
        out += part * s_groups[:, j].astype(np.float64)
    return out * r[..., None]


# ---------------------------------------------------------------------------
# Selective scan
# ---------------------------------------------------------------------------

def softplus(z: np.ndarray) -> np.ndarray:
    """softplus(z) = log(1 + e^z), written as max(z, 0) + log1p(e^-|z|) so it
    neither overflows nor loses the small-z tail."""
    z = np.asarray(z, dtype=np.float64)
    return np.maximum(z, 0.0) + np.log1p(np.exp(-np.abs(z)))


def selective_scan(u, delta, A, Bm, Cm, D, h0=None):
    """Sequential selective recurrence in float64 ([TriSSM] caption and
    "Repository structure": the BitSSM block's recurrence).

    u, delta: [B, L, E]; A: [E, N]; Bm, Cm: [B, L, N] (shared by all channels);
    D: [E]; h0: [B, E, N] or None (zero state).  For each step t:
        a_t = exp(delta_t[e] * A[e, n])
        h_t = a_t * h_{t-1} + delta_t[e] * B_t[n] * u_t[e]
        y_t[e] = sum_n C_t[n] * h_t[e, n] + D[e] * u_t[e]
    Returns (y [B, L, E], h_L [B, E, N]).
    """
    u = np.asarray(u, dtype=np.float64)
    delta = np.asarray(delta, dtype=np.float64)
    A = np.asarray(A, dtype=np.float64)
    Bm = np.asarray(Bm, dtype=np.float64)
    Cm = np.asarray(Cm, dtype=np.float64)
    D = np.asarray(D, dtype=np.float64)
    Bsz, L, E = u.shape
    N = A.shape[1]
    h = np.zeros((Bsz, E, N)) if h0 is None else np.array(h0, dtype=np.float64)
    y = np.zeros((Bsz, L, E))
    for t in range(L):
        dt = delta[:, t, :, None]
        a = np.exp(dt * A[None])
        b = dt * Bm[:, t, None, :] * u[:, t, :, None]
        h = a * h + b
        y[:, t] = (h * Cm[:, t, None, :]).sum(-1) + D[None] * u[:, t]
    return y, h


def selective_scan_associative(u, delta, A, Bm, Cm, D, h0=None, chunk=16):
    """The same recurrence evaluated as a chunked parallel associative scan
    ([TriSSM] caption: "parallel associative scan"; [TernarySSM] abstract).

    Each step is the affine map h -> a_t h + b_t, the pair (a_t, b_t).  Maps
    compose associatively: applying (a, b) and then (a', b') is
    (a' a, a' b + b').  Within each chunk of ``chunk`` steps the inclusive
    prefix compositions are formed by a Hillis-Steele scan (log2(chunk)
    rounds of pairwise composition); the state entering each chunk is then
    carried from chunk to chunk, and h_t = Acum_t * h_in + Bcum_t.
    """
    u = np.asarray(u, dtype=np.float64)
    delta = np.asarray(delta, dtype=np.float64)
    A = np.asarray(A, dtype=np.float64)
    Bm = np.asarray(Bm, dtype=np.float64)
    Cm = np.asarray(Cm, dtype=np.float64)
    D = np.asarray(D, dtype=np.float64)
    Bsz, L, E = u.shape
    N = A.shape[1]
    h_in = np.zeros((Bsz, E, N)) if h0 is None else np.array(h0, dtype=np.float64)
    y = np.zeros((Bsz, L, E))
    for c0 in range(0, L, chunk):
        c1 = min(c0 + chunk, L)
        dt = delta[:, c0:c1, :, None]                            # [B, l, E, 1]
        a = np.exp(dt * A[None, None])                           # [B, l, E, N]
        b = dt * Bm[:, c0:c1, None, :] * u[:, c0:c1, :, None]    # [B, l, E, N]
        step = 1
        while step < c1 - c0:
            a_prev = np.ones_like(a)
            b_prev = np.zeros_like(b)
            a_prev[:, step:] = a[:, :-step]
            b_prev[:, step:] = b[:, :-step]
            # compose: first the earlier map (a_prev, b_prev), then (a, b)
            b = a * b_prev + b
            a = a * a_prev
            step *= 2
        h = a * h_in[:, None] + b                                # [B, l, E, N]
        y[:, c0:c1] = (h * Cm[:, c0:c1, None, :]).sum(-1) + D[None, None] * u[:, c0:c1]
        h_in = h[:, -1]
    return y, h_in


# ---------------------------------------------------------------------------
# Mamba-1 block pieces: depthwise causal conv1d and SiLU
# ---------------------------------------------------------------------------

def causal_conv1d(v: np.ndarray, w: np.ndarray, b=None) -> np.ndarray:
    """Depthwise causal convolution along time, one filter per channel.

    v [B, L, E], w [E, K], b [E] or None.  out[:, l, e] = b[e] +
    sum_{k=0}^{K-1} w[e, k] * v[:, l - (K-1) + k, e], terms with a negative
    time index dropped (zero padding on the left): tap K-1 multiplies the
    current step, tap 0 the step K-1 earlier.  This is a width-K conv with
    K-1 zeros of left padding whose output is cut to the first L steps, the
    usual causal form.  float64.
    """
    v = np.asarray(v, dtype=np.float64)
    w = np.asarray(w, dtype=np.float64)
    Bsz, L, E = v.shape
    K = w.shape[1]
    out = np.zeros_like(v)
    if b is not None:
        out += np.asarray(b, dtype=np.float64)[None, None, :]
    for k in range(K):
        shift = K - 1 - k          # how many steps back tap k looks
        if shift >= L:
            continue
        out[:, shift:, :] += w[None, None, :, k] * v[:, :L - shift, :]
    return out


def silu(v: np.ndarray) -> np.ndarray:
    """SiLU(v) = v * sigmoid(v) = v / (1 + e^-v), float64; for v < 0 written
    as v e^v / (1 + e^v) so that e^-v cannot overflow."""
    v = np.asarray(v, dtype=np.float64)
    e = np.exp(-np.abs(v))                     # in (0, 1]
    return np.where(v >= 0, v / (1.0 + e), v * e / (1.0 + e))


# ---------------------------------------------------------------------------
# The BitSSM mixer and the stack
# ---------------------------------------------------------------------------

class TernaryLayer:
    """Ternarised weights of one mixer, from full-precision matrices."""

    def __init__(self, lw, act_mode: str = "A8"):
        self.act_mode = act_mode
        group = GROUP if act_mode == "A16" else 0
        self.group = group
        self.Wq, self.s = {}, {}
        for name in ("W_in", "W_dt_down", "W_B", "W_C", "W_dt_up", "W_out"):
            self.Wq[name], self.s[name] = absmean_ternary(getattr(lw, name), group)
        self.A = np.asarray(lw.A, dtype=np.float64)
        self.D = np.asarray(lw.D, dtype=np.float64)
        self.dt_bias = np.asarray(lw.dt_bias, dtype=np.float64)
        self.R = lw.W_dt_down.shape[0]
        self.N = lw.W_B.shape[0]
        # Mamba-1 block extras (None for the mixer)
        self.block = getattr(lw, "W_z", None) is not None
        if self.block:
            self.Wq["W_z"], self.s["W_z"] = absmean_ternary(lw.W_z, group)
            self.conv_w = np.asarray(lw.conv_w, dtype=np.float64)
            self.conv_b = (np.zeros(self.conv_w.shape[0]) if lw.conv_b is None
                           else np.asarray(lw.conv_b, dtype=np.float64))


def bitssm_layer_a8(x: np.ndarray, P: TernaryLayer, h0=None) -> tuple[np.ndarray, dict]:
    """One BitSSM mixer with int8 activations, x [B, L, d_model] -> out.
    h0 [B, d_inner, N] (None = zero) is the scan's starting state; the
    state after the last step is returned as stages["h_last"] (the recurrent
    form: [TernaryMamba] abstract, linear-time inference).

    Readings: in_proj and out_proj are ternary BitLinears too; the Delta path
    is low rank (d_inner -> dt_rank -> d_inner), both factors ternary;
    Delta-down, B and C share one RMSNorm + quantisation of u (unit-gain
    RMSNorms of one row are identical; reuse of quantised activations across
    modules: [SSDi8] abstract), each with its own weight scale; the codes fed
    to Delta-down/B/C and to Delta-up come from the integer rows of the
    projection before them (``bitlinear_a8_int_input``); out_proj quantises
    the scan output y from its float32 value.  No conv1d, no gate.
    """
    Bsz, L, d = x.shape
    T = Bsz * L
    xt = np.asarray(x).reshape(T, d)
    # in_proj
    u, st_in = bitlinear_a8(xt, P.Wq["W_in"], P.s["W_in"])
    c_u = np.float64(P.s["W_in"]) * st_in["deq"]                 # u = c_u * acc_in
    # x_proj: Delta-down | B | C on one shared quantisation of u
    W_x = np.concatenate([P.Wq["W_dt_down"], P.Wq["W_B"], P.Wq["W_C"]], axis=0)
    _, st_x = bitlinear_a8_int_input(st_in["acc"], c_u, W_x, 1.0)
    acc_x, deq_u = st_x["acc"], st_x["deq"]
    R, N = P.R, P.N
    dt_low = acc_x[:, :R] * np.float64(P.s["W_dt_down"]) * deq_u[:, None]
    Bm = acc_x[:, R:R + N] * np.float64(P.s["W_B"]) * deq_u[:, None]
    Cm = acc_x[:, R + N:R + 2 * N] * np.float64(P.s["W_C"]) * deq_u[:, None]
    # dt_proj on dt_low = (s_dt * deq_u) * acc_x[:, :R]
    c_dt = np.float64(P.s["W_dt_down"]) * deq_u
    delta_raw, st_dt = bitlinear_a8_int_input(acc_x[:, :R], c_dt, P.Wq["W_dt_up"],
                                              P.s["W_dt_up"])
    delta = softplus(delta_raw + P.dt_bias[None])
    E = u.shape[1]
    y, h_last = selective_scan(u.reshape(Bsz, L, E), delta.reshape(Bsz, L, E), P.A,
                               Bm.reshape(Bsz, L, N), Cm.reshape(Bsz, L, N), P.D, h0)
    out, st_out = bitlinear_a8(y.reshape(T, E), P.Wq["W_out"], P.s["W_out"])
    stages = dict(q_x=st_in["q"], deq_x=st_in["deq"], acc_in=st_in["acc"], u=u,
                  q_u=st_x["q"], deq_u=deq_u, acc_x=acc_x, Bm=Bm, Cm=Cm, dt_low=dt_low,
                  q_dt=st_dt["q"], deq_dt=st_dt["deq"], delta_raw=delta_raw, delta=delta,
                  y=y.reshape(T, E), q_y=st_out["q"], deq_y=st_out["deq"],
                  acc_out=st_out["acc"], h_last=h_last)
    return out.reshape(Bsz, L, -1), stages


def bitssm_layer_a16(x: np.ndarray, P: TernaryLayer, h0=None) -> tuple[np.ndarray, dict]:
    """One BitSSM mixer in W1.58A16 form ([TernaryMamba] abstract): every
    projection is ``bitlinear_a16`` on the 16-bit activation row before it.
    h0 / stages["h_last"]: the carried state, as in ``bitssm_layer_a8``."""
    Bsz, L, d = x.shape
    T = Bsz * L
    g = P.group
    xt = np.asarray(x, dtype=np.float64).reshape(T, d)
    u = bitlinear_a16(xt, P.Wq["W_in"], P.s["W_in"], g)
    R, N = P.R, P.N
    dt_low = bitlinear_a16(u, P.Wq["W_dt_down"], P.s["W_dt_down"], g)
    Bm = bitlinear_a16(u, P.Wq["W_B"], P.s["W_B"], g)
    Cm = bitlinear_a16(u, P.Wq["W_C"], P.s["W_C"], g)
    delta_raw = bitlinear_a16(dt_low, P.Wq["W_dt_up"], P.s["W_dt_up"], g)
    delta = softplus(delta_raw + P.dt_bias[None])
    E = u.shape[1]
    y, h_last = selective_scan(u.reshape(Bsz, L, E), delta.reshape(Bsz, L, E), P.A,
                               Bm.reshape(Bsz, L, N), Cm.reshape(Bsz, L, N), P.D, h0)
    out = bitlinear_a16(y.reshape(T, E), P.Wq["W_out"], P.s["W_out"], g)
    stages = dict(u=u, dt_low=dt_low, Bm=Bm, Cm=Cm, delta_raw=delta_raw, delta=delta,
                  y=y.reshape(T, E), h_last=h_last)
    return out.reshape(Bsz, L, -1), stages


def bitssm_block_a8(x: np.ndarray, P: TernaryLayer) -> tuple[np.ndarray, dict]:
    """The mixer in Mamba-1 block form with int8 activations, x [B, L, d] ->
    out [B, L, d], from a zero state.

    Steps (the mixer of ``bitssm_layer_a8`` with three additions):
      1. x-branch and gate branch: u_pre = BitLinear(x; W_in), z =
         BitLinear(x; W_z), two ternary projections of the same int8 codes of
         x (the two halves of Mamba's in_proj, each with its own absmean
         scale);
      2. u = SiLU(causal_conv1d(u_pre; conv_w, conv_b));
      3. x_proj (Delta-down | B | C) is a BitLinear on u; u is no longer a
         scaled integer row, so its codes are taken from its float32 value
         (``bitlinear_a8``), not from an integer row;
      4. Delta-up, softplus and the selective scan as in the mixer, on u;
      5. the gate: y_g = y * SiLU(z), and out_proj is a BitLinear on y_g.
    Readings: the conv acts on the full-precision u_pre; the codes of u and of
    y_g are decided in float32 (the precision of the kernel path).
    """
    if not P.block:
        raise ValueError("layer has no block weights")
    Bsz, L, d = x.shape
    T = Bsz * L
    xt = np.asarray(x).reshape(T, d)
    u_pre, st_in = bitlinear_a8(xt, P.Wq["W_in"], P.s["W_in"])
    acc_z = int_gemm(st_in["q"], P.Wq["W_z"])
    z = acc_z.astype(np.float64) * np.float64(P.s["W_z"]) * st_in["deq"][:, None]
    E = u_pre.shape[1]
    u = silu(causal_conv1d(u_pre.reshape(Bsz, L, E), P.conv_w, P.conv_b)).reshape(T, E)
    W_x = np.concatenate([P.Wq["W_dt_down"], P.Wq["W_B"], P.Wq["W_C"]], axis=0)
    _, st_x = bitlinear_a8(u, W_x, 1.0)
    acc_x, deq_u = st_x["acc"], st_x["deq"]
    R, N = P.R, P.N
    Bm = acc_x[:, R:R + N] * np.float64(P.s["W_B"]) * deq_u[:, None]
    Cm = acc_x[:, R + N:R + 2 * N] * np.float64(P.s["W_C"]) * deq_u[:, None]
    c_dt = np.float64(P.s["W_dt_down"]) * deq_u
    delta_raw, st_dt = bitlinear_a8_int_input(acc_x[:, :R], c_dt, P.Wq["W_dt_up"],
                                              P.s["W_dt_up"])
    delta = softplus(delta_raw + P.dt_bias[None])
    y, h_last = selective_scan(u.reshape(Bsz, L, E), delta.reshape(Bsz, L, E), P.A,
                               Bm.reshape(Bsz, L, N), Cm.reshape(Bsz, L, N), P.D)
    y = y.reshape(T, E)
    yg = y * silu(z)
    out, st_out = bitlinear_a8(yg, P.Wq["W_out"], P.s["W_out"])
    stages = dict(q_x=st_in["q"], deq_x=st_in["deq"], u_pre=u_pre, z=z, u=u,
                  q_u=st_x["q"], deq_u=deq_u, acc_x=acc_x, Bm=Bm, Cm=Cm,
                  q_dt=st_dt["q"], deq_dt=st_dt["deq"], delta=delta, y=y, yg=yg,
                  q_y=st_out["q"], deq_y=st_out["deq"], h_last=h_last)
    return out.reshape(Bsz, L, -1), stages


def bitssm_layer(x, P: TernaryLayer, h0=None):
    if getattr(P, "block", False):
        if P.act_mode != "A8" or h0 is not None:
            raise NotImplementedError("block form: A8 from a zero state only")
        return bitssm_block_a8(x, P)
    if P.act_mode == "A16":
        return bitssm_layer_a16(x, P, h0)
    return bitssm_layer_a8(x, P, h0)


def bitssm_step(x_t: np.ndarray, P: TernaryLayer, h: np.ndarray):
    """The decode step: one token per sequence, x_t [B, d_model], state h
    [B, d_inner, N] -> (out [B, d_model], new h).  The same layer with L = 1
    and the state carried (the recurrence is the only link between steps)."""
    out, st = bitssm_layer(np.asarray(x_t)[:, None, :], P, h)
    return out[:, 0, :], st["h_last"]


def round_bf16(a: np.ndarray) -> np.ndarray:
    """Round to the nearest bfloat16 (ties to even), returned as float64.
    The residual stream of the stack is stored in bf16."""
    a32 = np.asarray(a, dtype=np.float64).astype(F32)
    bits = a32.view(np.uint32).astype(np.uint64)
    bits = ((bits + 0x7FFF + ((bits >> 16) & 1)) >> 16) << 16
    return bits.astype(np.uint32).view(F32).astype(np.float64)


def bitssm_stack(x: np.ndarray, layers: list, io_bf16: bool = True):
    """Residual stack x <- x + BitSSM_l(x) over the layers ([TriSSM] Overview
    table: 12 layers at d = 256).  The pre-RMSNorm of each mixer is the one
    folded into its in_proj quantiser.  With ``io_bf16`` the residual stream
    is rounded to bf16 after every add.  Returns (x_final, [layer inputs])."""
    h = np.asarray(x, dtype=np.float64)
    inputs = []
    for P in layers:
        inputs.append(h)
        out, _ = bitssm_layer(h, P)
        h = h + out
        if io_bf16:
            h = round_bf16(h)
    return h, inputs
