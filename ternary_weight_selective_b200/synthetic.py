"""Seeded synthetic inputs for the BitSSM forward pass.

This module draws random numbers and nothing else: it holds none of the
method's arithmetic (no quantisation, no projection, no scan).  Both the CUDA
path and the CPU oracle take their inputs from here, so that the two see the
same bytes.

Workloads (the shapes the pages train and evaluate at):

* ``tiny``     B=1,  L=64,    d_model=64,   d_inner=128,  N=16, dt_rank=4,   fp32, int8 activations
* ``trissm``   B=64, L=256,   d_model=256,  d_inner=512,  N=16, dt_rank=16,  bf16, int8 activations
  (one mixer of the TriSSM model: d=256 in the README's Overview table; the
  64 x 256 batch of its "Train" section)
* ``stack12``  the same mixer, 12 layers with residual adds (the README's
  12-layer TriSSM), input = bf16 embeddings of uniform token ids over the
  8k vocabulary of its "Prepare the data" step
* ``mamba2_1p3b_a16``  B=4, L=2048, d_model=2048, d_inner=4096, N=16,
  dt_rank=128, bf16 activations without activation quantisation and
  per-group (128) weight scales: the W1.58A16 Mamba-2 1.3B setting of
  "Ternary Mamba: Grouped Quantization-Aware Training of W1.58A16 State
  Space Models" (abstract)
* ``long16k``  B=16, L=16384, the TriSSM mixer on a long sequence, input =
  embeddings of a uniform id stream
* ``trissm_block``  the ``trissm`` shapes as a Mamba-1 block: a depthwise
  causal conv1d of width 4 and a SiLU on the in_proj branch, and a SiLU gate
  from a second (ternary) in_proj branch z on the scan output

Draw order for seed s (numpy PCG64 ``default_rng(s)``): the input first
(x ~ N(0,1), or the embedding table ~ N(0,1) followed by the ids), then for
each layer W_in, W_dt_down, W_B, W_C, W_dt_up, W_out (all N(0, 0.02)),
A_log ~ U(log 1, log 16), dt_bias ~ U(log 1e-3, log 1e-1); D = 1.
A = -exp(A_log).  Block workloads then draw, per layer, W_z ~ N(0, 0.02)
[d_inner, d_model], the conv taps ~ U(-1/sqrt(w), 1/sqrt(w)) [d_inner, w]
and the conv bias ~ U(-1/sqrt(w), 1/sqrt(w)) [d_inner] (w = d_conv; the
usual fan-in bound of a depthwise conv).  Weights are returned as float32
full-precision matrices; ternarisation is the method's business, not this
module's.
"""

from __future__ import annotations

import dataclasses
import math

import numpy as np

VOCAB = 8192


@dataclasses.dataclass(frozen=True)
class Workload:
    name: str
    batch: int
    seqlen: int
    d_model: int
    d_inner: int
    d_state: int
    dt_rank: int
    io_dtype: str      # "f32" or "bf16": dtype of x / out at the boundary
    act_mode: str      # "A8" (int8 activation codes) or "A16" (bf16, grouped scales)
    layers: int = 1
    source: str = "gauss"  # "gauss": x ~ N(0,1); "embed": x = E[ids]
    block: bool = False    # Mamba-1 block: conv1d + SiLU on u, SiLU(z) gate on y
    d_conv: int = 4        # conv width (block workloads)

    @property
    def tokens(self) -> int:
        return self.batch * self.seqlen

    @property
    def weight_group(self) -> int:
        return 128 if self.act_mode == "A16" else 0


WORKLOADS = {
    "tiny": Workload("tiny", 1, 64, 64, 128, 16, 4, "f32", "A8"),
    "trissm": Workload("trissm", 64, 256, 256, 512, 16, 16, "bf16", "A8"),
    "stack12": Workload("stack12", 64, 256, 256, 512, 16, 16, "bf16", "A8", layers=12, source="embed"),
    "mamba2_1p3b_a16": Workload("mamba2_1p3b_a16", 4, 2048, 2048, 4096, 16, 128, "bf16", "A16"),
    "long16k": Workload("long16k", 16, 16384, 256, 512, 16, 16, "bf16", "A8", source="embed"),
    # decode: one token for each of 64 sequences, the state carried in h
    "trissm_decode": Workload("trissm_decode", 64, 1, 256, 512, 16, 16, "bf16", "A8"),
    # the Mamba-1 block form of the trissm mixer (conv1d, SiLU, z gate)
    "trissm_block": Workload("trissm_block", 64, 256, 256, 512, 16, 16, "bf16", "A8", block=True),
}


def round_to_bf16(a: np.ndarray) -> np.ndarray:
    """Round float32 values to the nearest bfloat16 (ties to even); returns float32.

    Data preparation only: bf16 inputs are stored as float32 values that are
    exactly representable in bf16, so both sides read identical numbers.
    """
    a = np.ascontiguousarray(a, dtype=np.float32)
    bits = a.view(np.uint32).astype(np.uint64)
    lsb = (bits >> 16) & 1
    rounded = ((bits + 0x7FFF + lsb) >> 16) << 16
    out = rounded.astype(np.uint32).view(np.float32)
    nan = np.isnan(a)
    if nan.any():
        out = out.copy()
        out[nan] = np.float32("nan")
    return out


def bf16_bits(a: np.ndarray) -> np.ndarray:
    """Upper 16 bits of float32 values that are already bf16-representable."""
    a = np.ascontiguousarray(a, dtype=np.float32)
    return (a.view(np.uint32) >> 16).astype(np.uint16)


@dataclasses.dataclass
class LayerWeights:
    W_in: np.ndarray       # [d_inner, d_model]
    W_dt_down: np.ndarray  # [dt_rank, d_inner]
    W_B: np.ndarray        # [d_state, d_inner]
    W_C: np.ndarray        # [d_state, d_inner]
    W_dt_up: np.ndarray    # [d_inner, dt_rank]
    W_out: np.ndarray      # [d_model, d_inner]
    A: np.ndarray          # [d_inner, d_state], negative
    D: np.ndarray          # [d_inner]
    dt_bias: np.ndarray    # [d_inner]
    W_z: np.ndarray | None = None     # [d_inner, d_model], block only
    conv_w: np.ndarray | None = None  # [d_inner, d_conv], block only
    conv_b: np.ndarray | None = None  # [d_inner], block only


def _layer(rng: np.random.Generator, wl: Workload) -> LayerWeights:
    d, E, N, R = wl.d_model, wl.d_inner, wl.d_state, wl.dt_rank

    def w(n_out, k_in):
        return rng.normal(0.0, 0.02, size=(n_out, k_in)).astype(np.float32)

    W_in = w(E, d)
    W_dt_down = w(R, E)
    W_B = w(N, E)
    W_C = w(N, E)
    W_dt_up = w(E, R)
    W_out = w(d, E)
    A_log = rng.uniform(math.log(1.0), math.log(16.0), size=(E, N))
    dt_bias = rng.uniform(math.log(1e-3), math.log(1e-1), size=(E,))
    A = (-np.exp(A_log)).astype(np.float32)
    D = np.ones((E,), dtype=np.float32)
    lw = LayerWeights(W_in, W_dt_down, W_B, W_C, W_dt_up, W_out, A, D,
                      dt_bias.astype(np.float32))
    if wl.block:
        K = wl.d_conv
        bound = 1.0 / math.sqrt(K)
        lw.W_z = w(E, d)
        lw.conv_w = rng.uniform(-bound, bound, size=(E, K)).astype(np.float32)
        lw.conv_b = rng.uniform(-bound, bound, size=(E,)).astype(np.float32)
    return lw


def make_inputs(wl: Workload, seed: int = 0, batch: int | None = None,
                seqlen: int | None = None):
    """Return (x, layers): x float32 [B, L, d_model] (bf16-representable when
    the workload's io dtype is bf16) and a list of LayerWeights.

    ``batch`` / ``seqlen`` override the workload's sizes (the draw order is
    unchanged, so a smaller sample is a different draw, not a slice).
    """
    rng = np.random.default_rng(seed)
    B = wl.batch if batch is None else batch
    L = wl.seqlen if seqlen is None else seqlen
    if wl.source == "embed":
        table = rng.normal(0.0, 1.0, size=(VOCAB, wl.d_model)).astype(np.float32)
        ids = rng.integers(0, VOCAB, size=(B, L))
        x = table[ids]
    else:
        x = rng.normal(0.0, 1.0, size=(B, L, wl.d_model)).astype(np.float32)
    if wl.io_dtype == "bf16":
        x = round_to_bf16(x)
    layers = [_layer(rng, wl) for _ in range(wl.layers)]
    return x, layers


def random_rows(seed: int, rows: int, cols: int, scale: float = 1.0,
                dtype: str = "f32", zero_rows=()) -> np.ndarray:
    """Gaussian test rows, optionally with all-zero rows (degenerate case)."""
    rng = np.random.default_rng(seed)
    a = (rng.normal(0.0, scale, size=(rows, cols))).astype(np.float32)
    for r in zero_rows:
        a[r] = 0.0
    if dtype == "bf16":
        a = round_to_bf16(a)
    return a


def random_scan_inputs(seed: int, B: int, L: int, E: int, N: int):
    """Inputs of the selective scan alone, drawn like the layer's:
    u ~ N(0,1), delta_raw ~ N(0, 0.5), B, C ~ N(0,1), A and dt_bias as above."""
    rng = np.random.default_rng(seed)
    u = rng.normal(0.0, 1.0, size=(B, L, E)).astype(np.float32)
    delta_raw = rng.normal(0.0, 0.5, size=(B, L, E)).astype(np.float32)
    Bm = rng.normal(0.0, 1.0, size=(B, L, N)).astype(np.float32)
    Cm = rng.normal(0.0, 1.0, size=(B, L, N)).astype(np.float32)
    A = (-np.exp(rng.uniform(0.0, math.log(16.0), size=(E, N)))).astype(np.float32)
    D = np.ones((E,), dtype=np.float32)
    dt_bias = rng.uniform(math.log(1e-3), math.log(1e-1), size=(E,)).astype(np.float32)
    return u, delta_raw, dt_bias, A, Bm, Cm, D


def random_ssd_inputs(seed: int, B: int, L: int, H: int, P: int, G: int, N: int):
    """Inputs of the SSD scan alone, drawn as Mamba-2 initialises them:
    x, B, C ~ N(0,1); the step dt log-uniform in [1e-3, 1e-1] (the range its
    dt bias is initialised to give); A = -U(1, 16) per head; D = 1.
    Returns float32 arrays x [B,L,H,P], dt [B,L,H], A [H], Bm, Cm [B,L,G,N], D [H]."""
    rng = np.random.default_rng(seed)
    x = rng.normal(0.0, 1.0, size=(B, L, H, P)).astype(np.float32)
    dt = np.exp(rng.uniform(math.log(1e-3), math.log(1e-1), size=(B, L, H))).astype(np.float32)
    A = (-rng.uniform(1.0, 16.0, size=(H,))).astype(np.float32)
    Bm = rng.normal(0.0, 1.0, size=(B, L, G, N)).astype(np.float32)
    Cm = rng.normal(0.0, 1.0, size=(B, L, G, N)).astype(np.float32)
    D = np.ones((H,), dtype=np.float32)
    return x, dt, A, Bm, Cm, D
