"""ctypes access to the C host oracle (oracle/c/bitssm_oracle.h).

TEST INFRASTRUCTURE ONLY, like the rest of oracle/.  The functions take
numpy arrays (host memory) and return numpy arrays."""

from __future__ import annotations

import ctypes

import numpy as np

from . import build_oracle

_lib = ctypes.CDLL(build_oracle.build())
_p = ctypes.c_void_p
_i = ctypes.c_int


class oracle_layer(ctypes.Structure):
    _fields_ = [(n, _p) for n in ("Wq_in", "Wq_dt_down", "Wq_b", "Wq_c", "Wq_dt_up", "Wq_out",
                                  "s_in", "s_dt_down", "s_b", "s_c", "s_dt_up", "s_out",
                                  "A", "D", "dt_bias")] + \
               [(n, _i) for n in ("d_model", "d_inner", "d_state", "dt_rank", "group")] + \
               [("Wq_z", _p), ("s_z", _p), ("conv_w", _p), ("conv_b", _p), ("d_conv", _i)]


_lib.oracle_absmean_ternary.argtypes = [_p, _i, _i, _i, _p, _p]
_lib.oracle_pack_ternary.argtypes = [_p, _i, _i, _p]
_lib.oracle_absmax_codes.argtypes = [_p, ctypes.c_long, _i, _p, _p]
_lib.oracle_bitlinear_forward.argtypes = [_p, _i, _i, _p, _p, _i, _i, _i, _p]
_lib.oracle_selective_scan_forward.argtypes = [_p] * 9 + [_i] * 4
_lib.oracle_bitssm_forward.argtypes = [ctypes.POINTER(oracle_layer), _p, _p, _i, _i, _i, _p, _p]
_lib.oracle_ssd_scan_forward.argtypes = [_p] * 9 + [_i] * 6
_lib.oracle_ssd_scan_forward.restype = _i
_lib.oracle_set_threads.argtypes = [_i]
_lib.oracle_set_threads.restype = _i


def set_threads(n: int) -> int:
    """Threads of the oracle's parallel loops from now on; returns the previous count."""
    return _lib.oracle_set_threads(n)


for _f in ("oracle_absmean_ternary", "oracle_pack_ternary", "oracle_absmax_codes",
           "oracle_bitlinear_forward", "oracle_selective_scan_forward", "oracle_bitssm_forward"):
    getattr(_lib, _f).restype = _i


def _c(a, dtype):
    return np.ascontiguousarray(a, dtype=dtype)


def _ptr(a):
    return None if a is None else a.ctypes.data


def _ok(rc, where):
    if rc != 0:
        raise ValueError(f"{where}: invalid argument")


def absmean_ternary(W, group=0):
    W = _c(W, np.float32)
    n, k = W.shape
    Wq = np.zeros((n, k), np.int8)
    s = np.zeros((1,) if group == 0 else (n, -(-k // group)), np.float32)
    _ok(_lib.oracle_absmean_ternary(_ptr(W), n, k, group, _ptr(Wq), _ptr(s)), "absmean_ternary")
    return Wq, (s.reshape(()) if group == 0 else s)


def pack_ternary(Wq):
    Wq = _c(Wq, np.int8)
    n, k = Wq.shape
    out = np.zeros((n, -(-k // 4)), np.uint8)
    _ok(_lib.oracle_pack_ternary(_ptr(Wq), n, k, _ptr(out)), "pack_ternary")
    return out


def absmax_codes(v):
    v = _c(v, np.float32)
    rows = int(np.prod(v.shape[:-1]))
    K = v.shape[-1]
    q = np.zeros(v.shape, np.int32)
    m = np.zeros(v.shape[:-1], np.float32)
    _ok(_lib.oracle_absmax_codes(_ptr(v), rows, K, _ptr(q), _ptr(m)), "absmax_codes")
    return q, m


def bitlinear(x, Wq, s, group, act_mode):
    x = _c(x, np.float32)
    M, K = x.shape
    Wq = _c(Wq, np.int8)
    s = _c(np.atleast_1d(s), np.float32)
    y = np.zeros((M, Wq.shape[0]), np.float64)
    _ok(_lib.oracle_bitlinear_forward(_ptr(x), M, K, _ptr(Wq), _ptr(s), Wq.shape[0], group,
                                      act_mode, _ptr(y)), "bitlinear_forward")
    return y


def selective_scan(u, delta, A, Bm, Cm, D, h0=None):
    u, delta, A, Bm, Cm, D = (_c(a, np.float64) for a in (u, delta, A, Bm, Cm, D))
    Bsz, L, E = u.shape
    N = A.shape[1]
    h0 = None if h0 is None else _c(h0, np.float64)
    y = np.zeros((Bsz, L, E))
    h = np.zeros((Bsz, E, N))
    _ok(_lib.oracle_selective_scan_forward(_ptr(u), _ptr(delta), _ptr(A), _ptr(Bm), _ptr(Cm),
                                           _ptr(D), _ptr(h0), _ptr(y), _ptr(h), Bsz, L, E, N),
        "selective_scan_forward")
    return y, h


class Layer:
    """Ternary codes and scales of one mixer, ternarised by the C oracle."""

    def __init__(self, lw, act_mode="A8"):
        self.act_mode = 0 if act_mode == "A8" else 1
        self.group = 0 if act_mode == "A8" else 128
        self.keep = {}
        names = ("W_in", "W_dt_down", "W_B", "W_C", "W_dt_up", "W_out")
        for n in names:
            self.keep[n] = absmean_ternary(getattr(lw, n), self.group)
        for n in ("A", "D", "dt_bias"):
            self.keep[n] = _c(getattr(lw, n), np.float32)
        qs = [self.keep[n] for n in names]
        self.s_arrays = [_c(np.atleast_1d(s), np.float32) for _, s in qs]
        self.c = oracle_layer(*[_ptr(q) for q, _ in qs], *[_ptr(s) for s in self.s_arrays],
                              _ptr(self.keep["A"]), _ptr(self.keep["D"]),
                              _ptr(self.keep["dt_bias"]),
                              lw.W_in.shape[1], lw.W_in.shape[0], lw.A.shape[1],
                              lw.W_dt_down.shape[0], self.group)
        if getattr(lw, "W_z", None) is not None:  # Mamba-1 block form
            self.keep["W_z"] = absmean_ternary(lw.W_z, self.group)
            self.keep["s_z"] = _c(np.atleast_1d(self.keep["W_z"][1]), np.float32)
            self.keep["conv_w"] = _c(lw.conv_w, np.float32)
            self.keep["conv_b"] = _c(lw.conv_b, np.float32)
            self.c.Wq_z = _ptr(self.keep["W_z"][0])
            self.c.s_z = _ptr(self.keep["s_z"])
            self.c.conv_w = _ptr(self.keep["conv_w"])
            self.c.conv_b = _ptr(self.keep["conv_b"])
            self.c.d_conv = lw.conv_w.shape[1]


def bitssm_forward(x, layer: Layer, h0=None):
    x = _c(x, np.float32)
    Bsz, L, d = x.shape
    out = np.zeros((Bsz, L, d), np.float64)
    E, N = layer.c.d_inner, layer.c.d_state
    h0 = None if h0 is None else _c(h0, np.float64)
    h = np.zeros((Bsz, E, N))
    _ok(_lib.oracle_bitssm_forward(ctypes.byref(layer.c), _ptr(x), _ptr(out), Bsz, L,
                                   layer.act_mode, _ptr(h0), _ptr(h)), "bitssm_forward")
    return out, h


def ssd_scan(x, dt, A, Bm, Cm, D, S0=None):
    x, dt, A, Bm, Cm, D = (_c(a, np.float64) for a in (x, dt, A, Bm, Cm, D))
    Bsz, L, H, P = x.shape
    G, N = Bm.shape[2], Bm.shape[3]
    S0 = None if S0 is None else _c(S0, np.float64)
    y = np.zeros_like(x)
    S = np.zeros((Bsz, H, P, N))
    _ok(_lib.oracle_ssd_scan_forward(_ptr(x), _ptr(dt), _ptr(A), _ptr(Bm), _ptr(Cm), _ptr(D),
                                     _ptr(S0), _ptr(y), _ptr(S), Bsz, L, H, P, G, N),
        "ssd_scan_forward")
    return y, S

