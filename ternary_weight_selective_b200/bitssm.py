"""ctypes binding of libbitssm.so (include/bitssm.h).

Argument marshalling only: every function here forwards to the C entry point
of the same name; every step of the computation runs in the library's CUDA
kernels.  Pointer arguments accept an ``int`` device address, ``None`` (a
null pointer), or any object with ``data_ptr()`` (a torch tensor).  Streams
accept an ``int`` handle, ``None`` or a ``torch.cuda.Stream``.

The library must exist: importing this module raises when it cannot be
loaded, and there is no fallback of any kind.
"""

from __future__ import annotations

import ctypes
import os

HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(HERE, "libbitssm.so")

OK = 0
ERR_INVALID_ARG = 1
ERR_UNSUPPORTED_SHAPE = 2
ERR_WORKSPACE = 3
ERR_CUDA = 4
ERR_TIMEOUT = 5
ERR_DEVICE_FLAG = 6

F32, BF16, I32, I16 = 0, 1, 2, 3
A8, A16 = 0, 1
KEEP_CODES = 1


class BitssmError(RuntimeError):
    def __init__(self, status: int, where: str):
        msg = f"{where}: {bitssm_status_string(status)} (status {status})"
        if status == ERR_CUDA:
            msg += f" [{bitssm_last_error()}]"
        super().__init__(msg)
        self.status = status


def _load():
    if not os.path.exists(LIB_PATH):
        raise ImportError(
            f"{LIB_PATH} is missing: build it with `python -m ternary_weight_selective_b200.build`")
    return ctypes.CDLL(LIB_PATH)


_lib = _load()

_vp = ctypes.c_void_p
_sz = ctypes.c_size_t
_i = ctypes.c_int


class bitssm_tw(ctypes.Structure):
    _fields_ = [("packed", _vp), ("scales", _vp), ("n_out", _i), ("k_in", _i), ("group", _i)]


class bitssm_layer(ctypes.Structure):
    _fields_ = [("in_proj", bitssm_tw), ("dt_down", bitssm_tw), ("b_proj", bitssm_tw),
                ("c_proj", bitssm_tw), ("dt_up", bitssm_tw), ("out_proj", bitssm_tw),
                ("A", _vp), ("D", _vp), ("dt_bias", _vp),
                ("d_model", _i), ("d_inner", _i), ("d_state", _i), ("dt_rank", _i),
                ("prepared", _vp), ("flags", _i),
                ("z_proj", bitssm_tw), ("conv_w", _vp), ("conv_b", _vp), ("d_conv", _i)]


class bitssm_ws_view(ctypes.Structure):
    _fields_ = [(n, _sz) for n in ("q_x", "deq_x", "u", "q_u", "deq_u", "Bm", "Cm", "q_dt",
                                   "deq_dt", "y", "q_y", "deq_y", "r_x", "dt_low", "r_dt",
                                   "delta_raw", "r_y", "u_scale", "delta", "u_pre", "z")] + \
               [("ld_qx", _i), ("ld_qu", _i), ("ld_qdt", _i), ("u_dtype", _i)]


_P_TW = ctypes.POINTER(bitssm_tw)
_P_LAYER = ctypes.POINTER(bitssm_layer)

_SIGS = {
    "bitssm_version": (_i, []),
    "bitssm_status_string": (ctypes.c_char_p, [_i]),
    "bitssm_last_error": (ctypes.c_char_p, []),
    "bitssm_device_error": (_i, [ctypes.POINTER(ctypes.c_uint), _i]),
    "bitssm_pack_workspace_size": (_i, [_i, _i, _i, ctypes.POINTER(_sz)]),
    "bitssm_pack_ternary": (_i, [_vp, _i, _i, _i, _vp, _vp, _vp, _sz, _vp]),
    "bitlinear_workspace_size": (_i, [_P_TW, _i, _i, ctypes.POINTER(_sz)]),
    "bitlinear_forward": (_i, [_P_TW, _vp, _i, _i, _vp, _i, _i, _vp, _sz, _vp]),
    "bitlinear_forward_noalloc": (_i, [_P_TW, _vp, _i, _i, _vp, _i, _i, _vp]),
    "selective_scan_forward": (_i, [_vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp,
                                    _i, _i, _i, _i, _i, _vp]),
    "bitssm_workspace_size": (_i, [_P_LAYER, _i, _i, _i, _i, ctypes.POINTER(_sz)]),
    "bitssm_forward": (_i, [_P_LAYER, _vp, _vp, _vp, _i, _i, _i, _i, _vp, _sz, _vp]),
    "bitssm_forward_state": (_i, [_P_LAYER, _vp, _vp, _vp, _vp, _i, _i, _i, _i, _vp, _sz, _vp]),
    "bitssm_step": (_i, [_P_LAYER, _vp, _vp, _vp, _vp, _i, _i, _i, _vp, _sz, _vp]),
    "bitssm_stack_forward": (_i, [_P_LAYER, _i, _vp, _vp, _i, _i, _i, _i, _vp, _sz, _vp]),
    "bitssm_forward_host": (_i, [_P_LAYER, _i, _vp, _vp, _i, _i, _i, _i, _vp, _vp, _vp, _sz, _i,
                                 _vp]),
    "bitssm_forward_launches": (_i, [_P_LAYER, _i, _i, _i]),
    "bitssm_selftest_wait": (_i, [ctypes.c_uint, _vp]),
    "ssd_scan_forward": (_i, [_vp] * 9 + [_i] * 6 + [_vp]),
    "bitssm_check_packed": (_i, [_vp, _i, _i, ctypes.POINTER(ctypes.c_long)]),
    "bitssm_forward_timed": (_i, [_P_LAYER, _vp, _vp, _vp, _i, _i, _i, _i, _vp, _sz,
                                  ctypes.POINTER(_vp), _i, _vp]),
    "bitssm_prepared_size": (_i, [_P_LAYER, _i, ctypes.POINTER(_sz)]),
    "bitssm_prepare_weights": (_i, [_P_LAYER, _i, _vp, _sz, _vp]),
    "bitssm_workspace_layout": (_i, [_P_LAYER, _i, _i, _i, _i, ctypes.POINTER(bitssm_ws_view)]),
}

EXPORTS = tuple(_SIGS)

for _name, (_res, _args) in _SIGS.items():
    _f = getattr(_lib, _name)
    _f.restype = _res
    _f.argtypes = _args


def _ptr(x):
    if x is None:
        return None
    if isinstance(x, int):
        return x
    return x.data_ptr()


def _stream(s):
    if s is None:
        return None
    if isinstance(s, int):
        return s
    return s.cuda_stream


def _check(rc: int, where: str):
    if rc != OK:
        raise BitssmError(rc, where)


def bitssm_version() -> int:
    return _lib.bitssm_version()


def bitssm_status_string(status: int) -> str:
    return _lib.bitssm_status_string(status).decode()


def bitssm_last_error() -> str:
    return _lib.bitssm_last_error().decode()


def bitssm_device_error(clear: bool = True) -> int:
    """Returns the device error word (after synchronising the device)."""
    v = ctypes.c_uint(0)
    rc = _lib.bitssm_device_error(ctypes.byref(v), int(clear))
    if rc not in (OK, ERR_TIMEOUT):
        _check(rc, "bitssm_device_error")
    return v.value


def bitssm_pack_workspace_size(n_out: int, k_in: int, group: int) -> int:
    n = _sz(0)
    _check(_lib.bitssm_pack_workspace_size(n_out, k_in, group, ctypes.byref(n)),
           "bitssm_pack_workspace_size")
    return n.value


def bitssm_pack_ternary(W, n_out, k_in, group, packed, scales, ws, ws_bytes, stream=None):
    _check(_lib.bitssm_pack_ternary(_ptr(W), n_out, k_in, group, _ptr(packed), _ptr(scales),
                                    _ptr(ws), ws_bytes, _stream(stream)), "bitssm_pack_ternary")


def bitlinear_workspace_size(w: bitssm_tw, M: int, act_mode: int) -> int:
    n = _sz(0)
    _check(_lib.bitlinear_workspace_size(ctypes.byref(w), M, act_mode, ctypes.byref(n)),
           "bitlinear_workspace_size")
    return n.value


def bitlinear_forward(w: bitssm_tw, x, M, x_dtype, y, y_dtype, act_mode, ws, ws_bytes,
                      stream=None):
    _check(_lib.bitlinear_forward(ctypes.byref(w), _ptr(x), M, x_dtype, _ptr(y), y_dtype,
                                  act_mode, _ptr(ws), ws_bytes, _stream(stream)),
           "bitlinear_forward")


NOALLOC_SCRATCH_BYTES = 16 << 20


def bitlinear_forward_noalloc(w: bitssm_tw, x, M, x_dtype, y, y_dtype, act_mode, stream=None):
    """bitlinear_forward on the library's built-in scratch array, for callers
    that cannot allocate device memory (see include/bitssm.h)."""
    _check(_lib.bitlinear_forward_noalloc(ctypes.byref(w), _ptr(x), M, x_dtype, _ptr(y), y_dtype,
                                          act_mode, _stream(stream)), "bitlinear_forward_noalloc")


def selective_scan_forward(u, delta_raw, delta_bias, A, Bm, Cm, D, h0, y, h_last,
                           B, L, E, N, dtype, stream=None):
    _check(_lib.selective_scan_forward(_ptr(u), _ptr(delta_raw), _ptr(delta_bias), _ptr(A),
                                       _ptr(Bm), _ptr(Cm), _ptr(D), _ptr(h0), _ptr(y),
                                       _ptr(h_last), B, L, E, N, dtype, _stream(stream)),
           "selective_scan_forward")


def bitssm_workspace_size(layer: bitssm_layer, B, L, dtype, act_mode) -> int:
    n = _sz(0)
    _check(_lib.bitssm_workspace_size(ctypes.byref(layer), B, L, dtype, act_mode,
                                      ctypes.byref(n)), "bitssm_workspace_size")
    return n.value


def bitssm_forward(layer: bitssm_layer, x, out, residual, B, L, dtype, act_mode, ws, ws_bytes,
                   stream=None):
    _check(_lib.bitssm_forward(ctypes.byref(layer), _ptr(x), _ptr(out), _ptr(residual), B, L,
                               dtype, act_mode, _ptr(ws), ws_bytes, _stream(stream)),
           "bitssm_forward")


def bitssm_forward_state(layer: bitssm_layer, x, out, residual, h, B, L, dtype, act_mode, ws,
                         ws_bytes, stream=None):
    _check(_lib.bitssm_forward_state(ctypes.byref(layer), _ptr(x), _ptr(out), _ptr(residual),
                                     _ptr(h), B, L, dtype, act_mode, _ptr(ws), ws_bytes,
                                     _stream(stream)),
           "bitssm_forward_state")


def bitssm_step(layer: bitssm_layer, x, out, residual, h, B, dtype, act_mode, ws, ws_bytes,
                stream=None):
    _check(_lib.bitssm_step(ctypes.byref(layer), _ptr(x), _ptr(out), _ptr(residual), _ptr(h), B,
                            dtype, act_mode, _ptr(ws), ws_bytes, _stream(stream)),
           "bitssm_step")


def bitssm_check_packed(packed_host, n_out: int, k_in: int) -> int:
    """Number of invalid codes in a packed matrix in host memory (a numpy
    uint8 array or an address); 0 when the matrix is valid."""
    bad = ctypes.c_long(0)
    addr = packed_host if isinstance(packed_host, int) else packed_host.ctypes.data
    rc = _lib.bitssm_check_packed(addr, n_out, k_in, ctypes.byref(bad))
    if rc not in (OK, ERR_INVALID_ARG) or (rc == ERR_INVALID_ARG and bad.value == 0):
        _check(rc, "bitssm_check_packed")
    return bad.value


def ssd_scan_forward(x, dt, A, Bm, Cm, D, S0, y, S_last, B, L, H, P, G, N, stream=None):
    _check(_lib.ssd_scan_forward(_ptr(x), _ptr(dt), _ptr(A), _ptr(Bm), _ptr(Cm), _ptr(D), _ptr(S0),
                                 _ptr(y), _ptr(S_last), B, L, H, P, G, N, _stream(stream)),
           "ssd_scan_forward")


def bitssm_selftest_wait(limit_us: int, stream=None):
    _check(_lib.bitssm_selftest_wait(limit_us, _stream(stream)), "bitssm_selftest_wait")


def bitssm_forward_launches(layer: bitssm_layer, B, L, act_mode) -> int:
    n = _lib.bitssm_forward_launches(ctypes.byref(layer), B, L, act_mode)
    if n < 0:
        raise BitssmError(ERR_INVALID_ARG, "bitssm_forward_launches")
    return n


def bitssm_forward_timed(layer: bitssm_layer, x, out, residual, B, L, dtype, act_mode, ws,
                         ws_bytes, events, stream=None):
    """``events``: cudaEvent_t handles (ints, e.g. torch.cuda.Event.cuda_event)."""
    arr = (_vp * len(events))(*events)
    _check(_lib.bitssm_forward_timed(ctypes.byref(layer), _ptr(x), _ptr(out), _ptr(residual), B,
                                     L, dtype, act_mode, _ptr(ws), ws_bytes, arr, len(events),
                                     _stream(stream)), "bitssm_forward_timed")


def bitssm_stack_forward(layers, x, out, B, L, dtype, act_mode, ws, ws_bytes, stream=None):
    arr = (bitssm_layer * len(layers))(*layers)
    _check(_lib.bitssm_stack_forward(arr, len(layers), _ptr(x), _ptr(out), B, L, dtype,
                                     act_mode, _ptr(ws), ws_bytes, _stream(stream)),
           "bitssm_stack_forward")


def bitssm_forward_host(layers, x_host, out_host, B, L, dtype, act_mode, x_dev, out_dev, ws,
                        ws_bytes, n_chunks, stream=None):
    """x_host / out_host: host tensors (page-locked for overlap); one layer
    struct or a list of them (a residual stack)."""
    if isinstance(layers, bitssm_layer):
        layers = [layers]
    arr = (bitssm_layer * len(layers))(*layers)
    _check(_lib.bitssm_forward_host(arr, len(layers), _ptr(x_host), _ptr(out_host), B, L, dtype,
                                    act_mode, _ptr(x_dev), _ptr(out_dev), _ptr(ws), ws_bytes,
                                    n_chunks, _stream(stream)),
           "bitssm_forward_host")


def bitssm_prepared_size(layer: bitssm_layer, act_mode) -> int:
    n = _sz(0)
    _check(_lib.bitssm_prepared_size(ctypes.byref(layer), act_mode, ctypes.byref(n)),
           "bitssm_prepared_size")
    return n.value


def bitssm_prepare_weights(layer: bitssm_layer, act_mode, dst, dst_bytes, stream=None):
    _check(_lib.bitssm_prepare_weights(ctypes.byref(layer), act_mode, _ptr(dst), dst_bytes,
                                       _stream(stream)), "bitssm_prepare_weights")


def bitssm_workspace_layout(layer: bitssm_layer, B, L, dtype, act_mode) -> bitssm_ws_view:
    v = bitssm_ws_view()
    _check(_lib.bitssm_workspace_layout(ctypes.byref(layer), B, L, dtype, act_mode,
                                        ctypes.byref(v)), "bitssm_workspace_layout")
    return v
