"""Device-side weights and buffers for the C ABI, held in torch CUDA memory.

PyTorch provides device memory and streams only; packing and every forward
step run in libbitssm.so through ``bitssm.py``.
"""

from __future__ import annotations

import numpy as np
import torch

from . import bitssm as abi


def aligned_empty(nbytes: int, device="cuda", align: int = 256):
    """uint8 device buffer of at least ``nbytes`` whose address is ``align``-aligned.
    Returns (buffer, aligned address)."""
    buf = torch.empty(max(1, nbytes) + align, dtype=torch.uint8, device=device)
    addr = buf.data_ptr()
    return buf, (addr + align - 1) // align * align


class PackedMatrix:
    """A ternary matrix packed on the device by ``bitssm_pack_ternary``."""

    def __init__(self, W: np.ndarray, group: int, device="cuda", stream=None):
        W = np.ascontiguousarray(W, dtype=np.float32)
        self.n_out, self.k_in = W.shape
        self.group = group
        Wd = torch.from_numpy(W).to(device)
        self.packed = torch.empty((self.n_out, (self.k_in + 3) // 4), dtype=torch.uint8, device=device)
        ns = 1 if group == 0 else self.n_out * ((self.k_in + group - 1) // group)
        self.scales = torch.empty((ns,), dtype=torch.float32, device=device)
        wsb = abi.bitssm_pack_workspace_size(self.n_out, self.k_in, group)
        self._ws, ws = aligned_empty(wsb, device)
        abi.bitssm_pack_ternary(Wd, self.n_out, self.k_in, group, self.packed, self.scales, ws, wsb,
                                stream)
        self.tw = abi.bitssm_tw(self.packed.data_ptr(), self.scales.data_ptr(), self.n_out,
                                self.k_in, group)


class DeviceLayer:
    """One BitSSM mixer's weights on the device (from float32 matrices)."""

    NAMES = ("W_in", "W_dt_down", "W_B", "W_C", "W_dt_up", "W_out")

    def __init__(self, lw, act_mode: int, device="cuda", stream=None):
        group = 128 if act_mode == abi.A16 else 0
        self.act_mode = act_mode
        self.mats = {n: PackedMatrix(getattr(lw, n), group, device, stream) for n in self.NAMES}
        self.A = torch.from_numpy(np.ascontiguousarray(lw.A, dtype=np.float32)).to(device)
        self.D = torch.from_numpy(np.ascontiguousarray(lw.D, dtype=np.float32)).to(device)
        self.dt_bias = torch.from_numpy(np.ascontiguousarray(lw.dt_bias, dtype=np.float32)).to(device)
        m = self.mats
        self.layer = abi.bitssm_layer(
            m["W_in"].tw, m["W_dt_down"].tw, m["W_B"].tw, m["W_C"].tw, m["W_dt_up"].tw,
            m["W_out"].tw, self.A.data_ptr(), self.D.data_ptr(), self.dt_bias.data_ptr(),
            lw.W_in.shape[1], lw.W_in.shape[0], lw.A.shape[1], lw.W_dt_down.shape[0], None, 0)
        if getattr(lw, "W_z", None) is not None:  # Mamba-1 block form
            self.mats["W_z"] = PackedMatrix(lw.W_z, group, device, stream)
            self.conv_w = torch.from_numpy(np.ascontiguousarray(lw.conv_w, dtype=np.float32)).to(device)
            self.conv_b = torch.from_numpy(np.ascontiguousarray(lw.conv_b, dtype=np.float32)).to(device)
            self.layer.z_proj = self.mats["W_z"].tw
            self.layer.conv_w = self.conv_w.data_ptr()
            self.layer.conv_b = self.conv_b.data_ptr()
            self.layer.d_conv = lw.conv_w.shape[1]
        self._prepared = None

    def prepare(self, stream=None):
        """Expand the packed weights once (``bitssm_prepare_weights``) and let the
        forward use the expanded copy."""
        n = abi.bitssm_prepared_size(self.layer, self.act_mode)
        self._prepared, addr = aligned_empty(n)
        abi.bitssm_prepare_weights(self.layer, self.act_mode, addr, n, stream)
        self.layer.prepared = addr
        return self

    def unprepare(self):
        self.layer.prepared = None
        self._prepared = None
        return self


class Workspace:
    """A reusable, 256-byte-aligned device workspace."""

    def __init__(self, nbytes: int, device="cuda"):
        self.nbytes = nbytes
        self.buf, self.addr = aligned_empty(nbytes, device)


def to_device_input(x: np.ndarray, dtype: int, device="cuda") -> torch.Tensor:
    t = torch.from_numpy(np.ascontiguousarray(x, dtype=np.float32))
    t = t.to(torch.bfloat16) if dtype == abi.BF16 else t
    return t.to(device)
