"""GPU checks of the carried-state forward and the decode step
(bitssm_forward_state / bitssm_step).

Every stage but the recurrence is token-local, and the kernels do the same
float32 arithmetic for a step whatever call it falls in, so a sequence run
in pieces, or one token at a time, with the state carried between calls
must reproduce one whole-sequence bitssm_forward bit for bit.  The carried
state itself is compared with the oracle's (float32 state, 1e-3), and the
decode outputs with the oracle's decode steps."""

import numpy as np
import pytest

from oracle import bitssm_oracle as O
from ternary_weight_selective_b200 import synthetic as S
from tests._helpers import TOL_BF16, TOL_F32, rel_err, to_np, ws_array

pytestmark = pytest.mark.gpu

# (workload, act): the fused three-kernel A8 path, the six-kernel A8 path
# (d_model = 64), and the W1.58A16 path
CASES = [
    (S.Workload("st_fused", 3, 40, 256, 512, 16, 16, "bf16", "A8"), "A8"),
    (S.Workload("st_six", 2, 37, 64, 128, 16, 4, "f32", "A8"), "A8"),
    (S.Workload("st_a16", 2, 33, 128, 256, 16, 16, "bf16", "A16"), "A16"),
]


@pytest.fixture(scope="module")
def env(cuda_ok):
    import torch
    from ternary_weight_selective_b200 import bitssm as abi
    from ternary_weight_selective_b200 import device as dev
    return torch, abi, dev


def _setup(env, wl, act):
    torch, abi, dev = env
    x, layers = S.make_inputs(wl, seed=11)
    amode = abi.A16 if act == "A16" else abi.A8
    dtype = abi.BF16 if wl.io_dtype == "bf16" else abi.F32
    dl = dev.DeviceLayer(layers[0], amode)
    return x, layers[0], dl, amode, dtype


def _ws(env, dl, B, L, dtype, amode):
    torch, abi, dev = env
    n = abi.bitssm_workspace_size(dl.layer, B, L, dtype, amode)
    return dev.Workspace(n), n


@pytest.mark.parametrize("wl,act", CASES, ids=[c[0].name for c in CASES])
def test_pieces_and_steps_reproduce_the_whole_call(env, wl, act):
    torch, abi, dev = env
    x, lw, dl, amode, dtype = _setup(env, wl, act)
    B, L, d = x.shape
    E, N = lw.W_in.shape[0], lw.A.shape[1]
    xd = dev.to_device_input(x, dtype)
    # one whole call
    ws, n = _ws(env, dl, B, L, dtype, amode)
    out_full = torch.zeros_like(xd)
    abi.bitssm_forward(dl.layer, xd, out_full, None, B, L, dtype, amode, ws.addr, n)
    h_full = torch.zeros((B, E, N), dtype=torch.float32, device="cuda")
    out_full2 = torch.zeros_like(xd)
    abi.bitssm_forward_state(dl.layer, xd, out_full2, None, h_full, B, L, dtype, amode, ws.addr, n)
    # two pieces with the state carried (a split inside a 16-step chunk)
    cut = 21
    h = torch.zeros((B, E, N), dtype=torch.float32, device="cuda")
    outs = []
    for a, b in ((0, cut), (cut, L)):
        xp = xd[:, a:b].contiguous()
        op = torch.zeros_like(xp)
        wsp, np_ = _ws(env, dl, B, b - a, dtype, amode)
        abi.bitssm_forward_state(dl.layer, xp, op, None, h, B, b - a, dtype, amode, wsp.addr, np_)
        outs.append(op)
    out_pieces = torch.cat(outs, dim=1)
    # one token at a time
    hs = torch.zeros((B, E, N), dtype=torch.float32, device="cuda")
    ws1, n1 = _ws(env, dl, B, 1, dtype, amode)
    steps = []
    for t in range(L):
        xt = xd[:, t].contiguous()
        ot = torch.zeros_like(xt)
        abi.bitssm_step(dl.layer, xt, ot, None, hs, B, dtype, amode, ws1.addr, n1)
        steps.append(ot[:, None])
    out_steps = torch.cat(steps, dim=1)
    torch.cuda.synchronize()
    assert abi.bitssm_device_error() == 0
    assert torch.equal(out_full2, out_full)
    assert torch.equal(out_pieces, out_full)
    assert torch.equal(h, h_full)
    assert torch.equal(out_steps, out_full)
    assert torch.equal(hs, h_full)
    # the carried state against the oracle's
    P = O.TernaryLayer(lw, act)
    ref_out, st = O.bitssm_layer(x, P)
    if act == "A8":
        # u, B, C and delta are exact or float32 on both sides
        assert rel_err(to_np(h_full), st["h_last"]) <= TOL_F32
    else:
        # A16 rounds u and dt_low to bf16 tensor-core operands, and that
        # rounding compounds through the recurrence: teacher-force the scan
        # with the GPU's own u, delta, B and C (the workspace of the last call)
        v = abi.bitssm_workspace_layout(dl.layer, B, L, dtype, amode)
        g = lambda off, dt, shape: ws_array(torch, ws, off, dt, shape)
        u = g(v.u, torch.bfloat16, (B, L, E))
        delta = g(v.delta, torch.float32, (B, L, E))
        Bm = g(v.Bm, torch.float32, (B, L, N))
        Cm = g(v.Cm, torch.float32, (B, L, N))
        _, h_tf = O.selective_scan(u, delta, lw.A, Bm, Cm, lw.D)
        assert rel_err(to_np(h_full), h_tf) <= TOL_F32
    if wl.io_dtype == "bf16":
        assert rel_err(to_np(out_full), ref_out) <= TOL_BF16


def test_decode_steps_against_oracle_steps(env):
    """Decode from a non-zero state: prefill 24 tokens, then 8 steps; each
    step's output and the final state against the oracle's decode steps
    started from the oracle's prefill state."""
    torch, abi, dev = env
    wl, act = CASES[0]
    x, lw, dl, amode, dtype = _setup(env, wl, act)
    B, L, d = x.shape
    E, N = lw.W_in.shape[0], lw.A.shape[1]
    P = O.TernaryLayer(lw, act)
    pre = 24
    xd = dev.to_device_input(x, dtype)
    h = torch.zeros((B, E, N), dtype=torch.float32, device="cuda")
    xp = xd[:, :pre].contiguous()
    op = torch.zeros_like(xp)
    wsp, npre = _ws(env, dl, B, pre, dtype, amode)
    abi.bitssm_forward_state(dl.layer, xp, op, None, h, B, pre, dtype, amode, wsp.addr, npre)
    _, st = O.bitssm_layer(x[:, :pre], P)
    h_ref = st["h_last"]
    ws1, n1 = _ws(env, dl, B, 1, dtype, amode)
    for t in range(pre, pre + 8):
        xt = xd[:, t].contiguous()
        ot = torch.zeros_like(xt)
        abi.bitssm_step(dl.layer, xt, ot, None, h, B, dtype, amode, ws1.addr, n1)
        o_ref, h_ref = O.bitssm_step(x[:, t], P, h_ref)
        torch.cuda.synchronize()
        assert rel_err(to_np(ot), o_ref) <= TOL_BF16
    assert rel_err(to_np(h), h_ref) <= TOL_F32
    assert abi.bitssm_device_error() == 0


def test_state_argument_errors(env):
    torch, abi, dev = env
    wl, act = CASES[0]
    x, lw, dl, amode, dtype = _setup(env, wl, act)
    B = x.shape[0]
    xt = dev.to_device_input(x[:, 0], dtype)
    ot = torch.zeros_like(xt)
    ws1, n1 = _ws(env, dl, B, 1, dtype, amode)
    with pytest.raises(abi.BitssmError):
        abi.bitssm_step(dl.layer, xt, ot, None, None, B, dtype, amode, ws1.addr, n1)
