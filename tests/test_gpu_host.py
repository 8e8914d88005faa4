"""GPU checks of bitssm_forward_host: the forward on host buffers with the
copies overlapped (chunks of whole sequences).  Sequences are independent,
so any chunking must reproduce the device-buffer forward bit for bit."""

import pytest

from ternary_weight_selective_b200 import synthetic as S

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def env(cuda_ok):
    import torch
    from ternary_weight_selective_b200 import bitssm as abi
    from ternary_weight_selective_b200 import device as dev
    return torch, abi, dev


CASES = [
    (S.Workload("h_fused", 5, 64, 256, 512, 16, 16, "bf16", "A8"), 1),
    (S.Workload("h_stack", 4, 48, 256, 512, 16, 16, "bf16", "A8", layers=2), 2),
    (S.Workload("h_a16", 3, 40, 128, 256, 16, 16, "bf16", "A16"), 1),
    (S.Workload("h_six", 3, 37, 64, 128, 16, 4, "f32", "A8"), 1),
]


@pytest.mark.parametrize("wl,n_layers", CASES, ids=[c[0].name for c in CASES])
@pytest.mark.parametrize("n_chunks,pinned", [(1, True), (3, True), (2, False)])
def test_host_forward_equals_device_forward(env, wl, n_layers, n_chunks, pinned):
    torch, abi, dev = env
    x, layers = S.make_inputs(wl, seed=5)
    amode = abi.A16 if wl.act_mode == "A16" else abi.A8
    dtype = abi.BF16 if wl.io_dtype == "bf16" else abi.F32
    dl = [dev.DeviceLayer(lw, amode).prepare() for lw in layers]
    B, L, d = x.shape
    xd = dev.to_device_input(x, dtype)
    n = abi.bitssm_workspace_size(dl[0].layer, B, L, dtype, amode)
    ws = dev.Workspace(n)
    ref = torch.zeros_like(xd)
    if n_layers == 1:
        abi.bitssm_forward(dl[0].layer, xd, ref, None, B, L, dtype, amode, ws.addr, n)
    else:
        abi.bitssm_stack_forward([t.layer for t in dl], xd, ref, B, L, dtype, amode, ws.addr, n)
    x_host = torch.empty(xd.shape, dtype=xd.dtype, pin_memory=pinned)
    x_host.copy_(xd.cpu())
    out_host = torch.zeros(xd.shape, dtype=xd.dtype, pin_memory=pinned)
    x_dev = torch.empty_like(xd)
    out_dev = torch.empty_like(xd)
    # a workspace for one chunk is enough
    bc = -(-B // min(n_chunks, B))
    nc = abi.bitssm_workspace_size(dl[0].layer, bc, L, dtype, amode)
    wsc = dev.Workspace(nc)
    abi.bitssm_forward_host([t.layer for t in dl], x_host, out_host, B, L, dtype, amode, x_dev,
                            out_dev, wsc.addr, nc, n_chunks)
    torch.cuda.synchronize()
    assert abi.bitssm_device_error() == 0
    assert torch.equal(out_host, ref.cpu())
    assert torch.equal(out_dev, ref)


def test_host_forward_unprepared_weights(env):
    """Without prepared weights every chunk expands them into its workspace."""
    torch, abi, dev = env
    wl = CASES[0][0]
    x, layers = S.make_inputs(wl, seed=9)
    d_l = dev.DeviceLayer(layers[0], abi.A8)
    B, L, d = x.shape
    xd = dev.to_device_input(x, abi.BF16)
    n = abi.bitssm_workspace_size(d_l.layer, B, L, abi.BF16, abi.A8)
    ws = dev.Workspace(n)
    ref = torch.zeros_like(xd)
    abi.bitssm_forward(d_l.layer, xd, ref, None, B, L, abi.BF16, abi.A8, ws.addr, n)
    xh = xd.cpu().pin_memory()
    oh = torch.zeros_like(xh).pin_memory()
    abi.bitssm_forward_host(d_l.layer, xh, oh, B, L, abi.BF16, abi.A8, torch.empty_like(xd),
                            torch.empty_like(xd), ws.addr, n, 2)
    torch.cuda.synchronize()
    assert torch.equal(oh, ref.cpu())


def test_host_forward_argument_errors(env):
    torch, abi, dev = env
    wl = CASES[0][0]
    x, layers = S.make_inputs(wl, seed=5)
    d_l = dev.DeviceLayer(layers[0], abi.A8).prepare()
    B, L, d = x.shape
    xd = dev.to_device_input(x, abi.BF16)
    n = abi.bitssm_workspace_size(d_l.layer, B, L, abi.BF16, abi.A8)
    ws = dev.Workspace(n)
    xh = xd.cpu().pin_memory()
    oh = torch.empty_like(xh).pin_memory()
    for bad_chunks in (0, 17):
        with pytest.raises(abi.BitssmError):
            abi.bitssm_forward_host(d_l.layer, xh, oh, B, L, abi.BF16, abi.A8, xd,
                                    torch.empty_like(xd), ws.addr, n, bad_chunks)
    with pytest.raises(abi.BitssmError):
        abi.bitssm_forward_host(d_l.layer, None, oh, B, L, abi.BF16, abi.A8, xd,
                                torch.empty_like(xd), ws.addr, n, 2)
    # too small a workspace for the chunk is reported, not written past
    with pytest.raises(abi.BitssmError):
        abi.bitssm_forward_host(d_l.layer, xh, oh, B, L, abi.BF16, abi.A8, xd,
                                torch.empty_like(xd), ws.addr, 256, 2)
    torch.cuda.synchronize()
