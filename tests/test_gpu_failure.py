"""The failure-detection path on the GPU, exercised without a fault: a wait
on a barrier that nothing completes runs out after its (short) limit, the
kernel records it in the device error word and returns, the host reads the
status, and the context keeps working."""

import pytest

from ternary_weight_selective_b200 import synthetic as S

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def env(cuda_ok):
    import torch
    from ternary_weight_selective_b200 import bitssm as abi
    from ternary_weight_selective_b200 import device as dev
    return torch, abi, dev


def test_bounded_wait_runs_out_and_is_reported(env):
    torch, abi, dev = env
    assert abi.bitssm_device_error(clear=True) == 0
    abi.bitssm_selftest_wait(2000)  # 2 ms
    torch.cuda.synchronize()
    flags = abi.bitssm_device_error(clear=True)
    assert flags == 8  # bit 3: the self-test wait; no other wait ran out
    assert abi.bitssm_device_error(clear=False) == 0  # cleared
    # the context is still usable: a forward runs and matches a second one
    wl = S.Workload("after_timeout", 2, 32, 256, 512, 16, 16, "bf16", "A8")
    x, layers = S.make_inputs(wl, seed=4)
    d_l = dev.DeviceLayer(layers[0], abi.A8).prepare()
    B, L, d = x.shape
    xd = dev.to_device_input(x, abi.BF16)
    n = abi.bitssm_workspace_size(d_l.layer, B, L, abi.BF16, abi.A8)
    ws = dev.Workspace(n)
    o1, o2 = torch.zeros_like(xd), torch.zeros_like(xd)
    abi.bitssm_forward(d_l.layer, xd, o1, None, B, L, abi.BF16, abi.A8, ws.addr, n)
    abi.bitssm_forward(d_l.layer, xd, o2, None, B, L, abi.BF16, abi.A8, ws.addr, n)
    torch.cuda.synchronize()
    assert abi.bitssm_device_error(clear=True) == 0
    assert torch.equal(o1, o2) and o1.abs().sum().item() > 0


def test_selftest_limit_is_checked(env):
    torch, abi, dev = env
    for bad in (0, 1000001):
        with pytest.raises(abi.BitssmError):
            abi.bitssm_selftest_wait(bad)
