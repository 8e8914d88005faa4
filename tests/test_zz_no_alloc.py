"""bitlinear_forward_noalloc: the BitLinear entry point for callers that
cannot allocate device memory (an operator inside a host framework whose
allocator owns every device byte, code held to a memory budget fixed at
start-up, latency-critical paths that must not pay for an allocation).  It
runs on a scratch array built into the library instead of a caller
workspace.

Checked through the C ABI against bitlinear_forward with a caller
workspace, on two calls in a row (different weights and inputs, so the
second call runs on scratch the first one left behind), plus the rejection
of a shape that needs more than the built-in array.  This file is collected
last so that a failure here stops a run only after every other test."""

import numpy as np
import pytest

from ternary_weight_selective_b200 import synthetic as S
from tests._helpers import TOL_F32, rel_err, to_np

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def env(cuda_ok):
    import torch
    from ternary_weight_selective_b200 import bitssm as abi
    from ternary_weight_selective_b200 import device as dev
    return torch, abi, dev


def _case(dev, seed, M, K, N, xdt, group):
    rng = np.random.default_rng(seed)
    W = rng.normal(0, 0.02, size=(N, K)).astype(np.float32)
    pm = dev.PackedMatrix(W, group)
    x = S.random_rows(seed + 1, M, K, dtype=xdt)
    return pm, x


def _with_workspace(torch, abi, dev, pm, xd, M, x_dtype, y_dtype, act):
    y = torch.zeros((M, pm.n_out), dtype={abi.F32: torch.float32, abi.I32: torch.int32}[y_dtype],
                    device="cuda")
    n = abi.bitlinear_workspace_size(pm.tw, M, act)
    ws = dev.Workspace(n)
    abi.bitlinear_forward(pm.tw, xd, M, x_dtype, y, y_dtype, act, ws.addr, n)
    torch.cuda.synchronize()
    return to_np(y)


def _no_alloc(torch, abi, pm, xd, M, x_dtype, y_dtype, act):
    y = torch.zeros((M, pm.n_out), dtype={abi.F32: torch.float32, abi.I32: torch.int32}[y_dtype],
                    device="cuda")
    abi.bitlinear_forward_noalloc(pm.tw, xd, M, x_dtype, y, y_dtype, act)
    torch.cuda.synchronize()
    return to_np(y)


def test_noalloc_matches_workspace_path_two_calls(env):
    torch, abi, dev = env
    cases = [
        # (seed, M, K, N, x dtype, act, y dtype)
        (1, 300, 512, 256, "bf16", abi.A8, abi.I32),
        (2, 1000, 256, 512, "f32", abi.A8, abi.F32),
    ]
    for seed, M, K, N, xdt, act, ydt in cases:
        pm, x = _case(dev, seed, M, K, N, xdt, 0)
        x_dtype = abi.BF16 if xdt == "bf16" else abi.F32
        xd = dev.to_device_input(x, x_dtype)
        got = _no_alloc(torch, abi, pm, xd, M, x_dtype, ydt, act)
        ref = _with_workspace(torch, abi, dev, pm, xd, M, x_dtype, ydt, act)
        if ydt == abi.I32:
            assert np.array_equal(got, ref)
        else:
            assert rel_err(got, ref) <= TOL_F32
    assert abi.bitssm_device_error() == 0


def test_noalloc_a16_and_repeat(env):
    torch, abi, dev = env
    pm, x = _case(dev, 3, 200, 512, 384, "bf16", 128)
    xd = dev.to_device_input(x, abi.BF16)
    a = _no_alloc(torch, abi, pm, xd, 200, abi.BF16, abi.F32, abi.A16)
    b = _no_alloc(torch, abi, pm, xd, 200, abi.BF16, abi.F32, abi.A16)
    ref = _with_workspace(torch, abi, dev, pm, xd, 200, abi.BF16, abi.F32, abi.A16)
    assert np.array_equal(a, b)
    assert rel_err(a, ref) <= TOL_F32


def test_noalloc_rejects_shapes_beyond_the_scratch(env):
    torch, abi, dev = env
    pm, _ = _case(dev, 4, 4, 512, 64, "f32", 0)
    M = 40000  # 40000 rows x 512 codes alone exceed 16 MiB
    assert abi.bitlinear_workspace_size(pm.tw, M, abi.A8) > abi.NOALLOC_SCRATCH_BYTES
    x = torch.zeros((M, 512), dtype=torch.float32, device="cuda")
    y = torch.zeros((M, 64), dtype=torch.float32, device="cuda")
    with pytest.raises(abi.BitssmError) as e:
        abi.bitlinear_forward_noalloc(pm.tw, x, M, abi.F32, y, abi.F32, abi.A8)
    assert e.value.status == abi.ERR_WORKSPACE
    assert "needs" in abi.bitssm_last_error()
