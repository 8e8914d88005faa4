"""GPU parity: ternary packing and the standalone BitLinear against the oracle.

Bit-exact: packed bytes, absmean scales, int32 accumulators.  Floating-point
outputs: within the tolerances of tests/_helpers.py."""

import numpy as np
import pytest

from oracle import bitssm_oracle as O
from ternary_weight_selective_b200 import synthetic as S
from tests._helpers import TOL_BF16, TOL_F32, rel_err, to_np

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def env(cuda_ok):
    import torch
    from ternary_weight_selective_b200 import bitssm as abi
    from ternary_weight_selective_b200 import device as dev
    return torch, abi, dev


@pytest.mark.parametrize("shape,group", [((37, 53), 0), ((512, 256), 0), ((48, 512), 0),
                                         ((256, 300), 128), ((160, 4096), 128), ((5, 4), 0)])
def test_pack_bit_exact(env, shape, group):
    torch, abi, dev = env
    rng = np.random.default_rng(sum(shape) + group)
    W = rng.normal(0, 0.02, size=shape).astype(np.float32)
    pm = dev.PackedMatrix(W, group)
    torch.cuda.synchronize()
    Wq, s = O.absmean_ternary(W, group)
    assert np.array_equal(to_np(pm.packed), O.pack_ternary(Wq))
    assert np.array_equal(to_np(pm.scales).reshape(np.shape(s) if group else ()), s)


def _bitlinear(env, x, W, act, x_dtype, y_dtype, group=0):
    torch, abi, dev = env
    pm = dev.PackedMatrix(W, group)
    M = x.shape[0]
    xd = dev.to_device_input(x, x_dtype)
    ty = {abi.F32: torch.float32, abi.BF16: torch.bfloat16, abi.I32: torch.int32}[y_dtype]
    y = torch.zeros((M, W.shape[0]), dtype=ty, device="cuda")
    n = abi.bitlinear_workspace_size(pm.tw, M, act)
    ws = dev.Workspace(n)
    abi.bitlinear_forward(pm.tw, xd, M, x_dtype, y, y_dtype, act, ws.addr, n)
    torch.cuda.synchronize()
    assert abi.bitssm_device_error() == 0
    return to_np(y)


A8_SHAPES = [(64, 64, 128), (200, 100, 48), (1, 256, 512), (300, 512, 256), (129, 512, 48),
             (16384, 256, 512), (257, 16, 512), (130, 4, 128), (77, 384, 640)]


@pytest.mark.parametrize("M,K,N", A8_SHAPES)
def test_bitlinear_a8_accumulators_bit_exact(env, M, K, N):
    torch, abi, dev = env
    rng = np.random.default_rng(M * 7 + K * 3 + N)
    x = S.random_rows(M + K, M, K, scale=2.0, zero_rows=(0,) if M > 2 else ())
    W = rng.normal(0, 0.02, size=(N, K)).astype(np.float32)
    acc = _bitlinear(env, x, W, abi.A8, abi.F32, abi.I32)
    Wq, s = O.absmean_ternary(W)
    _, st = O.bitlinear_a8(x, Wq, s)
    assert np.array_equal(acc.astype(np.int64), st["acc"])


@pytest.mark.parametrize("M,K,N", [(64, 64, 128), (200, 100, 48), (300, 512, 256)])
@pytest.mark.parametrize("xdt", ["f32", "bf16"])
def test_bitlinear_a8_outputs(env, M, K, N, xdt):
    torch, abi, dev = env
    rng = np.random.default_rng(M + K + N)
    x = S.random_rows(M * 3 + K, M, K, dtype=xdt)
    W = rng.normal(0, 0.02, size=(N, K)).astype(np.float32)
    Wq, s = O.absmean_ternary(W)
    ref, _ = O.bitlinear_a8(x, Wq, s)
    xd = abi.F32 if xdt == "f32" else abi.BF16
    y32 = _bitlinear(env, x, W, abi.A8, xd, abi.F32)
    assert rel_err(y32, ref) <= TOL_F32
    y16 = _bitlinear(env, x, W, abi.A8, xd, abi.BF16)
    assert rel_err(y16, ref) <= TOL_BF16


@pytest.mark.parametrize("M,K,N", [(64, 128, 64), (200, 256, 160), (130, 2048, 256), (64, 4096, 2048)])
def test_bitlinear_a16(env, M, K, N):
    torch, abi, dev = env
    rng = np.random.default_rng(M + 2 * K + N)
    x = S.random_rows(M + K + 5, M, K, dtype="bf16")
    W = rng.normal(0, 0.02, size=(N, K)).astype(np.float32)
    Wq, s = O.absmean_ternary(W, 128)
    ref = O.bitlinear_a16(x, Wq, s, 128)
    y = _bitlinear(env, x, W, abi.A16, abi.BF16, abi.F32, group=128)
    # bf16 group scales inside the operand: <= 2^-9 relative per group
    assert rel_err(y, ref) <= 1e-2
    yb = _bitlinear(env, x, W, abi.A16, abi.BF16, abi.BF16, group=128)
    assert rel_err(yb, ref) <= TOL_BF16


def test_bitlinear_empty_and_errors(env):
    torch, abi, dev = env
    W = np.random.default_rng(0).normal(0, 0.02, size=(32, 64)).astype(np.float32)
    pm = dev.PackedMatrix(W, 0)
    n = abi.bitlinear_workspace_size(pm.tw, 0, abi.A8)
    ws = dev.Workspace(n)
    abi.bitlinear_forward(pm.tw, None, 0, abi.F32, None, abi.F32, abi.A8, ws.addr, n)
    with pytest.raises(abi.BitssmError) as e:
        abi.bitlinear_forward(pm.tw, ws.addr, 4, abi.F32, ws.addr, abi.F32, abi.A8, ws.addr, 0)
    assert e.value.status == abi.ERR_WORKSPACE
    with pytest.raises(abi.BitssmError) as e:
        abi.bitlinear_forward(pm.tw, ws.addr, 4, 7, ws.addr, abi.F32, abi.A8, ws.addr, n)
    assert e.value.status == abi.ERR_INVALID_ARG
