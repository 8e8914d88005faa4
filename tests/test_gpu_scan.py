"""GPU parity: the standalone selective scan against the oracle's float64
sequential recurrence (fp32 <= 1e-3, bf16 <= 2e-2), with initial and final
states, ragged and degenerate sizes, and bit-exact causality and
determinism."""

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
    return torch, abi


def run_scan(env, u, dr, bias, A, Bm, Cm, D, h0=None, dtype="f32", want_h=True):
    torch, abi = env
    Bsz, L, E = u.shape
    N = A.shape[1]
    tdt = torch.float32 if dtype == "f32" else torch.bfloat16
    dev = lambda a, t=torch.float32: torch.from_numpy(np.ascontiguousarray(a, dtype=np.float32)).to("cuda").to(t)
    ud, drd = dev(u, tdt), dev(dr, tdt)
    y = torch.zeros((Bsz, L, E), dtype=tdt, device="cuda")
    hl = torch.zeros((Bsz, E, N), dtype=torch.float32, device="cuda") if want_h else None
    abi.selective_scan_forward(ud, drd, dev(bias), dev(A), dev(Bm), dev(Cm), dev(D),
                               None if h0 is None else dev(h0), y, hl, Bsz, L, E, N,
                               abi.F32 if dtype == "f32" else abi.BF16)
    torch.cuda.synchronize()
    return to_np(y), (to_np(hl) if want_h else None)


def oracle_scan(u, dr, bias, A, Bm, Cm, D, h0=None):
    delta = O.softplus(np.asarray(dr, np.float64) + np.asarray(bias, np.float64))
    return O.selective_scan(u, delta, A, Bm, Cm, D, h0)


# (B, L, E): covers 16, 8 and 4 states per thread (many to few channels),
# ragged L and E
SHAPES = [(1, 64, 128), (2, 37, 40), (3, 1, 16), (64, 256, 512), (1, 300, 8), (4, 2048, 96),
          (16, 33, 4096), (32, 20, 4096), (4, 70, 4096)]


@pytest.mark.parametrize("B,L,E", SHAPES)
def test_scan_fp32(env, B, L, E):
    args = S.random_scan_inputs(B * 1000 + L + E, B, L, E, 16)
    y, hl = run_scan(env, *args)
    yr, hr = oracle_scan(*args)
    assert rel_err(y, yr) <= TOL_F32
    assert rel_err(hl, hr) <= TOL_F32


@pytest.mark.parametrize("B,L,E", [(2, 100, 64), (64, 256, 512)])
def test_scan_bf16(env, B, L, E):
    from ternary_weight_selective_b200.synthetic import round_to_bf16
    u, dr, bias, A, Bm, Cm, D = S.random_scan_inputs(7 + L, B, L, E, 16)
    u, dr = round_to_bf16(u), round_to_bf16(dr)
    y, _ = run_scan(env, u, dr, bias, A, Bm, Cm, D, dtype="bf16")
    yr, _ = oracle_scan(u, dr, bias, A, Bm, Cm, D)
    assert rel_err(y, yr) <= TOL_BF16


def test_scan_initial_state_and_segmenting(env):
    B, L, E = 2, 90, 48
    u, dr, bias, A, Bm, Cm, D = S.random_scan_inputs(11, B, L, E, 16)
    h0 = np.random.default_rng(3).normal(size=(B, E, 16)).astype(np.float32)
    y, hl = run_scan(env, u, dr, bias, A, Bm, Cm, D, h0=h0)
    yr, hr = oracle_scan(u, dr, bias, A, Bm, Cm, D, h0)
    assert rel_err(y, yr) <= TOL_F32 and rel_err(hl, hr) <= TOL_F32
    # two GPU segments chained through h_last == one pass
    s = 41
    ya, ha = run_scan(env, u[:, :s], dr[:, :s], bias, A, Bm[:, :s], Cm[:, :s], D, h0=h0)
    yb, hb = run_scan(env, u[:, s:], dr[:, s:], bias, A, Bm[:, s:], Cm[:, s:], D, h0=ha)
    assert rel_err(np.concatenate([ya, yb], 1), yr) <= TOL_F32
    assert rel_err(hb, hr) <= TOL_F32


def test_scan_empty_sequence_copies_state(env):
    torch, abi = env
    h0 = torch.randn((2, 16, 16), device="cuda")
    hl = torch.zeros_like(h0)
    abi.selective_scan_forward(None, None, None, None, None, None, None, h0, None, hl, 2, 0, 16, 16,
                               abi.F32)
    torch.cuda.synchronize()
    assert torch.equal(h0, hl)


def test_scan_causality_and_determinism(env):
    B, L, E = 2, 128, 64
    args = list(S.random_scan_inputs(5, B, L, E, 16))
    y1, _ = run_scan(env, *args)
    y2, _ = run_scan(env, *args)
    assert np.array_equal(y1, y2)
    t0 = 70
    args[0] = args[0].copy()
    args[0][:, t0] += 4.0
    y3, _ = run_scan(env, *args)
    assert np.array_equal(y1[:, :t0], y3[:, :t0])
    assert not np.array_equal(y1[:, t0:], y3[:, t0:])


def test_scan_special_cases(env):
    # C = 0: y = D u exactly (up to the output rounding); A = 0: prefix sums
    B, L, E = 1, 50, 32
    u, dr, bias, A, Bm, Cm, D = S.random_scan_inputs(13, B, L, E, 16)
    y, _ = run_scan(env, u, dr, bias, A, Bm, np.zeros_like(Cm), D)
    assert np.allclose(y, D * u, rtol=0, atol=0)
    y, _ = run_scan(env, u, dr, bias, np.zeros_like(A), Bm, Cm, D)
    yr, _ = oracle_scan(u, dr, bias, np.zeros_like(A), Bm, Cm, D)
    assert rel_err(y, yr) <= TOL_F32
