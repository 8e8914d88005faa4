"""GPU parity of the SSD scan (ssd_scan_forward) against the oracle's
step-by-step recurrence: y and the final state within 1e-3 (float32
recurrence against float64), over head/group layouts, state sizes 16 to 128,
ragged lengths, a carried state (also updated in place), and the Mamba-2
1.3B shape (64 heads of 64, N = 128, 4 x 2048 tokens) on sampled sequences."""

import numpy as np
import pytest

from oracle import ssd_oracle as SSD
from ternary_weight_selective_b200 import synthetic as S
from tests._helpers import TOL_F32, rel_err, to_np

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def env(cuda_ok):
    import torch
    from ternary_weight_selective_b200 import bitssm as abi
    return torch, abi


def run_gpu(env, x, dt, A, Bm, Cm, D, S0=None, in_place=False):
    torch, abi = env
    Bsz, L, H, P = x.shape
    G, N = Bm.shape[2], Bm.shape[3]
    dev = lambda a: torch.from_numpy(np.ascontiguousarray(a, dtype=np.float32)).cuda()
    xd, dtd, Ad, Bd, Cd, Dd = map(dev, (x, dt, A, Bm, Cm, D))
    y = torch.full((Bsz, L, H, P), float("nan"), device="cuda")
    s0 = dev(S0) if S0 is not None else None
    s_last = s0 if in_place else torch.full((Bsz, H, P, N), float("nan"), device="cuda")
    abi.ssd_scan_forward(xd, dtd, Ad, Bd, Cd, Dd, s0, y, s_last, Bsz, L, H, P, G, N)
    torch.cuda.synchronize()
    return to_np(y), to_np(s_last)


@pytest.mark.parametrize("Bsz,L,H,P,G,N", [
    (2, 37, 4, 32, 2, 16),
    (3, 16, 6, 16, 3, 32),
    (1, 70, 2, 64, 1, 128),
    (2, 1, 4, 32, 4, 16),
    (1, 129, 8, 8, 2, 64),
])
def test_ssd_matches_oracle(env, Bsz, L, H, P, G, N):
    args = S.random_ssd_inputs(Bsz * 1000 + L, Bsz, L, H, P, G, N)
    y, s_last = run_gpu(env, *args)
    y_ref, s_ref = SSD.ssd_sequential(*args)
    assert rel_err(y, y_ref) <= TOL_F32
    assert rel_err(s_last, s_ref) <= TOL_F32


@pytest.mark.parametrize("in_place", [False, True])
def test_ssd_carried_state(env, in_place):
    Bsz, L, H, P, G, N = 2, 40, 4, 32, 1, 32
    x, dt, A, Bm, Cm, D = S.random_ssd_inputs(77, Bsz, L, H, P, G, N)
    S0 = np.random.default_rng(78).normal(size=(Bsz, H, P, N)).astype(np.float32)
    y, s_last = run_gpu(env, x, dt, A, Bm, Cm, D, S0=S0, in_place=in_place)
    y_ref, s_ref = SSD.ssd_sequential(x, dt, A, Bm, Cm, D, S0=S0)
    assert rel_err(y, y_ref) <= TOL_F32
    assert rel_err(s_last, s_ref) <= TOL_F32
    # zero length: the state passes through unchanged
    _, s_pass = run_gpu(env, x[:, :0], dt[:, :0], A, Bm[:, :0], Cm[:, :0], D, S0=S0)
    assert np.array_equal(s_pass, S0)


def test_ssd_mamba2_1p3b_shape_sampled(env):
    """64 heads x 64 channels, N = 128, one B/C group, 4 sequences of 2048:
    sequences 0 and 3 against the oracle (sequences are independent)."""
    Bsz, L, H, P, G, N = 4, 2048, 64, 64, 1, 128
    x, dt, A, Bm, Cm, D = S.random_ssd_inputs(5, Bsz, L, H, P, G, N)
    y, s_last = run_gpu(env, x, dt, A, Bm, Cm, D)
    assert np.isfinite(y).all()
    for b in (0, 3):
        sl = slice(b, b + 1)
        y_ref, s_ref = SSD.ssd_sequential(x[sl], dt[sl], A, Bm[sl], Cm[sl], D)
        assert rel_err(y[sl], y_ref) <= TOL_F32
        assert rel_err(s_last[sl], s_ref) <= TOL_F32
