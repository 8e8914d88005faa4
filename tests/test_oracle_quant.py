"""Pins of the oracle's quantisers and integer GEMM (CPU only).

Each expectation here comes from somewhere other than the oracle's own code:
hand-derived values, brute force in pure Python, closed forms of the weight
distribution, or a library routine in a special case.
"""

import math

import numpy as np
import pytest

from oracle import bitssm_oracle as O
from ternary_weight_selective_b200 import synthetic as S


# --- absmean ternary weights ------------------------------------------------

def test_absmean_hand_example():
    # s = (0.3 + 0.1 + 0.02 + 0.4) / 4 = 0.205; W / (s + 1e-5) =
    # [1.463, -0.488, 0.0975, -1.951] -> rint -> [1, -0, 0, -2] -> clip -> [1, 0, 0, -1]
    W = np.array([[0.3, -0.1, 0.02, -0.4]], dtype=np.float32)
    Wq, s = O.absmean_ternary(W)
    assert Wq.tolist() == [[1, 0, 0, -1]]
    assert abs(float(s) - 0.205) < 1e-7


def test_absmean_codes_and_scale_brute_force():
    rng = np.random.default_rng(1)
    W = rng.normal(0, 0.02, size=(37, 53)).astype(np.float32)
    Wq, s = O.absmean_ternary(W)
    assert set(np.unique(Wq).tolist()) <= {-1, 0, 1}
    mean_abs = math.fsum(abs(float(w)) for w in W.ravel()) / W.size
    assert abs(float(s) - mean_abs) <= np.spacing(np.float32(mean_abs))
    # brute-force code of every element from the definition
    denom = float(np.float32(np.float32(s) + np.float32(1e-5)))
    for (i, j), w in np.ndenumerate(W):
        t = float(np.float32(w) / np.float32(denom))
        code = max(-1, min(1, round(t)))  # Python round: half to even
        assert Wq[i, j] == code


def test_absmean_equal_magnitudes_give_sign():
    rng = np.random.default_rng(2)
    sign = rng.choice([-1.0, 1.0], size=(16, 40))
    W = (0.037 * sign).astype(np.float32)
    Wq, s = O.absmean_ternary(W)
    assert np.array_equal(Wq, sign.astype(np.int8))
    assert abs(float(s) - 0.037) <= 1e-8


def test_absmean_gaussian_statistics():
    # For W ~ N(0, sigma): E|W| = sigma sqrt(2/pi); a weight rounds to 0 when
    # |W| < s/2, probability erf((s/2) / (sigma sqrt 2)) = erf(sqrt(2/pi)/(2 sqrt 2)).
    sigma = 0.02
    rng = np.random.default_rng(3)
    W = rng.normal(0, sigma, size=(512, 512)).astype(np.float32)
    Wq, s = O.absmean_ternary(W)
    n = W.size
    exp_s = sigma * math.sqrt(2 / math.pi)
    assert abs(float(s) - exp_s) < 4 * sigma * math.sqrt(1 - 2 / math.pi) / math.sqrt(n)
    p0 = math.erf(math.sqrt(2 / math.pi) / (2 * math.sqrt(2)))
    assert abs(p0 - 0.3101) < 1e-4
    frac0 = float((Wq == 0).mean())
    assert abs(frac0 - p0) < 5 * math.sqrt(p0 * (1 - p0) / n) + 2e-3


def test_absmean_grouped():
    # two groups of 128 along K with very different magnitudes: each group is
    # scaled by its own mean, so both carry non-zero codes
    rng = np.random.default_rng(4)
    W = np.concatenate([rng.normal(0, 1.0, (8, 128)), rng.normal(0, 1e-3, (8, 128)),
                        rng.normal(0, 0.1, (8, 5))], axis=1).astype(np.float32)
    Wq, s = O.absmean_ternary(W, group=128)
    assert s.shape == (8, 3)
    for n in range(8):
        for j, (a, b) in enumerate([(0, 128), (128, 256), (256, 261)]):
            blk = W[n, a:b].astype(np.float64)
            assert abs(float(s[n, j]) - np.abs(blk).mean()) <= 2 * np.spacing(s[n, j])
            sub, _ = O.absmean_ternary(W[n:n + 1, a:b])
            assert np.array_equal(Wq[n, a:b], sub[0])
    assert (Wq[:, 128:256] != 0).mean() > 0.5


def test_pack_hand_example_and_brute_decode():
    # codes [1, 0, 0, -1] -> c = w+1 = [2, 1, 1, 0] -> 2 | 1<<2 | 1<<4 | 0<<6 = 22
    assert O.pack_ternary(np.array([[1, 0, 0, -1]])).tolist() == [[22]]
    # padding: a row of 5 codes fills the 2nd byte with c=1 (w=0) in slots 1..3
    p = O.pack_ternary(np.array([[-1, -1, -1, -1, 1]]))
    assert p.tolist() == [[0, 2 | (1 << 2) | (1 << 4) | (1 << 6)]]
    rng = np.random.default_rng(5)
    Wq = rng.integers(-1, 2, size=(19, 45))
    P = O.pack_ternary(Wq)
    assert P.shape == (19, 12) and P.dtype == np.uint8
    for i in range(19):
        for k in range(45):
            c = (int(P[i, k // 4]) >> (2 * (k % 4))) & 3
            assert c - 1 == Wq[i, k]
        for k in range(45, 48):
            assert (int(P[i, k // 4]) >> (2 * (k % 4))) & 3 == 1


# --- absmax int8 activations -----------------------------------------------

def test_absmax_hand_example_with_tie():
    # m = 4, sigma = 127/4 = 31.75, v*sigma = [31.75, -63.5, 15.875, 127]:
    # rint gives 32, -64 (tie -> even), 16, 127
    q, m = O.absmax_codes(np.array([[1.0, -2.0, 0.5, 4.0]], dtype=np.float32))
    assert q.tolist() == [[32, -64, 16, 127]]
    assert float(m[0]) == 4.0


def test_absmax_range_argmax_and_zero_rows():
    v = S.random_rows(6, 50, 333, zero_rows=(3, 17))
    q, m = O.absmax_codes(v)
    assert q.min() >= -128 and q.max() <= 127
    for i in range(50):
        if i in (3, 17):
            assert not q[i].any() and m[i] == 0
            continue
        k = int(np.argmax(np.abs(v[i])))
        assert abs(int(q[i, k])) == 127 and np.sign(q[i, k]) == np.sign(v[i, k])
        assert (np.abs(q[i]) <= 127).all()


def test_absmax_scale_invariance():
    v = S.random_rows(7, 40, 256)
    q, _ = O.absmax_codes(v)
    for c in (0.25, 2.0, 1024.0):   # powers of two: every float32 step is exact
        q2, _ = O.absmax_codes(v * np.float32(c))
        assert np.array_equal(q, q2)
    # an RMSNorm-like positive scale changes at most rare near-tie codes by 1
    r = (1.0 / np.sqrt((v.astype(np.float64) ** 2).mean(-1) + 1e-5)).astype(np.float32)
    q3, _ = O.absmax_codes(v * r[:, None])
    d = np.abs(q3 - q)
    assert d.max() <= 1 and (d > 0).mean() < 1e-3


def test_int_gemm_brute_force_and_library():
    rng = np.random.default_rng(8)
    q = rng.integers(-128, 128, size=(5, 7))
    W = rng.integers(-1, 2, size=(3, 7))
    acc = O.int_gemm(q, W)
    for i in range(5):
        for j in range(3):
            assert acc[i, j] == sum(int(q[i, k]) * int(W[j, k]) for k in range(7))
    q = rng.integers(-128, 128, size=(64, 512))
    W = rng.integers(-1, 2, size=(96, 512))
    assert np.array_equal(O.int_gemm(q, W), q.astype(np.int64) @ W.astype(np.int64).T)
    # extreme: all -128 against all -1 over K=4096 -> 128*4096
    assert O.int_gemm(np.full((1, 4096), -128), np.full((1, 4096), -1))[0, 0] == 524288


# --- BitLinear ---------------------------------------------------------------

def test_bitlinear_a8_hand_example():
    # v = [1, -2, 0.5, 4]: codes [32, -64, 16, 127], m = 4,
    # r = 1/sqrt((1 + 4 + 0.25 + 16)/4 + 1e-5) = 1/sqrt(5.31251)
    # W_q rows [1, 0, 0, -1] and [0, 1, 1, 1], s = 0.5:
    # acc = [32 - 127, -64 + 16 + 127] = [-95, 79]; out = acc * 0.5 * 4 r / 127
    v = np.array([[1.0, -2.0, 0.5, 4.0]], dtype=np.float32)
    Wq = np.array([[1, 0, 0, -1], [0, 1, 1, 1]], dtype=np.int8)
    out, st = O.bitlinear_a8(v, Wq, np.float32(0.5))
    r = 1.0 / math.sqrt(5.3125 + 1e-5)
    assert st["acc"].tolist() == [[-95, 79]]
    assert np.allclose(out, [[-95 * 0.5 * 4 * r / 127, 79 * 0.5 * 4 * r / 127]], rtol=1e-14)


def test_bitlinear_a8_equals_unfolded_rmsnorm_then_quant():
    # the oracle folds RMSNorm into the quantiser; compose it the long way
    rng = np.random.default_rng(9)
    v = S.random_rows(10, 64, 256, scale=3.0)
    Wf = rng.normal(0, 0.02, size=(96, 256)).astype(np.float32)
    Wq, s = O.absmean_ternary(Wf)
    out, _ = O.bitlinear_a8(v, Wq, s)
    v64 = v.astype(np.float64)
    n = v64 / np.sqrt((v64 ** 2).mean(-1, keepdims=True) + 1e-5)
    gamma = np.abs(n).max(-1, keepdims=True)
    qn = np.clip(np.rint(n * 127 / gamma), -128, 127)
    ref = (qn @ Wq.astype(np.float64).T) * float(s) * gamma / 127
    err = np.abs(out - ref).max() / np.abs(ref).max()
    assert err < 2e-3   # equal up to rare near-tie code flips


def test_bitlinear_int_input_matches_real_row():
    rng = np.random.default_rng(11)
    acc_in = rng.integers(-3000, 3000, size=(32, 512))
    c = rng.uniform(1e-4, 1e-3, size=32)
    Wq = rng.integers(-1, 2, size=(48, 512))
    out, st = O.bitlinear_a8_int_input(acc_in, c, Wq, 0.7)
    ref, st_ref = O.bitlinear_a8(c[:, None] * acc_in, Wq, 0.7)
    assert (st["q"] != st_ref["q"]).mean() < 1e-2
    assert np.abs(out - ref).max() / np.abs(ref).max() < 1e-2
    assert np.allclose(st["deq"], st_ref["deq"], rtol=1e-12)


def test_bitlinear_a16_brute_force():
    rng = np.random.default_rng(12)
    v = rng.normal(size=(3, 300))
    Wf = rng.normal(0, 0.02, size=(4, 300)).astype(np.float32)
    Wq, s = O.absmean_ternary(Wf, group=128)
    out = O.bitlinear_a16(v, Wq, s, 128)
    for i in range(3):
        r = 1.0 / math.sqrt(math.fsum(x * x for x in v[i]) / 300 + 1e-5)
        for n in range(4):
            tot = 0.0
            for k in range(300):
                tot += float(s[n, k // 128]) * int(Wq[n, k]) * v[i, k]
            assert abs(out[i, n] - r * tot) < 1e-12 * (1 + abs(r * tot))


def test_bf16_rounding_matches_torch():
    torch = pytest.importorskip("torch")
    rng = np.random.default_rng(13)
    a = (rng.normal(size=10000) * 10.0 ** rng.integers(-8, 8, size=10000)).astype(np.float32)
    ref = torch.from_numpy(a).to(torch.bfloat16).float().numpy()
    assert np.array_equal(S.round_to_bf16(a), ref)
    assert np.array_equal(O.round_bf16(a).astype(np.float32), ref)
