"""Pins of the CPU oracle against things other than itself.

Each test checks one part of the oracle against a closed form, a library
routine of different construction (SciPy's Sylvester Hadamard matrix, float64
BLAS), brute force, or the hand-derived worked example in tests/golden. The
mutation tests at the end plant plausible mistakes in the oracle and check
that at least one pin catches each.
"""
import math

import numpy as np
import pytest
import scipy.linalg

import conftest
import oracle
from hadamard_bit_quant_hbl_b200 import inputs

RNG = np.random.default_rng(12345)


# ---------------------------------------------------------------- transform

@pytest.mark.parametrize("n", [1, 2, 4, 8, 64, 256, 1024])
def test_fwht_equals_scipy_sylvester_matrix(n):
    # fwht of the identity rows gives the columns of H_n / sqrt(n); SciPy builds H_n by the
    # Sylvester recursion directly (no butterflies).
    got = oracle.fwht(np.eye(n))
    want = scipy.linalg.hadamard(n).astype(np.float64) / math.sqrt(n)
    np.testing.assert_allclose(got, want.T, rtol=0, atol=1e-12)


def test_fwht_walsh_closed_form():
    # Sylvester-ordered Hadamard entry: H[i, j] = (-1)^popcount(i & j).
    n = 4096
    for j in RNG.integers(0, n, size=6):
        e = np.zeros(n)
        e[j] = 1.0
        got = oracle.fwht(e) * math.sqrt(n)
        i = np.arange(n)
        want = np.array([(-1.0) ** bin(int(ii) & int(j)).count("1") for ii in i])
        np.testing.assert_array_equal(got, want)


def test_fwht_orthogonal_involution_parseval():
    n = 8192
    x = RNG.standard_normal((3, n))
    y = oracle.fwht(x)
    np.testing.assert_allclose(np.linalg.norm(y, axis=1), np.linalg.norm(x, axis=1), rtol=1e-12)
    np.testing.assert_allclose(oracle.fwht(y), x, rtol=0, atol=1e-11)
    # H H^T = n I, exactly in integers, on a 256-point matrix built by the oracle
    H = np.rint(oracle.fwht(np.eye(256)) * 16).astype(np.int64)
    np.testing.assert_array_equal(H @ H.T, 256 * np.eye(256, dtype=np.int64))


def test_fwht_delta_and_constant():
    n = 2048
    e0 = np.zeros(n)
    e0[0] = 1
    np.testing.assert_allclose(oracle.fwht(e0), np.full(n, 1 / math.sqrt(n)), rtol=1e-13)
    np.testing.assert_allclose(oracle.fwht(np.ones(n)), math.sqrt(n) * e0, atol=1e-11)


def test_fwht_rejects_non_power_of_two():
    with pytest.raises(ValueError):
        oracle.fwht(np.ones(12))


def test_block_diagonal_transform_matches_kron():
    blk = 256
    nb = 6
    x = RNG.standard_normal((4, nb * blk))
    dense = np.kron(np.eye(nb), scipy.linalg.hadamard(blk) / 16.0)
    np.testing.assert_allclose(oracle.hadamard_transform(x, blk), x @ dense.T, atol=1e-12)
    # 43 blocks (K = 11008), checked block by block against the dense 256-point matrix
    x = RNG.standard_normal((2, 43 * blk))
    got = oracle.hadamard_transform(x, blk)
    H = scipy.linalg.hadamard(blk) / 16.0
    for b in range(43):
        sl = slice(b * blk, (b + 1) * blk)
        np.testing.assert_allclose(got[:, sl], x[:, sl] @ H.T, atol=1e-12)


def test_block_of_one_is_identity():
    # kron(I_K, H_1) with H_1 = [1]: the block-diagonal transform with blocks of one feature
    # leaves every row unchanged (plain BitLinear, no rotation)
    x = RNG.standard_normal((3, 768))
    np.testing.assert_array_equal(oracle.hadamard_transform(x, 1), x)


# ---------------------------------------------------------------- bf16 input

def test_bf16_to_f64_known_patterns():
    bits = np.array([0x3F80, 0xC000, 0x0001, 0x8001, 0x7F7F, 0x0000, 0x8000, 0x4049, 0x0080], dtype=np.uint16)
    want = [1.0, -2.0, 2.0 ** -133, -(2.0 ** -133), (2.0 - 2.0 ** -7) * 2.0 ** 127, 0.0, -0.0,
            3.140625, 2.0 ** -126]
    got = oracle.bf16_to_f64(bits)
    assert got.dtype == np.float64
    np.testing.assert_array_equal(got, want)
    assert math.copysign(1.0, got[6]) == -1.0


def test_bf16_to_f64_matches_torch():
    torch = pytest.importorskip("torch")
    bits = np.arange(1 << 16, dtype=np.uint32).astype(np.uint16)
    ref = torch.from_numpy(bits.view(np.int16)).view(torch.bfloat16).to(torch.float64).numpy()
    got = oracle.bf16_to_f64(bits)
    nan = np.isnan(ref)
    np.testing.assert_array_equal(np.isnan(got), nan)
    np.testing.assert_array_equal(got[~nan], ref[~nan])


# ---------------------------------------------------------------- norm

def test_rmsnorm_unit_rms_and_gain():
    x = RNG.laplace(0, 0.1, size=(5, 512))
    y = oracle.rmsnorm(x, None, eps=0.0)
    np.testing.assert_allclose(np.sqrt(np.mean(y ** 2, axis=1)), 1.0, rtol=1e-13)
    # the output is x divided by a positive per-row factor
    ratio = y / x
    np.testing.assert_allclose(ratio, ratio[:, :1] * np.ones_like(ratio), rtol=1e-12)
    g = RNG.uniform(0.5, 2.0, size=512)
    np.testing.assert_allclose(oracle.rmsnorm(x, g, eps=0.0), y * g, rtol=1e-13)
    # eps enters under the square root: a zero row stays zero
    np.testing.assert_array_equal(oracle.rmsnorm(np.zeros((1, 8)), None, 1e-6), np.zeros((1, 8)))


def test_rmsnorm_eps_under_the_square_root():
    # x = [3, 4]: mean(x^2) = 12.5. With eps = 11.5 under the square root r = sqrt(24), so
    # y = [3, 4] / sqrt(24). Eps added outside the root would give r = sqrt(12.5) + 11.5, eps on
    # the mean before squaring something else again; both differ here by far more than rounding.
    y = oracle.rmsnorm(np.array([[3.0, 4.0]]), None, eps=11.5)
    np.testing.assert_allclose(y[0], np.array([3.0, 4.0]) / math.sqrt(24.0), rtol=1e-15)
    assert abs(y[0, 0] - 3.0 / (math.sqrt(12.5) + 11.5)) > 0.1
    # the gain multiplies after the division
    y = oracle.rmsnorm(np.array([[3.0, 4.0]]), np.array([2.0, -1.0]), eps=11.5)
    np.testing.assert_allclose(y[0], np.array([6.0, -4.0]) / math.sqrt(24.0), rtol=1e-15)


def test_rms_is_preserved_by_the_orthonormal_transform():
    x = RNG.standard_normal((3, 1024))
    np.testing.assert_allclose(np.mean(oracle.fwht(x) ** 2, axis=1), np.mean(x ** 2, axis=1), rtol=1e-12)


# ---------------------------------------------------------------- quantisers

QUANTS = [(8, "absmax", 127, -128, 127), (4, "absmean", math.sqrt(7), -8, 7), (4, "absmax", 7, -8, 7)]


@pytest.mark.parametrize("abits,mode,Q,lo,hi", QUANTS)
def test_quantiser_defining_properties(abits, mode, Q, lo, hi):
    x = RNG.laplace(0, 1.0, size=(64, 256))
    x[:, 7] *= 30  # an outlier channel
    q, s = oracle.quantize(x, abits, mode)
    assert q.dtype == np.int8 and q.min() >= lo and q.max() <= hi
    a = np.abs(x)
    # the scale is the row statistic divided by the code range, computed independently here
    stat = a.max(axis=1) if mode == "absmax" else a.sum(axis=1) / a.shape[1]
    np.testing.assert_allclose(s * Q, stat, rtol=1e-13)
    # rounding to nearest: every unclipped code is within half a step of x / s
    v = x / s[:, None]
    unclipped = (v > lo - 0.5) & (v < hi + 0.5)
    assert np.all(np.abs(v[unclipped] - q[unclipped]) <= 0.5 + 1e-5)
    # clipped codes sit at the bound on the correct side
    assert np.all(q[v >= hi + 0.5] == hi) and np.all(q[v <= lo - 0.5] == lo)
    if mode == "absmax":
        # the largest magnitude maps to +-Q exactly
        am = np.argmax(a, axis=1)
        np.testing.assert_array_equal(np.abs(q[np.arange(64), am]), int(Q))


def test_quantiser_ties_go_to_even():
    # exact ties in float64: a4 absmax with gamma = 7 maps x to x itself, so x = +-2.5, 3.5, 0.5
    # sit on .5 boundaries; nearest-even gives 2, 4, 0 (round-half-away would give 3, 4, 1,
    # floor 2, 3, 0, and a float32 detour cannot move them: every value here is exact)
    x = np.array([[2.5, -2.5, 3.5, 0.5, -0.5, 7.0]])
    q, s = oracle.quantize(x, 4, "absmax")
    np.testing.assert_array_equal(q[0], [2, -2, 4, 0, 0, 7])
    assert s[0] == 1.0
    # a8 absmax: gamma = 127 maps x to x; 126.5 -> 126, -127.5 cannot occur (|x| <= gamma)
    x = np.array([[126.5, -1.5, 127.0, 64.5]])
    q, _ = oracle.quantize(x, 8, "absmax")
    np.testing.assert_array_equal(q[0], [126, -2, 127, 64])


def test_quantiser_eps_q_closed_form():
    # reading R4 with eps: q = RoundClip(Q x / (stat + eps), lo, hi), s = stat / Q (no eps in s)
    x = np.array([[1.0, -2.0, 3.0, -4.0]])
    # a4 absmean: beta = 2.5; eps = 1.5 gives multiplier sqrt7 / 4 = 0.6614...:
    # [0.661, -1.323, 1.984, -2.646] -> [1, -1, 2, -3]; without eps sqrt7 / 2.5 gives [1, -2, 3, -4]
    q, s = oracle.quantize(x, 4, "absmean", eps_q=1.5)
    np.testing.assert_array_equal(q[0], [1, -1, 2, -3])
    assert s[0] == pytest.approx(2.5 / math.sqrt(7), rel=1e-15)
    q0, _ = oracle.quantize(x, 4, "absmean")
    np.testing.assert_array_equal(q0[0], [1, -2, 3, -4])
    # a8 absmax: gamma = 4, eps = 1: 127 x / 5 = [25.4, -50.8, 76.2, -101.6] -> [25, -51, 76, -102]
    q, s = oracle.quantize(x, 8, "absmax", eps_q=1.0)
    np.testing.assert_array_equal(q[0], [25, -51, 76, -102])
    assert s[0] == pytest.approx(4.0 / 127.0, rel=1e-15)
    # a4 absmax: gamma = 4, eps = 4: 7 x / 8 = [0.875, -1.75, 2.625, -3.5] -> [1, -2, 3, -4] (-3.5 is a tie: even)
    q, _ = oracle.quantize(x, 4, "absmax", eps_q=4.0)
    np.testing.assert_array_equal(q[0], [1, -2, 3, -4])
    # with eps > 0 a zero row is still all zeros, with s = 0
    q, s = oracle.quantize(np.zeros((1, 4)), 4, "absmean", eps_q=0.5)
    assert not q.any() and s[0] == 0.0


@pytest.mark.parametrize("abits,mode,Q,lo,hi", QUANTS)
def test_quantiser_brute_force_nearest_code(abits, mode, Q, lo, hi):
    # brute force: among all codes in [lo, hi] the oracle picks the one nearest to Q x / stat
    # (ties to the even code), found here by searching every code rather than rounding.
    x = RNG.standard_normal((8, 32))
    q, s = oracle.quantize(x, abits, mode)
    for m in range(8):
        row = [abs(float(v)) for v in x[m]]
        stat = max(row) if mode == "absmax" else sum(row) / len(row)
        for k in range(32):
            vv = Q * float(x[m, k]) / stat
            best = min(range(lo, hi + 1), key=lambda c: (abs(vv - c), c % 2))
            assert q[m, k] == best, (m, k, vv, q[m, k], best)


def test_quantiser_zero_row_and_scale_invariance():
    x = np.zeros((2, 64))
    x[1] = RNG.standard_normal(64)
    for abits, mode, *_ in QUANTS:
        q, s = oracle.quantize(x, abits, mode)
        assert np.all(q[0] == 0) and s[0] == 0.0
        q4, s4 = oracle.quantize(4.0 * x, abits, mode)  # power of two: exact scaling
        np.testing.assert_array_equal(q4, q)
        np.testing.assert_array_equal(s4, 4.0 * s)


def test_quantiser_rejects_unknown_modes():
    with pytest.raises(ValueError):
        oracle.quantize(np.ones((1, 4)), 8, "absmean")
    with pytest.raises(ValueError):
        oracle.quantize(np.ones((1, 4)), 2, "absmax")


# ---------------------------------------------------------------- weights

def test_ternarize_constant_and_brute_force():
    for c in (0.3, -0.07):
        t, alpha = oracle.absmean_ternarize(np.full((4, 6), c))
        assert alpha == pytest.approx(abs(c), rel=1e-15)
        np.testing.assert_array_equal(t, np.sign(c) * np.ones((4, 6)))
    W = RNG.standard_normal((16, 8)) * 0.02
    t, alpha = oracle.absmean_ternarize(W)
    assert set(np.unique(t)) <= {-1, 0, 1}
    assert alpha == pytest.approx(np.abs(W).sum() / W.size, rel=1e-14)
    for (k, n), w in np.ndenumerate(W):
        best = min((-1, 0, 1), key=lambda c: abs(w / alpha - c))
        assert t[k, n] == best
    t0, a0 = oracle.absmean_ternarize(np.zeros((3, 3)))
    assert a0 == 0.0 and not t0.any()


def test_ternarize_eps_w_closed_form():
    # alpha = mean|W| = 1.0 / 4 = 0.25. Without eps W / alpha = [0.8, -1.2, 2.0, 0] -> [1, -1, 1, 0];
    # with eps_w = 0.2 the divisor is 0.45: [0.444, -0.667, 1.11, 0] -> [0, -1, 1, 0]. alpha itself
    # does not include eps.
    W = np.array([[0.2, -0.3], [0.5, 0.0]])
    t, alpha = oracle.absmean_ternarize(W)
    np.testing.assert_array_equal(t, [[1, -1], [1, 0]])
    assert alpha == pytest.approx(0.25, rel=1e-15)
    t, alpha = oracle.absmean_ternarize(W, eps_w=0.2)
    np.testing.assert_array_equal(t, [[0, -1], [1, 0]])
    assert alpha == pytest.approx(0.25, rel=1e-15)
    # an all-zero W with eps > 0 gives t = 0 as well
    t, alpha = oracle.absmean_ternarize(np.zeros((2, 2)), eps_w=0.1)
    assert not t.any() and alpha == 0.0


def test_rotate_weights_undoes_a_rotation():
    # W = (H / sqrt n) T c along K: rotating it again gives T c (the orthonormal Sylvester matrix
    # is its own inverse), whose absmean ternarisation is T with alpha = c * mean|T|. A missing
    # rotation, a transform along N instead of K, or a missing 1/sqrt(n) breaks one of these.
    K, N, c = 256, 40, 0.013
    T = RNG.integers(-1, 2, size=(K, N)).astype(np.int8)
    H = scipy.linalg.hadamard(K) / math.sqrt(K)
    W = H @ (T.astype(np.float64) * c)
    Wr = oracle.rotate_weights(W)
    np.testing.assert_allclose(Wr, T * c, atol=1e-14)
    t, alpha = oracle.absmean_ternarize(Wr)
    np.testing.assert_array_equal(t, T)
    assert alpha == pytest.approx(c * np.abs(T).mean(), rel=1e-12)
    # block-diagonal: each 256-slice of the K column is rotated on its own
    W2 = np.kron(np.eye(3), H) @ (np.tile(T, (3, 1)).astype(np.float64) * c)
    np.testing.assert_allclose(oracle.rotate_weights(W2, 256), np.tile(T, (3, 1)) * c, atol=1e-14)


def test_rotate_weights_columns_closed_form():
    # a unit column e_j becomes column j of the orthonormal Walsh matrix: (-1)^popcount(i & j) / sqrt(n)
    n, j = 1024, 613
    W = np.zeros((n, 3))
    W[j, 1] = 1.0
    got = oracle.rotate_weights(W)
    i = np.arange(n)
    want = np.array([(-1.0) ** bin(int(ii) & j).count("1") for ii in i]) / math.sqrt(n)
    np.testing.assert_array_equal(got[:, 1], want)
    assert not got[:, 0].any() and not got[:, 2].any()


def test_rotated_layer_keeps_the_full_precision_product():
    # (H x)^T (H W) = x^T W: rotating both sides leaves the full-precision layer unchanged
    x = RNG.standard_normal((5, 512))
    W = RNG.standard_normal((512, 7))
    xr = oracle.hadamard_transform(x)
    np.testing.assert_allclose(xr @ oracle.rotate_weights(W), x @ W, rtol=1e-10, atol=1e-10)
    np.testing.assert_allclose(oracle.hadamard_transform(x, 256) @ oracle.rotate_weights(W, 256), x @ W,
                               rtol=1e-10, atol=1e-10)


# ---------------------------------------------------------------- product

def test_ternary_matmul_brute_force_and_blas():
    q = RNG.integers(-8, 8, size=(5, 37)).astype(np.int8)
    t = RNG.integers(-1, 2, size=(37, 6)).astype(np.int8)
    acc = oracle.ternary_matmul(q, t)
    for m in range(5):
        for n in range(6):
            assert acc[m, n] == sum(int(q[m, k]) * int(t[k, n]) for k in range(37))
    # float64 BLAS is exact here (integers far below 2^53), and computes in another order
    q = RNG.integers(-128, 128, size=(64, 4096)).astype(np.int8)
    t = RNG.integers(-1, 2, size=(4096, 48)).astype(np.int8)
    np.testing.assert_array_equal(oracle.ternary_matmul(q, t),
                                  (q.astype(np.float64) @ t.astype(np.float64)).astype(np.int64))
    # and numpy's integer matmul (a third routine)
    np.testing.assert_array_equal(oracle.ternary_matmul(q, t), q.astype(np.int64) @ t.astype(np.int64))


# ---------------------------------------------------------------- worked example

@pytest.mark.parametrize("abits,mode,key", [(8, "absmax", "a8"), (4, "absmean", "a4_absmean"),
                                            (4, "absmax", "a4_absmax")])
def test_worked_example(golden, abits, mode, key):
    g = golden("worked_example_k4.txt")
    x = np.array([g["x"]])
    W = np.array(g["W"]).reshape(4, 2)
    out = oracle.h_bitlinear_forward(x, W, None, 0, abits, mode, eps_norm=0.0)
    xr = oracle.hadamard_transform(oracle.rmsnorm(x, None, 0.0))
    np.testing.assert_allclose(xr[0], g["xr"], rtol=1e-14, atol=1e-15)
    np.testing.assert_array_equal(out["t"].ravel(), np.array(g["t"]))
    assert out["alpha"] == pytest.approx(g["alpha"][0], rel=1e-14)
    np.testing.assert_array_equal(out["q"][0], np.array(g[f"{key}_q"]))
    assert out["s"][0] == pytest.approx(g[f"{key}_s"][0], rel=1e-13)
    np.testing.assert_array_equal(out["acc"][0], np.array(g[f"{key}_acc"]))
    np.testing.assert_allclose(out["y"][0], g[f"{key}_y"], rtol=1e-13)


# ---------------------------------------------------------------- whole layer

def test_forward_equals_dense_dequantised_product():
    # The layer's output written the way the method states it, Q_w(W) . Q(Hadamard(LN(X))),
    # with dense matrices: dequantised activations times dequantised weights.
    K, N, M = 512, 24, 9
    x = RNG.laplace(0, 0.05, size=(M, K))
    x[:, 3] *= 50
    W = RNG.standard_normal((K, N)) * 0.02
    out = oracle.h_bitlinear_forward(x, W, None, 0, 4, "absmean")
    xn = x / np.sqrt((x ** 2).mean(axis=1, keepdims=True) + 1e-6)
    xr = xn @ (scipy.linalg.hadamard(K) / math.sqrt(K)).T
    np.testing.assert_allclose(xr, oracle.hadamard_transform(oracle.rmsnorm(x)), atol=1e-12)
    Xq = out["q"].astype(np.float64) * out["s"][:, None]
    Wq = out["t"].astype(np.float64) * out["alpha"]
    np.testing.assert_allclose(out["y"], Xq @ Wq, rtol=1e-12, atol=1e-14)


def test_transform_flattens_outliers_on_workload_inputs():
    # Property of the method (BitNet v2 abstract; walkthrough Figs. 2-3): after the transform
    # the outlier-heavy activations are far less heavy-tailed. Sanity only, not parity.
    spec = inputs.WORKLOADS["wo_1p3b_a4"].with_m(32)
    x = oracle.bf16_to_f64(inputs.activations(spec))

    def kurt(a):
        a = a - a.mean(axis=1, keepdims=True)
        return np.mean(a ** 4, axis=1) / np.mean(a ** 2, axis=1) ** 2

    xr = oracle.hadamard_transform(oracle.rmsnorm(x))
    assert np.median(kurt(x)) > 20 * np.median(kurt(xr))
    assert np.median(kurt(xr)) < 4.0


# ---------------------------------------------------------------- planted mistakes

_REAL_FWHT = oracle.fwht


def _fwht_no_scale(x):
    return _REAL_FWHT(x) * math.sqrt(np.asarray(x).shape[-1])


def _fwht_reversed_order(x):
    return _REAL_FWHT(x)[..., ::-1].copy()


@pytest.mark.parametrize("mutant", [_fwht_no_scale, _fwht_reversed_order])
def test_planted_transform_mistakes_are_caught(monkeypatch, mutant):
    monkeypatch.setattr(oracle.hbl_oracle, "fwht", mutant)
    monkeypatch.setattr(oracle, "fwht", mutant)
    caught = 0
    for check in (lambda: test_fwht_equals_scipy_sylvester_matrix(8),
                  lambda: test_worked_example(conftest.load_golden, 8, "absmax", "a8")):
        try:
            check()
        except AssertionError:
            caught += 1
    assert caught >= 1


def test_planted_quantiser_mistake_is_caught(monkeypatch):
    real = oracle.hbl_oracle.quantize

    def floor_instead_of_round(xr, abits, mode, eps_q=0.0):
        q, s = real(xr, abits, mode, eps_q)
        v = np.asarray(xr) / np.where(s > 0, s, 1)[:, None]
        return np.clip(np.floor(v), -8 if abits == 4 else -128, 7 if abits == 4 else 127).astype(np.int8), s

    monkeypatch.setattr(oracle, "quantize", floor_instead_of_round)
    with pytest.raises(AssertionError):
        test_quantiser_defining_properties(4, "absmean", math.sqrt(7), -8, 7)


def test_planted_norm_and_rounding_mistakes_are_caught(monkeypatch):
    real_rms = oracle.hbl_oracle.rmsnorm

    def eps_outside_root(x, gain=None, eps=1e-6):
        x = np.asarray(x, dtype=np.float64)
        y = x / (np.sqrt(np.mean(x * x, axis=-1, keepdims=True)) + eps)
        return y if gain is None else y * gain

    monkeypatch.setattr(oracle, "rmsnorm", eps_outside_root)
    with pytest.raises(AssertionError):
        test_rmsnorm_eps_under_the_square_root()
    monkeypatch.setattr(oracle, "rmsnorm", real_rms)

    def half_away(v, lo, hi):
        return np.clip(np.sign(v) * np.floor(np.abs(v) + 0.5), lo, hi).astype(np.int8)

    monkeypatch.setattr(oracle.hbl_oracle, "_round_clip", half_away)
    with pytest.raises(AssertionError):
        test_quantiser_ties_go_to_even()



# ---------------------------------------------------------------- QKV states after RoPE

def test_rope_identity_norm_and_inverse():
    x = RNG.standard_normal((6, 3, 128))
    pos = np.array([0, 1, 7, 100, 4095, 8191])
    y = oracle.rope(x, pos)
    np.testing.assert_array_equal(y[0], x[0])  # position 0: angle 0
    # every (f, f + D/2) pair keeps its length
    n_x = x[..., :64] ** 2 + x[..., 64:] ** 2
    n_y = y[..., :64] ** 2 + y[..., 64:] ** 2
    np.testing.assert_allclose(n_y, n_x, rtol=1e-12)
    # rotating by -pos undoes it
    np.testing.assert_allclose(oracle.rope(y, -pos), x, atol=1e-12)


def test_rope_one_hot_closed_form():
    D, f, p, theta = 64, 5, 37, 10000.0
    x = np.zeros((1, 1, D))
    x[0, 0, f] = 1.0
    y = oracle.rope(x, np.array([p]), theta)[0, 0]
    a = p * theta ** (-2.0 * f / D)
    want = np.zeros(D)
    want[f], want[f + D // 2] = math.cos(a), math.sin(a)
    np.testing.assert_allclose(y, want, atol=1e-15)
    x = np.zeros((1, 1, D))
    x[0, 0, f + D // 2] = 1.0  # the second feature of the pair turns the other way
    y = oracle.rope(x, np.array([p]), theta)[0, 0]
    want = np.zeros(D)
    want[f], want[f + D // 2] = -math.sin(a), math.cos(a)
    np.testing.assert_allclose(y, want, atol=1e-15)


def test_rope_depends_on_relative_position():
    # <rope(q, p), rope(k, p')> depends on p - p' only (brute force over position pairs)
    q = RNG.standard_normal((1, 1, 128))
    k = RNG.standard_normal((1, 1, 128))
    for p, pp in ((10, 3), (1000, 993), (5, -2)):
        a = np.sum(oracle.rope(q, np.array([p])) * oracle.rope(k, np.array([pp])))
        b = np.sum(oracle.rope(q, np.array([p - pp])) * k)
        assert a == pytest.approx(b, rel=1e-10)


@pytest.mark.parametrize("bits", [2, 3, 4, 8])
def test_unsigned_quantiser_properties(bits):
    L = (1 << bits) - 1
    x = RNG.standard_normal((40, 4, 128))
    u, g = oracle.quantize_unsigned_absmax(x, bits)
    assert u.dtype == np.uint8 and u.min() >= 0 and u.max() <= L
    np.testing.assert_array_equal(g, np.abs(x).max(axis=-1))
    # the element of largest magnitude maps to an end of the range
    am = np.abs(x).argmax(axis=-1)
    ext = np.take_along_axis(u, am[..., None], axis=-1)[..., 0]
    sgn = np.sign(np.take_along_axis(x, am[..., None], axis=-1)[..., 0])
    np.testing.assert_array_equal(ext, np.where(sgn > 0, L, 0))
    # dequantised values lie within half a step (gamma / L) of x, and the code is the nearest
    # level, found here by searching all 2^b levels
    xd = oracle.dequantize_unsigned(u, g, bits)
    assert np.all(np.abs(xd - x) <= g[..., None] / L * (1 + 1e-12))
    levels = (2.0 * np.arange(L + 1) - L) / L
    xs, gs, us = x[:2].reshape(-1, 128), g[:2].reshape(-1), u[:2].reshape(-1, 128)
    for h in range(xs.shape[0]):
        for d in range(128):
            best = int(np.argmin(np.abs(levels * gs[h] - xs[h, d])))
            assert us[h, d] == best


def test_unsigned_quantiser_closed_form():
    # b = 3: [-gamma, gamma] onto 0..7, step 2 gamma / 7. x = [-1, 1, 0, 0.5, -0.25] (gamma = 1):
    # 3.5 (x + 1) = [0, 7, 3.5, 5.25, 2.625] -> [0, 7, 4 (tie to even), 5, 3]
    u, g = oracle.quantize_unsigned_absmax(np.array([[-1.0, 1.0, 0.0, 0.5, -0.25]]), 3)
    np.testing.assert_array_equal(u[0], [0, 7, 4, 5, 3])
    assert g[0] == 1.0
    np.testing.assert_allclose(oracle.dequantize_unsigned(u, g, 3)[0], [-1, 1, 1 / 7, 3 / 7, -1 / 7], rtol=1e-15)
    # a zero head takes the middle code and dequantises to 0
    u, g = oracle.quantize_unsigned_absmax(np.zeros((1, 8)), 3)
    assert np.all(u == 4) and g[0] == 0.0
    assert not oracle.dequantize_unsigned(u, g, 3).any()
    # exact ties at b = 8 go to the even code: with gamma = 1.5625 (all values bf16), 255 (x + gamma)
    # / (2 gamma) is exactly 178.5, 76.5, 229.5 and 25.5 for x = 0.625, -0.625, 1.25, -1.25
    u, _ = oracle.quantize_unsigned_absmax(np.array([[1.5625, 0.625, -0.625, 1.25, -1.25, 0.0]]), 8)
    np.testing.assert_array_equal(u[0], [255, 178, 76, 230, 26, 128])
