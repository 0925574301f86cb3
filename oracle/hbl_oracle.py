"""Plain CPU oracle of the H-BitLinear forward pass (BitNet v2).

TEST INFRASTRUCTURE ONLY. Only the tests, the smoke check and the benchmark's
CPU-baseline leg may import this module. The product path (the CUDA library
and its Python binding) never calls it and shares no code with it.

It is written to be checked by eye against the sources, not to be fast:
floating point in float64, integer matmul in int64, numpy library calls as
single steps, no blocking or fusion beyond what the method states.

Sources (the pages on the method; every formula on them was lost when the
pages were extracted, the surrounding words survive):
  [ABS]  "BitNet v2: Native 4-bit Activations with Hadamard Transformation
         for 1-bit LLMs" (arXiv 2504.18415), abstract as shown on the
         fugumt.com summary page.
  [ART]  Chinese walkthrough of the BitNet v2 paper (m.jxzklqfsx.com,
         article 817179), sections "BitNet v2：原生4位激活" and
         "H-BitLinear模塊".
  [B158] bitnet.cpp / BitNet b1.58 news article (gubiw.cn, 336601), section
         "6 页论文，引入 1 bit LLM".

Readings taken where the pages are silent or the formulas were dropped
(each is a reading of a passage whose formula was lost):
  R1 weights: per-tensor absmean alpha = mean|W|; t = RoundClip(W/(alpha+eps_w), -1, 1).
  R2 norm: RMSNorm over the K features of a token, x / sqrt(mean(x^2) + eps_n),
     optional per-feature gain; eps_n defaults to 1e-6.
  R3 transform: Sylvester-ordered Walsh-Hadamard matrix scaled by 1/sqrt(n)
     (orthonormal); when K is not a power of two, the same transform is applied
     to each consecutive block of n features (block-diagonal).
  R4 activation quantisers, per token row:
       a8 absmax : gamma = max|x|, q = RoundClip(127 x/(gamma+eps), -128, 127), s = gamma/127
       a4 absmean: beta = mean|x|, q = RoundClip(sqrt7 x/(beta+eps), -8, 7), s = beta/sqrt7
       a4 absmax : gamma = max|x|, q = RoundClip(7 x/(gamma+eps), -8, 7),    s = gamma/7
     A row whose statistic is zero (and eps = 0) gives q = 0 and s = 0.
  R5 RoundClip rounds to nearest, ties to even, and clips to the code range.
     The pages fix no precision for any step, so every step here, the rounding
     decision included, is taken in float64 on the float64 values of the steps
     before it: q = clip(rint(Q * x / (stat + eps)), lo, hi).
  R6 output: y[m, n] = s[m] * alpha * sum_k q[m, k] t[k, n], evaluated in float64.
  R7 rotated weights (optional): W' = H W along K with the activations' transform,
     then R1 on W'.
  R8 RoPE on the Q and K states (LLaMA-like parts): the rotate-half form, frequency f of
     a head of D features pairing features f and f + D/2 with the angle
     pos * theta^(-2f/D); theta is a parameter (10000 by default).
  R9 QKV quantisation after RoPE to unsigned b-bit integers with an absmax scale, per
     token and head: gamma = max|x| over the head's D values, the interval
     [-gamma, gamma] mapped linearly onto [0, L], L = 2^b - 1:
       u = RoundClip(L (x + gamma) / (2 gamma), 0, L),   x~ = (2u - L) gamma / L;
     a head whose gamma is 0 takes u = RoundClip(L / 2).

Parity status: every function below names the tests that pin it against
something other than itself (closed forms, a dense Sylvester matrix from
SciPy, torch's bf16 widening, brute force on small inputs, a hand-derived
worked example). The choice of readings R1-R7 themselves is not pinned by any
number on the pages, which print none: against the published method the
oracle is "parity unpinned" in that sense only.
"""
from __future__ import annotations

import math

import numpy as np

SQRT7 = math.sqrt(7.0)

__all__ = [
    "bf16_to_f64",
    "absmean_ternarize",
    "rmsnorm",
    "fwht",
    "hadamard_transform",
    "quantize",
    "rotate_weights",
    "norm_fht_quant",
    "ternary_matmul",
    "dequant",
    "h_bitlinear_forward",
    "rope",
    "quantize_unsigned_absmax",
    "dequantize_unsigned",
    "qkv_quant",
]


def bf16_to_f64(bits: np.ndarray) -> np.ndarray:
    """bf16 bit patterns (uint16) -> float64, exactly (bf16 is the top half of a float32).

    Pinned by test_bf16_to_f64_known_patterns (1.0, -2.0, the smallest subnormal, the largest
    finite value, signed zero) and test_bf16_to_f64_matches_torch (all 65536 patterns against
    torch's own bf16 -> float conversion).
    """
    b = np.asarray(bits, dtype=np.uint16)
    with np.errstate(invalid="ignore"):  # NaN patterns stay NaN
        return (b.astype(np.uint32) << 16).view(np.float32).astype(np.float64)


def absmean_ternarize(W: np.ndarray, eps_w: float = 0.0) -> tuple[np.ndarray, float]:
    """Per-tensor absmean ternarisation of the weights (reading R1).

    [ART] "H-BitLinear模塊": the weights are ternarised to {-1, 0, 1} with a
    per-tensor absmean scale. [B158] "6 页论文，引入 1 bit LLM": the weight
    matrix is scaled by its mean absolute value and each entry is rounded to the
    nearest of -1, 0, 1.

    Returns (t int8 with the shape of W, alpha); alpha does not include eps_w.
    Pinned by test_ternarize_constant_and_brute_force (constant matrices, brute-force
    nearest of {-1, 0, 1}, all-zero W) and test_ternarize_eps_w_closed_form.
    """
    W = np.asarray(W, dtype=np.float64)
    alpha = float(np.sum(np.abs(W)) / W.size)
    denom = alpha + eps_w
    if denom == 0.0:
        return np.zeros(W.shape, dtype=np.int8), alpha
    t = np.clip(np.rint(W / denom), -1, 1).astype(np.int8)
    return t, alpha


def rmsnorm(x: np.ndarray, gain: np.ndarray | None = None, eps: float = 1e-6) -> np.ndarray:
    """RMSNorm of each row over its K features (reading R2).

    [ART] "BitNet v2：原生4位激活": the model is built from LLaMA-like parts
    including RMS normalisation; "H-BitLinear模塊" names the normalisation
    applied inside the layer before the Hadamard transform.

    Pinned by test_rmsnorm_unit_rms_and_gain (unit RMS, per-row factor, gain) and
    test_rmsnorm_eps_under_the_square_root (a closed form that separates eps inside the
    square root from eps added outside it or to the mean before squaring).
    """
    x = np.asarray(x, dtype=np.float64)
    r = np.sqrt(np.mean(x * x, axis=-1, keepdims=True) + eps)
    y = x / r
    if gain is not None:
        y = y * np.asarray(gain, dtype=np.float64)
    return y


def fwht(x: np.ndarray) -> np.ndarray:
    """Orthonormal fast Walsh-Hadamard transform along the last axis (reading R3).

    [ART] "H-BitLinear模塊": the product with the Hadamard matrix is computed by
    the fast Hadamard transform in O(n log n); the matrix has entries +-1 and
    mutually orthogonal rows. This is the Sylvester construction
    H_2n = [[H_n, H_n], [H_n, -H_n]], realised as log2(n) butterfly stages: at
    stage h the pair (x[j], x[j+h]) inside each block of 2h becomes
    (x[j] + x[j+h], x[j] - x[j+h]). The result is scaled by 1/sqrt(n).

    Pinned by test_fwht_equals_scipy_sylvester_matrix, test_fwht_walsh_closed_form,
    test_fwht_orthogonal_involution_parseval and test_fwht_delta_and_constant.
    """
    y = np.array(x, dtype=np.float64, copy=True)
    n = y.shape[-1]
    if n < 1 or n & (n - 1):
        raise ValueError(f"transform length {n} is not a power of two")
    lead = y.shape[:-1]
    h = 1
    while h < n:
        v = y.reshape(*lead, n // (2 * h), 2, h)
        a = v[..., 0, :].copy()
        b = v[..., 1, :].copy()
        v[..., 0, :] = a + b
        v[..., 1, :] = a - b
        h *= 2
    return y / math.sqrt(n)


def hadamard_transform(x: np.ndarray, block: int = 0) -> np.ndarray:
    """Hadamard transform of each row: over all of K (block = 0) or block-diagonal.

    Block-diagonal (reading R3): K = nb * block, and each consecutive slice of
    `block` features is transformed on its own, i.e. the matrix is
    kron(I_nb, H_block / sqrt(block)). A block of 1 is the identity (H_1 = [1]).

    Pinned by test_block_diagonal_transform_matches_kron and test_block_of_one_is_identity.
    """
    x = np.asarray(x, dtype=np.float64)
    K = x.shape[-1]
    if block == 0 or block == K:
        return fwht(x)
    if K % block:
        raise ValueError(f"K={K} is not a multiple of block={block}")
    lead = x.shape[:-1]
    return fwht(x.reshape(*lead, K // block, block)).reshape(*lead, K)


def _round_clip(v: np.ndarray, lo: int, hi: int) -> np.ndarray:
    """RoundClip (reading R5): nearest integer, ties to even, clipped to [lo, hi]."""
    return np.clip(np.rint(v), lo, hi).astype(np.int8)


def quantize(xr: np.ndarray, abits: int, scale_mode: str, eps_q: float = 0.0
             ) -> tuple[np.ndarray, np.ndarray]:
    """Per-token activation quantisation without zero point (reading R4).

    [ART] "H-BitLinear模塊": separate strategies for INT8 and INT4 activations
    (formulas dropped in extraction). [B158] "6 页论文，引入 1 bit LLM":
    activations are scaled into [-Q_b, Q_b], which removes the zero point.

    Returns (q int8 [M, K], s float64 [M]); s does not include eps_q.
    Pinned by test_quantiser_defining_properties, test_quantiser_brute_force_nearest_code,
    test_quantiser_ties_go_to_even, test_quantiser_eps_q_closed_form and
    test_quantiser_zero_row_and_scale_invariance.
    """
    xr = np.asarray(xr, dtype=np.float64)
    a = np.abs(xr)
    if abits == 8 and scale_mode == "absmax":
        stat, qmul, lo, hi = a.max(axis=-1), 127.0, -128, 127
    elif abits == 4 and scale_mode == "absmean":
        stat, qmul, lo, hi = a.mean(axis=-1), SQRT7, -8, 7
    elif abits == 4 and scale_mode == "absmax":
        stat, qmul, lo, hi = a.max(axis=-1), 7.0, -8, 7
    else:
        raise ValueError(f"unsupported quantiser abits={abits} scale_mode={scale_mode!r}")
    denom = stat + eps_q
    live = denom > 0.0
    v = np.where(live[..., None], qmul * xr / np.where(live, denom, 1.0)[..., None], 0.0)
    q = _round_clip(v, lo, hi)
    s = np.where(live, stat / qmul, 0.0)
    return q, s


def norm_fht_quant(x: np.ndarray, gain: np.ndarray | None, had_block: int, abits: int,
                   scale_mode: str, eps_norm: float = 1e-6, eps_q: float = 0.0
                   ) -> tuple[np.ndarray, np.ndarray]:
    """Activation side of H-BitLinear: Q(Hadamard(RMSNorm(x))) per token row.

    [ABS]: an online Hadamard transformation is applied before activation
    quantisation. [ART] "H-BitLinear模塊": the layer computes
    Q_w(W) . Q_INT8/INT4(Hadamard(LN(X))).

    x: float64 values (or bf16 bit patterns as uint16) [M, K].
    Pinned through its parts and by test_worked_example (hand-derived K = 4 example).
    """
    if x.dtype == np.uint16:
        x = bf16_to_f64(x)
    xr = hadamard_transform(rmsnorm(x, gain, eps_norm), had_block)
    return quantize(xr, abits, scale_mode, eps_q)


def rotate_weights(W: np.ndarray, block: int = 0) -> np.ndarray:
    """Weight-side Hadamard rotation, W' = H W along K (reading R7).

    [ART] section "與其他後訓練量化方法的對比", Table 5: the Hadamard rotation applied to the
    weights and the activations, or to the activations only, both stabilise low-bit training.
    With rotated weights each column of W (the K weights of one output feature) goes through the
    same transform as the activations, so that (H x)^T (H W) = x^T W in exact arithmetic.

    Pinned by test_rotate_weights_undoes_a_rotation (W = H T c ternarises back to T with
    alpha = c * mean|T|), test_rotate_weights_columns_closed_form (a unit column gives the Walsh
    column) and test_rotated_layer_keeps_the_full_precision_product.
    """
    W = np.asarray(W, dtype=np.float64)
    return hadamard_transform(W.T, block).T


def ternary_matmul(q: np.ndarray, t: np.ndarray) -> np.ndarray:
    """acc[m, n] = sum_k q[m, k] * t[k, n] in exact int64 arithmetic (the sum written as an einsum).

    Pinned by test_ternary_matmul_brute_force_and_blas (a triple loop, float64 BLAS, np.matmul).
    """
    return np.einsum("mk,kn->mn", np.asarray(q, dtype=np.int64), np.asarray(t, dtype=np.int64))


def dequant(acc: np.ndarray, s: np.ndarray, alpha: float) -> np.ndarray:
    """y[m, n] = acc[m, n] * s[m] * alpha in float64 (reading R6).

    Pinned by test_worked_example and test_forward_equals_dense_dequantised_product.
    """
    return np.asarray(acc, dtype=np.float64) * np.asarray(s, dtype=np.float64)[:, None] * float(alpha)


def h_bitlinear_forward(x: np.ndarray, W: np.ndarray, gain: np.ndarray | None = None,
                        had_block: int = 0, abits: int = 4, scale_mode: str | None = None,
                        eps_norm: float = 1e-6, eps_q: float = 0.0, eps_w: float = 0.0,
                        rotate_w: bool = False) -> dict:
    """The whole layer: weights ternarised, activations normed/rotated/quantised, product, dequant.

    had_block = 1 is the plain BitLinear (no rotation). rotate_w rotates the latent weights with
    the same transform before ternarising them (reading R7).
    Returns a dict with every intermediate (t, alpha, q, s, acc, y) for parity checks.
    """
    if scale_mode is None:
        scale_mode = "absmax" if abits == 8 else "absmean"
    t, alpha = absmean_ternarize(rotate_weights(W, had_block) if rotate_w else W, eps_w)
    q, s = norm_fht_quant(x, gain, had_block, abits, scale_mode, eps_norm, eps_q)
    acc = ternary_matmul(q, t)
    return {"t": t, "alpha": alpha, "q": q, "s": s, "acc": acc, "y": dequant(acc, s, alpha)}


def rope(x: np.ndarray, pos: np.ndarray, theta: float = 10000.0) -> np.ndarray:
    """Rotary position embedding of x [M, H, D] at token positions pos [M] (reading R8).

    [ART] section "實驗結果": the QKV states are quantised after RoPE (rotary position
    embedding); the model is LLaMA-like ("BitNet v2：原生4位激活"), whose RoPE rotates the pair
    of features (f, f + D/2) of every head by the angle pos * theta^(-2f/D).

    Pinned by test_rope_identity_norm_and_inverse (position 0, pair norms, rotating back),
    test_rope_one_hot_closed_form and test_rope_depends_on_relative_position.
    """
    x = np.asarray(x, dtype=np.float64)
    D = x.shape[-1]
    half = D // 2
    inv = np.float64(theta) ** (-2.0 * np.arange(half) / D)
    ang = np.asarray(pos, dtype=np.float64)[:, None] * inv[None, :]
    c = np.cos(ang)[:, None, :]
    s = np.sin(ang)[:, None, :]
    x1, x2 = x[..., :half], x[..., half:]
    return np.concatenate([x1 * c - x2 * s, x1 * s + x2 * c], axis=-1)


def quantize_unsigned_absmax(x: np.ndarray, bits: int) -> tuple[np.ndarray, np.ndarray]:
    """Per-head absmax quantisation to unsigned b-bit integers (reading R9).

    [ART] section "實驗結果": the QKV heads are quantised directly to unsigned integers with
    the absmax function, with no calibration set; a 3-bit KV cache matches full precision.
    x: [..., D]. Returns (u uint8 [..., D], gamma float64 [...]).

    Pinned by test_unsigned_quantiser_properties (range, extremes, half-step error bound,
    brute-force nearest level) and test_unsigned_quantiser_closed_form.
    """
    x = np.asarray(x, dtype=np.float64)
    L = (1 << bits) - 1
    g = np.abs(x).max(axis=-1)[..., None]
    live = g > 0
    gs = np.where(live, g, 1.0)
    # L (x + gamma) / (2 gamma) in one division: for bf16 inputs the numerator is exact in float64,
    # so a value exactly on a .5 boundary is represented exactly and goes to the even code
    v = np.where(live, (L * x + L * gs) / (2.0 * gs), L / 2.0)
    u = np.clip(np.rint(v), 0, L).astype(np.uint8)
    return u, g[..., 0]


def dequantize_unsigned(u: np.ndarray, gamma: np.ndarray, bits: int) -> np.ndarray:
    """x~ = (2u - (2^b - 1)) * gamma / (2^b - 1) (reading R9).

    Pinned by test_unsigned_quantiser_properties (dequantised values within half a step of x) and
    test_unsigned_quantiser_closed_form (the b = 3 levels, a zero head dequantising to 0).
    """
    L = (1 << bits) - 1
    return (2.0 * np.asarray(u, dtype=np.float64) - L) * np.asarray(gamma, dtype=np.float64)[..., None] / L


def qkv_quant(x: np.ndarray, pos: np.ndarray | None, bits: int, theta: float = 10000.0
              ) -> tuple[np.ndarray, np.ndarray]:
    """RoPE (when pos is given: the Q and K states; V takes none) then per-head unsigned absmax
    quantisation of x [M, H, D] (float64 values or bf16 bit patterns). Returns (u, gamma).

    Pinned through its parts (the rope and quantiser pins above) and bf16_to_f64's pins.
    """
    if x.dtype == np.uint16:
        x = bf16_to_f64(x)
    if pos is not None:
        x = rope(x, pos, theta)
    return quantize_unsigned_absmax(x, bits)
