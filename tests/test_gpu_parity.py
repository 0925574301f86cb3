"""Parity of the CUDA path (through the C ABI) with the CPU oracle, element by element.

Bars (fixed here, derived from the method's arithmetic):
  * weight codes and every integer accumulator: bit-exact;
  * activation codes: equal except for at most 1e-4 of them (at least one allowed), each off by
    one step: a code flips only where the fp32 value lies within rounding noise of a .5 boundary;
  * alpha and s_x: relative 1e-6 / 1e-5 (fp32 on the GPU, fp64 in the oracle);
  * outputs: per token row, ||y_gpu - y_oracle|| <= 1e-3 ||y_oracle|| plus the exact effect of the
    permitted code flips (sum over flipped k of |dq| * s * alpha * ||t[k, :]||); and, with the
    GPU's own codes fed to the oracle's product, per-row relative error <= 1e-5.
"""
import dataclasses

import numpy as np
import pytest
import torch

import oracle
import hadamard_bit_quant_hbl_b200 as hbl
from hadamard_bit_quant_hbl_b200 import inputs
from formats import code_flips, decode_blob, pack_int4, row_rel_err, unpack_int4

pytestmark = pytest.mark.gpu

QUANT_NAME = {hbl.HBL_Q_A8_ABSMAX: (8, "absmax"), hbl.HBL_Q_A4_ABSMEAN: (4, "absmean"),
              hbl.HBL_Q_A4_ABSMAX: (4, "absmax")}


@pytest.fixture(scope="module", autouse=True)
def _gpu():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    torch.cuda.set_device(0)
    hbl.lib()
    yield
    assert hbl.hbl_device_status() == hbl.HBL_OK


def spec_like(name, **kw):
    return dataclasses.replace(inputs.WORKLOADS[name], **kw)


def to_dev_bf16(bits):
    return torch.from_numpy(bits.view(np.int16)).cuda().view(torch.bfloat16)


def gpu_codes(x_bits, gain, had_block, quant, fmt, eps_norm=1e-6, eps_q=0.0):
    M, K = x_bits.shape
    X = to_dev_bf16(x_bits)
    g = None if gain is None else torch.from_numpy(gain.astype(np.float32)).cuda()
    codes, s = hbl.hbl_norm_fht_quant(X, g, had_block, quant, eps_norm, eps_q, fmt)
    torch.cuda.synchronize()
    c = codes.cpu().numpy()
    abits = QUANT_NAME[quant][0]
    q = unpack_int4(c, K) if (fmt == hbl.HBL_CODES_PACKED and abits == 4) else c.view(np.int8)
    return q, s.cpu().numpy().astype(np.float64)


def assert_codes_close(q_gpu, q_ora):
    flips, worst = code_flips(q_gpu, q_ora)
    allowed = max(1, int(1e-4 * q_ora.size))
    assert flips <= allowed and worst <= 1, f"{flips} flipped codes (allowed {allowed}), max step {worst}"


# ---------------------------------------------------------------- fused norm / transform / quant

NFQ_CASES = [
    # (K, had_block, M, quant, fmt, gain)
    (256, 0, 16, hbl.HBL_Q_A8_ABSMAX, hbl.HBL_CODES_PACKED, False),
    (256, 0, 37, hbl.HBL_Q_A4_ABSMEAN, hbl.HBL_CODES_PACKED, True),
    (512, 0, 21, hbl.HBL_Q_A4_ABSMAX, hbl.HBL_CODES_I8, False),
    (1024, 0, 37, hbl.HBL_Q_A4_ABSMEAN, hbl.HBL_CODES_PACKED, False),
    (2048, 0, 37, hbl.HBL_Q_A4_ABSMEAN, hbl.HBL_CODES_I8, True),
    (2048, 0, 9, hbl.HBL_Q_A8_ABSMAX, hbl.HBL_CODES_PACKED, False),
    (4096, 0, 37, hbl.HBL_Q_A4_ABSMEAN, hbl.HBL_CODES_PACKED, False),
    (4096, 0, 5, hbl.HBL_Q_A4_ABSMAX, hbl.HBL_CODES_PACKED, True),
    (8192, 0, 37, hbl.HBL_Q_A4_ABSMEAN, hbl.HBL_CODES_PACKED, False),
    (8192, 0, 7, hbl.HBL_Q_A8_ABSMAX, hbl.HBL_CODES_I8, False),
    (16384, 0, 19, hbl.HBL_Q_A4_ABSMEAN, hbl.HBL_CODES_PACKED, False),
    # few rows run on CUDA cores (the tensor-core kernels start at 17 rows of 16384 features, 65
    # of 8192, 257 of 4096 and of block-diagonal rows)
    (4096, 0, 3, hbl.HBL_Q_A4_ABSMEAN, hbl.HBL_CODES_I8, False),
    (8192, 0, 1, hbl.HBL_Q_A8_ABSMAX, hbl.HBL_CODES_PACKED, False),
    (16384, 0, 1, hbl.HBL_Q_A4_ABSMAX, hbl.HBL_CODES_I8, False),
    (16384, 0, 3, hbl.HBL_Q_A4_ABSMEAN, hbl.HBL_CODES_I8, True),
    (768, 256, 37, hbl.HBL_Q_A4_ABSMEAN, hbl.HBL_CODES_PACKED, False),
    (11008, 256, 23, hbl.HBL_Q_A4_ABSMEAN, hbl.HBL_CODES_PACKED, False),
    (11008, 256, 5, hbl.HBL_Q_A8_ABSMAX, hbl.HBL_CODES_I8, True),
    (2560, 512, 11, hbl.HBL_Q_A4_ABSMEAN, hbl.HBL_CODES_PACKED, False),
    (12288, 4096, 6, hbl.HBL_Q_A4_ABSMEAN, hbl.HBL_CODES_PACKED, False),
    (32768, 16384, 3, hbl.HBL_Q_A4_ABSMEAN, hbl.HBL_CODES_PACKED, False),
    (32768, 256, 3, hbl.HBL_Q_A4_ABSMEAN, hbl.HBL_CODES_PACKED, False),
    # the tensor-core kernels at their smallest row counts, the 4- and 2-row groups with a ragged
    # last group of one row
    (16384, 0, 17, hbl.HBL_Q_A4_ABSMAX, hbl.HBL_CODES_I8, False),
    (8192, 0, 67, hbl.HBL_Q_A4_ABSMEAN, hbl.HBL_CODES_PACKED, False),
    (4096, 0, 261, hbl.HBL_Q_A4_ABSMEAN, hbl.HBL_CODES_I8, False),
    (4096, 0, 257, hbl.HBL_Q_A8_ABSMAX, hbl.HBL_CODES_PACKED, False),
    (11008, 256, 257, hbl.HBL_Q_A4_ABSMAX, hbl.HBL_CODES_I8, False),
    # more row groups than resident CTAs (two per SM): every CTA of the tensor-core kernel walks
    # three or more groups, through both TMEM accumulators and the refill of its copy buffer
    (16384, 0, 1000, hbl.HBL_Q_A4_ABSMEAN, hbl.HBL_CODES_I8, False),
    (8192, 0, 2000, hbl.HBL_Q_A4_ABSMAX, hbl.HBL_CODES_PACKED, False),
    (4096, 0, 4000, hbl.HBL_Q_A8_ABSMAX, hbl.HBL_CODES_I8, False),
    # and the CUDA-core kernel over thousands of row groups
    (2048, 0, 3000, hbl.HBL_Q_A4_ABSMEAN, hbl.HBL_CODES_I8, False),
    (11008, 256, 700, hbl.HBL_Q_A4_ABSMEAN, hbl.HBL_CODES_I8, False),
]


@pytest.mark.parametrize("K,had_block,M,quant,fmt,use_gain", NFQ_CASES)
def test_norm_fht_quant_matches_oracle(K, had_block, M, quant, fmt, use_gain):
    spec = spec_like("wo_7b_a4", K=K, M=M, seed=100 + K + had_block)
    x = inputs.activations(spec)
    gain = np.random.default_rng(K).uniform(0.5, 1.5, size=K).astype(np.float32) if use_gain else None
    abits, mode = QUANT_NAME[quant]
    q_ref, s_ref = oracle.norm_fht_quant(x, gain, had_block, abits, mode)
    q, s = gpu_codes(x, gain, had_block, quant, fmt)
    assert_codes_close(q, q_ref)
    np.testing.assert_allclose(s, s_ref, rtol=1e-5)


# plain BitLinear (had_block = 1: blocks of one feature, no rotation), the other linears' inputs
NQ_CASES = [
    (256, 16, hbl.HBL_Q_A8_ABSMAX, hbl.HBL_CODES_PACKED, False),
    (768, 37, hbl.HBL_Q_A4_ABSMEAN, hbl.HBL_CODES_PACKED, True),
    (2304, 9, hbl.HBL_Q_A4_ABSMAX, hbl.HBL_CODES_I8, False),
    (4096, 300, hbl.HBL_Q_A4_ABSMEAN, hbl.HBL_CODES_I8, False),
    (4096, 5, hbl.HBL_Q_A8_ABSMAX, hbl.HBL_CODES_I8, True),
    (8448, 7, hbl.HBL_Q_A4_ABSMEAN, hbl.HBL_CODES_PACKED, False),
    (11008, 33, hbl.HBL_Q_A4_ABSMEAN, hbl.HBL_CODES_I8, True),
    (16384, 3, hbl.HBL_Q_A4_ABSMAX, hbl.HBL_CODES_PACKED, False),
    (17152, 2, hbl.HBL_Q_A4_ABSMEAN, hbl.HBL_CODES_I8, False),
    (32768, 4, hbl.HBL_Q_A8_ABSMAX, hbl.HBL_CODES_I8, True),
]


@pytest.mark.parametrize("K,M,quant,fmt,use_gain", NQ_CASES)
def test_norm_quant_without_transform_matches_oracle(K, M, quant, fmt, use_gain):
    spec = spec_like("wo_7b_a4", K=K, M=M, seed=7 + K)
    x = inputs.activations(spec)
    gain = np.random.default_rng(K + 1).uniform(0.5, 1.5, size=K).astype(np.float32) if use_gain else None
    abits, mode = QUANT_NAME[quant]
    q_ref, s_ref = oracle.norm_fht_quant(x, gain, 1, abits, mode)
    q, s = gpu_codes(x, gain, 1, quant, fmt)
    assert_codes_close(q, q_ref)
    np.testing.assert_allclose(s, s_ref, rtol=1e-5)


def test_norm_quant_without_transform_degenerate_rows_and_eps():
    K = 4096
    x = np.zeros((5, K), dtype=np.float32)
    x[1, 5] = 3.0
    x[2] = -1.0
    x[3, ::2] = 1e-30
    x[4] = 60000.0 * np.sign(np.sin(np.arange(K)))
    bits = inputs.f32_to_bf16_bits(x)
    for quant in QUANT_NAME:
        abits, mode = QUANT_NAME[quant]
        for eps_norm, eps_q in ((1e-6, 0.0), (1e-2, 1e-3)):
            q_ref, s_ref = oracle.norm_fht_quant(bits, None, 1, abits, mode, eps_norm=eps_norm, eps_q=eps_q)
            q, s = gpu_codes(bits, None, 1, quant, hbl.HBL_CODES_I8, eps_norm=eps_norm, eps_q=eps_q)
            assert_codes_close(q, q_ref)
            assert np.all(q[0] == 0) and s[0] == 0.0
            np.testing.assert_allclose(s[1:], s_ref[1:], rtol=1e-5)


@pytest.mark.parametrize("K,fmt", [(2048, hbl.HBL_CODES_I8), (16384, hbl.HBL_CODES_I8),
                                   (16384, hbl.HBL_CODES_PACKED)])
def test_norm_fht_quant_degenerate_rows(K, fmt):
    # at K = 16384 the constant row's transform is one spike of sqrt(7) K > 2^15 codes before
    # clamping: the 16384-wide tensor-core kernel must take its clamp for rounded values outside
    # int16 (the six rows are repeated to 18 so that 16384 features run on that kernel)
    x = np.zeros((6, K), dtype=np.float32)
    x[1, 5] = 3.0                      # single spike: transform is flat, all |codes| equal
    x[2] = -1.0                        # constant row: transform is a single spike
    x[3] = np.linspace(-1, 1, K)
    x[4, ::2] = 1e-30                  # tiny values
    x[5] = 60000.0 * np.sign(np.sin(np.arange(K)))  # large values
    if K == 16384:
        x = np.tile(x, (3, 1))
    bits = inputs.f32_to_bf16_bits(x)
    for quant in QUANT_NAME:
        abits, mode = QUANT_NAME[quant]
        q_ref, s_ref = oracle.norm_fht_quant(bits, None, 0, abits, mode)
        q, s = gpu_codes(bits, None, 0, quant, fmt)
        assert_codes_close(q, q_ref)
        zero = np.all(x == 0, axis=1)
        assert np.all(q[zero] == 0) and np.all(s[zero] == 0.0)
        np.testing.assert_allclose(s[~zero], s_ref[~zero], rtol=1e-5)


@pytest.mark.parametrize("K,had_block,M", [(2048, 0, 13), (4096, 0, 261), (8192, 0, 67), (16384, 0, 19),
                                           (11008, 256, 259), (16384, 0, 13)])
def test_norm_fht_quant_eps_q_and_eps_norm(K, had_block, M):
    # eps under the RMS root and in the quantiser's divisor, on the CUDA-core kernel (2048; 16384
    # at 13 rows) and on every tensor-core form (one block of 4096 / 8192 / 16384, blocks of 256)
    spec = spec_like("wo_7b_a4", K=K, M=M, had_block=had_block, seed=K + 5)
    x = inputs.activations(spec)
    for quant in QUANT_NAME:
        abits, mode = QUANT_NAME[quant]
        q_ref, s_ref = oracle.norm_fht_quant(x, None, had_block, abits, mode, eps_norm=1e-2, eps_q=1e-3)
        q, s = gpu_codes(x, None, had_block, quant, hbl.HBL_CODES_I8, eps_norm=1e-2, eps_q=1e-3)
        assert_codes_close(q, q_ref)
        np.testing.assert_allclose(s, s_ref, rtol=1e-5)


# ---------------------------------------------------------------- weights

@pytest.mark.parametrize("K,N", [(256, 256), (2048, 520), (11008, 64)])
def test_pack_weights_matches_oracle(K, N):
    W = np.random.default_rng(K + N).standard_normal((K, N)).astype(np.float32) * 0.02
    t_ref, alpha_ref = oracle.absmean_ternarize(W)
    packed, alpha = hbl.hbl_pack_weights(torch.from_numpy(W).cuda())
    torch.cuda.synchronize()
    assert alpha == pytest.approx(alpha_ref, rel=1e-6)
    t2, t8, colsum = decode_blob(packed.cpu().numpy(), K, N)
    np.testing.assert_array_equal(t2, t8)
    near_half = np.abs(np.abs(W.astype(np.float64) / alpha_ref) - 0.5) < 1e-6
    assert np.all((t8 == t_ref) | near_half)
    np.testing.assert_array_equal(colsum, t8.astype(np.int64).sum(axis=0))


@pytest.mark.parametrize("K,N,had_block", [(256, 256, 0), (2048, 520, 0), (16384, 64, 0), (11008, 64, 256),
                                           (12288, 40, 4096), (4096, 136, 1), (8192, 2560, 0)])
def test_pack_weights_rotated_matches_oracle(K, N, had_block):
    W = np.random.default_rng(K + N + had_block).standard_normal((K, N)).astype(np.float32) * 0.02
    Wr_ref = oracle.rotate_weights(W, had_block)
    t_ref, alpha_ref = oracle.absmean_ternarize(Wr_ref)
    packed, alpha = hbl.hbl_pack_weights_rotated(torch.from_numpy(W).cuda(), had_block)
    torch.cuda.synchronize()
    assert alpha == pytest.approx(alpha_ref, rel=1e-6)
    t2, t8, colsum = decode_blob(packed.cpu().numpy(), K, N)
    np.testing.assert_array_equal(t2, t8)
    # the rotation runs in fp32 (relative error ~1e-6 of the column scale): a weight within that
    # of a rounding boundary may land on either side
    near_half = np.abs(np.abs(Wr_ref / alpha_ref) - 0.5) < 2e-5
    assert np.all((t8 == t_ref) | near_half)
    assert np.count_nonzero(t8 != t_ref) <= max(1, int(1e-4 * t8.size))
    np.testing.assert_array_equal(colsum, t8.astype(np.int64).sum(axis=0))


def test_pack_ternary_roundtrip_and_bad_codes():
    K, N = 512, 40
    t = np.random.default_rng(3).integers(-1, 2, size=(K, N)).astype(np.int8)
    packed = hbl.hbl_pack_ternary(torch.from_numpy(t).cuda())
    t2, t8, colsum = decode_blob(packed.cpu().numpy(), K, N)
    np.testing.assert_array_equal(t2, t)
    np.testing.assert_array_equal(t8, t)
    np.testing.assert_array_equal(colsum, t.astype(np.int64).sum(axis=0))
    assert hbl.hbl_device_status() == hbl.HBL_OK
    bad = t.copy()
    bad[7, 3] = 2
    hbl.hbl_pack_ternary(torch.from_numpy(bad).cuda())
    assert hbl.hbl_device_status() == hbl.HBL_EINVAL   # flagged, clamped, no trap
    assert hbl.hbl_device_status() == hbl.HBL_OK       # the flag was cleared


def test_all_zero_weights():
    K, N = 256, 16
    packed, alpha = hbl.hbl_pack_weights(torch.zeros((K, N), device="cuda"))
    assert alpha == 0.0
    t2, t8, colsum = decode_blob(packed.cpu().numpy(), K, N)
    assert not t2.any() and not t8.any() and not colsum.any()


# ---------------------------------------------------------------- integer product (bit-exact)

def run_gemm_with_oracle_codes(q, t, s, alpha, fmt, abits):
    M, K = q.shape
    N = t.shape[1]
    codes = pack_int4(q) if (fmt == hbl.HBL_CODES_PACKED and abits == 4) else q.view(np.uint8)
    codes_d = torch.from_numpy(np.ascontiguousarray(codes)).cuda()
    packed = hbl.hbl_pack_ternary(torch.from_numpy(t).cuda())
    s_d = torch.from_numpy(s.astype(np.float32)).cuda()
    acc = torch.empty((M, N), dtype=torch.int32, device="cuda")
    Y = hbl.hbl_ternary_gemm(codes_d, fmt, abits, s_d, packed, alpha, N, K, acc_debug=acc)
    torch.cuda.synchronize()
    return acc.cpu().numpy(), Y.cpu().numpy()


GEMM_CASES = [
    # (M, K, N, abits, fmt)  -- int8 codes: M <= 4 on CUDA cores, up to 256 on swapped tcgen05
    # tiles, larger M on SM pairs; packed int4 codes: M <= 8 on CUDA cores
    (1, 256, 8, 4, hbl.HBL_CODES_PACKED),
    (1, 16384, 264, 4, hbl.HBL_CODES_PACKED),
    (2, 4096, 128, 8, hbl.HBL_CODES_PACKED),
    (3, 11008, 72, 4, hbl.HBL_CODES_I8),
    (5, 2048, 520, 4, hbl.HBL_CODES_PACKED),
    (8, 32768, 24, 4, hbl.HBL_CODES_PACKED),
    (1, 4096, 4096, 4, hbl.HBL_CODES_I8),
    (7, 16384, 136, 4, hbl.HBL_CODES_I8),
    (9, 256, 8, 4, hbl.HBL_CODES_I8),
    (16, 4096, 264, 4, hbl.HBL_CODES_I8),
    (64, 16384, 128, 4, hbl.HBL_CODES_I8),
    (255, 2048, 136, 8, hbl.HBL_CODES_I8),
    (128, 1024, 256, 8, hbl.HBL_CODES_I8),
    (300, 2048, 520, 4, hbl.HBL_CODES_I8),
    (257, 11008, 264, 4, hbl.HBL_CODES_I8),
    (200, 4096, 1032, 8, hbl.HBL_CODES_I8),
    # swapped tiles over a long K: several batches per CTA, so that every ring and tensor-memory
    # slot wraps (16, 112 and 256 padded tokens)
    (16, 16384, 4096, 4, hbl.HBL_CODES_I8),
    (100, 16384, 1024, 8, hbl.HBL_CODES_I8),
    (256, 16384, 256, 4, hbl.HBL_CODES_I8),
    # more 256 x 256 pair tiles than SM pairs: clusters walk two or more tiles, alternating their
    # two TMEM accumulators (80 and 160 tiles for 74 pairs)
    (2560, 512, 2048, 4, hbl.HBL_CODES_I8),
    (2560, 256, 4096, 8, hbl.HBL_CODES_I8),
    # few tiles over a long K: two SM pairs per tile, the second pair's partial sums added through
    # distributed shared memory (ragged rows and columns)
    (512, 16384, 1032, 4, hbl.HBL_CODES_I8),
    (700, 8192, 264, 8, hbl.HBL_CODES_I8),
]


@pytest.mark.parametrize("M,K,N,abits,fmt", GEMM_CASES)
def test_ternary_gemm_bit_exact(M, K, N, abits, fmt):
    rng = np.random.default_rng(M * 7 + K + N)
    lo, hi = (-8, 7) if abits == 4 else (-128, 127)
    q = rng.integers(lo, hi + 1, size=(M, K)).astype(np.int8)
    q[0, :] = hi                           # extreme row: largest positive sum
    if M > 2:
        q[-1, :] = lo
    t = rng.integers(-1, 2, size=(K, N)).astype(np.int8)
    t[:, 0] = 1
    s = rng.uniform(0.01, 0.1, size=M)
    alpha = 0.0173
    acc, Y = run_gemm_with_oracle_codes(q, t, s, alpha, fmt, abits)
    acc_ref = oracle.ternary_matmul(q, t)
    np.testing.assert_array_equal(acc.astype(np.int64), acc_ref)
    y_ref = oracle.dequant(acc_ref, s.astype(np.float32).astype(np.float64), np.float32(alpha))
    np.testing.assert_allclose(Y, y_ref, rtol=2e-6, atol=1e-30)


def test_tensor_core_path_needs_int8_codes():
    q = np.zeros((64, 256), dtype=np.int8)
    with pytest.raises(hbl.HblError) as e:
        run_gemm_with_oracle_codes(q, np.zeros((256, 8), np.int8), np.ones(64), 1.0, hbl.HBL_CODES_PACKED, 4)
    assert e.value.status == hbl.HBL_EUNSUPPORTED


def test_bf16_output():
    rng = np.random.default_rng(5)
    for M in (4, 200):
        q = rng.integers(-8, 8, size=(M, 1024)).astype(np.int8)
        t = rng.integers(-1, 2, size=(1024, 264)).astype(np.int8)
        s = rng.uniform(0.01, 0.1, size=M)
        packed = hbl.hbl_pack_ternary(torch.from_numpy(t).cuda())
        codes = torch.from_numpy(q.view(np.uint8)).cuda()
        Y = hbl.hbl_ternary_gemm(codes, hbl.HBL_CODES_I8, 4, torch.from_numpy(s.astype(np.float32)).cuda(), packed,
                                 0.02, 264, 1024, out_dtype=hbl.HBL_OUT_BF16)
        y_ref = oracle.dequant(oracle.ternary_matmul(q, t), s.astype(np.float32), np.float32(0.02))
        y = Y.float().cpu().numpy()
        np.testing.assert_allclose(y, y_ref, rtol=2 ** -8, atol=1e-6)


# ---------------------------------------------------------------- whole layer

def fused_forward(spec):
    """hbl_forward_decode (the decode kernel computing its own activation side) takes one token
    with K a power of two up to 8192: one transform block, blocks of a power of two, or none."""
    K = spec.K
    n = K if spec.had_block == 0 else spec.had_block
    return (spec.M == 1 and K <= 8192 and K & (K - 1) == 0
            and (n == 1 or (n & (n - 1) == 0 and 256 <= n <= 16384 and K % n == 0)))


def check_forward(spec, rows=None, out_dtype=hbl.HBL_OUT_F32):
    """Run hbl_forward on the full spec; compare `rows` (default: all) with the oracle."""
    x = inputs.activations(spec)
    W = inputs.weights(spec)
    quant = hbl.HBL_Q_A8_ABSMAX if spec.abits == 8 else hbl.HBL_Q_A4_ABSMEAN
    abits, mode = QUANT_NAME[quant]
    packed, alpha = hbl.hbl_pack_weights(torch.from_numpy(W).cuda())
    X = to_dev_bf16(x)
    Y = hbl.hbl_forward(X, packed, alpha, spec.N, None, spec.had_block, quant, out_dtype=out_dtype)
    fmt = hbl.HBL_CODES_PACKED if spec.M <= 8 else hbl.HBL_CODES_I8
    codes, s_x = hbl.hbl_norm_fht_quant(X, None, spec.had_block, quant, fmt=fmt)
    torch.cuda.synchronize()
    y = Y.float().cpu().numpy()
    assert np.all(np.isfinite(y))
    sel = np.arange(spec.M) if rows is None else np.asarray(rows)
    c = codes.cpu().numpy()[sel]
    q_gpu = unpack_int4(c, spec.K) if (fmt == hbl.HBL_CODES_PACKED and abits == 4) else c.view(np.int8)
    s_gpu = s_x.cpu().numpy()[sel].astype(np.float64)
    ref = oracle.h_bitlinear_forward(x[sel], W, None, spec.had_block, abits, mode)
    assert alpha == pytest.approx(ref["alpha"], rel=1e-6)
    assert_codes_close(q_gpu, ref["q"])
    np.testing.assert_allclose(s_gpu, ref["s"], rtol=1e-5)
    ys = y[sel]
    tnorm = np.linalg.norm(ref["t"].astype(np.float64), axis=1)
    rel = 1e-3 if out_dtype == hbl.HBL_OUT_F32 else 4e-3
    err = np.linalg.norm(ys - ref["y"], axis=1)
    # exact product of the GPU's own codes, oracle weights and scales
    y_own = oracle.dequant(oracle.ternary_matmul(q_gpu, ref["t"]), ref["s"], ref["alpha"])
    tol_own = 1e-5 if out_dtype == hbl.HBL_OUT_F32 else 2 ** -8
    assert np.all(row_rel_err(ys, y_own) <= tol_own)
    # end to end against the oracle, with the permitted flips accounted for exactly
    dq = np.abs(q_gpu.astype(np.float64) - ref["q"])
    flip_part = (dq @ tnorm) * ref["s"] * ref["alpha"]
    bound = rel * np.linalg.norm(ref["y"], axis=1) + flip_part
    assert np.all(err <= bound + 1e-30)


@pytest.mark.parametrize("name,M", [("single_a8_16x256", None), ("wo_1p3b_a4", 67), ("wdown_3b_a4", 130),
                                    ("wo_7b_a4", 5), ("wdown_7b_a4", 2), ("wdown_nonpow2_a4", 40)])
def test_forward_small(name, M):
    spec = inputs.WORKLOADS[name] if M is None else inputs.WORKLOADS[name].with_m(M)
    check_forward(spec)


@pytest.mark.parametrize("M,quant", [(1, hbl.HBL_Q_A4_ABSMEAN), (3, hbl.HBL_Q_A8_ABSMAX), (64, hbl.HBL_Q_A4_ABSMEAN),
                                     (300, hbl.HBL_Q_A8_ABSMAX), (1024, hbl.HBL_Q_A4_ABSMEAN)])
def test_plain_bitlinear_forward_qkv_shape(M, quant):
    # a QKV-like projection 4096 -> 12288 with no rotation (had_block = 1), all rows
    spec = spec_like("wo_7b_a4", M=M, N=12288, had_block=1, abits=QUANT_NAME[quant][0], seed=11)
    x = inputs.activations(spec)
    W = inputs.weights(spec)
    abits, mode = QUANT_NAME[quant]
    packed, alpha = hbl.hbl_pack_weights(torch.from_numpy(W).cuda())
    X = to_dev_bf16(x)
    Y = hbl.hbl_forward(X, packed, alpha, spec.N, None, 1, quant, out_dtype=hbl.HBL_OUT_F32)
    codes, s_x = hbl.hbl_norm_fht_quant(X, None, 1, quant, fmt=hbl.HBL_CODES_I8)
    torch.cuda.synchronize()
    q_gpu = codes.cpu().numpy().view(np.int8)
    ref = oracle.h_bitlinear_forward(x, W, None, 1, abits, mode)
    assert_codes_close(q_gpu, ref["q"])
    y = Y.cpu().numpy()
    y_own = oracle.dequant(oracle.ternary_matmul(q_gpu, ref["t"]), ref["s"], ref["alpha"])
    assert np.all(row_rel_err(y, y_own) <= 1e-5)
    dq = np.abs(q_gpu.astype(np.float64) - ref["q"])
    flip_part = (dq @ np.linalg.norm(ref["t"].astype(np.float64), axis=1)) * ref["s"] * ref["alpha"]
    err = np.linalg.norm(y - ref["y"], axis=1)
    assert np.all(err <= 1e-3 * np.linalg.norm(ref["y"], axis=1) + flip_part + 1e-30)


@pytest.mark.parametrize("name,M", [("wdown_3b_a4", 300), ("wdown_nonpow2_a4", 20), ("wo_7b_a4", 2)])
def test_forward_with_rotated_weights(name, M):
    # the weights-and-activations variant: weights rotated by the packer, activations by the layer
    spec = inputs.WORKLOADS[name].with_m(M)
    x = inputs.activations(spec)
    W = inputs.weights(spec)
    packed, alpha = hbl.hbl_pack_weights_rotated(torch.from_numpy(W).cuda(), spec.had_block)
    X = to_dev_bf16(x)
    Y = hbl.hbl_forward(X, packed, alpha, spec.N, None, spec.had_block, hbl.HBL_Q_A4_ABSMEAN)
    codes, _ = hbl.hbl_norm_fht_quant(X, None, spec.had_block, hbl.HBL_Q_A4_ABSMEAN, fmt=hbl.HBL_CODES_I8)
    torch.cuda.synchronize()
    ref = oracle.h_bitlinear_forward(x, W, None, spec.had_block, 4, "absmean", rotate_w=True)
    assert alpha == pytest.approx(ref["alpha"], rel=1e-6)
    t2, t8, _ = decode_blob(packed.cpu().numpy(), spec.K, spec.N)
    q_gpu = codes.cpu().numpy().view(np.int8)
    assert_codes_close(q_gpu, ref["q"])
    y = Y.cpu().numpy()
    # the product of the GPU's own codes with its own weight codes, through the oracle
    y_own = oracle.dequant(oracle.ternary_matmul(q_gpu, t8), ref["s"], ref["alpha"])
    assert np.all(row_rel_err(y, y_own) <= 1e-5)
    # against the oracle end to end: flipped activation codes and weight codes accounted exactly
    dq = np.abs(q_gpu.astype(np.float64) - ref["q"])
    dt = np.abs(t8.astype(np.float64) - ref["t"])
    flip = (dq @ np.linalg.norm(ref["t"].astype(np.float64), axis=1)
            + np.abs(q_gpu.astype(np.float64)) @ dt.sum(axis=1)) * ref["s"] * ref["alpha"]
    err = np.linalg.norm(y - ref["y"], axis=1)
    assert np.all(err <= 1e-3 * np.linalg.norm(ref["y"], axis=1) + flip + 1e-30)


FUSED_CASES = [
    # (K, N, had_block, M, quant, gain, eps_norm, eps_q)
    (4096, 4096, 0, 1, hbl.HBL_Q_A4_ABSMEAN, False, 1e-6, 0.0),
    (8192, 520, 0, 1, hbl.HBL_Q_A8_ABSMAX, True, 1e-6, 0.0),
    (4096, 4096, 0, 1, hbl.HBL_Q_A4_ABSMAX, False, 1e-2, 1e-3),
    (4096, 264, 256, 1, hbl.HBL_Q_A4_ABSMEAN, True, 1e-6, 0.0),
    (8192, 2560, 2048, 1, hbl.HBL_Q_A4_ABSMEAN, False, 1e-6, 0.0),
    (2048, 2048, 0, 1, hbl.HBL_Q_A8_ABSMAX, False, 1e-6, 1e-3),
    (256, 256, 0, 1, hbl.HBL_Q_A8_ABSMAX, False, 1e-6, 0.0),
    (8192, 136, 4096, 1, hbl.HBL_Q_A4_ABSMEAN, False, 1e-6, 0.0),
    (4096, 12288, 1, 1, hbl.HBL_Q_A4_ABSMEAN, True, 1e-6, 0.0),
    (1024, 128, 1, 1, hbl.HBL_Q_A8_ABSMAX, False, 1e-6, 0.0),
]


@pytest.mark.parametrize("K,N,had_block,M,quant,use_gain,eps_norm,eps_q", FUSED_CASES)
def test_fused_decode_forward(K, N, had_block, M, quant, use_gain, eps_norm, eps_q):
    # one launch per layer for one token (hbl_forward_decode): the product kernel computes each
    # CTA's slice of the activation codes itself (transform stages across slices as signed sums, statistics reduced
    # over the cluster); compared with the oracle per row with the one-step flip budget
    abits, mode = QUANT_NAME[quant]
    spec = spec_like("wdown_7b_a4", K=K, N=N, M=M, had_block=had_block, abits=abits, seed=K + N + M)
    assert fused_forward(spec)
    x = inputs.activations(spec)
    W = inputs.weights(spec)
    gain = np.random.default_rng(K).uniform(0.5, 1.5, size=K).astype(np.float32) if use_gain else None
    packed, alpha = hbl.hbl_pack_weights(torch.from_numpy(W).cuda())
    g = None if gain is None else torch.from_numpy(gain).cuda()
    Y = hbl.hbl_forward_decode(to_dev_bf16(x), packed, alpha, N, g, had_block, quant, eps_norm, eps_q)
    torch.cuda.synchronize()
    y = Y.cpu().numpy()
    ref = oracle.h_bitlinear_forward(x, W, gain, had_block, abits, mode, eps_norm=eps_norm, eps_q=eps_q)
    tnorm = np.linalg.norm(ref["t"].astype(np.float64), axis=1)
    flips = max(1, int(1e-4 * K))
    bound = 1e-3 * np.linalg.norm(ref["y"], axis=1) + flips * tnorm.max() * ref["s"] * ref["alpha"]
    err = np.linalg.norm(y - ref["y"], axis=1)
    assert np.all(err <= bound + 1e-30), (err / np.linalg.norm(ref["y"], axis=1))


FULL = [("single_a8_16x256", None), ("wo_1p3b_a4", None), ("wdown_3b_a4", None), ("wo_7b_a4", 8192),
        ("wdown_7b_a4", 8192), ("wo_7b_a4", 1), ("wdown_7b_a4", 1), ("wdown_7b_a4", 16), ("wo_7b_a4", 64),
        ("wdown_7b_a4", 64), ("wdown_7b_a4", 512), ("wdown_nonpow2_a4", None)]


@pytest.mark.parametrize("name,M", FULL)
def test_forward_full_size_sampled_rows(name, M):
    # the benchmark's launch configuration (bf16 output); the oracle checks a sample of rows
    spec = inputs.WORKLOADS[name] if M is None else inputs.WORKLOADS[name].with_m(M)
    picks = [0, 1, spec.M // 2, spec.M - 1] + list(np.random.default_rng(spec.M).integers(0, spec.M, 4))
    rows = sorted(set(int(r) for r in picks if r < spec.M))
    check_forward(spec, rows=rows, out_dtype=hbl.HBL_OUT_BF16)


@pytest.mark.parametrize("name,M", [("wdown_7b_a4", 8192), ("wo_7b_a4", 8192)])
def test_norm_fht_quant_full_size_every_row(name, M):
    # the activation kernel exactly as the benchmark launches it (a4 absmean, int8 codes) at full
    # size: every code and every scale against the oracle, rows checked in chunks
    spec = inputs.WORKLOADS[name].with_m(M)
    x = inputs.activations(spec)
    q, s = gpu_codes(x, None, spec.had_block, hbl.HBL_Q_A4_ABSMEAN, hbl.HBL_CODES_I8)
    flips = 0
    for r0 in range(0, M, 1024):
        q_ref, s_ref = oracle.norm_fht_quant(x[r0:r0 + 1024], None, spec.had_block, 4, "absmean")
        d = np.abs(q[r0:r0 + 1024].astype(np.int32) - q_ref)
        assert d.max() <= 1
        flips += int(np.count_nonzero(d))
        np.testing.assert_allclose(s[r0:r0 + 1024], s_ref, rtol=1e-5)
    assert flips <= max(1, int(1e-4 * M * spec.K)), flips


@pytest.mark.parametrize("M", [1, 3, 16, 64, 300])
def test_chained_layers_read_the_previous_output(M):
    # Two layers on one stream, the second fed by the first's output: the second layer's kernels
    # may launch before the first layer's product has finished (programmatic dependent launch)
    # and must wait for it before reading. Every kernel reduces in a fixed order, so the result
    # equals, bit for bit, the second layer run after an explicit synchronisation.
    spec = inputs.WORKLOADS["wo_7b_a4"].with_m(M)
    X = to_dev_bf16(inputs.activations(spec))
    W1 = inputs.weights(spec)
    W2 = np.ascontiguousarray(W1[::-1, ::-1])
    p1, a1 = hbl.hbl_pack_weights(torch.from_numpy(W1).cuda())
    p2, a2 = hbl.hbl_pack_weights(torch.from_numpy(W2).cuda())
    q = hbl.HBL_Q_A4_ABSMEAN
    Y1 = hbl.hbl_forward(X, p1, a1, spec.N, None, 0, q, out_dtype=hbl.HBL_OUT_BF16)
    Y2 = hbl.hbl_forward(Y1, p2, a2, spec.N, None, 0, q, out_dtype=hbl.HBL_OUT_F32)
    torch.cuda.synchronize()
    Y1c = Y1.clone()
    torch.cuda.synchronize()
    Y2_ref = hbl.hbl_forward(Y1c, p2, a2, spec.N, None, 0, q, out_dtype=hbl.HBL_OUT_F32)
    torch.cuda.synchronize()
    assert torch.equal(Y2, Y2_ref)
    assert hbl.hbl_device_status() == hbl.HBL_OK
