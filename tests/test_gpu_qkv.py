"""Parity of the post-RoPE QKV quantiser (unsigned absmax, per head) with the CPU oracle.

Bars: the per-head scales gamma within relative 2e-6 (max of fp32 values against the fp64
oracle); the unsigned codes equal except for at most 1e-4 of them (at least one), each off by one
step (fp32 rotation and rounding against fp64); dequantised bf16 values equal to the oracle's
dequantisation of the GPU's own codes within bf16 rounding.
"""
import numpy as np
import pytest
import torch

import oracle
import hadamard_bit_quant_hbl_b200 as hbl
from hadamard_bit_quant_hbl_b200 import inputs
from formats import unpack_bitstream

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _gpu():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    torch.cuda.set_device(0)
    hbl.lib()
    yield
    assert hbl.hbl_device_status() == hbl.HBL_OK


def run(x_bits, H, D, bits, pos, theta=10000.0):
    M, stride = x_bits.shape
    X = torch.from_numpy(x_bits.view(np.int16)).cuda().view(torch.bfloat16)
    P = None if pos is None else torch.from_numpy(pos.astype(np.int32)).cuda()
    codes, gamma = hbl.hbl_qkv_quant(X, H, D, bits, pos=P, rope_theta=theta, row_stride=stride)
    Y = hbl.hbl_qkv_dequant(codes, gamma, D, bits)
    torch.cuda.synchronize()
    u = unpack_bitstream(codes.cpu().numpy(), D, bits)
    return u, gamma.cpu().numpy().astype(np.float64), Y.float().cpu().numpy()


def check(x_bits, H, D, bits, pos, theta=10000.0):
    M = x_bits.shape[0]
    u, g, y = run(x_bits, H, D, bits, pos, theta)
    xh = x_bits[:, :H * D].reshape(M, H, D)
    u_ref, g_ref = oracle.qkv_quant(xh, pos, bits, theta)
    np.testing.assert_allclose(g, g_ref, rtol=2e-6)
    d = np.abs(u.astype(np.int32) - u_ref.astype(np.int32))
    assert d.max() <= 1
    assert np.count_nonzero(d) <= max(1, int(1e-4 * d.size)), np.count_nonzero(d)
    y_own = oracle.dequantize_unsigned(u, g, bits)
    np.testing.assert_allclose(y, y_own, rtol=2 ** -8, atol=1e-30)
    return u, g


CASES = [
    # (M, H, D, bits, rope, row_stride)
    (7, 4, 128, 3, True, None),
    (33, 32, 128, 3, True, None),
    (5, 3, 64, 4, True, None),
    (9, 2, 256, 2, True, None),
    (17, 8, 128, 8, False, None),
    (4, 8, 128, 3, True, 3 * 8 * 128),   # the Q slice of a fused QKV row
    (6, 1, 64, 3, False, 200),
    (3, 12, 256, 4, False, None),
]


@pytest.mark.parametrize("M,H,D,bits,use_rope,stride", CASES)
def test_qkv_quant_matches_oracle(M, H, D, bits, use_rope, stride):
    x = inputs.qkv_states(M, H, D, seed=M + D + bits, row_stride=stride)
    pos = np.random.default_rng(M).integers(0, 32768, size=M) if use_rope else None
    check(x, H, D, bits, pos)


def test_qkv_quant_degenerate_heads_and_theta():
    M, H, D = 3, 4, 128
    x = np.zeros((M, H * D), dtype=np.float32)
    x[1, 128 + 7] = -2.5           # one spike: gamma = 2.5, every other feature the middle code
    x[2, :128] = 1.0               # a constant head
    x[2, 256:384] = np.linspace(-3, 3, 128)
    x[0, 384:390] = [1.5625, 0.625, -0.625, 1.25, -1.25, 0.0]  # exact .5 ties at 8 bits (no rotation)
    bits = inputs.f32_to_bf16_bits(x)
    pos = np.array([0, 5, 4000])
    for b in (2, 3, 4, 8):
        u, g = check(bits, H, D, b, pos, theta=500000.0)
        assert np.all(g[0, :3] == 0.0)
        assert np.all(u[0, :3] == (1 << (b - 1)))  # zero heads: the code nearest the middle (ties to even)
        u, g = check(bits, H, D, b, None)  # no rotation: the ties of row 0, head 3 are exact
        if b == 8:
            np.testing.assert_array_equal(u[0, 3, :6], [255, 178, 76, 230, 26, 128])


def test_qkv_quant_full_size_7b_heads():
    # 8192 tokens of a 7B-like attention (32 heads of 128), K states with RoPE at positions
    # 0..8191, 3-bit codes: every code and scale against the oracle
    M, H, D = 8192, 32, 128
    x = inputs.qkv_states(M, H, D)
    check(x, H, D, 3, np.arange(M))
