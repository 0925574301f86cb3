"""Bit-level identities the CUDA kernels rely on, checked on the CPU with numpy (no GPU, no oracle):
the swapped-operand product's widening of 2-bit weight codes to int8 64 t, the decode kernel's
per-plane masking with exact recombination, and rounding onto 1.5 * 2^23 in fp32."""
import numpy as np

RNG = np.random.default_rng(20241203)


def _pack_words(codes):
    """codes [n, 16] in {0, 1, 2} (c' = t + 1) -> uint32 words, code k = 4 s + b at bits 8 b + 2 s
    (the blob's section-0 layout within one word)."""
    w = np.zeros(codes.shape[0], dtype=np.uint64)
    for s in range(4):
        for b in range(4):
            w |= codes[:, 4 * s + b].astype(np.uint64) << np.uint64(8 * b + 2 * s)
    return w.astype(np.uint32)


def test_widening_to_64t_is_exact():
    # (w * 2^(6 - 2 s) + 0xc0c0c0c0) & 0xc0c0c0c0 gives, in byte b, the int8 value 64 t of code
    # 4 s + b: the carries out of a byte land in the next byte's bits 0..5, which the mask drops,
    # and never reach its bits 6..7 (bits 0..5 hold at most three codes, each <= 2: 0b101010 + 1)
    codes = RNG.integers(0, 3, size=(200000, 16))
    codes[:3] = [[0] * 16, [1] * 16, [2] * 16]
    w = _pack_words(codes).astype(np.uint64)
    for s in range(4):
        o = ((w * np.uint64(1 << (6 - 2 * s)) + np.uint64(0xC0C0C0C0)) & np.uint64(0xC0C0C0C0)).astype(np.uint32)
        got = o.view(np.uint8).reshape(-1, 4).view(np.int8).astype(np.int64)  # little-endian bytes b = 0..3
        want = 64 * (codes[:, 4 * s:4 * s + 4] - 1)
        np.testing.assert_array_equal(got, want)


def test_64t_sums_fit_int32_and_divide_exactly():
    # |64 sum_k t q| <= 64 * 32768 * 128 = 2^28 for the largest K and a8 codes; the sum of 64 t q is
    # a multiple of 64, so the arithmetic shift by 6 returns sum t q exactly
    assert 64 * 32768 * 128 == 2 ** 28 < 2 ** 31
    t = RNG.integers(-1, 2, size=(64, 4096))
    q = RNG.integers(-128, 128, size=(4096,))
    s64 = (64 * t) @ q
    np.testing.assert_array_equal(s64.astype(np.int32) >> 6, t @ q)


def test_plane_masking_recombines_exactly():
    # the decode kernel masks plane s in place (bytes c' * 4^s), multiplies by the activation of
    # k-group s, and recombines acc0 + acc1 / 4 + acc2 / 16 + acc3 / 64; minus sum q gives sum t q
    codes = RNG.integers(0, 3, size=(5000, 16))
    q = RNG.integers(-128, 128, size=(5000, 16))
    w = _pack_words(codes)
    total = np.zeros(5000, dtype=np.int64)
    for s in range(4):
        masked = (w & np.uint32(0x03030303 << (2 * s))).view(np.uint8).reshape(-1, 4).astype(np.int64)
        acc = (masked * q[:, 4 * s:4 * s + 4]).sum(axis=1)
        assert np.all(acc % (4 ** s) == 0)
        total += acc // (4 ** s)
    np.testing.assert_array_equal(total - q.sum(axis=1), ((codes - 1) * q).sum(axis=1))


def test_rounding_onto_the_magic_number():
    # fp32 t + 1.5 * 2^23 rounds t to the nearest integer (ties to even) for |t| < 2^22, and the
    # low mantissa bits (minus the magic) are that integer: the codes' rounding in every kernel
    magic = np.float32(12582912.0)
    t = np.concatenate([RNG.uniform(-2 ** 21, 2 ** 21, 100000), RNG.uniform(-300, 300, 100000),
                        np.arange(-200, 200) + 0.5]).astype(np.float32)
    y = (t + magic).astype(np.float32)
    got = (y - magic).astype(np.float64)
    np.testing.assert_array_equal(got, np.rint(t.astype(np.float64)))
    n = np.rint(t.astype(np.float64)).astype(np.int64)
    bits = y.view(np.uint32).astype(np.int64)
    np.testing.assert_array_equal((bits & 0x7FFFFF) - (1 << 22), n)  # mantissa = 2^22 + n
    small = np.abs(n) < 2 ** 15  # the low 16 bits are n as an int16 (the kernels' int16 lanes)
    np.testing.assert_array_equal((bits[small] & 0xFFFF).astype(np.uint16).view(np.int16), n[small])
