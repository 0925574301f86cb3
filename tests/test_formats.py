"""The test-side readers of the library's byte formats (tests/formats.py), checked on the CPU against
element-by-element writers of the layouts documented in include/hbl.h, so that a mistake in a
reader cannot hide a mistake on the GPU side."""
import numpy as np

from formats import blob_offsets, decode_blob, pack_int4, unpack_bitstream, unpack_int4

RNG = np.random.default_rng(7)


def test_int4_nibbles():
    # element 2j in the low nibble of byte j, two's complement
    q = np.array([[1, -1, 7, -8, 0, 5]], dtype=np.int8)
    packed = pack_int4(q)
    assert packed.tolist() == [[0xF1, 0x87, 0x50]]
    np.testing.assert_array_equal(unpack_int4(packed, 6), q)
    allq = RNG.integers(-8, 8, size=(5, 64)).astype(np.int8)
    np.testing.assert_array_equal(unpack_int4(pack_int4(allq), 64), allq)


def _blob_by_element(t: np.ndarray) -> np.ndarray:
    """t [K, N] in {-1, 0, 1} -> blob, one element at a time from the documented layout: section 0
    tile-major 2-bit words (tile of 128 features x 128 k = 4 KB; feature row r of the tile at 32 bytes
    per row; code k = 16w + 4s + b of the k-block at bits 8b + 2s of word w; c = t + 1; features
    padded to a multiple of 128 with t = 0), section 1 int8 t as [N][K], section 2 int32 column
    sums of t."""
    K, N = t.shape
    o0, o1, o2, end = blob_offsets(K, N)
    NP = (N + 127) // 128 * 128
    words = np.zeros((NP // 128) * (K // 128) * 128 * 8, dtype=np.uint32)
    for n in range(NP):
        for k in range(K):
            c = (int(t[k, n]) if n < N else 0) + 1
            tile, row, kb, kk = n // 128, n % 128, k // 128, k % 128
            w, rem = kk // 16, kk % 16
            s, b = rem // 4, rem % 4
            idx = ((tile * (K // 128) + kb) * 128 + row) * 8 + w
            words[idx] |= np.uint32(c << (8 * b + 2 * s))
    blob = np.zeros(end, dtype=np.uint8)
    blob[o0:o0 + words.nbytes] = words.view(np.uint8)
    blob[o1:o1 + N * K] = t.T.astype(np.int8).reshape(-1).view(np.uint8)
    blob[o2:o2 + 4 * N] = t.sum(axis=0).astype(np.int32).view(np.uint8)
    return blob


def test_decode_blob_reads_the_documented_layout():
    K, N = 256, 136  # two k-blocks, one full and one padded feature tile
    t = RNG.integers(-1, 2, size=(K, N)).astype(np.int8)
    t2, t8, colsum = decode_blob(_blob_by_element(t), K, N)
    np.testing.assert_array_equal(t2, t)
    np.testing.assert_array_equal(t8, t)
    np.testing.assert_array_equal(colsum, t.sum(axis=0))


def test_unpack_bitstream_reads_little_endian_codes():
    # code d of a head at bits [b d, b d + b) of its little-endian bit string (bit i = bit i % 8 of
    # byte i / 8)
    for bits in (2, 3, 4, 8):
        D = 64
        codes = RNG.integers(0, 2 ** bits, size=(3, 2, D))
        packed = np.zeros((3, 2, D * bits // 8), dtype=np.uint8)
        for i in np.ndindex(3, 2):
            for d in range(D):
                for j in range(bits):
                    if (codes[i][d] >> j) & 1:
                        pos = bits * d + j
                        packed[i][pos // 8] |= np.uint8(1 << (pos % 8))
        np.testing.assert_array_equal(unpack_bitstream(packed, D, bits), codes)
    # a hand-made example: b = 3, codes 0..7 -> 0b[111 110 101 100 011 010 001 000] read upwards
    assert unpack_bitstream(np.array([[0x88, 0xC6, 0xFA]], dtype=np.uint8), 8, 3).tolist() == [list(range(8))]
