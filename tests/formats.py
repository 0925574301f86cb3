"""Test-side readers and writers of the library's documented byte formats (include/hbl.h).

Independent of both the oracle and the CUDA code: they only move bits between the documented
layouts and plain integer arrays, so that the tests can compare the two sides element by element.
"""
import numpy as np


def unpack_int4(packed: np.ndarray, K: int) -> np.ndarray:
    """[M, K/2] uint8, element 2j in the low nibble of byte j -> int8 [M, K]."""
    p = np.asarray(packed, dtype=np.uint8)
    lo = (p & 0x0F).astype(np.int16)
    hi = (p >> 4).astype(np.int16)
    out = np.empty((p.shape[0], K), dtype=np.int16)
    out[:, 0::2] = lo
    out[:, 1::2] = hi
    out[out >= 8] -= 16
    return out.astype(np.int8)


def pack_int4(q: np.ndarray) -> np.ndarray:
    """int8 [M, K] in [-8, 7] -> [M, K/2] uint8 (element 2j low nibble of byte j)."""
    q = np.asarray(q, dtype=np.int16)
    assert q.min() >= -8 and q.max() <= 7
    u = (q & 0x0F).astype(np.uint8)
    return (u[:, 0::2] | (u[:, 1::2] << 4)).astype(np.uint8)


def blob_offsets(K: int, N: int):
    r = lambda v: (v + 255) // 256 * 256  # noqa: E731
    off1 = r((N + 127) // 128 * 128 * K // 4)
    off2 = off1 + r(N * K)
    return 0, off1, off2, off2 + r(4 * N)


def decode_blob(blob: np.ndarray, K: int, N: int):
    """Packed weight blob -> (t from the 2-bit section [K, N], t from the int8 section [K, N], column sums)."""
    o0, o1, o2, _ = blob_offsets(K, N)
    b = np.asarray(blob, dtype=np.uint8)
    NP = (N + 127) // 128 * 128
    # tile-major: [N/128 tiles][K/128 blocks][128 rows][8 words] -> [NP rows][K/16 words]
    tiles = b[o0:o0 + NP * K // 4].view(np.uint32).reshape(NP // 128, K // 128, 128, 8)
    words = tiles.transpose(0, 2, 1, 3).reshape(NP, K // 16)[:N]
    t2 = np.empty((N, K), dtype=np.int8)
    for s in range(4):
        for bb in range(4):
            c = ((words >> (8 * bb + 2 * s)) & 3).astype(np.int8) - 1
            t2[:, 4 * s + bb::16] = c
    t8 = b[o1:o1 + N * K].view(np.int8).reshape(N, K)
    colsum = b[o2:o2 + 4 * N].view(np.int32)
    return t2.T.copy(), t8.T.copy(), colsum.copy()


def code_flips(a: np.ndarray, b: np.ndarray):
    """(number of differing codes, largest absolute difference)."""
    d = np.abs(a.astype(np.int32) - b.astype(np.int32))
    return int(np.count_nonzero(d)), int(d.max()) if d.size else 0


def row_rel_err(y: np.ndarray, ref: np.ndarray) -> np.ndarray:
    """Per token row: ||y - ref||_2 / ||ref||_2 (0 where the reference row is all zero and y matches)."""
    num = np.linalg.norm(np.asarray(y, np.float64) - ref, axis=1)
    den = np.linalg.norm(ref, axis=1)
    return np.where(den > 0, num / np.where(den > 0, den, 1), num)


def unpack_bitstream(packed: np.ndarray, D: int, bits: int) -> np.ndarray:
    """Codes of hbl_qkv_quant: [..., D*bits/8] bytes, code d at bits [bits*d, bits*d + bits) of the
    little-endian bit string of each head -> uint8 [..., D]."""
    p = np.asarray(packed, dtype=np.uint8)
    lead = p.shape[:-1]
    bitarr = np.unpackbits(p.reshape(-1, p.shape[-1]), axis=-1, bitorder="little")  # [n, D*bits]
    bitarr = bitarr.reshape(-1, D, bits).astype(np.uint16)
    vals = (bitarr << np.arange(bits, dtype=np.uint16)).sum(axis=-1)
    return vals.astype(np.uint8).reshape(*lead, D)
