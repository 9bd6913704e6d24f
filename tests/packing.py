"""Test-side encoder for the canonical block formats.

It writes codes into bytes (the inverse direction of every decoder), so a test
can build a packed matrix from known integer codes and known fp16 scales and
compare any decoder against the dense matrix those codes and scales define.
It shares nothing with the oracle or the CUDA library.
"""
import numpy as np


def pack(fmt: str, q: np.ndarray) -> np.ndarray:
    """q int [rows, K] (K multiple of 32) -> uint8 [rows, K/32, B]."""
    rows, K = q.shape
    nb = K // 32
    q = q.reshape(rows, nb, 32).astype(np.uint8)
    if fmt == "q4":
        assert q.max() <= 15
        return (q[..., 0::2] | (q[..., 1::2] << 4)).astype(np.uint8)
    if fmt == "q2":
        assert q.max() <= 3
        return (q[..., 0::4] | (q[..., 1::4] << 2) | (q[..., 2::4] << 4) | (q[..., 3::4] << 6)).astype(np.uint8)
    assert q.max() <= 7
    bits = np.zeros((rows, nb, 96), dtype=np.uint8)
    for t in range(3):
        bits[..., t::3] = (q >> t) & 1          # code j -> bits 3j, 3j+1, 3j+2
    return np.packbits(bits, axis=-1, bitorder="little")


def dense(fmt: str, q: np.ndarray, scale_bits: np.ndarray) -> np.ndarray:
    """W[r, k] = s[r, k//32] * (q[r, k] - zero) in fp64."""
    zero = {"q4": 8, "q3": 4, "q2": 2}[fmt]
    s = scale_bits.astype(np.uint16).view(np.float16).astype(np.float64)
    return np.repeat(s, 32, axis=1) * (q.astype(np.float64) - zero)


def random_matrix(rng, fmt: str, rows: int, K: int, lo=0.005, hi=0.02):
    qmax = {"q4": 16, "q3": 8, "q2": 4}[fmt]
    q = rng.integers(0, qmax, size=(rows, K))
    s = rng.uniform(lo, hi, size=(rows, K // 32)).astype(np.float16).view(np.uint16)
    return q, s, pack(fmt, q), dense(fmt, q, s)
