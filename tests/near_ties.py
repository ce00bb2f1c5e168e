"""Inputs on which rounding the product twice and rounding it once differ.

The quantiser rounds the product z * inv to f32 first and only then to an
integer, ties to even.  These rows make the f32 product land exactly on 63.5
while the exact product lies a little below it: two roundings give 64, a
multiply-add that rounds the exact product once gives 63.

Block 128: each rotated block is z = (A, 0, ..., +-A/2 at one position, ...,
0) with A even in [128, 255], so x = H z / 128 has entries (A +- A/2) / 128;
A is kept only where 3A/2 and A/2 have at most 8 significant bits, so x is
exact in bf16 (and in f32) and an f32 transform of it (sums of small
integers) gives z back exactly.  Then amax = A, inv = f32(127 / A), and for
the A kept, f32((A/2) * inv) = 63.5 although (A/2) * inv != 63.5.
Block 0 (no rotation): x = (a, a/2, -a/2, 0, ...) with a bf16 amax a for
which f32((a/2) * f32(127/a)) = 63.5 likewise.

Only input construction lives here; the expected codes come from the oracle.
"""
import numpy as np


def is_near_tie(a: float) -> bool:
    inv = np.float32(127) / np.float32(a)
    exact = (a / 2) * float(inv)
    p = float(np.float32(exact))
    return p == 63.5 and exact != p and np.rint(p) != np.rint(exact)


def fits_bf16(v: int) -> bool:
    while v % 2 == 0:
        v //= 2
    return v < 256


def rotated_rows(K: int = 1024) -> np.ndarray:
    """Rows whose every block is z = (A, +-A/2 at position j), as exact x."""
    As = [A for A in range(128, 256, 2)
          if is_near_tie(float(A)) and fits_bf16(3 * A // 2) and fits_bf16(A // 2)]
    assert len(As) >= 10
    # Sylvester H_128: H[i][j] = (-1)^popcount(i & j)
    H = np.array([[1 - 2 * (bin(i & j).count("1") & 1) for j in range(128)] for i in range(128)], dtype=np.int64)
    rows = []
    for r, A in enumerate(As):
        x = np.zeros(K, dtype=np.float64)
        for b in range(K // 128):
            z = np.zeros(128, dtype=np.int64)
            z[0] = A
            j = 1 + (7 * b + 13 * r) % 127
            z[j] = (A // 2) * (1 if (b + r) % 2 == 0 else -1)
            x[b * 128:(b + 1) * 128] = (H @ z) / 128.0
        rows.append(x)
    return np.array(rows)


def plain_rows(K: int = 256) -> np.ndarray:
    bf16 = (np.arange(0x3F80, 0x4380, dtype=np.uint32) << 16).view(np.float32)
    amaxes = [float(a) for a in bf16 if is_near_tie(float(a))]
    assert len(amaxes) >= 20
    rows = np.zeros((len(amaxes), K))
    for r, a in enumerate(amaxes):
        rows[r, 0] = a
        rows[r, 1 + r % (K - 2)] = a / 2
        rows[r, 2 + (5 * r) % (K - 3)] = -a / 2
    return rows
