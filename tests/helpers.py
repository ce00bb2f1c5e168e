"""Comparison rules shared by the GPU parity tests.

Codes and scales: bit-exact.  The one tolerated exception (never relied on so
far) is a code off by one unit on at most 1e-4 of the elements, and only where
the exact pre-rounding value z*127/amax lies within 1e-6 of a .5 boundary.
Accumulators: bit-exact.  bf16 outputs: relative L2 <= 1e-2 and cosine
>= 0.9999 against the oracle's fp64 dequantisation.
"""
import numpy as np
import torch

from oracle import oracle as O

REL_L2_MAX = 1e-2
COS_MIN = 0.9999
TIE_WINDOW = 1e-6
MISMATCH_FRACTION_MAX = 1e-4


def bits(x: torch.Tensor) -> np.ndarray:
    return O.bf16_bits(x)


def f32_of_bf16(x: torch.Tensor) -> np.ndarray:
    return x.detach().float().cpu().numpy()


def assert_codes_match(q_gpu: np.ndarray, s_gpu: np.ndarray, q_ref: np.ndarray, s_ref: np.ndarray,
                       x_f32: np.ndarray | None = None, block: int = 128, rows: np.ndarray | None = None,
                       regular: bool = False) -> int:
    """Scales bit-exact; codes bit-exact up to the tie exception above.

    x_f32 (the input rows, same rows as q_ref) lets the exception be checked
    against the exact rotation (block b, Sylvester or, with `regular`, the
    regular H_4^(x)k).  Returns the number of codes that differ."""
    assert s_gpu.shape == s_ref.shape
    bad_s = np.flatnonzero(s_gpu.view(np.uint32) != s_ref.view(np.uint32))
    assert bad_s.size == 0, f"{bad_s.size} scales differ, first rows {bad_s[:5]}: gpu {s_gpu[bad_s[:5]]} ref {s_ref[bad_s[:5]]}"
    diff = q_gpu.astype(np.int16) - q_ref.astype(np.int16)
    bad = np.argwhere(diff != 0)
    if bad.size == 0:
        return 0
    assert np.abs(diff).max() <= 1, "a code differs by more than one unit"
    assert bad.shape[0] <= MISMATCH_FRACTION_MAX * q_ref.size, f"{bad.shape[0]} codes differ"
    assert x_f32 is not None, f"{bad.shape[0]} codes differ and no input to check the tie rule"
    for m, k in bad:
        z = O.rotate_explicit_f64(x_f32[m:m + 1], block, regular)[0]
        amax = float(s_ref[m]) * 127.0
        v = z[k] * 127.0 / amax
        frac = abs(abs(v) - np.floor(abs(v)) - 0.5)
        assert frac <= TIE_WINDOW, f"code ({m},{k}) differs but {v} is not within {TIE_WINDOW} of a tie"
    return int(bad.shape[0])


def assert_close_bf16(y_gpu: np.ndarray, y_ref: np.ndarray, what: str = ""):
    y = y_gpu.astype(np.float64).ravel()
    r = y_ref.astype(np.float64).ravel()
    assert np.isfinite(y).all(), f"{what}: non-finite output"
    nr = np.linalg.norm(r)
    rel = np.linalg.norm(y - r) / max(nr, 1e-300)
    cos = float(y @ r / max(np.linalg.norm(y) * nr, 1e-300))
    assert rel <= REL_L2_MAX, f"{what}: rel-L2 {rel:.3e}"
    assert cos >= COS_MIN, f"{what}: cosine {cos:.8f}"
    return rel, cos
