"""The GELU epilogue's erfc (gemm_core.cuh, gelu_pair) against its derivation:
the coefficients in the kernel source are the ones fit_gelu_erfc.py fits, and
GELU evaluated the kernel's way in float32 stays within 2e-5 of the exact-erf
GELU in float64 (bf16 keeps 2^-9)."""
import os
import re

import numpy as np
from scipy.special import erfc

from w8a8_int8_quantized_block_b200 import fit_gelu_erfc as F

SRC = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))), "w8a8_int8_quantized_block_b200",
                   "csrc", "gemm_core.cuh")


def _kernel_coefficients():
    body = open(SRC).read()
    body = body[body.index("__device__ __forceinline__ void gelu_pair("):]
    body = body[:body.index("const uint64_t a = pk2f(a0, a1);")]
    # every pk2f(c, c) literal pair of the Horner chain, highest degree first
    vals = re.findall(r"pk2f\(\s*(-?[0-9.]+e[-+][0-9]+)f,\s*(-?[0-9.]+e[-+][0-9]+)f\)", body)
    assert all(a == b for a, b in vals)
    return np.array([np.float32(a) for a, _ in vals], dtype=np.float32)


def test_kernel_coefficients_are_the_fit():
    k = _kernel_coefficients()
    c = F.fit()
    assert k.size == F.DEG + 1
    assert np.array_equal(k, c[::-1].astype(np.float32))


def test_gelu_error_bound():
    c = F.fit()
    y = np.concatenate([np.linspace(-30, 30, 200001), -np.logspace(-8, 1.5, 5001), np.logspace(-8, 1.5, 5001)])
    ref = 0.5 * y * erfc(-y / np.sqrt(2.0))
    got = F.gelu_f32(y, c).astype(np.float64)
    ok = np.abs(ref) > 1e-30
    assert (np.abs(got[ok] - ref[ok]) / np.abs(ref[ok])).max() < 2e-5
    # exact at 0 and GELU(y) -> y, 0 far out
    assert F.gelu_f32(np.array([0.0]), c)[0] == 0.0
    assert F.gelu_f32(np.array([40.0]), c)[0] == np.float32(40.0)
    assert F.gelu_f32(np.array([-40.0]), c)[0] == 0.0
