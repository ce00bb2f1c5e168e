"""Python face of the CPU oracle (``convrot_oracle.c``) plus pure-Python
references used only on tiny inputs.

TEST INFRASTRUCTURE ONLY: imported by tests/, ``__graft_entry__.smoke()`` and
the CPU-baseline leg of ``bench.py``.  It shares no code with the CUDA path and
never imports the product package's arithmetic.

Every function cites the passage it follows (page title and section):

* block-diagonal Hadamard rotation -- lehuy.net "Nen mo hinh video khuech tan
  31B xuong 14B chi voi 6 buoc", section "Cach nen hoat dong";
* rowwise int8 activation quantisation -- MiniMax-H3-Rung-Omega README,
  "Technical Architecture Overview", item 2 (Floor 1);
* per-output-channel F32 weight scales, [output, input] storage -- "MiniMax H3 -
  pruned INT8 ConvRot - input-major", section "Input-major checkpoint";
* exact undo of the rotation -- "HyperFlow H3 Flash MLX", section "How to run";
* W8A8 INT8 -- HyperFlow H3 Flash card, "Choose a Weight Format";
* the activation prologue of the down projection ("SwiGLU + ConvRot64 +
  Rowwise INT8 Quantize" in MLP.fc2) -- MiniMax-H3-Rung-Omega README,
  "Technical Architecture Overview", item 2;
* int8 attention ("sageattn_qk_int8_pv_fp16_cuda" in the Rung-Omega engine's
  Floor 1 -- MiniMax-H3-Rung-Omega README, "Technical Architecture
  Overview", item 2): Q and K quantised per token row to int8, P V in
  16-bit floating point;
* the regular rotation H_4^(x)k ("DC-balanced regular orthogonal Hadamard
  matrix H_256 = H_4^(x)4") -- MiniMax-H3-Rung-Omega README, "Technical
  Architecture Overview", item 1.

Readings where the pages are silent: Sylvester
order H[i][j] = (-1)^popcount(i & j); unnormalised transform with the 1/b
folded into the dequantisation; fp32 butterflies in ascending stage order;
s = amax/127 and q = rne(z * (127/amax)) in f32; a zero row has s = 0;
regular H_4 = J - 2I, its fp32 stages in ascending digit stride, each group
t = (x0 + x1) + (x2 + x3), x_i -> t - 2 x_i.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
from fractions import Fraction

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "convrot_oracle.c")
# CONVROT_ORACLE_LIB points the wrapper at another build of the oracle; the
# mutation tests use it to check that the pins catch planted mistakes.
_LIB_PATH = os.environ.get("CONVROT_ORACLE_LIB") or os.path.join(_HERE, "liboracle.so")
CFLAGS = ["-O2", "-fopenmp", "-ffp-contract=off", "-fno-fast-math", "-fPIC", "-shared"]

__all__ = [
    "build", "lib", "num_threads", "hadamard", "hadamard_sylvester", "hadamard_regular_kron", "fwht",
    "quantize_rows", "quantize_act", "act_f32", "act_quantize", "ACT_NONE", "ACT_GELU", "ACT_SWIGLU",
    "pack_weight", "igemm", "igemm_pairs", "attention", "attention_rows",
    "dequant", "dequant_pairs", "linear", "rotate_explicit_f64",
    "bf16_bits", "bf16_bits_to_f32", "py_fwht_exact", "py_quantize_row_exact",
    "py_igemm",
]


def build(force: bool = False) -> str:
    """Compile the C oracle into ``oracle/liboracle.so`` (gcc, no fast-math)."""
    if os.environ.get("CONVROT_ORACLE_LIB"):
        return _LIB_PATH  # an explicitly chosen build is used as it is
    if force or not os.path.exists(_LIB_PATH) or os.path.getmtime(_LIB_PATH) < os.path.getmtime(_SRC):
        subprocess.check_call(["gcc", *CFLAGS, "-o", _LIB_PATH, _SRC, "-lm"])
    return _LIB_PATH


_lib = None


def lib() -> ctypes.CDLL:
    global _lib
    if _lib is None:
        build()
        L = ctypes.CDLL(_LIB_PATH)
        P = ctypes.c_void_p
        I64 = ctypes.c_int64
        I32 = ctypes.c_int
        L.oracle_hadamard_entry.argtypes = [I64, I64]
        L.oracle_hadamard_entry.restype = I32
        L.oracle_num_threads.restype = I32
        L.oracle_regular_entry.argtypes = [I64, I64, I32]
        L.oracle_regular_entry.restype = I32
        L.oracle_fwht_f32.argtypes = [P, I64, I32]
        L.oracle_rotate_f32.argtypes = [P, I64, I32, I32]
        L.oracle_quantize_rows_f32.argtypes = [P, I64, I64, I64, P, I64, P]
        L.oracle_quantize_act_bf16.argtypes = [P, I64, I64, I64, I32, I32, P, I64, P]
        L.oracle_pack_weight_f32.argtypes = [P, I64, I64, I32, I32, P, P]
        L.oracle_act_f32.argtypes = [P, I64, I64, I64, I32, P]
        L.oracle_act_quantize_bf16.argtypes = [P, I64, I64, I64, I32, I32, I32, P, I64, P]
        L.oracle_igemm_s64.argtypes = [P, I64, P, I64, I64, I64, I64, P, I64]
        L.oracle_igemm_s64_pairs.argtypes = [P, I64, P, I64, I64, P, P, I64, P]
        L.oracle_dequant_f64.argtypes = [P, I64, I64, P, P, P, ctypes.c_double, I32, P]
        L.oracle_dequant_pairs_f64.argtypes = [P, P, P, I64, P, P, P, ctypes.c_double, I32, P]
        L.oracle_rotate_explicit_f64.argtypes = [P, I64, I64, I32, I32, P]
        _lib = L
    return _lib


def _p(a: np.ndarray | None):
    return None if a is None else a.ctypes.data_as(ctypes.c_void_p)


def num_threads() -> int:
    """OpenMP threads the oracle uses."""
    return int(lib().oracle_num_threads())


# ---------------------------------------------------------------- Hadamard


def hadamard(b: int, regular: bool = False) -> np.ndarray:
    """H_b from its entry definition, via the C oracle: Sylvester
    (-1)^popcount(i & j), or the regular H_4^(x)k digit by digit."""
    L = lib()
    if regular:
        return np.array([[L.oracle_regular_entry(i, j, b) for j in range(b)] for i in range(b)], dtype=np.int64)
    return np.array([[L.oracle_hadamard_entry(i, j) for j in range(b)] for i in range(b)], dtype=np.int64)


def hadamard_sylvester(b: int) -> list[list[int]]:
    """Independent construction: H_1 = [1], H_2n = [[H, H], [H, -H]] (pure Python)."""
    H = [[1]]
    while len(H) < b:
        H = [r + r for r in H] + [r + [-v for v in r] for r in H]
    if len(H) != b:
        raise ValueError("b must be a power of two")
    return H


def hadamard_regular_kron(b: int) -> np.ndarray:
    """Independent construction of the regular matrix: Kronecker powers of
    H_4 = J - 2I (numpy), b = 4^k."""
    H4 = np.ones((4, 4), dtype=np.int64) - 2 * np.eye(4, dtype=np.int64)
    H = np.ones((1, 1), dtype=np.int64)
    while H.shape[0] < b:
        H = np.kron(H, H4)
    if H.shape[0] != b:
        raise ValueError("b must be a power of four")
    return H


def fwht(x: np.ndarray, b: int, regular: bool = False) -> np.ndarray:
    """Block-diagonal rotation of the last axis of a float32 array (canonical order)."""
    v = np.ascontiguousarray(x, dtype=np.float32).copy()
    if regular:
        lib().oracle_rotate_f32(_p(v), v.size, b, 1)
    else:
        lib().oracle_fwht_f32(_p(v), v.size, b)
    return v


def rotate_explicit_f64(x: np.ndarray, b: int, regular: bool = False) -> np.ndarray:
    """z = blockdiag(H_b) x by the explicit matrix, fp64 accumulation."""
    x = np.ascontiguousarray(x, dtype=np.float32)
    M, K = x.shape
    z = np.empty((M, K), dtype=np.float64)
    lib().oracle_rotate_explicit_f64(_p(x), M, K, b, int(regular), _p(z))
    return z


# ---------------------------------------------------------------- quantisers


def bf16_bits(x) -> np.ndarray:
    """Raw uint16 bits of a torch bfloat16 tensor (CPU)."""
    import torch

    t = x.detach().to("cpu").contiguous()
    assert t.dtype == torch.bfloat16
    return t.view(torch.int16).numpy().view(np.uint16)


def bf16_bits_to_f32(bits: np.ndarray) -> np.ndarray:
    return (bits.astype(np.uint32) << 16).view(np.float32)


def quantize_rows(z: np.ndarray):
    """Rowwise symmetric int8 of already-rotated f32 rows -> (q int8, s f32)."""
    z = np.ascontiguousarray(z, dtype=np.float32)
    M, K = z.shape
    q = np.empty((M, K), dtype=np.int8)
    s = np.empty((M,), dtype=np.float32)
    lib().oracle_quantize_rows_f32(_p(z), M, K, K, _p(q), K, _p(s))
    return q, s


def _require_finite_bf16(bits: np.ndarray, what: str) -> None:
    """Non-finite inputs are outside the method's contract (the pages quantise
    finite activations and weights only): refuse them rather than compute."""
    if bool(((bits & 0x7F80) == 0x7F80).any()):
        raise ValueError(f"{what}: non-finite bf16 input (inf or NaN) is outside the contract")


def quantize_act(x_bits: np.ndarray, b: int, regular: bool = False):
    """bf16 activations (uint16 bits [M, K]) -> rotate (block b) -> (q, s_x)."""
    x_bits = np.ascontiguousarray(x_bits, dtype=np.uint16)
    _require_finite_bf16(x_bits, "quantize_act")
    M, K = x_bits.shape
    q = np.empty((M, K), dtype=np.int8)
    s = np.empty((M,), dtype=np.float32)
    lib().oracle_quantize_act_bf16(_p(x_bits), M, K, K, b, int(regular), _p(q), K, _p(s))
    return q, s


ACT_NONE, ACT_GELU, ACT_SWIGLU = 0, 1, 2


def _act_width(h_bits: np.ndarray, act: int) -> int:
    cols = h_bits.shape[1]
    if act == ACT_SWIGLU:
        assert cols % 2 == 0
        return cols // 2
    return cols


def act_f32(h_bits: np.ndarray, act: int) -> np.ndarray:
    """The activation alone: x = gelu(h) or silu(g) * u ([g | u] = h's halves),
    each value computed in fp64 and rounded once to f32."""
    h_bits = np.ascontiguousarray(h_bits, dtype=np.uint16)
    M = h_bits.shape[0]
    K = _act_width(h_bits, act)
    x = np.empty((M, K), dtype=np.float32)
    lib().oracle_act_f32(_p(h_bits), M, K, h_bits.shape[1], act, _p(x))
    return x


def act_quantize(h_bits: np.ndarray, act: int, b: int, regular: bool = False):
    """Activation prologue + rotation + rowwise int8: the down projection's
    (q, s_x) from the up projection's bf16 output h ([M, K] or [M, 2K])."""
    h_bits = np.ascontiguousarray(h_bits, dtype=np.uint16)
    _require_finite_bf16(h_bits, "act_quantize")
    M = h_bits.shape[0]
    K = _act_width(h_bits, act)
    q = np.empty((M, K), dtype=np.int8)
    s = np.empty((M,), dtype=np.float32)
    lib().oracle_act_quantize_bf16(_p(h_bits), M, K, h_bits.shape[1], act, b, int(regular), _p(q), K, _p(s))
    return q, s


def pack_weight(w: np.ndarray, b: int, regular: bool = False):
    """f32 weights [N, K] -> rotate along K -> per-output-channel (q_w, s_w)."""
    w = np.ascontiguousarray(w, dtype=np.float32)
    if not bool(np.isfinite(w).all()):
        raise ValueError("pack_weight: non-finite weights (inf or NaN) are outside the contract")
    N, K = w.shape
    q = np.empty((N, K), dtype=np.int8)
    s = np.empty((N,), dtype=np.float32)
    lib().oracle_pack_weight_f32(_p(w), N, K, b, int(regular), _p(q), _p(s))
    return q, s


# ---------------------------------------------------------------- GEMM + epilogue


def igemm(qa: np.ndarray, qb: np.ndarray) -> np.ndarray:
    """acc = qa @ qb.T exactly in int64 (qa [M, K], qb [N, K], int8)."""
    qa = np.ascontiguousarray(qa, dtype=np.int8)
    qb = np.ascontiguousarray(qb, dtype=np.int8)
    M, K = qa.shape
    N, K2 = qb.shape
    assert K == K2
    c = np.empty((M, N), dtype=np.int64)
    lib().oracle_igemm_s64(_p(qa), K, _p(qb), K, M, N, K, _p(c), N)
    return c


def igemm_pairs(qa: np.ndarray, qb: np.ndarray, mi: np.ndarray, ni: np.ndarray) -> np.ndarray:
    """acc[t] = qa[mi[t]] . qb[ni[t]] exactly in int64."""
    qa = np.ascontiguousarray(qa, dtype=np.int8)
    qb = np.ascontiguousarray(qb, dtype=np.int8)
    mi = np.ascontiguousarray(mi, dtype=np.int64)
    ni = np.ascontiguousarray(ni, dtype=np.int64)
    K = qa.shape[1]
    out = np.empty(mi.shape, dtype=np.int64)
    lib().oracle_igemm_s64_pairs(_p(qa), K, _p(qb), K, K, _p(mi), _p(ni), mi.size, _p(out))
    return out


def _alpha(b: int) -> float:
    return 1.0 / b if b > 1 else 1.0


def dequant(acc: np.ndarray, s_a: np.ndarray, s_b: np.ndarray, bias: np.ndarray | None,
            b: int, gelu: bool = False) -> np.ndarray:
    """y = acc * s_a[m] * s_b[n] / b + bias[n] in fp64 (optional exact GELU)."""
    acc = np.ascontiguousarray(acc, dtype=np.int64)
    M, N = acc.shape
    s_a = np.ascontiguousarray(s_a, dtype=np.float32)
    s_b = np.ascontiguousarray(s_b, dtype=np.float32)
    bias = None if bias is None else np.ascontiguousarray(bias, dtype=np.float32)
    y = np.empty((M, N), dtype=np.float64)
    lib().oracle_dequant_f64(_p(acc), M, N, _p(s_a), _p(s_b), _p(bias), _alpha(b), int(gelu), _p(y))
    return y


def dequant_pairs(acc, mi, ni, s_a, s_b, bias, b: int, gelu: bool = False) -> np.ndarray:
    acc = np.ascontiguousarray(acc, dtype=np.int64)
    mi = np.ascontiguousarray(mi, dtype=np.int64)
    ni = np.ascontiguousarray(ni, dtype=np.int64)
    s_a = np.ascontiguousarray(s_a, dtype=np.float32)
    s_b = np.ascontiguousarray(s_b, dtype=np.float32)
    bias = None if bias is None else np.ascontiguousarray(bias, dtype=np.float32)
    y = np.empty(acc.shape, dtype=np.float64)
    lib().oracle_dequant_pairs_f64(_p(acc), _p(mi), _p(ni), acc.size, _p(s_a), _p(s_b), _p(bias),
                                   _alpha(b), int(gelu), _p(y))
    return y


def linear(x_bits: np.ndarray, w: np.ndarray, bias: np.ndarray | None, b: int, gelu: bool = False,
           regular: bool = False):
    """Whole path on the CPU: returns (y fp64, q_x, s_x, q_w, s_w, acc).  Both
    H_b H_b^T = b I kinds share alpha = 1/b."""
    qx, sx = quantize_act(x_bits, b, regular)
    qw, sw = pack_weight(w, b, regular)
    acc = igemm(qx, qw)
    y = dequant(acc, sx, sw, bias, b, gelu)
    return y, qx, sx, qw, sw, acc


# ---------------------------------------------------------------- attention


def _attention_head(qx, sq, kx, sk, v, scale):
    """One head: S = (q . k) s_q s_k scale from exact int64 dot products,
    P = softmax over the keys, O = P V, all in fp64."""
    S = igemm(qx, kx).astype(np.float64) * sq.astype(np.float64)[:, None] * sk.astype(np.float64)[None, :] * scale
    S -= S.max(axis=1, keepdims=True)
    P = np.exp(S)
    P /= P.sum(axis=1, keepdims=True)
    return P @ v


def attention(q_bits: np.ndarray, k_bits: np.ndarray, v_bits: np.ndarray, scale: float | None = None):
    """int8 attention: q, k, v bf16 bits [H, L, d] (k and v share their L).
    Q and K are quantised per token row (the rowwise int8 quantiser, no
    rotation); O = softmax(S) V with S = (q . k) s_q s_k * scale, scale
    1/sqrt(d) unless given; returns O fp64 [H, Lq, d] and the codes and
    scales (qx, sq, kx, sk)."""
    H, Lq, d = q_bits.shape
    _require_finite_bf16(np.asarray(v_bits, dtype=np.uint16), "attention (v)")  # q, k: checked by the quantiser
    scale = 1.0 / np.sqrt(d) if scale is None else scale
    qx, sq = quantize_act(q_bits.reshape(H * Lq, d), 0)
    kx, sk = quantize_act(k_bits.reshape(-1, d), 0)
    Lk = k_bits.shape[1]
    qx, sq = qx.reshape(H, Lq, d), sq.reshape(H, Lq)
    kx, sk = kx.reshape(H, Lk, d), sk.reshape(H, Lk)
    v = bf16_bits_to_f32(v_bits).astype(np.float64)
    O = np.stack([_attention_head(qx[h], sq[h], kx[h], sk[h], v[h], scale) for h in range(H)])
    return O, (qx, sq, kx, sk)


def attention_rows(qx, sq, kx, sk, v_bits, heads: np.ndarray, rows: np.ndarray, scale: float) -> np.ndarray:
    """O for a sample of (head, query row) pairs, from given codes and scales
    (qx [H, Lq, d], kx [H, Lk, d] int8; sq, sk f32): each row in full."""
    out = np.empty((len(heads), qx.shape[2]), dtype=np.float64)
    for t, (h, i) in enumerate(zip(heads, rows)):
        v = bf16_bits_to_f32(v_bits[h]).astype(np.float64)
        out[t] = _attention_head(qx[h, i:i + 1], sq[h, i:i + 1], kx[h], sk[h], v, scale)[0]
    return out


# ---------------------------------------------------------------- pure-Python references (tiny inputs)


def py_fwht_exact(x: list, b: int, regular: bool = False) -> list:
    """Explicit H_b x per block with exact rational arithmetic (no rounding)."""
    if regular:
        H = hadamard_regular_kron(b).tolist()
    else:
        H = hadamard_sylvester(b) if b > 1 else [[1]]
    bb = max(b, 1)
    out = []
    for o in range(0, len(x), bb):
        blk = [Fraction(v) for v in x[o:o + bb]]
        out.extend(sum(H[i][j] * blk[j] for j in range(bb)) for i in range(bb))
    return out


def _round_to_f32(r: Fraction) -> Fraction:
    """Round a rational to the nearest float32 value (ties to even), exactly."""
    if r == 0:
        return Fraction(0)
    sign = -1 if r < 0 else 1
    a = abs(r)
    e = a.numerator.bit_length() - a.denominator.bit_length()
    if Fraction(2) ** e > a:
        e -= 1
    e = max(e, -126)  # subnormal range keeps the -149 quantum
    quantum = Fraction(2) ** (e - 23)
    n = a / quantum
    fl = n.numerator // n.denominator
    rem = n - fl
    if rem > Fraction(1, 2) or (rem == Fraction(1, 2) and fl % 2 == 1):
        fl += 1
    return sign * fl * quantum


def _rne_int(r: Fraction) -> int:
    fl = r.numerator // r.denominator
    rem = r - fl
    if rem > Fraction(1, 2) or (rem == Fraction(1, 2) and fl % 2 == 1):
        fl += 1
    return fl


def py_quantize_row_exact(z: list):
    """Quantiser of one row with exact rational arithmetic standing in for f32:
    inv = f32(127/amax), v = f32(z*inv), q = ties-to-even(v) clamped to +-127,
    s = f32(amax/127).  Returns (codes, scale as Fraction)."""
    zq = [Fraction(v) for v in z]
    amax = max((abs(v) for v in zq), default=Fraction(0))
    if amax == 0:
        return [0] * len(zq), Fraction(0)
    inv = _round_to_f32(Fraction(127) / amax)
    s = _round_to_f32(amax / 127)
    codes = []
    for v in zq:
        c = _rne_int(_round_to_f32(v * inv))
        codes.append(max(-127, min(127, c)))
    return codes, s


def py_igemm(qa: list, qb: list) -> list:
    """Brute-force integer dot products in Python ints."""
    return [[sum(int(a) * int(b) for a, b in zip(ra, rb)) for rb in qb] for ra in qa]


def py_attention_exact_scores(qx: list, sq: list, kx: list, sk: list, v: list, scale: float) -> list:
    """One head by plain Python loops (math.exp), for tiny inputs."""
    import math
    out = []
    for i in range(len(qx)):
        s = [sum(a * b for a, b in zip(qx[i], kx[j])) * sq[i] * sk[j] * scale for j in range(len(kx))]
        m = max(s)
        e = [math.exp(x - m) for x in s]
        t = sum(e)
        out.append([sum(e[j] * v[j][c] for j in range(len(kx))) / t for c in range(len(v[0]))])
    return out
