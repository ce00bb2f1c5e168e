"""Thin ctypes binding over ``libconvrot.so`` (include/convrot.h).

Argument marshalling only: every step of the path runs in the library's
sm_100a kernels.  Tensors are torch CUDA tensors (torch supplies device memory
and streams); outputs are allocated here when not given.  There is no CPU
fallback: if the library cannot be loaded, every call raises.
"""
from __future__ import annotations

import ctypes
import os
from dataclasses import dataclass

import torch

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "libconvrot.so")

OK, EINVAL, EUNSUPPORTED, ELAYOUT, ECUDA, ETIMEOUT, ETOOLARGE = range(7)
EPI_NONE, EPI_GELU = 0, 1
WDESC_MAGIC = 0x52564E43
WDESC_VERSION = 1
LAYOUT_OUTPUT_MAJOR = 1
# Block values: 0 = no rotation, 64/128/256 = Sylvester H_b, REGULAR | 16/64/256
# = the regular H_4^(x)k (H_4 = J - 2I).
REGULAR = 0x10000
BLOCKS = (0, 64, 128, 256, REGULAR | 16, REGULAR | 64, REGULAR | 256)
# Activation prologues of a down projection (convrot_act_quantize).
ACT_NONE, ACT_GELU, ACT_SWIGLU = 0, 1, 2


def block_length(block: int) -> int:
    """b of a block value (1 for no rotation)."""
    n = block & ~REGULAR
    return n if n > 1 else 1

# Every symbol include/convrot.h declares.
EXPORTS = (
    "convrot_status_string", "convrot_abi_version", "convrot_pack_weight", "convrot_quantize_act",
    "convrot_w8a8_linear", "convrot_workspace_bytes", "convrot_linear_fused", "convrot_linear_fused_host",
    "convrot_w8a8_bmm", "convrot_igemm_s32", "convrot_last_device_status", "convrot_set_wait_limit_ns",
    "convrot_selftest_wait_timeout", "convrot_linear_fused_noalloc", "convrot_act_quantize", "convrot_linear_act",
    "convrot_attention_workspace_bytes", "convrot_attention", "convrot_attention_split_bytes",
    "convrot_attention_int8", "convrot_fused_workspace_bytes",
)


class ConvrotError(RuntimeError):
    def __init__(self, fn: str, status: int, msg: str):
        super().__init__(f"{fn}: {msg} (status {status})")
        self.status = status


class WDesc(ctypes.Structure):
    _fields_ = [("magic", ctypes.c_uint32), ("version", ctypes.c_uint32), ("layout", ctypes.c_uint32),
                ("block", ctypes.c_int32), ("N", ctypes.c_int64), ("K", ctypes.c_int64)]


_lib = None


def load(path: str | None = None) -> ctypes.CDLL:
    """Load (building first if it is missing or stale) the CUDA library."""
    global _lib
    if _lib is not None:
        return _lib
    p = path or LIB_PATH
    if path is None:
        from . import build as _build
        try:
            _build.build()
        except OSError as e:  # no nvcc here: only an existing library will do
            if not os.path.exists(p):
                raise RuntimeError(f"libconvrot.so is missing and could not be built: {e}") from e
        # (a failed compile or link raises: a library older than its sources is never used)
    if not os.path.exists(p):
        raise RuntimeError(f"libconvrot.so not found at {p}; run `python -m w8a8_int8_quantized_block_b200.build`")
    L = ctypes.CDLL(p)
    P, I64, I32, U64 = ctypes.c_void_p, ctypes.c_int64, ctypes.c_int32, ctypes.c_uint64
    sig = {
        "convrot_status_string": ([ctypes.c_int], ctypes.c_char_p),
        "convrot_abi_version": ([], ctypes.c_int),
        "convrot_pack_weight": ([P, I64, I64, I32, P, P, ctypes.POINTER(WDesc), P], ctypes.c_int),
        "convrot_quantize_act": ([P, I64, I64, I64, I32, P, P, P], ctypes.c_int),
        "convrot_w8a8_linear": ([P, P, P, P, ctypes.POINTER(WDesc), P, I32, I64, P, I64, P], ctypes.c_int),
        "convrot_workspace_bytes": ([I64, I64], ctypes.c_size_t),
        "convrot_fused_workspace_bytes": ([I64, I64], ctypes.c_size_t),
        "convrot_linear_fused": ([P, I64, I64, P, P, ctypes.POINTER(WDesc), P, I32, P, ctypes.c_size_t, P, I64, P],
                                 ctypes.c_int),
        "convrot_linear_fused_host": ([P, I64, P, P, ctypes.POINTER(WDesc), P, I32, P, P, ctypes.c_size_t, P, P, P],
                                      ctypes.c_int),
        "convrot_w8a8_bmm": ([P, P, P, P, I64, I64, I64, I64, P, P], ctypes.c_int),
        "convrot_igemm_s32": ([P, P, I64, I64, I64, I64, P, P], ctypes.c_int),
        "convrot_last_device_status": ([P, ctypes.POINTER(ctypes.c_uint32)], ctypes.c_int),
        "convrot_set_wait_limit_ns": ([U64], None),
        "convrot_selftest_wait_timeout": ([U64, P], ctypes.c_int),
        "convrot_linear_fused_noalloc": ([P, I64, I64, P, P, ctypes.POINTER(WDesc), P, I32, P, I64, P],
                                         ctypes.c_int),
        "convrot_act_quantize": ([P, I64, I64, I64, I32, I32, P, P, P], ctypes.c_int),
        "convrot_attention_workspace_bytes": ([I64, I64, I64], ctypes.c_size_t),
        "convrot_attention": ([P, P, P, I64, I64, I64, ctypes.c_float, P, ctypes.c_size_t, P, P], ctypes.c_int),
        "convrot_attention_split_bytes": ([I64, I64, I64], ctypes.c_size_t),
        "convrot_attention_int8": ([P, P, P, P, P, I64, I64, I64, ctypes.c_float, P, ctypes.c_size_t, P, P],
                                   ctypes.c_int),
        "convrot_linear_act": ([P, I64, I64, I32, P, P, ctypes.POINTER(WDesc), P, I32, P, ctypes.c_size_t, P, I64,
                                P], ctypes.c_int),
    }
    for name, (args, res) in sig.items():
        f = getattr(L, name)
        f.argtypes = args
        f.restype = res
    _lib = L
    return L


def _check(fn: str, st: int):
    if st != OK:
        raise ConvrotError(fn, st, load().convrot_status_string(st).decode())


def _ptr(t: torch.Tensor | None):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(stream=None):
    s = stream if stream is not None else torch.cuda.current_stream()
    return ctypes.c_void_p(s.cuda_stream)


def _need(t: torch.Tensor, dtype, name: str, cuda: bool = True):
    if t.dtype != dtype:
        raise TypeError(f"{name} must be {dtype}, got {t.dtype}")
    if cuda and not t.is_cuda:
        raise TypeError(f"{name} must be a CUDA tensor")


@dataclass
class PackedWeight:
    """Offline-packed weights: int8 codes [N, K], f32 scales [N], descriptor."""
    q: torch.Tensor
    s: torch.Tensor
    desc: WDesc

    @property
    def N(self) -> int:
        return int(self.desc.N)

    @property
    def K(self) -> int:
        return int(self.desc.K)

    @property
    def block(self) -> int:
        return int(self.desc.block)


def pack_weight(w: torch.Tensor, block: int = 128, stream=None) -> PackedWeight:
    _need(w, torch.float32, "w")
    w = w.contiguous()
    N, K = w.shape
    q = torch.empty((N, K), dtype=torch.int8, device=w.device)
    s = torch.empty((N,), dtype=torch.float32, device=w.device)
    d = WDesc()
    _check("convrot_pack_weight", load().convrot_pack_weight(_ptr(w), N, K, block, _ptr(q), _ptr(s),
                                                             ctypes.byref(d), _stream(stream)))
    return PackedWeight(q, s, d)


def quantize_act(x: torch.Tensor, block: int = 128, q: torch.Tensor | None = None, s: torch.Tensor | None = None,
                 stream=None):
    _need(x, torch.bfloat16, "x")
    if x.dim() != 2 or x.stride(1) != 1:
        raise ValueError("x must be 2-D with unit column stride")
    M, K = x.shape
    q = torch.empty((M, K), dtype=torch.int8, device=x.device) if q is None else q
    s = torch.empty((M,), dtype=torch.float32, device=x.device) if s is None else s
    _check("convrot_quantize_act", load().convrot_quantize_act(_ptr(x), M, K, x.stride(0), block, _ptr(q), _ptr(s),
                                                               _stream(stream)))
    return q, s


def _act_width(h: torch.Tensor, act: int) -> int:
    if h.dim() != 2 or h.stride(1) != 1:
        raise ValueError("h must be 2-D with unit column stride")
    if act == ACT_SWIGLU:
        if h.shape[1] % 2:
            raise ValueError("a SwiGLU input holds gate and up halves: an even number of columns")
        return h.shape[1] // 2
    return h.shape[1]


def act_quantize(h: torch.Tensor, act: int, block: int = 128, q: torch.Tensor | None = None,
                 s: torch.Tensor | None = None, stream=None):
    """The down projection's input: rotate + quantise act(h) (ACT_GELU on
    h [M, K], or ACT_SWIGLU on h [M, 2K] = [gate | up]) -> (q [M, K], s [M])."""
    _need(h, torch.bfloat16, "h")
    K = _act_width(h, act)
    M = h.shape[0]
    q = torch.empty((M, K), dtype=torch.int8, device=h.device) if q is None else q
    s = torch.empty((M,), dtype=torch.float32, device=h.device) if s is None else s
    _check("convrot_act_quantize", load().convrot_act_quantize(_ptr(h), M, K, h.stride(0), act, block, _ptr(q),
                                                               _ptr(s), _stream(stream)))
    return q, s


def linear_act(h: torch.Tensor, act: int, pw: PackedWeight, bias: torch.Tensor | None = None, gelu: bool = False,
               workspace: torch.Tensor | None = None, out: torch.Tensor | None = None, stream=None) -> torch.Tensor:
    """Down projection with the activation prologue: y = act(h) W^T (+ bias)."""
    _need(h, torch.bfloat16, "h")
    K = _act_width(h, act)
    if K != pw.K:
        raise ValueError(f"act(h) has {K} columns, the weights {pw.K}")
    M = h.shape[0]
    ws = alloc_workspace(M, pw.K, h.device) if workspace is None else workspace
    y = torch.empty((M, pw.N), dtype=torch.bfloat16, device=h.device) if out is None else out
    _check("convrot_linear_act", load().convrot_linear_act(
        _ptr(h), M, h.stride(0), act, _ptr(pw.q), _ptr(pw.s), ctypes.byref(pw.desc), _ptr(bias),
        EPI_GELU if gelu else EPI_NONE, _ptr(ws), ws.numel(), _ptr(y), y.stride(0), _stream(stream)))
    return y


def attention(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, scale: float | None = None,
              workspace: torch.Tensor | None = None, out: torch.Tensor | None = None, stream=None) -> torch.Tensor:
    """int8 attention: q [H, Lq, 128], k and v [H, Lk, 128] bf16 -> O [H, Lq, 128]
    bf16 (scale defaults to 1/sqrt(128))."""
    for t, n in ((q, "q"), (k, "k"), (v, "v")):
        _need(t, torch.bfloat16, n)
    H, Lq, d = q.shape
    Lk = k.shape[1]
    if d != 128 or tuple(k.shape) != (H, Lk, d) or tuple(v.shape) != (H, Lk, d):
        raise ValueError("q [H, Lq, 128], k and v [H, Lk, 128]")
    q, k, v = q.contiguous(), k.contiguous(), v.contiguous()
    L = load()
    if workspace is None:
        workspace = torch.empty((L.convrot_attention_workspace_bytes(H, Lq, Lk),), dtype=torch.uint8, device=q.device)
    o = torch.empty((H, Lq, d), dtype=torch.bfloat16, device=q.device) if out is None else out
    _check("convrot_attention", L.convrot_attention(_ptr(q), _ptr(k), _ptr(v), H, Lq, Lk,
                                                    (d ** -0.5) if scale is None else scale, _ptr(workspace),
                                                    workspace.numel(), _ptr(o), _stream(stream)))
    return o


def attention_split_bytes(H: int, Lq: int, Lk: int) -> int:
    """Bytes of the buffer that lets attention_int8 split the last wave's units
    over their keys on the current device (0: nothing to split)."""
    return int(load().convrot_attention_split_bytes(H, Lq, Lk))


def attention_int8(qx, sq, kx, sk, vt, scale: float | None = None, out: torch.Tensor | None = None,
                   stream=None, split_ws: torch.Tensor | None = None) -> torch.Tensor:
    """The attention kernel on quantised inputs: qx [H, Lq, 128] int8, sq [H, Lq],
    kx [H, Lk, 128] int8, sk [H, Lk], vt = V^T [H, 128, Lk] bf16.  split_ws
    (attention_split_bytes bytes, optional) lets the last wave's units run
    split over their keys."""
    H, Lq, d = qx.shape
    Lk = kx.shape[1]
    o = torch.empty((H, Lq, d), dtype=torch.bfloat16, device=qx.device) if out is None else out
    _check("convrot_attention_int8", load().convrot_attention_int8(
        _ptr(qx), _ptr(sq), _ptr(kx), _ptr(sk), _ptr(vt), H, Lq, Lk, (d ** -0.5) if scale is None else scale,
        _ptr(split_ws), 0 if split_ws is None else split_ws.numel() * split_ws.element_size(), _ptr(o),
        _stream(stream)))
    return o


def w8a8_linear(qx: torch.Tensor, sx: torch.Tensor, pw: PackedWeight, bias: torch.Tensor | None = None,
                gelu: bool = False, out: torch.Tensor | None = None, stream=None) -> torch.Tensor:
    _need(qx, torch.int8, "qx")
    M = qx.shape[0]
    y = torch.empty((M, pw.N), dtype=torch.bfloat16, device=qx.device) if out is None else out
    _check("convrot_w8a8_linear", load().convrot_w8a8_linear(
        _ptr(qx.contiguous()), _ptr(sx), _ptr(pw.q), _ptr(pw.s), ctypes.byref(pw.desc), _ptr(bias),
        EPI_GELU if gelu else EPI_NONE, M, _ptr(y), y.stride(0), _stream(stream)))
    return y


def workspace_bytes(M: int, K: int) -> int:
    """Workspace bytes for either path of linear_fused (the whole codes array)."""
    return int(load().convrot_workspace_bytes(M, K))


def fused_workspace_bytes(M: int, K: int) -> int:
    """Workspace bytes for linear_fused's one-kernel path (its codes ring)."""
    return int(load().convrot_fused_workspace_bytes(M, K))


def alloc_workspace(M: int, K: int, device=None, one_kernel_only: bool = False) -> torch.Tensor:
    """Caller-owned workspace for linear_fused (torch allocations are 512-byte
    aligned); one_kernel_only: just the one-kernel path's size."""
    n = fused_workspace_bytes(M, K) if one_kernel_only else workspace_bytes(M, K)
    return torch.empty((n,), dtype=torch.uint8, device=device or "cuda")


def _r256(n: int) -> int:
    return (n + 255) // 256 * 256


def workspace_scales(ws: torch.Tensor, M: int) -> torch.Tensor:
    """The f32 [M] scales region of a linear workspace (it comes first)."""
    return ws[:4 * M].view(torch.float32)


def workspace_codes(ws: torch.Tensor, M: int, K: int, rows: int | None = None) -> torch.Tensor:
    """The int8 codes region of a linear workspace as [rows, K] (default M
    rows: the two-kernel path's whole array; the one-kernel path's ring holds
    fewer).  It follows the scales and the one-kernel path's counters."""
    panels = (M + 255) // 256
    off = _r256(4 * M) + _r256(4 * (2 * panels + 1))
    rows = M if rows is None else rows
    return ws[off:off + rows * K].view(torch.int8).view(rows, K)


def linear_fused(x: torch.Tensor, pw: PackedWeight, bias: torch.Tensor | None = None, gelu: bool = False,
                 workspace: torch.Tensor | None = None, out: torch.Tensor | None = None, stream=None) -> torch.Tensor:
    _need(x, torch.bfloat16, "x")
    if x.dim() != 2 or x.stride(1) != 1:
        raise ValueError("x must be 2-D with unit column stride")
    M = x.shape[0]
    ws = alloc_workspace(M, pw.K, x.device) if workspace is None else workspace
    y = torch.empty((M, pw.N), dtype=torch.bfloat16, device=x.device) if out is None else out
    _check("convrot_linear_fused", load().convrot_linear_fused(
        _ptr(x), M, x.stride(0), _ptr(pw.q), _ptr(pw.s), ctypes.byref(pw.desc), _ptr(bias),
        EPI_GELU if gelu else EPI_NONE, _ptr(ws), ws.numel(), _ptr(y), y.stride(0), _stream(stream)))
    return y


def linear_fused_noalloc(x: torch.Tensor, pw: PackedWeight, bias: torch.Tensor | None = None, gelu: bool = False,
                         out: torch.Tensor | None = None, stream=None) -> torch.Tensor:
    """The fused linear without a workspace, for callers that cannot allocate
    device scratch (the codes and scales go to the library's fixed 32 MiB
    array; the output tensor is still the caller's).  Raises ConvrotError with
    status ETOOLARGE beyond that size.  Calls that overlap on the GPU race."""
    _need(x, torch.bfloat16, "x")
    if x.dim() != 2 or x.stride(1) != 1:
        raise ValueError("x must be 2-D with unit column stride")
    M = x.shape[0]
    y = torch.empty((M, pw.N), dtype=torch.bfloat16, device=x.device) if out is None else out
    _check("convrot_linear_fused_noalloc", load().convrot_linear_fused_noalloc(
        _ptr(x), M, x.stride(0), _ptr(pw.q), _ptr(pw.s), ctypes.byref(pw.desc), _ptr(bias),
        EPI_GELU if gelu else EPI_NONE, _ptr(y), y.stride(0), _stream(stream)))
    return y


def linear_fused_host(x_host: torch.Tensor, pw: PackedWeight, bias, gelu: bool, x_dev: torch.Tensor,
                      workspace: torch.Tensor, y_dev: torch.Tensor, y_host: torch.Tensor, stream=None) -> None:
    """Host bf16 activations in, host bf16 outputs out (copies enqueued on `stream`)."""
    _need(x_host, torch.bfloat16, "x_host", cuda=False)
    _need(y_host, torch.bfloat16, "y_host", cuda=False)
    M = x_host.shape[0]
    _check("convrot_linear_fused_host", load().convrot_linear_fused_host(
        _ptr(x_host), M, _ptr(pw.q), _ptr(pw.s), ctypes.byref(pw.desc), _ptr(bias), EPI_GELU if gelu else EPI_NONE,
        _ptr(x_dev), _ptr(workspace), workspace.numel(), _ptr(y_dev), _ptr(y_host), _stream(stream)))


def w8a8_bmm(qa: torch.Tensor, sa: torch.Tensor, qb: torch.Tensor, sb: torch.Tensor,
             out: torch.Tensor | None = None, stream=None) -> torch.Tensor:
    _need(qa, torch.int8, "qa")
    _need(qb, torch.int8, "qb")
    B, M, K = qa.shape
    N = qb.shape[1]
    y = torch.empty((B, M, N), dtype=torch.bfloat16, device=qa.device) if out is None else out
    _check("convrot_w8a8_bmm", load().convrot_w8a8_bmm(_ptr(qa), _ptr(sa), _ptr(qb), _ptr(sb), B, M, N, K, _ptr(y),
                                                       _stream(stream)))
    return y


def igemm_s32(qa: torch.Tensor, qb: torch.Tensor, stream=None) -> torch.Tensor:
    """Raw int32 accumulators (test hook); qa [B, M, K] or [M, K], qb likewise."""
    _need(qa, torch.int8, "qa")
    _need(qb, torch.int8, "qb")
    squeeze = qa.dim() == 2
    a = qa.unsqueeze(0) if squeeze else qa
    b = qb.unsqueeze(0) if squeeze else qb
    B, M, K = a.shape
    N = b.shape[1]
    acc = torch.empty((B, M, N), dtype=torch.int32, device=qa.device)
    _check("convrot_igemm_s32", load().convrot_igemm_s32(_ptr(a.contiguous()), _ptr(b.contiguous()), B, M, N, K,
                                                         _ptr(acc), _stream(stream)))
    return acc[0] if squeeze else acc


def last_device_status(stream=None):
    code = ctypes.c_uint32(0)
    st = load().convrot_last_device_status(_stream(stream), ctypes.byref(code))
    return st, code.value


def set_wait_limit_ns(ns: int) -> None:
    load().convrot_set_wait_limit_ns(ns)


def selftest_wait_timeout(limit_ns: int, stream=None) -> None:
    _check("convrot_selftest_wait_timeout", load().convrot_selftest_wait_timeout(limit_ns, _stream(stream)))
