"""Writes stay inside their outputs.  Each entry point writes into a view of a
larger device buffer filled with a sentinel byte: a guard region before and
after the view, and, where the API takes a row stride, padding columns at the
end of every row.  Every byte outside the logical output must still hold the
sentinel afterwards.  (No sanitizer runs on this pool; this catches stores
past a ragged edge, including the tensor-memory-accelerator stores of the
epilogues, on shapes whose last tiles are partial.)"""
import ctypes

import numpy as np
import pytest
import torch

from w8a8_int8_quantized_block_b200 import convrot as C
from w8a8_int8_quantized_block_b200 import workloads as W

pytestmark = pytest.mark.gpu
DEV = "cuda"
SENT = 0x5A
GUARD = 4096  # bytes before and after every view


def _guarded(nbytes: int):
    buf = torch.full((GUARD + nbytes + GUARD,), SENT, dtype=torch.uint8, device=DEV)
    return buf, buf[GUARD:GUARD + nbytes]


def _guards_intact(buf: torch.Tensor, nbytes: int, what: str):
    b = buf.cpu().numpy()
    assert (b[:GUARD] == SENT).all(), f"{what}: bytes written before the output"
    assert (b[GUARD + nbytes:] == SENT).all(), f"{what}: bytes written after the output"


def _strided_bf16(M: int, N: int, ldy: int):
    buf, body = _guarded(M * ldy * 2)
    y = body.view(torch.bfloat16).view(M, ldy)[:, :N]
    return buf, body, y


def _padding_intact(body: torch.Tensor, M: int, N: int, ldy: int, what: str):
    rows = body.cpu().numpy().reshape(M, ldy * 2)
    assert (rows[:, 2 * N:] == SENT).all(), f"{what}: bytes written into a row's padding"


@pytest.mark.parametrize("M,K,N,ldx_pad", [(300, 640, 264, 0), (300, 640, 264, 8), (7000, 512, 72, 0),
                                            (3500, 5376, 264, 0)])
def test_linear_fused_writes_stay_inside(M, K, N, ldx_pad):
    # ldx_pad 0: the one-kernel path, in a workspace of exactly its own size
    # (7000 and 3500 rows: its codes ring wraps, and the workspace is shorter
    # than a whole codes array); 8: the two-kernel path in the full size
    spec, (x, w, bias) = W.custom_linear(M, K, N, seed=M + ldx_pad, n_out=2)
    xp = torch.zeros(M, K + ldx_pad, dtype=torch.bfloat16)
    xp[:, :K] = x
    xd = xp.to(DEV)[:, :K]
    pw = C.pack_weight(w.to(DEV), 128)
    ldy = N + 24
    ybuf, ybody, y = _strided_bf16(M, N, ldy)
    nws = C.fused_workspace_bytes(M, K) if ldx_pad == 0 else C.workspace_bytes(M, K)
    wbuf, ws = _guarded(nws)
    C.linear_fused(xd, pw, bias.to(DEV), workspace=ws, out=y)
    torch.cuda.synchronize()
    assert C.last_device_status() == (C.OK, 0)
    _guards_intact(ybuf, M * ldy * 2, "linear_fused y")
    _padding_intact(ybody, M, N, ldy, "linear_fused y")
    _guards_intact(wbuf, nws, "linear_fused workspace")
    y_ref = C.linear_fused(xd, pw, bias.to(DEV))
    assert torch.equal(y.contiguous().view(torch.int16), y_ref.view(torch.int16))


def test_quantize_and_linear_writes_stay_inside():
    M, K, N = 129, 1024, 392
    spec, (x, w, bias) = W.custom_linear(M, K, N, seed=5, n_out=3)
    pw = C.pack_weight(w.to(DEV), 128)
    qbuf, qbody = _guarded(M * K)
    sbuf, sbody = _guarded(M * 4)
    q, s = C.quantize_act(x.to(DEV), 128, qbody.view(torch.int8).view(M, K), sbody.view(torch.float32))
    ldy = N + 8
    ybuf, ybody, y = _strided_bf16(M, N, ldy)
    C.w8a8_linear(q, s, pw, bias.to(DEV), out=y)
    torch.cuda.synchronize()
    assert C.last_device_status() == (C.OK, 0)
    _guards_intact(qbuf, M * K, "quantize_act codes")
    _guards_intact(sbuf, M * 4, "quantize_act scales")
    _guards_intact(ybuf, M * ldy * 2, "w8a8_linear y")
    _padding_intact(ybody, M, N, ldy, "w8a8_linear y")


def test_pack_weight_writes_stay_inside():
    N, K = 200, 768
    w = torch.randn(N, K, generator=torch.Generator().manual_seed(3)).to(DEV) * 0.02
    qbuf, qbody = _guarded(N * K)
    sbuf, sbody = _guarded(N * 4)
    d = C.WDesc()
    L = C.load()
    st = L.convrot_pack_weight(ctypes.c_void_p(w.data_ptr()), N, K, 128, ctypes.c_void_p(qbody.data_ptr()),
                               ctypes.c_void_p(sbody.data_ptr()), ctypes.byref(d), C._stream(None))
    assert st == C.OK
    torch.cuda.synchronize()
    _guards_intact(qbuf, N * K, "pack_weight codes")
    _guards_intact(sbuf, N * 4, "pack_weight scales")


def test_bmm_writes_stay_inside():
    B, M, N, K = 3, 200, 136, 128
    g = torch.Generator().manual_seed(9)
    qa = torch.randint(-127, 128, (B, M, K), generator=g, dtype=torch.int8).to(DEV)
    qb = torch.randint(-127, 128, (B, N, K), generator=g, dtype=torch.int8).to(DEV)
    sa = torch.rand(B, M, generator=g).to(DEV)
    sb = torch.rand(B, N, generator=g).to(DEV)
    ybuf, ybody = _guarded(B * M * N * 2)
    C.w8a8_bmm(qa, sa, qb, sb, out=ybody.view(torch.bfloat16).view(B, M, N))
    torch.cuda.synchronize()
    assert C.last_device_status() == (C.OK, 0)
    _guards_intact(ybuf, B * M * N * 2, "w8a8_bmm y")


@pytest.mark.parametrize("H,Lq,Lk", [(3, 384, 1024), (2, 256, 256)])
def test_attention_writes_stay_inside(H, Lq, Lk):
    # (3, 384, 1024): 6 units split 4 ways over their keys (parts + combine);
    # (2, 256, 256): whole units only
    g = torch.Generator().manual_seed(H + Lq)
    q = torch.randn(H, Lq, 128, generator=g).to(torch.bfloat16).to(DEV)
    k = torch.randn(H, Lk, 128, generator=g).to(torch.bfloat16).to(DEV)
    v = torch.randn(H, Lk, 128, generator=g).to(torch.bfloat16).to(DEV)
    nws = C.load().convrot_attention_workspace_bytes(H, Lq, Lk)
    wbuf, ws = _guarded(nws)
    obuf, obody = _guarded(H * Lq * 128 * 2)
    C.attention(q, k, v, workspace=ws, out=obody.view(torch.bfloat16).view(H, Lq, 128))
    torch.cuda.synchronize()
    assert C.last_device_status() == (C.OK, 0)
    _guards_intact(obuf, H * Lq * 128 * 2, "attention O")
    _guards_intact(wbuf, nws, "attention workspace")
