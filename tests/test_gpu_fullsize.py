"""GPU parity at the workloads' full sizes, in the launch configuration the
benchmark times (the fused entry point, one call per batch).

Codes and scales are compared for every row (the oracle's quantiser is cheap);
outputs are compared on sampled rows and on random (row, column) pairs whose
dot products the oracle computes one by one.
"""
import numpy as np
import pytest
import torch

from oracle import oracle as O
from w8a8_int8_quantized_block_b200 import convrot as C
from w8a8_int8_quantized_block_b200 import workloads as W

from helpers import assert_close_bf16, assert_codes_match, bits, f32_of_bf16

pytestmark = pytest.mark.gpu
RING = 12  # panel slots of the one-kernel linear's codes ring (kFusedRingPanels)


def _sample(M, N, rows, pairs, seed):
    rng = np.random.default_rng(seed)
    r = np.unique(np.concatenate([[0, M - 1], rng.choice(M, rows, replace=False)]))
    mi = rng.integers(0, M, pairs).astype(np.int64)
    ni = rng.integers(0, N, pairs).astype(np.int64)
    return r.astype(np.int64), mi, ni


def _check_outputs(y_gpu, qx, sx, qw, sw, bias, block, rows, mi, ni, gelu=False, what=""):
    """Sampled whole rows and random pairs of y against the oracle's fp64 dequant."""
    accr = O.igemm(qx[rows], qw)
    yr = O.dequant(accr, sx[rows], sw, bias, block, gelu)
    assert_close_bf16(f32_of_bf16(y_gpu[torch.from_numpy(rows).to(y_gpu.device)]), yr, f"{what} rows")
    accp = O.igemm_pairs(qx, qw, mi, ni)
    yp = O.dequant_pairs(accp, mi, ni, sx, sw, bias, block, gelu)
    yg = f32_of_bf16(y_gpu[torch.from_numpy(mi).to(y_gpu.device), torch.from_numpy(ni).to(y_gpu.device)])
    assert_close_bf16(yg, yp, f"{what} pairs")


def test_proj_768p_full_size():
    spec = W.PROJ_768P
    x, w, bias = W.linear_inputs(spec)
    pw = C.pack_weight(w.cuda(), spec.block)
    xd = x.cuda()
    # the one-kernel path's own workspace size: scales, counters, then the
    # codes ring (about 17 MB, not the 208 MB of a whole codes array)
    ws = C.alloc_workspace(spec.M, spec.K, one_kernel_only=True)
    assert ws.numel() < 20 << 20
    y = C.linear_fused(xd, pw, bias.cuda(), workspace=ws)
    torch.cuda.synchronize()
    assert C.last_device_status() == (C.OK, 0)
    # The one-kernel path keeps the codes of RING row panels of 256 at a time
    # (panel p in slot p % RING), so after the call the slots hold the last
    # RING panels; every row's scale is there.
    sx = C.workspace_scales(ws, spec.M).cpu().numpy()
    xb = bits(x)
    qxr, sxr = O.quantize_act(xb, spec.block)
    ring = C.workspace_codes(ws, spec.M, spec.K, rows=RING * 256).cpu().numpy()
    panels = (spec.M + 255) // 256
    qx = np.zeros_like(qxr)
    held = np.zeros(spec.M, dtype=bool)
    for p in range(panels - RING, panels):
        r0, r1 = p * 256, min(spec.M, (p + 1) * 256)
        qx[r0:r1] = ring[(p % RING) * 256:(p % RING) * 256 + (r1 - r0)]
        held[r0:r1] = True
    assert_codes_match(qx[held], sx[held], qxr[held], sxr[held], None, spec.block)
    bad = np.nonzero(sx.view(np.uint32) != sxr.view(np.uint32))[0]
    assert bad.size == 0, f"{bad.size} scales differ"
    # every row's codes: the standalone quantiser (the same arithmetic; the
    # fused and two-kernel outputs are compared bit for bit in test_gpu_parity)
    q2, s2 = C.quantize_act(xd, spec.block)
    torch.cuda.synchronize()
    assert_codes_match(q2.cpu().numpy(), s2.cpu().numpy(), qxr, sxr, None, spec.block)
    qwr, swr = O.pack_weight(w.numpy(), spec.block)
    assert_codes_match(pw.q.cpu().numpy(), pw.s.cpu().numpy(), qwr, swr)
    rows, mi, ni = _sample(spec.M, spec.N, 48, 8192, 1)
    _check_outputs(y, qxr, sxr, qwr, swr, bias.numpy(), spec.block, rows, mi, ni, what="768p")


def test_proj_768p_one_kernel_equals_two_kernels_bitwise():
    # At 768p the one-kernel path's codes ring (12 panel slots for 151 panels)
    # turns over 12 times; its output must equal the two-kernel path's
    # (standalone quantiser into a full [M][K] array, then the GEMM) bit for bit.
    spec = W.PROJ_768P
    x, w, bias = W.linear_inputs(spec)
    pw = C.pack_weight(w.cuda(), spec.block)
    xd, bd = x.cuda(), bias.cuda()
    y1 = C.linear_fused(xd, pw, bd)
    q, s = C.quantize_act(xd, spec.block)
    y2 = C.w8a8_linear(q, s, pw, bd)
    torch.cuda.synchronize()
    assert C.last_device_status() == (C.OK, 0)
    differ = (y1.view(torch.int16) != y2.view(torch.int16)).sum().item()
    assert differ == 0, f"{differ} of {y1.numel()} outputs differ"


def test_proj_4k_full_size():
    spec = W.PROJ_4K
    x, w, bias = W.linear_inputs(spec)
    pw = C.pack_weight(w.cuda(), spec.block)
    y = C.linear_fused(x.cuda(), pw, bias.cuda())
    q, s = C.quantize_act(x.cuda(), spec.block)
    torch.cuda.synchronize()
    qxr, sxr = O.quantize_act(bits(x), spec.block)
    assert_codes_match(q.cpu().numpy(), s.cpu().numpy(), qxr, sxr, None, spec.block)
    qwr, swr = O.pack_weight(w.numpy(), spec.block)
    rows, mi, ni = _sample(spec.M, spec.N, 64, 8192, 2)
    _check_outputs(y, qxr, sxr, qwr, swr, bias.numpy(), spec.block, rows, mi, ni, what="4k")


def test_mlp_pair_full_size_stagewise():
    # Layer 2 is checked stage-wise: the oracle's quantiser is fed the GPU's own
    # bf16 GELU output, so layer-2 codes stay comparable bit for bit (the pages'
    # own check feeds each block the same input).
    spec = W.MLP_768P
    x, w_up, w_down = W.mlp_inputs(spec)
    pw1 = C.pack_weight(w_up.cuda(), spec.block)
    pw2 = C.pack_weight(w_down.cuda(), spec.block)
    h = C.linear_fused(x.cuda(), pw1, None, gelu=True)
    q2, s2 = C.quantize_act(h, spec.block)
    y = C.linear_fused(h, pw2, None)
    torch.cuda.synchronize()
    assert C.last_device_status() == (C.OK, 0)
    qxr, sxr = O.quantize_act(bits(x), spec.block)
    q1w, s1w = O.pack_weight(w_up.numpy(), spec.block)
    assert_codes_match(pw1.q.cpu().numpy(), pw1.s.cpu().numpy(), q1w, s1w)
    rows, mi, ni = _sample(spec.M, spec.H, 16, 4096, 3)
    _check_outputs(h, qxr, sxr, q1w, s1w, None, spec.block, rows, mi, ni, gelu=True, what="mlp up+gelu")
    hb = bits(h)
    del h
    q2r, s2r = O.quantize_act(hb, spec.block)
    assert_codes_match(q2.cpu().numpy(), s2.cpu().numpy(), q2r, s2r, None, spec.block)
    q2w, s2w = O.pack_weight(w_down.numpy(), spec.block)
    rows, mi, ni = _sample(spec.M, spec.K, 16, 4096, 4)
    _check_outputs(y, q2r, s2r, q2w, s2w, None, spec.block, rows, mi, ni, what="mlp down")


def test_qk_bmm_full_size():
    spec = W.QK_BMM
    q, k = W.bmm_inputs(spec)
    B, M, K = q.shape
    N = k.shape[1]
    qa, sa = C.quantize_act(q.cuda().view(B * M, K), 0)
    qb, sb = C.quantize_act(k.cuda().view(B * N, K), 0)
    y = C.w8a8_bmm(qa.view(B, M, K), sa, qb.view(B, N, K), sb)
    torch.cuda.synchronize()
    assert C.last_device_status() == (C.OK, 0)
    qar, sar = O.quantize_act(bits(q.view(B * M, K)), 0)
    qbr, sbr = O.quantize_act(bits(k.view(B * N, K)), 0)
    assert_codes_match(qa.cpu().numpy(), sa.cpu().numpy(), qar, sar)
    assert_codes_match(qb.cpu().numpy(), sb.cpu().numpy(), qbr, sbr)
    rng = np.random.default_rng(5)
    bi = rng.integers(0, B, 16384)
    mi = rng.integers(0, M, 16384)
    ni = rng.integers(0, N, 16384)
    acc = O.igemm_pairs(qar, qbr, bi * M + mi, bi * N + ni)
    yr = O.dequant_pairs(acc, bi * M + mi, bi * N + ni, sar, sbr, None, 0)
    yg = f32_of_bf16(y[torch.from_numpy(bi).cuda(), torch.from_numpy(mi).cuda(), torch.from_numpy(ni).cuda()])
    assert_close_bf16(yg, yr, "qk pairs")
    # one whole head, every element
    b = int(rng.integers(0, B))
    accb = O.igemm(qar[b * M:(b + 1) * M][:512], qbr[b * N:(b + 1) * N])
    yrb = O.dequant(accb, sar[b * M:(b + 1) * M][:512], sbr[b * N:(b + 1) * N], None, 0)
    assert_close_bf16(f32_of_bf16(y[b, :512]), yrb, "qk head rows")
