"""GPU parity of the down projection's activation prologue ("SwiGLU +
ConvRot64 + Rowwise INT8 Quantize" fused in MLP.fc2 -- MiniMax-H3-Rung-Omega
README, "Technical Architecture Overview", item 2): x = gelu(h) or
x = silu(g) * u from the up projection's bf16 output, then the rotation and
the rowwise quantiser.

The oracle computes each x in fp64 and rounds it once to f32; the kernel
evaluates it in f32 with CUDA's erfcf / expf and an IEEE division.  Its
relative error per element is a few ulp, plus what rounding the argument
does in a steep tail: erfc(t) at t = -h/sqrt 2 moves by 2 t |dt| relative,
about h^2 2^-24 for negative h; e^-g by |g| 2^-24 for negative g.  Everything
after x is the same f32 arithmetic in the same order, so a code may differ
only where that error in x (summed over the block, plus one rounding of the
perturbed partial sums per butterfly stage) can carry v = z * 127 / amax
across a rounding tie; the scale may move by the error of amax's block.
"""
import numpy as np
import pytest
import torch

from oracle import oracle as O
from w8a8_int8_quantized_block_b200 import convrot as C
from w8a8_int8_quantized_block_b200 import workloads as W

from helpers import assert_close_bf16, bits, f32_of_bf16

pytestmark = pytest.mark.gpu
DEV = "cuda"
ULPS = 8.0


def _h(M, K, act, seed):
    g = torch.Generator().manual_seed(seed)
    cols = 2 * K if act == C.ACT_SWIGLU else K
    h = torch.randn(M, cols, generator=g) * 1.5
    h[:, 3] *= 6  # an outlier channel
    h[0] = 0.0    # a zero row: s = 0, codes 0
    h[1, :] = -9.0  # deep in GELU's tail
    return h.to(torch.bfloat16)


def _oracle_kind(block):
    return C.block_length(block), bool(block & C.REGULAR)


def assert_prologue_codes(q, s, h, act, block):
    b, reg = _oracle_kind(block)
    hb = bits(h)
    qr, sr = O.act_quantize(hb, act, b, reg)
    x = O.act_f32(hb, act).astype(np.float64)
    M, K = x.shape
    bb = max(b, 1)
    hf = O.bf16_bits_to_f32(hb).astype(np.float64)
    if act == C.ACT_GELU:
        tail = np.where(hf < 0, hf * hf, 0.0)
    else:
        g = hf[:, :K]
        tail = np.where(g < 0, -g, 0.0)
    err = (ULPS * 2.0 ** -23 + tail * 2.0 ** -24) * np.abs(x)  # per-element bound on |dx|
    stages = int(np.log2(bb)) + 1
    blk = (err.reshape(M, K // bb, bb).sum(-1)
           + stages * 2.0 ** -24 * np.abs(x).reshape(M, K // bb, bb).sum(-1))  # bound on |dz| per block
    z = O.rotate_explicit_f64(x.astype(np.float32), b, reg)
    amax = np.abs(z).max(axis=1)
    amax_blk = blk[np.arange(M), np.abs(z).argmax(axis=1) // bb]
    s_tol = (amax_blk + 2.0 ** -22 * amax) / 127.0
    assert (np.abs(s.astype(np.float64) - sr.astype(np.float64)) <= s_tol + 1e-45).all()
    diff = q.astype(np.int16) - qr.astype(np.int16)
    assert np.abs(diff).max(initial=0) <= 1, "a code moved by more than one unit"
    bad = np.argwhere(diff != 0)
    for m, k in bad:
        v = z[m, k] * 127.0 / amax[m]
        room = 127.0 / amax[m] * (blk[m, k // bb] + amax_blk[m]) + abs(v) * 2.0 ** -22
        frac = abs(abs(v) - np.floor(abs(v)) - 0.5)
        assert frac <= room, f"code ({m},{k}) differs but v = {v} is {frac} from a tie (bound {room})"
    assert bad.shape[0] <= 1e-3 * q.size


@pytest.mark.parametrize("act", [C.ACT_GELU, C.ACT_SWIGLU], ids=["gelu", "swiglu"])
@pytest.mark.parametrize("block", [64, 128, C.REGULAR | 256, 0], ids=["syl64", "syl128", "reg256", "none"])
@pytest.mark.parametrize("M,K", [(37, 1024), (130, 5376)])
def test_act_quantize_matches_oracle(act, block, M, K):
    h = _h(M, K, act, seed=M + K + act)
    q, s = C.act_quantize(h.to(DEV), act, block)
    torch.cuda.synchronize()
    assert C.last_device_status() == (C.OK, 0)
    q, s = q.cpu().numpy(), s.cpu().numpy()
    assert s[0] == 0.0 and not q[0].any()
    assert_prologue_codes(q, s, h, act, block)


@pytest.mark.parametrize("act", [C.ACT_GELU, C.ACT_SWIGLU], ids=["gelu", "swiglu"])
def test_act_quantize_long_rows(act):
    # the MLP's down projection width: 21504 (several boxes per row)
    h = _h(40, 21504, act, seed=7 + act)
    q, s = C.act_quantize(h.to(DEV), act, 128)
    torch.cuda.synchronize()
    assert C.last_device_status() == (C.OK, 0)
    assert_prologue_codes(q.cpu().numpy(), s.cpu().numpy(), h, act, 128)


def test_act_quantize_strided_swiglu_rows():
    # h with a row stride wider than 2K (a slice of a bigger buffer)
    M, K = 50, 2048
    hfull = _h(M, K + 64, C.ACT_SWIGLU, seed=11)
    g, u = hfull[:, :K], hfull[:, K + 64:2 * K + 64]
    h = torch.cat([g, u], dim=1)
    big = torch.zeros(M, 2 * K + 256, dtype=torch.bfloat16)
    big[:, :2 * K] = h
    q, s = C.act_quantize(big.to(DEV)[:, :2 * K], C.ACT_SWIGLU, 64)
    torch.cuda.synchronize()
    assert_prologue_codes(q.cpu().numpy(), s.cpu().numpy(), h, C.ACT_SWIGLU, 64)


@pytest.mark.parametrize("act", [C.ACT_GELU, C.ACT_SWIGLU], ids=["gelu", "swiglu"])
def test_down_projection_with_prologue_matches_oracle(act):
    M, K, N = 300, 1536, 520
    h = _h(M, K, act, seed=21 + act)
    w = torch.randn(N, K, generator=torch.Generator().manual_seed(5)) * 0.02
    bias = torch.randn(N, generator=torch.Generator().manual_seed(6)) * 0.01
    pw = C.pack_weight(w.to(DEV), 64)
    ws = C.alloc_workspace(M, K)
    y = C.linear_act(h.to(DEV), act, pw, bias.to(DEV), workspace=ws)
    torch.cuda.synchronize()
    assert C.last_device_status() == (C.OK, 0)
    qr, sr = O.act_quantize(bits(h), act, 64)
    qw, sw = O.pack_weight(w.numpy(), 64)
    yr = O.dequant(O.igemm(qr, qw), sr, sw, bias.numpy(), 64)
    assert_close_bf16(f32_of_bf16(y), yr, "down projection with prologue")
    qx = ws[:M * K].view(torch.int8).view(M, K).cpu().numpy()
    off = (M * K + 255) // 256 * 256
    sx = ws[off:off + 4 * M].view(torch.float32).cpu().numpy()
    assert_prologue_codes(qx, sx, h, act, 64)


def test_gelu_prologue_equals_gelu_epilogue_route_on_the_mlp():
    # Two routes through an MLP's middle: GELU in the up projection's epilogue
    # then the plain quantiser, or the plain up projection then the GELU
    # prologue.  They round differently (bf16 after GELU vs bf16 before it),
    # so the down projection's outputs agree to the bf16 tolerance only.
    spec = W.MLP_768P
    M, K, H = 512, spec.K, spec.H
    x, w1, w2 = W.mlp_inputs(spec, M=M)
    p1 = C.pack_weight(w1.to(DEV), 128)
    p2 = C.pack_weight(w2.to(DEV), 128)
    xd = x.to(DEV)
    y_epi = C.linear_fused(C.linear_fused(xd, p1, gelu=True), p2)
    h = C.linear_fused(xd, p1)
    y_pro = C.linear_act(h, C.ACT_GELU, p2)
    torch.cuda.synchronize()
    a, b = y_epi.float().cpu().numpy().ravel(), y_pro.float().cpu().numpy().ravel()
    assert np.linalg.norm(a - b) / np.linalg.norm(a) < 1e-2
