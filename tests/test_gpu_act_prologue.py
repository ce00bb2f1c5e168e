"""GPU parity of the down projection's activation prologue ("SwiGLU +
ConvRot64 + Rowwise INT8 Quantize" fused in MLP.fc2 -- MiniMax-H3-Rung-Omega
README, "Technical Architecture Overview", item 2): x = gelu(h) or
x = silu(g) * u from the up projection's bf16 output, then the rotation and
the rowwise quantiser.

Both sides evaluate each x in double precision and round it once to f32 (the
kernel with CUDA's double erfc / exp, the oracle with the C library's), then
run the same f32 rotation and quantiser.  So the bar is the one every other
quantiser meets: scales bit-exact, codes bit-exact except at most one unit on
at most 1e-4 of them, and only where the exact pre-rounding value lies within
1e-6 of a .5 tie (helpers.assert_codes_match).
"""
import numpy as np
import pytest
import torch

from oracle import oracle as O
from w8a8_int8_quantized_block_b200 import convrot as C
from w8a8_int8_quantized_block_b200 import workloads as W

from helpers import assert_close_bf16, assert_codes_match, bits, f32_of_bf16

pytestmark = pytest.mark.gpu
DEV = "cuda"


def _h(M, K, act, seed):
    g = torch.Generator().manual_seed(seed)
    cols = 2 * K if act == C.ACT_SWIGLU else K
    h = torch.randn(M, cols, generator=g) * 1.5
    h[:, 3] *= 6  # an outlier channel
    h[0] = 0.0    # a zero row: s = 0, codes 0
    h[1, :] = -9.0  # deep in GELU's tail
    if M > 2:
        # inputs outside the kernel's tables of common values (tiny, huge, the
        # edges of each range, zero), which it evaluates directly
        odd = torch.tensor([1e-9, -3e-7, 9.5e-7, -9.6e-7, 1.5e-5, -1.6e-5, 255.0, -257.0, 4095.0, -4097.0,
                            5000.0, -7000.0, 300.0, -1e4, 0.0, 2.0e-38])
        h[2] = odd.repeat(cols // odd.numel() + 1)[:cols]
    return h.to(torch.bfloat16)


def _oracle_kind(block):
    return C.block_length(block), bool(block & C.REGULAR)


def assert_prologue_codes(q, s, h, act, block, rows=None):
    """The GPU's codes and scales of act(h) against the oracle's, by the
    strict rule; `rows` (indices into h) restricts the check to those rows
    (q and s then hold only them).  Returns the number of codes that differ."""
    b, reg = _oracle_kind(block)
    hb = bits(h) if rows is None else bits(h[torch.from_numpy(rows)])
    qr, sr = O.act_quantize(hb, act, b, reg)
    x = O.act_f32(hb, act)
    return assert_codes_match(q, s, qr, sr, x, b, regular=reg)


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
    qx = C.workspace_codes(ws, M, K).cpu().numpy()
    sx = C.workspace_scales(ws, M).cpu().numpy()
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


def _check_rows_in_chunks(q_dev, s_dev, h, act, block, chunk=4096):
    """Every row of the GPU's codes and scales against the oracle, a chunk of
    rows at a time (bounded host memory); returns the codes that differ."""
    M = h.shape[0]
    differ = 0
    for r0 in range(0, M, chunk):
        r1 = min(M, r0 + chunk)
        rows = np.arange(r0, r1)
        differ += assert_prologue_codes(q_dev[r0:r1].cpu().numpy(), s_dev[r0:r1].cpu().numpy(), h, act, block,
                                        rows=rows)
    return differ


def test_mlp_down_prologue_full_size():
    # The 768p MLP's down projection by the prologue route, in the launch
    # configuration `bench.py --workload mlp` times: gelu(h) rotated and
    # quantised (M = 38656 rows of K = 21504), then the GEMM.  h is the GPU's
    # own plain up projection (stage-wise, as the other MLP checks).  Every
    # row's codes and scales are checked; the output on sampled rows.
    spec = W.MLP_768P
    x, w_up, w_down = W.mlp_inputs(spec)
    pw1 = C.pack_weight(w_up.to(DEV), spec.block)
    pw2 = C.pack_weight(w_down.to(DEV), spec.block)
    del w_up
    h = C.linear_fused(x.to(DEV), pw1, None)
    ws = C.alloc_workspace(spec.M, spec.H)
    y = C.linear_act(h, C.ACT_GELU, pw2, None, workspace=ws)
    torch.cuda.synchronize()
    assert C.last_device_status() == (C.OK, 0)
    q = C.workspace_codes(ws, spec.M, spec.H)
    s = C.workspace_scales(ws, spec.M)
    h_cpu = h.cpu()
    del h
    differ = _check_rows_in_chunks(q, s, h_cpu, C.ACT_GELU, spec.block)
    print(f"gelu prologue, {spec.M} x {spec.H}: {differ} of {spec.M * spec.H} codes differ from the oracle")
    rng = np.random.default_rng(8)
    rows = np.unique(np.concatenate([[0, spec.M - 1], rng.choice(spec.M, 14, replace=False)]))
    qr, sr = O.act_quantize(bits(h_cpu[torch.from_numpy(rows)]), C.ACT_GELU, spec.block)
    qw, sw = O.pack_weight(w_down.numpy(), spec.block)
    yr = O.dequant(O.igemm(qr, qw), sr, sw, None, spec.block)
    assert_close_bf16(f32_of_bf16(y[torch.from_numpy(rows).to(DEV)]), yr, "mlp down by the prologue route")


def test_swiglu_prologue_full_width():
    # SwiGLU at the MLP's hidden width (K = 21504, rows of 2K = 43008 bf16),
    # 4096 rows, every row checked.
    M, K = 4096, 21504
    h = _h(M, K, C.ACT_SWIGLU, seed=29)
    q, s = C.act_quantize(h.to(DEV), C.ACT_SWIGLU, 128)
    torch.cuda.synchronize()
    assert C.last_device_status() == (C.OK, 0)
    differ = _check_rows_in_chunks(q, s, h, C.ACT_SWIGLU, 128)
    print(f"swiglu prologue, {M} x {K}: {differ} of {M * K} codes differ from the oracle")
