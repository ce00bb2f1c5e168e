"""GPU parity: the CUDA path through the C ABI against the CPU oracle, element
by element, on seeded inputs that span several tiles and a ragged tail."""
import numpy as np
import pytest
import torch

from oracle import oracle as O
from w8a8_int8_quantized_block_b200 import convrot as C
from w8a8_int8_quantized_block_b200 import workloads as W

from helpers import assert_close_bf16, assert_codes_match, bits, f32_of_bf16

pytestmark = pytest.mark.gpu
DEV = "cuda"


def _act(M, K, seed, n_out=0, out_scale=10.0, token_scale=False):
    spec, (x, _, _) = W.custom_linear(M, K, 8, seed, n_out=n_out, out_scale=out_scale, token_scale=token_scale)
    return x


# ------------------------------------------------------------------ rotate + quantise


@pytest.mark.parametrize("M,K,block", [
    (256, 512, 128), (1, 5376, 128), (127, 5376, 128), (129, 512, 128), (300, 21504, 128),
    (200, 128, 128), (64, 128, 0), (77, 1024, 128), (33, 384, 128), (5, 640, 0), (3, 32768, 128),
])
def test_quantize_act_bitexact(M, K, block):
    x = _act(M, K, seed=M + K, n_out=max(1, K // 100), token_scale=True)
    q, s = C.quantize_act(x.to(DEV), block)
    torch.cuda.synchronize()
    qr, sr = O.quantize_act(bits(x), block)
    assert_codes_match(q.cpu().numpy(), s.cpu().numpy(), qr, sr, f32_of_bf16(x), block)
    assert C.last_device_status() == (C.OK, 0)


def test_quantize_act_strided_rows():
    x = _act(150, 5376 + 64, seed=9, n_out=20)
    xs = x[:, 32:32 + 5376]  # row stride 5440, offset 64 bytes
    q, s = C.quantize_act(x.to(DEV)[:, 32:32 + 5376], 128)
    qr, sr = O.quantize_act(bits(xs.contiguous()), 128)
    assert_codes_match(q.cpu().numpy(), s.cpu().numpy(), qr, sr, f32_of_bf16(xs.contiguous()), 128)


def test_quantize_act_special_rows():
    K = 1024
    x = torch.randn(16, K, generator=torch.Generator().manual_seed(3))
    x[0] = 0.0                              # zero row
    x[1] = 0.0
    x[1, 517] = -7.5                        # spike
    x[2] = 1.0                              # constant row (DC of every block)
    x[3] = 1e-30                            # tiny values
    x[4] = 3.0e38 / 2 ** 10                 # large values, no overflow after 128-sums
    x[5, ::2] *= -1
    x = x.to(torch.bfloat16)
    q, s = C.quantize_act(x.to(DEV), 128)
    qr, sr = O.quantize_act(bits(x), 128)
    assert_codes_match(q.cpu().numpy(), s.cpu().numpy(), qr, sr, f32_of_bf16(x), 128)
    assert s[0].item() == 0.0 and not q[0].any()


@pytest.mark.parametrize("N,K", [(512, 512), (384, 5376), (5376, 5376), (1000, 21504), (3, 128)])
def test_pack_weight_bitexact(N, K):
    w = torch.randn(N, K, generator=torch.Generator().manual_seed(N + K)) * 0.02
    w[:, 7] *= 30
    pw = C.pack_weight(w.to(DEV), 128)
    qr, sr = O.pack_weight(w.numpy(), 128)
    assert (pw.desc.magic, pw.desc.version, pw.desc.layout, pw.desc.block, pw.desc.N, pw.desc.K) == (
        C.WDESC_MAGIC, C.WDESC_VERSION, C.LAYOUT_OUTPUT_MAJOR, 128, N, K)
    assert_codes_match(pw.q.cpu().numpy(), pw.s.cpu().numpy(), qr, sr)


# ------------------------------------------------------------------ int8 GEMM accumulators


def _codes(shape, seed):
    g = torch.Generator().manual_seed(seed)
    return torch.randint(-127, 128, shape, generator=g, dtype=torch.int8)


@pytest.mark.parametrize("B,M,N,K", [
    (1, 128, 256, 128), (1, 1, 8, 16), (1, 127, 260, 528), (1, 129, 512, 512), (1, 300, 1000, 5376),
    (3, 200, 264, 128), (1, 1024, 768, 1024), (1, 64, 4, 48),
])
def test_igemm_s32_bitexact(B, M, N, K):
    qa = _codes((B, M, K), M * 7 + K)
    qb = _codes((B, N, K), N * 3 + K + 1)
    acc = C.igemm_s32(qa.to(DEV), qb.to(DEV))
    torch.cuda.synchronize()
    for b in range(B):
        ref = O.igemm(qa[b].numpy(), qb[b].numpy())
        assert (acc[b].cpu().numpy().astype(np.int64) == ref).all()


@pytest.mark.parametrize("B,M,N,K", [(8, 2048, 336, 128), (4, 1536, 80, 256), (2, 2048, 592, 384)])
def test_igemm_s32_many_ragged_tiles(B, M, N, K):
    # More tiles than CTA pairs, each ending in a part-filled column tile (an
    # odd number of 32-column chunks), so every epilogue warp cycles its
    # staging buffers across tiles of uneven length, and prefetches the next
    # tile's scales while it drains one that ends short.
    qa = _codes((B, M, K), 11 + N)
    qb = _codes((B, N, K), 12 + N)
    acc = C.igemm_s32(qa.to(DEV), qb.to(DEV)).cpu().numpy().astype(np.int64)
    assert C.last_device_status() == (C.OK, 0)
    for b in range(B):
        assert (acc[b] == O.igemm(qa[b].numpy(), qb[b].numpy())).all(), f"batch {b}"


def test_bmm_many_ragged_tiles_matches_oracle():
    B, M, N, K = 8, 2048, 336, 128
    q, k = W.bmm_inputs(W.QK_BMM, M=M, N=N)
    q, k = q[:B], k[:B]
    qa, sa = C.quantize_act(q.to(DEV).reshape(B * M, K), 0)
    qb, sb = C.quantize_act(k.to(DEV).reshape(B * N, K), 0)
    y = C.w8a8_bmm(qa.view(B, M, K), sa, qb.view(B, N, K), sb)
    torch.cuda.synchronize()
    assert C.last_device_status() == (C.OK, 0)
    qar, sar = O.quantize_act(bits(q.reshape(B * M, K)), 0)
    qbr, sbr = O.quantize_act(bits(k.reshape(B * N, K)), 0)
    for b in range(B):
        acc = O.igemm(qar[b * M:(b + 1) * M], qbr[b * N:(b + 1) * N])
        yr = O.dequant(acc, sar[b * M:(b + 1) * M], sbr[b * N:(b + 1) * N], None, 0)
        assert_close_bf16(f32_of_bf16(y[b]), yr, f"bmm head {b}")


def test_igemm_s32_extreme_accumulators():
    K = 21504
    qa = torch.full((1, 130, K), -127, dtype=torch.int8)
    qa[0, 1] = 127
    qa[0, 2, ::2] = 127
    qb = torch.full((1, 260, K), 127, dtype=torch.int8)
    acc = C.igemm_s32(qa.to(DEV), qb.to(DEV)).cpu().numpy().astype(np.int64)
    assert (acc[0, 0] == -127 * 127 * K).all()
    assert (acc[0, 1] == 127 * 127 * K).all()
    assert (acc[0, 2] == 0).all()


# ------------------------------------------------------------------ the linear


def _run_linear(spec_or_args, fused=True, gelu=False):
    x, w, bias = spec_or_args
    pw = C.pack_weight(w.to(DEV), 128)
    b = None if bias is None else bias.to(DEV)
    if fused:
        y = C.linear_fused(x.to(DEV), pw, b, gelu=gelu)
    else:
        q, s = C.quantize_act(x.to(DEV), 128)
        y = C.w8a8_linear(q, s, pw, b, gelu=gelu)
    torch.cuda.synchronize()
    return y, pw


def test_linear_tiny_matches_oracle():
    x, w, bias = W.linear_inputs(W.TINY)
    y, pw = _run_linear((x, w, bias), fused=True)
    yr, qx, sx, qw, sw, acc = O.linear(bits(x), w.numpy(), bias.numpy(), 128)
    assert_codes_match(pw.q.cpu().numpy(), pw.s.cpu().numpy(), qw, sw)
    assert_close_bf16(f32_of_bf16(y), yr, "tiny linear")
    assert C.last_device_status() == (C.OK, 0)


def test_linear_fused_equals_two_step_bitwise():
    x, w, bias = W.linear_inputs(W.TINY)
    y1, _ = _run_linear((x, w, bias), fused=True)
    y2, _ = _run_linear((x, w, bias), fused=False)
    assert torch.equal(y1.view(torch.int16), y2.view(torch.int16))


@pytest.mark.parametrize("M,K,N", [(7937, 5376, 264), (16000, 256, 64)])
def test_linear_fused_codes_ring_equals_two_step_bitwise(M, K, N):
    # More than 12 row panels: the one-kernel path reuses its ring of code
    # slots (7937 rows: 31 panels, the last of one row; 16000 rows: 63 panels
    # of one column tile each, so every slot turns over five times).  The
    # two-kernel path keeps every row's codes, so any slot overwritten too
    # early or read stale changes outputs.
    spec, (x, w, bias) = W.custom_linear(M, K, N, seed=M + 11, n_out=3, token_scale=True)
    y1, _ = _run_linear((x, w, bias), fused=True)
    y2, _ = _run_linear((x, w, bias), fused=False)
    assert C.last_device_status() == (C.OK, 0)
    assert torch.equal(y1.view(torch.int16), y2.view(torch.int16))


@pytest.mark.parametrize("M,K,N", [(5000, 5376, 9488), (600, 6144, 8208)])
def test_grouped_tile_order_one_kernel_equals_two_kernels(M, K, N):
    # Weights over 48 MiB (N K = 51.0 / 50.4 MB): the two-kernel GEMM walks
    # the row panels in groups of 8 per column tile, the one-kernel path in
    # groups of half its codes ring.  5000 rows: 20 panels; two-kernel groups
    # 8, 8, 4; one-kernel groups 6, 6, 6, 2 with a ring of 12 slots that wraps.
    # 600 rows: 3 panels, one short group.  N ends in a part-filled column tile.
    spec, (x, w, bias) = W.custom_linear(M, K, N, seed=M + 17, n_out=3, token_scale=True)
    y1, pw = _run_linear((x, w, bias), fused=True)
    y2, _ = _run_linear((x, w, bias), fused=False)
    assert C.last_device_status() == (C.OK, 0)
    assert torch.equal(y1.view(torch.int16), y2.view(torch.int16))
    rows = np.unique(np.random.default_rng(M).choice(M, 24, replace=False))
    yr, *_ = O.linear(bits(x[torch.from_numpy(rows)]), w.numpy(), bias.numpy(), 128)
    assert_close_bf16(f32_of_bf16(y1[torch.from_numpy(rows).to(DEV)]), yr, "grouped tile order")


def test_igemm_s32_grouped_tile_order_bitexact():
    # N K = 8208 x 6144 = 50.4 MB: the accumulators of a grouped tile order
    # (3 row panels of 256 in one short group, 33 column tiles, the last
    # part-filled), every element against the exact int64 product
    M, N, K = 700, 8208, 6144
    qa = _codes((1, M, K), 31)
    qb = _codes((1, N, K), 32)
    acc = C.igemm_s32(qa.to(DEV), qb.to(DEV)).cpu().numpy().astype(np.int64)
    assert C.last_device_status() == (C.OK, 0)
    assert (acc[0] == O.igemm(qa[0].numpy(), qb[0].numpy())).all()


def test_linear_fused_long_rows_match_oracle():
    # K > 6144 (the MLP down projection's 21504): linear_fused runs the
    # quantiser and the GEMM as two kernels
    M, K, N = 257, 21504, 136
    spec, (x, w, bias) = W.custom_linear(M, K, N, seed=23, n_out=30, token_scale=True)
    y, pw = _run_linear((x, w, bias), fused=True)
    assert C.last_device_status() == (C.OK, 0)
    yr, *_ = O.linear(bits(x), w.numpy(), bias.numpy(), 128)
    assert_close_bf16(f32_of_bf16(y), yr, "linear K=21504")


@pytest.mark.parametrize("M,K,N", [(1, 128, 8), (127, 512, 384), (129, 640, 264), (257, 5376, 520),
                                   (1000, 1024, 2048)])
def test_linear_ragged_shapes(M, K, N):
    spec, (x, w, bias) = W.custom_linear(M, K, N, seed=M + N, n_out=max(1, K // 100))
    y, pw = _run_linear((x, w, bias), fused=True)
    yr, *_ = O.linear(bits(x), w.numpy(), bias.numpy(), 128)
    assert_close_bf16(f32_of_bf16(y), yr, f"linear {M}x{K}x{N}")


def test_linear_fused_many_ragged_tiles():
    # 32 row panels x 3 column tiles (256, 256, 80 columns): more tiles than
    # CTA pairs, and every third tile drains an odd number of 32-column chunks
    # through the epilogue's two staging buffers.
    M, K, N = 8192, 512, 592
    spec, (x, w, bias) = W.custom_linear(M, K, N, seed=17, n_out=5, token_scale=True)
    y, pw = _run_linear((x, w, bias), fused=True)
    assert C.last_device_status() == (C.OK, 0)
    yr, *_ = O.linear(bits(x), w.numpy(), bias.numpy(), 128)
    assert_close_bf16(f32_of_bf16(y), yr, "linear 8192x512x592")


@pytest.mark.parametrize("pad", [8, 16])
def test_linear_fused_strided_rows(pad):
    # Row stride K + 8 (16-byte aligned rows) takes the two-kernel path, K + 16
    # (32-byte aligned) the one-kernel path; both must match the oracle.
    M, K, N = 300, 5376, 512
    spec, (x, w, bias) = W.custom_linear(M, K, N, seed=pad, n_out=20, token_scale=True)
    xp = torch.zeros(M, K + pad, dtype=torch.bfloat16)
    xp[:, :K] = x
    pw = C.pack_weight(w.to(DEV), 128)
    y = C.linear_fused(xp.to(DEV)[:, :K], pw, bias.to(DEV))
    torch.cuda.synchronize()
    assert C.last_device_status() == (C.OK, 0)
    yr, *_ = O.linear(bits(x), w.numpy(), bias.numpy(), 128)
    assert_close_bf16(f32_of_bf16(y), yr, f"strided linear pad {pad}")
    y2 = C.linear_fused(x.to(DEV), pw, bias.to(DEV))
    assert torch.equal(y.view(torch.int16), y2.view(torch.int16))


def test_linear_gelu_epilogue():
    spec, (x, w, bias) = W.custom_linear(300, 1024, 768, seed=5, n_out=10)
    y, pw = _run_linear((x, w, bias), fused=True, gelu=True)
    yr, *_ = O.linear(bits(x), w.numpy(), bias.numpy(), 128, gelu=True)
    assert_close_bf16(f32_of_bf16(y), yr, "gelu linear")


def test_linear_epilogue_on_identical_codes_is_tight():
    # Same codes on both sides: the only error left is the f32 epilogue and the
    # final bf16 rounding (<= 2^-8 relative per element plus f32 noise).
    x, w, bias = W.linear_inputs(W.TINY)
    pw = C.pack_weight(w.to(DEV), 128)
    q, s = C.quantize_act(x.to(DEV), 128)
    y = C.w8a8_linear(q, s, pw, bias.to(DEV))
    acc = O.igemm(q.cpu().numpy(), pw.q.cpu().numpy())
    yr = O.dequant(acc, s.cpu().numpy(), pw.s.cpu().numpy(), bias.numpy(), 128)
    err = np.abs(f32_of_bf16(y).astype(np.float64) - yr)
    assert (err <= np.abs(yr) * 2.0 ** -8 + 1e-6).all()


def test_gelu_epilogue_rounds_like_the_exact_gelu():
    # Same codes on both sides, pre-activations spread over about [-12, 12] by
    # the bias, so the negative tail is exercised (there GELU(y) is
    # 0.5 y erfc(|y| / sqrt 2), many binades below y): nearly every output is
    # the correctly rounded bf16 of the oracle's fp64 GELU of its fp64
    # pre-activation, and none is further off than the f32 epilogue allows.
    # (The f32 rounding of y^2 alone moves 2^(-log2(e) y^2 / 2) by ~6e-6 at
    # y = -10, so a few in a thousand roundings may go the other way; the form
    # 0.5 y (1 + erf(y / sqrt 2)) in f32 rounds about a third of them wrongly.)
    x, w, _ = W.linear_inputs(W.TINY)
    bias = torch.linspace(-12.0, 12.0, w.shape[0], dtype=torch.float32)
    pw = C.pack_weight(w.to(DEV), 128)
    q, s = C.quantize_act(x.to(DEV), 128)
    y = C.w8a8_linear(q, s, pw, bias.to(DEV), gelu=True)
    torch.cuda.synchronize()
    assert C.last_device_status() == (C.OK, 0)
    acc = O.igemm(q.cpu().numpy(), pw.q.cpu().numpy())
    yr = O.dequant(acc, s.cpu().numpy(), pw.s.cpu().numpy(), bias.numpy(), 128, gelu=True)
    got = f32_of_bf16(y).astype(np.float64)
    nearest = torch.from_numpy(yr).to(torch.bfloat16).double().numpy()
    assert (yr < -1e-6).mean() > 0.2  # the tail is really there
    assert np.mean(got == nearest) >= 0.998
    assert (np.abs(got - yr) <= np.abs(yr) * 2.0 ** -8 + 1e-5).all()


# ------------------------------------------------------------------ batched skinny-K GEMM


def test_bmm_small_batch_matches_oracle():
    spec = W.QK_BMM
    q, k = W.bmm_inputs(spec, M=512, N=384)
    q = q[:3]
    k = k[:3]
    B, M, K = q.shape
    N = k.shape[1]
    qa, sa = C.quantize_act(q.to(DEV).reshape(B * M, K), 0)
    qb, sb = C.quantize_act(k.to(DEV).reshape(B * N, K), 0)
    y = C.w8a8_bmm(qa.view(B, M, K), sa, qb.view(B, N, K), sb)
    torch.cuda.synchronize()
    qar, sar = O.quantize_act(bits(q.reshape(B * M, K)), 0)
    qbr, sbr = O.quantize_act(bits(k.reshape(B * N, K)), 0)
    assert_codes_match(qa.cpu().numpy(), sa.cpu().numpy(), qar, sar)
    assert_codes_match(qb.cpu().numpy(), sb.cpu().numpy(), qbr, sbr)
    for b in range(B):
        acc = O.igemm(qar[b * M:(b + 1) * M], qbr[b * N:(b + 1) * N])
        yr = O.dequant(acc, sar[b * M:(b + 1) * M], sbr[b * N:(b + 1) * N], None, 0)
        assert_close_bf16(f32_of_bf16(y[b]), yr, f"bmm head {b}")


# ------------------------------------------------------------------ failure path


def test_bounded_wait_times_out_cleanly():
    assert C.last_device_status() == (C.OK, 0)
    C.selftest_wait_timeout(2_000_000)  # 2 ms
    st, code = C.last_device_status()
    assert st == C.ETIMEOUT and code == 6
    assert C.last_device_status() == (C.OK, 0)  # cleared, context still usable
    x = torch.ones(4, 128, dtype=torch.bfloat16, device=DEV)
    q, s = C.quantize_act(x, 128)
    torch.cuda.synchronize()
    assert q[:, 0].tolist() == [127] * 4
