"""GPU parity for every rotation: Sylvester H_b (b = 64, 128, 256) and the
regular H_4^(x)k (b = 16, 64, 256) -- the block-diagonal Hadamard rotation of
lehuy.net "Nen mo hinh video khuech tan 31B xuong 14B", section "Cach nen hoat
dong", with the "ConvRot64" block and the "DC-balanced regular orthogonal
Hadamard matrix H_256 = H_4^(x)4" of the MiniMax-H3-Rung-Omega README,
"Technical Architecture Overview", items 1-2.

Both sides run the same fp32 operations in the same order, so codes and
scales must match the oracle exactly (no tie allowance).
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

KINDS = [64, 128, 256, C.REGULAR | 16, C.REGULAR | 64, C.REGULAR | 256]


def _ids(block):
    return ("reg" if block & C.REGULAR else "syl") + str(C.block_length(block))


def _oracle_kind(block):
    return C.block_length(block), bool(block & C.REGULAR)


def _act(M, K, seed):
    spec, (x, _, _) = W.custom_linear(M, K, 8, seed, n_out=max(1, K // 100), token_scale=True)
    return x


# K = 768: 12 threads per row (short rows, 16-lane groups with 4 idle lanes);
# K = 2304: 36 threads per row, seven rows packed into eight warps;
# K = 5376: 84 threads per row, three rows packed into eight warps;
# K = 6144: 96 threads per row (whole warps).
@pytest.mark.parametrize("block", KINDS, ids=_ids)
@pytest.mark.parametrize("M,K", [(33, 768), (61, 2304), (130, 5376), (9, 6144)])
def test_quantize_act_every_rotation_exact(block, M, K):
    x = _act(M, K, seed=M + K + block % 977)
    q, s = C.quantize_act(x.to(DEV), block)
    torch.cuda.synchronize()
    assert C.last_device_status() == (C.OK, 0)
    b, reg = _oracle_kind(block)
    qr, sr = O.quantize_act(bits(x), b, reg)
    assert np.array_equal(s.cpu().numpy().view(np.uint32), sr.view(np.uint32))
    assert np.array_equal(q.cpu().numpy(), qr)


@pytest.mark.parametrize("block", KINDS, ids=_ids)
def test_pack_weight_every_rotation_exact(block):
    N, K = 300, 2304
    w = torch.randn(N, K, generator=torch.Generator().manual_seed(block % 1000)) * 0.02
    w[:, 17] *= 40
    pw = C.pack_weight(w.to(DEV), block)
    torch.cuda.synchronize()
    assert pw.block == block
    b, reg = _oracle_kind(block)
    qr, sr = O.pack_weight(w.numpy(), b, reg)
    assert np.array_equal(pw.s.cpu().numpy().view(np.uint32), sr.view(np.uint32))
    assert np.array_equal(pw.q.cpu().numpy(), qr)


@pytest.mark.parametrize("block", KINDS, ids=_ids)
@pytest.mark.parametrize("fused", [True, False], ids=["one_kernel", "two_kernels"])
def test_linear_every_rotation_matches_oracle(block, fused):
    M, K, N = 300, 1536, 520
    spec, (x, w, bias) = W.custom_linear(M, K, N, seed=block % 991, n_out=15, token_scale=True)
    pw = C.pack_weight(w.to(DEV), block)
    ws = C.alloc_workspace(M, K)
    if fused:
        y = C.linear_fused(x.to(DEV), pw, bias.to(DEV), workspace=ws)
    else:
        q, s = C.quantize_act(x.to(DEV), block)
        y = C.w8a8_linear(q, s, pw, bias.to(DEV))
    torch.cuda.synchronize()
    assert C.last_device_status() == (C.OK, 0)
    b, reg = _oracle_kind(block)
    yr, qxr, sxr, *_ = O.linear(bits(x), w.numpy(), bias.numpy(), b, regular=reg)
    assert_close_bf16(f32_of_bf16(y), yr, f"linear {_ids(block)}")
    if fused:
        # the one-kernel path leaves its codes in the workspace: exact too
        qx = C.workspace_codes(ws, M, K).cpu().numpy()
        sx = C.workspace_scales(ws, M).cpu().numpy()
        assert np.array_equal(qx, qxr)
        assert np.array_equal(sx.view(np.uint32), sxr.view(np.uint32))


def test_regular_rotation_keeps_a_constant_row_constant():
    # DC-balanced: a constant block stays constant, so every code is 127
    for b in (16, 64, 256):
        x = torch.full((3, 1024), 0.75, dtype=torch.bfloat16)
        q, s = C.quantize_act(x.to(DEV), C.REGULAR | b)
        torch.cuda.synchronize()
        assert (q.cpu() == 127).all()
        assert np.allclose(s.cpu().numpy(), 0.75 * b ** 0.5 / 127, rtol=1e-6)
