"""GPU parity of the int8 attention ("sageattn_qk_int8_pv_fp16_cuda" in the
Rung-Omega engine -- MiniMax-H3-Rung-Omega README, "Technical Architecture
Overview", item 2) against the oracle's fp64 softmax(S) V.

The Q and K codes and scales are the rowwise quantiser's and must match the
oracle exactly.  The output is floating point: the kernel rounds P to bf16
for the P V product and evaluates 2^x on the special-function unit, so O is
compared with the bf16 tolerance (relative L2 <= 1e-2, cosine >= 0.9999).
"""
import numpy as np
import pytest
import torch

from oracle import oracle as O
from w8a8_int8_quantized_block_b200 import convrot as C
from w8a8_int8_quantized_block_b200 import workloads as W

from helpers import assert_close_bf16, bits

pytestmark = pytest.mark.gpu
DEV = "cuda"


def _qkv(H, Lq, Lk, seed, qscale=1.0):
    g = torch.Generator().manual_seed(seed)
    q = (torch.randn(H, Lq, 128, generator=g) * qscale).to(torch.bfloat16)
    k = torch.randn(H, Lk, 128, generator=g).to(torch.bfloat16)
    v = torch.randn(H, Lk, 128, generator=g).to(torch.bfloat16)
    return q, k, v


def _run(q, k, v, scale=None):
    H, Lq, _ = q.shape
    Lk = k.shape[1]
    ws = torch.empty((C.load().convrot_attention_workspace_bytes(H, Lq, Lk),), dtype=torch.uint8, device=DEV)
    o = C.attention(q.to(DEV), k.to(DEV), v.to(DEV), scale, workspace=ws)
    torch.cuda.synchronize()
    assert C.last_device_status() == (C.OK, 0)
    return o, ws


def _check_codes(ws, q, k):
    H, Lq, _ = q.shape
    Lk = k.shape[1]
    r = lambda n: (n + 255) // 256 * 256
    qx = ws[:H * Lq * 128].view(torch.int8).cpu().numpy().reshape(H * Lq, 128)
    o1 = r(H * Lq * 128)
    sq = ws[o1:o1 + 4 * H * Lq].view(torch.float32).cpu().numpy()
    o2 = o1 + r(4 * H * Lq)
    kx = ws[o2:o2 + H * Lk * 128].view(torch.int8).cpu().numpy().reshape(H * Lk, 128)
    o3 = o2 + r(H * Lk * 128)
    sk = ws[o3:o3 + 4 * H * Lk].view(torch.float32).cpu().numpy()
    qr, sqr = O.quantize_act(bits(q.reshape(H * Lq, 128)), 0)
    kr, skr = O.quantize_act(bits(k.reshape(H * Lk, 128)), 0)
    assert np.array_equal(qx, qr) and np.array_equal(sq.view(np.uint32), sqr.view(np.uint32))
    assert np.array_equal(kx, kr) and np.array_equal(sk.view(np.uint32), skr.view(np.uint32))


@pytest.mark.parametrize("H,Lq,Lk", [(2, 256, 384), (1, 128, 128), (3, 128, 1024), (2, 640, 256), (1, 384, 512)])
def test_attention_matches_oracle(H, Lq, Lk):
    q, k, v = _qkv(H, Lq, Lk, seed=H * 1000 + Lq + Lk)
    o, ws = _run(q, k, v)
    _check_codes(ws, q, k)
    ref, _ = O.attention(bits(q), bits(k), bits(v))
    assert_close_bf16(o.float().cpu().numpy(), ref, f"attention {H}x{Lq}x{Lk}")


def test_attention_many_key_tiles_rescale_the_partial_output():
    # 64 key tiles; the queries are scaled up so that the running maximum keeps
    # growing over the tiles (the O rescaling runs often)
    q, k, v = _qkv(1, 128, 8192, seed=5, qscale=3.0)
    k[:, ::97] *= 2.5
    o, _ = _run(q, k, v)
    ref, _ = O.attention(bits(q), bits(k), bits(v))
    assert_close_bf16(o.float().cpu().numpy(), ref, "attention 64 key tiles")


def test_attention_zero_queries_and_sharp_softmax():
    q, k, v = _qkv(2, 256, 512, seed=6, qscale=2.0)
    q[0, :5] = 0.0  # s_q = 0: uniform weights, O = mean of V
    o, _ = _run(q, k, v, scale=0.5)  # a sharper softmax than 1/sqrt(128)
    ref, _ = O.attention(bits(q), bits(k), bits(v), scale=0.5)
    assert_close_bf16(o.float().cpu().numpy(), ref, "attention sharp")
    mean_v = v[0].float().mean(0).numpy()
    assert np.abs(o[0, :5].float().cpu().numpy() - mean_v).max() < 2e-2


def test_attention_full_size_sampled_rows():
    # the 42-head, 8192-token workload: O checked on sampled rows
    spec = W.QK_BMM
    q, k = W.bmm_inputs(spec)
    v = torch.randn(spec.batch, spec.N, spec.K, generator=torch.Generator().manual_seed(44)).to(torch.bfloat16)
    o, ws = _run(q, k, v)
    H, L = spec.batch, spec.M
    qx, sq = O.quantize_act(bits(q.reshape(H * L, 128)), 0)
    kx, sk = O.quantize_act(bits(k.reshape(H * L, 128)), 0)
    rng = np.random.default_rng(7)
    heads = rng.integers(0, H, 48)
    rows = rng.integers(0, L, 48)
    ref = O.attention_rows(qx.reshape(H, L, 128), sq.reshape(H, L), kx.reshape(H, L, 128), sk.reshape(H, L),
                           bits(v), heads, rows, 128 ** -0.5)
    got = o[torch.from_numpy(heads).to(DEV), torch.from_numpy(rows).to(DEV)].float().cpu().numpy()
    assert_close_bf16(got, ref, "attention full size (sampled rows)")


def test_attention_splits_the_last_wave_over_the_keys():
    # 150 units (heads x query-tile pairs) on 148 SMs: 148 run whole, the last
    # two are split over their 4 key tiles and combined; rows of both kinds
    # are checked against the oracle
    H, Lq, Lk = 150, 256, 512
    q, k, v = _qkv(H, Lq, Lk, seed=8)
    sms = torch.cuda.get_device_properties(0).multi_processor_count
    o, ws = _run(q, k, v)
    assert C.attention_split_bytes(H, Lq, Lk) > 0 or sms >= H
    qx, sq = O.quantize_act(bits(q.reshape(H * Lq, 128)), 0)
    kx, sk = O.quantize_act(bits(k.reshape(H * Lk, 128)), 0)
    rng = np.random.default_rng(9)
    heads = np.concatenate([np.full(12, H - 1), np.full(12, H - 2), rng.integers(0, H - 2, 12)])
    rows = rng.integers(0, Lq, heads.size)
    ref = O.attention_rows(qx.reshape(H, Lq, 128), sq.reshape(H, Lq), kx.reshape(H, Lk, 128), sk.reshape(H, Lk),
                           bits(v), heads, rows, 128 ** -0.5)
    got = o[torch.from_numpy(heads).to(DEV), torch.from_numpy(rows).to(DEV)].float().cpu().numpy()
    assert_close_bf16(got, ref, "attention, split last wave")


def test_attention_int8_with_and_without_the_split_buffer():
    # the kernel entry on quantised inputs: the split path (parts + combine)
    # and every unit whole both match the oracle
    H, Lq, Lk = 2, 256, 2048
    q, k, v = _qkv(H, Lq, Lk, seed=10)
    qx, sq = C.quantize_act(q.reshape(H * Lq, 128).to(DEV), 0)
    kx, sk = C.quantize_act(k.reshape(H * Lk, 128).to(DEV), 0)
    vt = v.transpose(1, 2).contiguous().to(DEV)
    nbytes = C.attention_split_bytes(H, Lq, Lk)
    assert nbytes > 0  # 2 units on one wave: split 8 ways over 16 key tiles
    split_ws = torch.empty((nbytes,), dtype=torch.uint8, device=DEV)
    args = (qx.view(H, Lq, 128), sq.view(H, Lq), kx.view(H, Lk, 128), sk.view(H, Lk), vt)
    o_split = C.attention_int8(*args, split_ws=split_ws)
    o_whole = C.attention_int8(*args)
    torch.cuda.synchronize()
    assert C.last_device_status() == (C.OK, 0)
    ref, _ = O.attention(bits(q), bits(k), bits(v))
    assert_close_bf16(o_split.float().cpu().numpy(), ref, "attention_int8 split")
    assert_close_bf16(o_whole.float().cpu().numpy(), ref, "attention_int8 whole")


def test_attention_int8_split_buffer_16_byte_aligned():
    # the entry asks only 16-byte alignment of the split buffer: one that is not
    # 32-byte aligned gives the same output as an aligned one
    H, Lq, Lk = 2, 256, 2048
    q, k, v = _qkv(H, Lq, Lk, seed=12)
    qx, sq = C.quantize_act(q.reshape(H * Lq, 128).to(DEV), 0)
    kx, sk = C.quantize_act(k.reshape(H * Lk, 128).to(DEV), 0)
    vt = v.transpose(1, 2).contiguous().to(DEV)
    nbytes = C.attention_split_bytes(H, Lq, Lk)
    buf = torch.empty((nbytes + 64,), dtype=torch.uint8, device=DEV)
    assert buf.data_ptr() % 256 == 0
    args = (qx.view(H, Lq, 128), sq.view(H, Lq), kx.view(H, Lk, 128), sk.view(H, Lk), vt)
    o_16 = C.attention_int8(*args, split_ws=buf[16:16 + nbytes])
    o_256 = C.attention_int8(*args, split_ws=buf[:nbytes])
    torch.cuda.synchronize()
    assert C.last_device_status() == (C.OK, 0)
    assert torch.equal(o_16, o_256)
