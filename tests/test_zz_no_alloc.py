"""The allocation-free entry point, convrot_linear_fused_noalloc.

It exists for callers that cannot call cudaMalloc (a runtime that owns every
device allocation, or a loop that cannot afford cudaMalloc's latency and
synchronisation): the codes and scales go to the library's fixed scratch
array instead of a caller workspace.  It must give the same result as
convrot_linear_fused, call after call, since every call reuses that array.

This file is named to be collected last, so that a run stopping at the first
failure has already run every other test.
"""
import pytest
import torch

from w8a8_int8_quantized_block_b200 import convrot as C
from w8a8_int8_quantized_block_b200 import workloads as W

from helpers import assert_close_bf16, f32_of_bf16

pytestmark = pytest.mark.gpu


def _case(M, K, N, seed):
    spec, (x, w, bias) = W.custom_linear(M, K, N, seed=seed, n_out=max(1, K // 100), token_scale=True)
    pw = C.pack_weight(w.cuda(), 128)
    return x.cuda(), pw, bias.cuda()


def test_noalloc_matches_workspace_entry_point_on_consecutive_calls():
    # Two calls in a row with different inputs (the second must not see the
    # first call's leftovers in the shared scratch), each checked against the
    # workspace entry point on the same inputs.
    for M, K, N, seed, gelu in ((1000, 5376, 1024, 21, False), (6236, 5376, 512, 22, True)):
        x, pw, bias = _case(M, K, N, seed)
        y_noalloc = C.linear_fused_noalloc(x, pw, bias, gelu=gelu)
        y_ref = C.linear_fused(x, pw, bias, gelu=gelu)
        torch.cuda.synchronize()
        assert C.last_device_status() == (C.OK, 0)
        assert_close_bf16(f32_of_bf16(y_noalloc), f32_of_bf16(y_ref).astype("float64"), f"noalloc M={M}")
        assert torch.equal(y_noalloc.view(torch.int16), y_ref.view(torch.int16))


def test_noalloc_takes_large_problems_on_the_one_kernel_path():
    # The one-kernel path keeps only a ring of row panels' codes, so the
    # scratch holds problems far larger than a whole codes array would allow
    # (here 38656 rows: a 208 MB codes array, a 16.5 MB ring).
    for M, seed in ((38656, 24), (9000, 25)):
        x, pw, bias = _case(M, 5376, 264, seed)
        y_noalloc = C.linear_fused_noalloc(x, pw, bias)
        y_ref = C.linear_fused(x, pw, bias)
        torch.cuda.synchronize()
        assert C.last_device_status() == (C.OK, 0)
        assert torch.equal(y_noalloc.view(torch.int16), y_ref.view(torch.int16))


def test_noalloc_rejects_problems_beyond_its_scratch():
    # On the two-kernel path the whole codes array must fit: rows of K = 21504
    # (past the one-kernel path's 6144) allow at most 1560 rows, and rows that
    # are 16- but not 32-byte aligned at K = 5376 at most 6236.
    x, pw, bias = _case(1561, 21504, 64, 23)
    xs = torch.empty(6237 * 5376 + 8, dtype=torch.bfloat16, device="cuda")[8:].view(6237, 5376)
    xs.copy_(torch.randn(6237, 5376, device="cuda").to(torch.bfloat16))
    _, pw2, bias2 = _case(8, 5376, 64, 26)
    for xx, ww, bb in ((x, pw, bias), (xs, pw2, bias2)):
        y = torch.full((xx.shape[0], 64), 7.0, dtype=torch.bfloat16, device="cuda")
        with pytest.raises(C.ConvrotError) as e:
            C.linear_fused_noalloc(xx, ww, bb, out=y)
        assert e.value.status == C.ETOOLARGE
        torch.cuda.synchronize()
        assert bool((y == 7.0).all())  # nothing was launched
