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


def test_noalloc_rejects_problems_beyond_its_scratch():
    x, pw, bias = _case(6237, 5376, 64, 23)
    y = torch.full((6237, 64), 7.0, dtype=torch.bfloat16, device="cuda")
    with pytest.raises(C.ConvrotError) as e:
        C.linear_fused_noalloc(x, pw, bias, out=y)
    assert e.value.status == C.ETOOLARGE
    torch.cuda.synchronize()
    assert bool((y == 7.0).all())  # nothing was launched
