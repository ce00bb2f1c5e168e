"""The quantiser rounds the product z * inv to f32 first and only then to an
integer ("Rowwise INT8 Quantize", MiniMax-H3-Rung-Omega README, "Technical
Architecture Overview", item 2: a symmetric per-row scale and round-to-nearest
of the scaled value, computed in single precision).

These rows are built so that the f32 product lands exactly on 63.5 while the
exact product is a little below it: the two-step rounding gives 64 (ties to
even), a multiply-add that rounds the exact product once gives 63.  Every
kernel must reproduce the oracle exactly here -- no tie allowance.

The rows come from near_ties.py, which explains the construction.
"""
import numpy as np
import pytest
import torch

from oracle import oracle as O
from w8a8_int8_quantized_block_b200 import convrot as C

from helpers import bits
from near_ties import plain_rows, rotated_rows

pytestmark = pytest.mark.gpu
DEV = "cuda"


def _oracle_has_two_step_codes(q: np.ndarray):
    # the test only means something if the oracle rounds twice: +-64, never +-63
    assert (np.abs(q) == 64).sum() >= q.shape[0]
    assert not (np.abs(q) == 63).any()


@pytest.mark.parametrize("block", [128, 0])
def test_quantize_act_double_rounding_exact(block):
    xr = rotated_rows() if block == 128 else plain_rows()
    x = torch.from_numpy(xr).to(torch.bfloat16)
    assert np.array_equal(x.double().numpy(), xr)  # exact in bf16
    qr, sr = O.quantize_act(bits(x), block)
    _oracle_has_two_step_codes(qr)
    q, s = C.quantize_act(x.to(DEV), block)
    torch.cuda.synchronize()
    assert C.last_device_status() == (C.OK, 0)
    assert np.array_equal(q.cpu().numpy(), qr)
    assert np.array_equal(s.cpu().numpy().view(np.uint32), sr.view(np.uint32))


def test_pack_weight_double_rounding_exact():
    w = torch.from_numpy(rotated_rows()).to(torch.float32)
    qr, sr = O.pack_weight(w.numpy(), 128)
    _oracle_has_two_step_codes(qr)
    pw = C.pack_weight(w.to(DEV), 128)
    torch.cuda.synchronize()
    assert np.array_equal(pw.q.cpu().numpy(), qr)
    assert np.array_equal(pw.s.cpu().numpy().view(np.uint32), sr.view(np.uint32))


def test_one_kernel_linear_codes_double_rounding_exact():
    # The quantiser warps inside the one-kernel linear write the same codes to
    # the workspace (every row's codes while the panels fit the ring).
    xr = rotated_rows()
    M, K = xr.shape
    x = torch.from_numpy(xr).to(torch.bfloat16)
    w = torch.randn(256, K, generator=torch.Generator().manual_seed(5)) * 0.02
    pw = C.pack_weight(w.to(DEV), 128)
    ws = C.alloc_workspace(M, K)
    C.linear_fused(x.to(DEV), pw, None, workspace=ws)
    torch.cuda.synchronize()
    assert C.last_device_status() == (C.OK, 0)
    qr, sr = O.quantize_act(bits(x), 128)
    q = C.workspace_codes(ws, M, K).cpu().numpy()
    s = C.workspace_scales(ws, M).cpu().numpy()
    assert np.array_equal(q, qr)
    assert np.array_equal(s.view(np.uint32), sr.view(np.uint32))
