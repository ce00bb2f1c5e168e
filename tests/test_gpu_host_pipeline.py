"""convrot_linear_fused_host: host buffers in and out, the rows in chunks
whose copies in, compute and copies out overlap on separate streams.  Rows are
independent through the whole linear, so the chunked result equals the
device-resident call on the same input bit for bit (that call is checked
against the oracle in test_gpu_parity.py)."""
import numpy as np
import pytest
import torch

from w8a8_int8_quantized_block_b200 import convrot as C
from w8a8_int8_quantized_block_b200 import workloads as W

pytestmark = pytest.mark.gpu
DEV = "cuda"


@pytest.mark.parametrize("M,gelu", [(7000, False), (6657, True), (700, False)])
def test_host_pipeline_equals_device_call(M, gelu):
    # K = 5376: 3328 rows per 32 MiB chunk, so 7000 and 6657 rows run in three
    # chunks (the last one ragged, down to a single row) and 700 rows in one piece
    K, N = 5376, 320
    spec, (x, w, bias) = W.custom_linear(M, K, N, seed=M + 3)
    pw = C.pack_weight(w.to(DEV), 128)
    b = bias.to(DEV)
    ws = C.alloc_workspace(M, K)
    y_ref = C.linear_fused(x.to(DEV), pw, b, gelu=gelu, workspace=ws)
    x_host = x.contiguous().pin_memory()
    y_host = torch.empty(M, N, dtype=torch.bfloat16).pin_memory()
    x_dev = torch.empty(M, K, dtype=torch.bfloat16, device=DEV)
    y_dev = torch.empty(M, N, dtype=torch.bfloat16, device=DEV)
    stream = torch.cuda.current_stream()
    for _ in range(2):  # twice in a row: the second call reuses the library's streams and events
        y_host.zero_()
        C.linear_fused_host(x_host, pw, b, gelu, x_dev, ws, y_dev, y_host, stream=stream)
        stream.synchronize()
        assert C.last_device_status() == (C.OK, 0)
        assert np.array_equal(y_host.view(torch.int16).numpy(), y_ref.cpu().view(torch.int16).numpy())
