"""Host-side tests of the C ABI: the library loads, exports every symbol the
header declares, and rejects bad arguments before touching the GPU."""
import ctypes
import os
import re

import pytest

from w8a8_int8_quantized_block_b200 import convrot as C

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "convrot.h")


def _declared_symbols():
    src = open(HEADER).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"\b(convrot_[a-z0-9_]+)\s*\(", src)))


def test_library_builds_and_exports_every_declared_symbol():
    L = C.load()
    declared = _declared_symbols()
    assert len(declared) >= 13
    for name in declared:
        assert hasattr(L, name), name
    assert sorted(C.EXPORTS) == declared


def test_library_matches_its_sources():
    # the library that loads is the one built from the sources in this tree
    # (a compile or link failure raises instead of leaving an older library)
    from w8a8_int8_quantized_block_b200 import build as B
    C.load()
    assert B.is_current()


def test_abi_version_and_status_strings():
    L = C.load()
    assert L.convrot_abi_version() == 1
    for st in range(6):
        s = L.convrot_status_string(st)
        assert isinstance(s, bytes) and len(s) > 0
    assert L.convrot_status_string(99) == b"unknown status"


def test_workspace_bytes():
    L = C.load()
    # scales, two counters per 256-row panel plus one, then the codes, each
    # rounded to 256 bytes; the codes are the whole [M][K] array (either path)
    # or the one-kernel path's ring of min(M, slots * 256) rows
    r = lambda v: (v + 255) // 256 * 256
    head = r(38656 * 4) + r((2 * 151 + 1) * 4)
    assert L.convrot_workspace_bytes(38656, 5376) == head + 38656 * 5376
    assert L.convrot_fused_workspace_bytes(38656, 5376) == head + 12 * 256 * 5376   # 12 slots, ~17 MB
    assert L.convrot_fused_workspace_bytes(38656, 6144) == r(38656 * 4) + r(303 * 4) + 10 * 256 * 6144
    assert L.convrot_fused_workspace_bytes(38656, 512) == r(38656 * 4) + r(303 * 4) + 12 * 256 * 512
    assert L.convrot_fused_workspace_bytes(38656, 21504) == L.convrot_workspace_bytes(38656, 21504)  # two kernels
    assert L.convrot_fused_workspace_bytes(1000, 5376) == L.convrot_workspace_bytes(1000, 5376)  # 4 panels fit
    assert L.convrot_fused_workspace_bytes(3073, 5376) == r(3073 * 4) + r(27 * 4) + 12 * 256 * 5376
    assert L.convrot_workspace_bytes(1, 128) == 256 + 256 + 256
    assert L.convrot_workspace_bytes(0, 128) == 0 and L.convrot_fused_workspace_bytes(0, 128) == 0


def test_noalloc_limits_follow_the_path():
    # the allocation-free entry point's 32 MiB scratch holds the workspace of
    # the path taken: the whole codes array on the two-kernel path, the ring on
    # the one-kernel path
    L, lim = C.load(), 32 << 20
    assert L.convrot_workspace_bytes(6236, 5376) <= lim < L.convrot_workspace_bytes(6237, 5376)
    assert L.convrot_workspace_bytes(1560, 21504) <= lim < L.convrot_workspace_bytes(1561, 21504)
    assert L.convrot_fused_workspace_bytes(4_000_000, 5376) <= lim < L.convrot_fused_workspace_bytes(4_300_000, 5376)


FAKE = ctypes.c_void_p(0x100000)  # never dereferenced: validation fails first


@pytest.mark.parametrize("M,K,ldx,block,expect", [
    (0, 512, 512, 128, C.EINVAL),
    (-3, 512, 512, 128, C.EINVAL),
    (4, 100, 100, 0, C.EINVAL),        # K % 64
    (4, 192, 192, 128, C.EINVAL),      # K % block
    (4, 512, 500, 128, C.EINVAL),      # ldx < K
    (4, 512, 516, 128, C.EINVAL),      # ldx % 8
    (4, 65536, 65536, 128, C.EINVAL),  # K too large
    (4, 512, 512, 32, C.EUNSUPPORTED),                # no 32-point rotation
    (4, 512, 512, 512, C.EUNSUPPORTED),
    (4, 512, 512, C.REGULAR | 128, C.EUNSUPPORTED),   # no regular Hadamard of order 128
    (4, 512, 512, C.REGULAR, C.EUNSUPPORTED),
    (4, 384, 384, 256, C.EINVAL),                     # K % 256
    (4, 384, 384, C.REGULAR | 256, C.EINVAL),
])
def test_quantize_act_rejects_bad_arguments(M, K, ldx, block, expect):
    st = C.load().convrot_quantize_act(FAKE, M, K, ldx, block, FAKE, FAKE, None)
    assert st == expect


def _skip_if_gpu():
    # With a GPU these calls would pass validation and launch on fake pointers.
    try:
        import torch
        if torch.cuda.is_available():
            pytest.skip("a GPU is present")
    except ImportError:
        pass


@pytest.mark.parametrize("block", C.BLOCKS)
def test_every_block_value_passes_validation(block):
    # a valid block gets past the argument checks to the device query, which
    # fails without a GPU: ECUDA, never EUNSUPPORTED or EINVAL
    _skip_if_gpu()
    st = C.load().convrot_quantize_act(FAKE, 4, 512, 512, block, FAKE, FAKE, None)
    assert st == C.ECUDA


def test_regular_flag_matches_the_header():
    hdr = open(os.path.join(ROOT, "include", "convrot.h")).read()
    m = re.search(r"#define CONVROT_HADAMARD_REGULAR (0x[0-9a-fA-F]+)", hdr)
    assert m and int(m.group(1), 16) == C.REGULAR
    assert [C.block_length(b) for b in C.BLOCKS] == [1, 64, 128, 256, 16, 64, 256]


def test_activation_prologue_rejects_bad_arguments():
    L = C.load()
    # unknown activation, and "none" (that is convrot_quantize_act's job)
    assert L.convrot_act_quantize(FAKE, 4, 512, 512, 7, 128, FAKE, FAKE, None) == C.EINVAL
    assert L.convrot_act_quantize(FAKE, 4, 512, 512, C.ACT_NONE, 128, FAKE, FAKE, None) == C.EINVAL
    # SwiGLU rows hold 2K elements: ldh must reach them
    assert L.convrot_act_quantize(FAKE, 4, 512, 512, C.ACT_SWIGLU, 128, FAKE, FAKE, None) == C.EINVAL
    assert L.convrot_act_quantize(FAKE, 4, 512, 512, C.ACT_GELU, 32, FAKE, FAKE, None) == C.EUNSUPPORTED
    d = _desc()
    assert L.convrot_linear_act(FAKE, 16, 512, 9, FAKE, FAKE, ctypes.byref(d), None, 0, FAKE, 1 << 20, FAKE, 512,
                                None) == C.EINVAL
    assert L.convrot_linear_act(FAKE, 16, 512, C.ACT_GELU, FAKE, FAKE, ctypes.byref(d), None, 0, FAKE, 16, FAKE,
                                512, None) == C.EINVAL  # workspace too small


def test_activation_prologue_valid_call_without_a_gpu_reports_cuda_error():
    _skip_if_gpu()
    L = C.load()
    assert L.convrot_act_quantize(FAKE, 4, 512, 1024, C.ACT_SWIGLU, 64, FAKE, FAKE, None) == C.ECUDA
    assert L.convrot_act_quantize(FAKE, 4, 512, 512, C.ACT_GELU, C.REGULAR | 256, FAKE, FAKE, None) == C.ECUDA


def test_null_pointers_rejected():
    L = C.load()
    assert L.convrot_quantize_act(None, 4, 512, 512, 128, FAKE, FAKE, None) == C.EINVAL
    assert L.convrot_pack_weight(FAKE, 4, 512, 128, FAKE, FAKE, None, None) == C.EINVAL
    assert L.convrot_igemm_s32(None, FAKE, 1, 4, 4, 16, FAKE, None) == C.EINVAL
    assert L.convrot_w8a8_bmm(FAKE, None, FAKE, FAKE, 1, 4, 8, 16, FAKE, None) == C.EINVAL


def test_misaligned_pointer_rejected():
    L = C.load()
    bad = ctypes.c_void_p(0x100008)
    assert L.convrot_quantize_act(bad, 4, 512, 512, 128, FAKE, FAKE, None) == C.EINVAL
    assert L.convrot_igemm_s32(FAKE, bad, 1, 4, 4, 16, FAKE, None) == C.EINVAL


def test_codes_output_must_be_32_byte_aligned():
    # the quantisers write the codes in 32-byte stores: a codes pointer that is
    # only 16-byte aligned is refused before any device work
    L = C.load()
    q16 = ctypes.c_void_p(0x100010)
    assert L.convrot_quantize_act(FAKE, 4, 512, 512, 128, q16, FAKE, None) == C.EINVAL
    assert L.convrot_pack_weight(FAKE, 4, 512, 128, q16, FAKE, ctypes.byref(C.WDesc()), None) == C.EINVAL
    assert L.convrot_act_quantize(FAKE, 4, 512, 512, C.ACT_GELU, 128, q16, FAKE, None) == C.EINVAL
    # a 32-byte aligned codes pointer passes validation: without a GPU the
    # device query fails (ECUDA); with one, the fake pointers must not launch
    _skip_if_gpu()
    q32 = ctypes.c_void_p(0x100020)
    assert L.convrot_quantize_act(FAKE, 4, 512, 512, 128, q32, FAKE, None) == C.ECUDA


def _desc(**kw):
    d = C.WDesc(C.WDESC_MAGIC, C.WDESC_VERSION, C.LAYOUT_OUTPUT_MAJOR, 128, 512, 512)
    for k, v in kw.items():
        setattr(d, k, v)
    return d


@pytest.mark.parametrize("field,value", [("magic", 0x12345678), ("version", 2), ("layout", 0), ("block", 32),
                                         ("block", C.REGULAR | 128), ("N", 0), ("K", 100), ("K", 320)])
def test_bad_weight_descriptor_is_a_layout_error(field, value):
    d = _desc(**{field: value})
    st = C.load().convrot_w8a8_linear(FAKE, FAKE, FAKE, FAKE, ctypes.byref(d), None, 0, 16, FAKE, 512, None)
    assert st == C.ELAYOUT


def test_linear_rejects_bad_output_stride_and_epilogue():
    L = C.load()
    d = _desc()
    assert L.convrot_w8a8_linear(FAKE, FAKE, FAKE, FAKE, ctypes.byref(d), None, 0, 16, FAKE, 500, None) == C.EINVAL
    assert L.convrot_w8a8_linear(FAKE, FAKE, FAKE, FAKE, ctypes.byref(d), None, 7, 16, FAKE, 512, None) == C.EINVAL
    ws = ctypes.c_void_p(0x100000)
    assert L.convrot_linear_fused(FAKE, 16, 512, FAKE, FAKE, ctypes.byref(d), None, 0, ws, 10, FAKE, 512,
                                  None) == C.EINVAL


def test_bmm_and_igemm_shape_rules():
    L = C.load()
    assert L.convrot_w8a8_bmm(FAKE, FAKE, FAKE, FAKE, 1, 4, 12, 16, FAKE, None) == C.EINVAL   # N % 8
    assert L.convrot_w8a8_bmm(FAKE, FAKE, FAKE, FAKE, 1, 4, 16, 24, FAKE, None) == C.EINVAL   # K % 16
    assert L.convrot_igemm_s32(FAKE, FAKE, 0, 4, 4, 16, FAKE, None) == C.EINVAL
    assert L.convrot_igemm_s32(FAKE, FAKE, 1, 4, 6, 16, FAKE, None) == C.EINVAL               # N % 4


def test_valid_call_without_a_gpu_reports_cuda_error():
    _skip_if_gpu()
    st = C.load().convrot_quantize_act(FAKE, 4, 512, 512, 128, FAKE, FAKE, None)
    assert st == C.ECUDA
