"""The C ABI on the host: the library loads, exports every symbol include/axr.h
declares, and rejects bad arguments before touching the GPU.  No kernel runs here."""
import ctypes
import os
import re

import numpy as np
import pytest
import torch

import oracle
from lut_attention_b200 import axr

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "axr.h")


def declared_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(axr_\w+)\s*\(", text)))


def test_header_declares_the_boundary():
    names = declared_functions()
    for required in ("axr_make_codebook", "axr_quantize_keys", "axr_scores", "axr_status_string"):
        assert required in names


def test_library_exports_every_declared_symbol(axr_lib):
    names = declared_functions()
    assert names
    for name in names:
        assert hasattr(axr_lib, name), name
        assert name in axr.SIGNATURES, name


def test_status_strings(axr_lib):
    for code in (0, -1, -2, -3):
        assert axr_lib.axr_status_string(code).startswith(b"AXR_")
    assert axr_lib.axr_version() >= 100


@pytest.mark.parametrize("d", [8, 16, 32, 64, 128, 256, 512])
@pytest.mark.parametrize("b", [1, 2, 3, 4])
def test_library_codebook_equals_oracle_codebook(axr_lib, d, b):
    """The library solves Lloyd-Max itself (positive half-line, long double); its
    fp32 codebook must equal the oracle's bit for bit."""
    c1, b1 = axr.axr_make_codebook(d, b)
    c2, b2 = oracle.codebook(d, b)
    assert np.array_equal(c1.view(np.uint32), c2.view(np.uint32))
    assert np.array_equal(b1.view(np.uint32), b2.view(np.uint32))


@pytest.mark.parametrize("d,b", [(100, 4), (4, 2), (1024, 2), (128, 0), (128, 5)])
def test_make_codebook_rejects_unsupported(axr_lib, d, b):
    cent = np.zeros(32, np.float32)
    assert axr_lib.axr_make_codebook(d, b, cent.ctypes.data, None) == axr.AXR_EUNSUPPORTED


def test_make_codebook_null_output(axr_lib):
    assert axr_lib.axr_make_codebook(128, 4, None, None) == axr.AXR_EINVAL


def test_quantize_argument_errors(axr_lib):
    q = axr_lib.axr_quantize_keys
    host = np.zeros(4096, np.uint8)
    p = host.ctypes.data
    assert q(p, 2, 10, 100, 4, p, p, p, None) == axr.AXR_EUNSUPPORTED    # d not a power of two
    assert q(p, 2, 10, 128, 5, p, p, p, None) == axr.AXR_EUNSUPPORTED    # b > 4
    assert q(p, 7, 10, 128, 4, p, p, p, None) == axr.AXR_EINVAL          # bad dtype
    assert q(p, 2, -1, 128, 4, p, p, p, None) == axr.AXR_EINVAL          # n < 0
    assert q(None, 2, 0, 128, 4, None, None, None, None) == axr.AXR_OK   # n == 0: no-op
    assert q(None, 2, 10, 128, 4, p, p, p, None) == axr.AXR_EINVAL       # NULL K
    assert q(p + 1, 2, 10, 128, 4, p, p, p, None) == axr.AXR_EINVAL      # misaligned K
    assert q(p, 2, 10, 128, 4, p, p, p, None) == axr.AXR_EINVAL          # host (not device) memory
    assert b"device" in axr_lib.axr_last_error()


def test_scores_argument_errors(axr_lib):
    s = axr_lib.axr_scores
    host = np.zeros(4096, np.uint8)
    p = host.ctypes.data
    assert s(p, 2, p, p, 10, 1, 9, 128, 4, p, p, None) == axr.AXR_EUNSUPPORTED  # group > 8
    assert s(p, 2, p, p, 10, 0, 1, 128, 4, p, p, None) == axr.AXR_EINVAL       # heads < 1
    assert s(p, 2, p, p, 10, 1, 0, 128, 4, p, p, None) == axr.AXR_EINVAL       # group < 1
    assert s(p, 2, p, p, 10, 1, 1, 96, 4, p, p, None) == axr.AXR_EUNSUPPORTED  # d
    assert s(p, 3, p, p, 10, 1, 1, 128, 4, p, p, None) == axr.AXR_EINVAL       # dtype
    assert s(None, 2, None, None, 0, 1, 1, 128, 4, None, None, None) == axr.AXR_OK
    assert s(p, 2, p + 8, p, 10, 1, 1, 128, 4, p, p, None) == axr.AXR_EINVAL   # misaligned idx
    assert s(p, 2, p, p, 10, 1, 1, 128, 4, p, p, None) == axr.AXR_EINVAL       # host memory


def test_append_argument_errors(axr_lib):
    f = axr_lib.axr_append_scores
    host = np.zeros(4096, np.uint8)
    p = host.ctypes.data
    # (k_new, kdtype, q, qdtype, idx, norms, capacity, pos, heads, group, d, b, signs, scores, stream)
    assert f(p, 2, p, 2, p, p, 16, 16, 1, 1, 128, 4, p, p, None) == axr.AXR_EINVAL        # pos == capacity
    assert f(p, 2, p, 2, p, p, 16, -1, 1, 1, 128, 4, p, p, None) == axr.AXR_EINVAL        # pos < 0
    assert f(p, 2, p, 2, p, p, 0, 0, 1, 1, 128, 4, p, p, None) == axr.AXR_EINVAL          # empty cache
    assert f(p, 2, p, 2, p, p, 16, 3, 0, 1, 128, 4, p, p, None) == axr.AXR_EINVAL         # heads < 1
    assert f(p, 2, p, 2, p, p, 16, 3, 1, 9, 128, 4, p, p, None) == axr.AXR_EUNSUPPORTED   # group > 8
    assert f(p, 2, p, 2, p, p, 16, 3, 1, 1, 96, 4, p, p, None) == axr.AXR_EUNSUPPORTED    # d
    assert f(p, 5, p, 2, p, p, 16, 3, 1, 1, 128, 4, p, p, None) == axr.AXR_EINVAL         # key dtype
    assert f(p, 2, p, 7, p, p, 16, 3, 1, 1, 128, 4, p, p, None) == axr.AXR_EINVAL         # query dtype
    assert f(p + 4, 2, p, 2, p, p, 16, 3, 1, 1, 128, 4, p, p, None) == axr.AXR_EINVAL     # misaligned k_new
    assert f(p, 2, p, 2, p, p, 16, 3, 1, 1, 128, 4, p, p, None) == axr.AXR_EINVAL         # host memory


def test_attention_workspace_and_argument_errors(axr_lib):
    # 32 heads x 64 chunks of 1024 keys x 4 queries x (128 + 2) floats
    assert axr.axr_attention_workspace_bytes(131072, 32, 4, 128) == 32 * 128 * 4 * 130 * 4
    assert axr.axr_attention_workspace_bytes(1, 1, 3, 64) == 1 * 1 * 4 * 66 * 4      # group padded to 4
    out = ctypes.c_int64(0)
    assert axr_lib.axr_attention_workspace_bytes(100, 1, 1, 16, ctypes.byref(out)) == axr.AXR_EUNSUPPORTED
    f = axr_lib.axr_attention
    host = np.zeros(4096, np.uint8)
    p = host.ctypes.data
    # (q, qdt, idx, norms, V, vdt, n, heads, group, d, b, signs, scores, ws, ws_bytes, out, stream)
    assert f(p, 2, p, p, p, 2, 0, 1, 1, 128, 4, p, p, p, 1 << 20, p, None) == axr.AXR_EINVAL       # n = 0
    assert f(p, 2, p, p, p, 2, 10, 1, 1, 16, 4, p, p, p, 1 << 20, p, None) == axr.AXR_EUNSUPPORTED  # d < 32
    assert f(p, 2, p, p, p, 9, 10, 1, 1, 128, 4, p, p, p, 1 << 20, p, None) == axr.AXR_EINVAL      # V dtype
    assert f(p, 2, p, p, p, 2, 10, 1, 1, 128, 4, p, p, p, 8, p, None) == axr.AXR_EINVAL            # workspace
    assert f(p, 2, p, p, p, 2, 10, 1, 1, 128, 4, p, p, p, 1 << 20, p, None) == axr.AXR_EINVAL      # host memory


def test_select_signs_argument_errors(axr_lib):
    f = axr_lib.axr_select_signs
    host = np.zeros(4096, np.uint8)
    p = host.ctypes.data
    # (K, kdt, q, qdt, n, samples, heads, group, d, b, candidates, C, errors, best, stream)
    assert f(p, 2, p, 2, 0, 8, 8, 4, 128, 4, p, 200, p, p, None) == axr.AXR_EINVAL            # no keys
    assert f(p, 2, p, 2, 64, 0, 8, 4, 128, 4, p, 200, p, p, None) == axr.AXR_EINVAL           # samples
    assert f(p, 2, p, 2, 64, 8, 0, 4, 128, 4, p, 200, p, p, None) == axr.AXR_EINVAL           # heads
    assert f(p, 2, p, 2, 64, 8, 8, 0, 128, 4, p, 200, p, p, None) == axr.AXR_EINVAL           # group
    assert f(p, 2, p, 2, 64, 8, 8, 4, 128, 4, p, 0, p, p, None) == axr.AXR_EINVAL             # no candidates
    assert f(p, 2, p, 2, 64, 8, 8, 9, 128, 4, p, 200, p, p, None) == axr.AXR_EUNSUPPORTED     # group > 8
    assert f(p, 2, p, 2, 64, 8, 8, 4, 100, 4, p, 200, p, p, None) == axr.AXR_EUNSUPPORTED     # d
    assert f(p, 2, p, 2, 64, 8, 8, 4, 128, 5, p, 200, p, p, None) == axr.AXR_EUNSUPPORTED     # b
    assert f(p, 2, p, 2, 64, 8, 1 << 20, 4, 128, 4, p, 1 << 12, p, p, None) == axr.AXR_EINVAL  # 2^32 pairs
    assert f(p, 6, p, 2, 64, 8, 8, 4, 128, 4, p, 200, p, p, None) == axr.AXR_EINVAL           # key dtype
    assert f(p + 8, 2, p, 2, 64, 8, 8, 4, 128, 4, p, 200, p, p, None) == axr.AXR_EINVAL       # misaligned K
    assert f(p, 2, p, 2, 64, 8, 8, 4, 128, 4, p, 200, p, p, None) == axr.AXR_EINVAL           # host memory
    assert f(None, 2, p, 2, 64, 8, 8, 4, 128, 4, p, 200, p, p, None) == axr.AXR_EINVAL        # NULL K


def test_block_rotation_argument_errors(axr_lib):
    fq = axr_lib.axr_quantize_keys_block
    fs = axr_lib.axr_scores_block
    host = np.zeros(4096, np.uint8)
    p = host.ctypes.data
    # (K, kdt, n, d, b, quats, idx, norms, stream)
    assert fq(p, 2, 0, 128, 4, p, p, p, None) == axr.AXR_OK                  # n = 0: no-op
    assert fq(p, 2, -1, 128, 4, p, p, p, None) == axr.AXR_EINVAL             # n < 0
    assert fq(p, 2, 10, 96, 4, p, p, p, None) == axr.AXR_EUNSUPPORTED        # d
    assert fq(p, 2, 10, 128, 0, p, p, p, None) == axr.AXR_EUNSUPPORTED       # b
    assert fq(p, 4, 10, 128, 4, p, p, p, None) == axr.AXR_EINVAL             # key dtype
    assert fq(p, 2, 10, 128, 4, None, p, p, None) == axr.AXR_EINVAL          # NULL quats
    assert fq(p, 2, 10, 128, 4, p, p, p, None) == axr.AXR_EINVAL             # host memory
    # (q, qdt, idx, norms, n, heads, group, d, b, quats, scores, stream)
    assert fs(p, 2, p, p, 0, 1, 1, 128, 4, p, p, None) == axr.AXR_OK          # n = 0: no-op
    assert fs(p, 2, p, p, 10, 0, 1, 128, 4, p, p, None) == axr.AXR_EINVAL     # heads
    assert fs(p, 2, p, p, 10, 1, 9, 128, 4, p, p, None) == axr.AXR_EUNSUPPORTED   # group > 8
    assert fs(p, 2, p, p, 10, 1, 1, 128, 4, None, p, None) == axr.AXR_EINVAL  # NULL quats
    assert fs(p, 2, p, p, 10, 1, 1, 128, 4, p, p, None) == axr.AXR_EINVAL     # host memory


def test_binding_refuses_cpu_tensors():
    """No CPU path: the binding raises instead of computing on the host."""
    K = torch.zeros(4, 128)
    s = torch.ones(128, dtype=torch.int8)
    with pytest.raises(ValueError, match="CUDA"):
        axr.axr_quantize_keys(K, 4, s)
    with pytest.raises(ValueError, match="CUDA"):
        axr.axr_scores(torch.zeros(1, 128), torch.zeros(1, 4, 64, dtype=torch.uint8),
                       torch.zeros(1, 4), 1, 4, s)


def test_debug_library_exports_every_declared_symbol_and_says_so(axr_lib):
    """libaxr_debug.so (-DAXR_DEBUG) has the same boundary; axr_debug_build tells
    the two apart and the span slack exists only in the debug build."""
    from lut_attention_b200 import build

    if not os.path.exists(build.DEBUG_LIB_PATH):
        build.build(debug=True)
    dbg = ctypes.CDLL(build.DEBUG_LIB_PATH)
    for name in declared_functions():
        assert hasattr(dbg, name), name
    dbg.axr_debug_build.restype = ctypes.c_int
    dbg.axr_debug_set_span_slack.restype = ctypes.c_int
    dbg.axr_debug_set_span_slack.argtypes = [ctypes.c_int64]
    assert dbg.axr_debug_build() == 1
    assert dbg.axr_debug_set_span_slack(-1) == axr.AXR_EINVAL
    assert dbg.axr_debug_set_span_slack(4) == axr.AXR_OK
    assert dbg.axr_debug_set_span_slack(0) == axr.AXR_OK
    assert axr_lib.axr_debug_build() == int(axr.DEBUG)
    if not axr.DEBUG:
        assert axr_lib.axr_debug_set_span_slack(0) == axr.AXR_EUNSUPPORTED
        assert b"debug build" in axr_lib.axr_last_error()
