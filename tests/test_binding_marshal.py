"""The Python binding passes every library call the argument list its C
signature declares, on the tensors' device (CPU only).

A fake library stands in for libaxr: it records each call.  torch's CUDA device
guard and current stream, and the binding's CUDA-tensor check, are stubbed so
that the binding's own code runs on CPU tensors.  No kernel runs here; the GPU
tests cover the real calls.
"""
import contextlib

import pytest
import torch

from lut_attention_b200 import axr, workloads


class _FakeLib:
    def __init__(self):
        self.calls = []

    def __getattr__(self, name):
        def fn(*args):
            self.calls.append((name, args))
            return axr.AXR_OK
        return fn


class _Stream:
    cuda_stream = 12345


@pytest.fixture
def fake(monkeypatch):
    lib = _FakeLib()
    devices = []

    @contextlib.contextmanager
    def device(d):
        devices.append(d)
        yield

    monkeypatch.setattr(axr, "library", lambda: lib)
    monkeypatch.setattr(axr, "_require_cuda", lambda t, name: None)
    monkeypatch.setattr(torch.cuda, "device", device)
    monkeypatch.setattr(torch.cuda, "current_stream", lambda dev=None: _Stream())
    lib.devices = devices
    return lib


def _check(lib, name, expect):
    """The last call is `name`, with as many arguments as its C signature and the
    given values at the given positions; the stream comes last."""
    got, args = lib.calls[-1]
    assert got == name
    assert len(args) == len(axr.SIGNATURES[name][1]), (name, len(args))
    for pos, val in expect.items():
        assert args[pos] == val, (name, pos, args[pos], val)
    assert args[-1] == _Stream.cuda_stream
    assert lib.devices and lib.devices[-1] == torch.device("cpu")


def test_write_and_read_calls(fake):
    d, b, heads, group, n = 128, 4, 3, 4, 257
    K = torch.zeros((heads, n, d), dtype=torch.bfloat16)
    signs = torch.ones(d, dtype=torch.int8)
    idx, norms = axr.axr_quantize_keys(K, b, signs)
    assert idx.shape == (heads, n, d * b // 8) and norms.shape == (heads, n)
    _check(fake, "axr_quantize_keys", {1: axr.AXR_BF16, 2: heads * n, 3: d, 4: b})
    q = torch.zeros((heads * group, d), dtype=torch.float16)
    scores = axr.axr_scores(q, idx, norms, group, b, signs)
    assert scores.shape == (heads * group, n)
    _check(fake, "axr_scores", {1: axr.AXR_F16, 4: n, 5: heads, 6: group, 7: d, 8: b})


def test_block_calls(fake):
    d, b, heads, group, n = 64, 3, 2, 2, 100
    quats = workloads.make_block_quats(workloads.GQA_DECODE_128K.with_(d=d))
    K = torch.zeros((heads, n, d), dtype=torch.float32)
    idx, norms = axr.axr_quantize_keys_block(K, b, quats)
    _check(fake, "axr_quantize_keys_block", {1: axr.AXR_F32, 2: heads * n, 3: d, 4: b})
    q = torch.zeros((heads * group, d), dtype=torch.float32)
    axr.axr_scores_block(q, idx, norms, group, b, quats)
    _check(fake, "axr_scores_block", {4: n, 5: heads, 6: group, 7: d, 8: b})


def test_decode_step_and_attention_calls(fake):
    d, b, heads, group, cap, pos = 128, 2, 2, 4, 300, 77
    idx = torch.zeros((heads, cap, d * b // 8), dtype=torch.uint8)
    norms = torch.zeros((heads, cap), dtype=torch.float32)
    signs = torch.ones(d, dtype=torch.int8)
    k_new = torch.zeros((heads, d), dtype=torch.bfloat16)
    q = torch.zeros((heads * group, d), dtype=torch.bfloat16)
    scores = axr.axr_append_scores(k_new, q, idx, norms, pos, group, b, signs)
    assert scores.shape == (heads * group, pos + 1)
    _check(fake, "axr_append_scores", {6: cap, 7: pos, 8: heads, 9: group, 10: d, 11: b})
    V = torch.zeros((heads, cap, d), dtype=torch.bfloat16)
    out, sc = axr.axr_attention(q, idx, norms, V, group, b, signs)
    assert out.shape == (heads * group, d) and sc.shape == (heads * group, cap)
    _check(fake, "axr_attention", {6: cap, 7: heads, 8: group, 9: d, 10: b})
    axr.axr_attention_static(q, idx, norms, V, group, b, signs, sc, out)
    _check(fake, "axr_attention_static", {6: cap, 7: heads, 8: group, 9: d, 10: b})


def test_sign_choice_call(fake):
    S, H, G, n, d, b, C = 2, 3, 4, 50, 64, 4, 5
    K = torch.zeros((S, H, n, d), dtype=torch.float32)
    q = torch.zeros((S, H * G, d), dtype=torch.float32)
    cand = torch.ones((C, d), dtype=torch.int8)
    errors, best = axr.axr_select_signs(K, q, G, b, cand)
    assert errors.shape == (C, H) and best.shape == (1,)
    _check(fake, "axr_select_signs", {4: n, 5: S, 6: H, 7: G, 8: d, 9: b, 11: C})
