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


def _decode_inputs(d=128, b=4, heads=2, group=4, n=300):
    idx = torch.zeros((heads, n, d * b // 8), dtype=torch.uint8)
    norms = torch.zeros((heads, n), dtype=torch.float32)
    q = torch.zeros((heads * group, d), dtype=torch.bfloat16)
    V = torch.zeros((heads, n, d), dtype=torch.bfloat16)
    scores = torch.zeros((heads * group, n), dtype=torch.float32)
    out = torch.zeros((heads * group, d), dtype=torch.float32)
    return idx, norms, q, V, scores, out


def test_static_attention_refuses_wrongly_typed_operands(fake):
    """The kernels read 4*n bytes of norms and n*P bytes of codes through raw
    pointers: a half-precision norms tensor of the right shape would be read past
    its end, so the binding refuses it before any call."""
    d, b, group = 128, 4, 4
    idx, norms, q, V, scores, out = _decode_inputs(d, b, group=group)
    signs = torch.ones(d, dtype=torch.int8)
    for bad in (dict(norms=norms.half()), dict(norms=norms.bfloat16()), dict(idx=idx.to(torch.int16)),
                dict(signs=signs.to(torch.int32))):
        a = dict(idx=idx, norms=norms, signs=signs) | bad
        with pytest.raises(ValueError):
            axr.axr_attention_static(q, a["idx"], a["norms"], V, group, b, a["signs"], scores, out)
    assert not fake.calls


def test_every_call_refuses_a_short_sign_pattern(fake):
    """The kernels read d entries of the sign pattern D."""
    d, b, group = 128, 4, 4
    idx, norms, q, V, scores, out = _decode_inputs(d, b, group=group)
    short = torch.ones(d - 1, dtype=torch.int8)
    K = torch.zeros((5, d), dtype=torch.bfloat16)
    k_new = torch.zeros((idx.shape[0], d), dtype=torch.bfloat16)
    calls = [
        lambda: axr.axr_quantize_keys(K, b, short),
        lambda: axr.axr_scores(q, idx, norms, group, b, short),
        lambda: axr.axr_append_scores(k_new, q, idx, norms, 3, group, b, short),
        lambda: axr.axr_attention(q, idx, norms, V, group, b, short),
        lambda: axr.axr_attention_static(q, idx, norms, V, group, b, short, scores, out),
    ]
    for call in calls:
        with pytest.raises(ValueError, match="signs"):
            call()
    assert not fake.calls


def test_read_calls_refuse_wrongly_typed_codes_and_norms(fake):
    d, b, group = 128, 4, 4
    idx, norms, q, V, scores, out = _decode_inputs(d, b, group=group)
    signs = torch.ones(d, dtype=torch.int8)
    quats = workloads.make_block_quats(workloads.GQA_DECODE_128K.with_(d=d))
    k_new = torch.zeros((idx.shape[0], d), dtype=torch.bfloat16)
    for bad_idx, bad_norms in ((idx, norms.half()), (idx.to(torch.int8), norms)):
        calls = [
            lambda: axr.axr_scores(q, bad_idx, bad_norms, group, b, signs),
            lambda: axr.axr_scores_block(q, bad_idx, bad_norms, group, b, quats),
            lambda: axr.axr_append_scores(k_new, q, bad_idx, bad_norms, 3, group, b, signs),
            lambda: axr.axr_attention(q, bad_idx, bad_norms, V, group, b, signs),
            lambda: axr.axr_quantize_keys(torch.zeros((idx.shape[0], idx.shape[1], d), dtype=torch.bfloat16),
                                          b, signs, idx=bad_idx, norms=bad_norms),
        ]
        for call in calls:
            with pytest.raises(ValueError):
                call()
    assert not fake.calls
