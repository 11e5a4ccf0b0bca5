"""Parity of decode attention (axr_attention) with the CPU oracle.

Two comparisons:
  * the softmax and value sum alone: the oracle's attention of the GPU's own
    scores; only fp32 arithmetic separates the two, so the bound is
    ATTN_TOL * max |V| of the head;
  * end to end: the oracle's attention of the oracle's scores.  Scores may differ
    by at most delta = 1e-4 * ||q|| * max_t ||k_t|| / sqrt(d) (the score bound), which
    moves every softmax weight by a factor within e^(+-2 delta), hence the output
    by at most (e^(2 delta) - 1) * max |V|; ATTN_TOL * max |V| is added for fp32.
"""
import math

import numpy as np
import pytest
import torch

import oracle
from lut_attention_b200 import axr, workloads

pytestmark = pytest.mark.gpu
DEV = "cuda"
ATTN_TOL = 2e-5


@pytest.fixture(autouse=True, scope="module")
def _libs(axr_lib, oracle_lib):
    return axr_lib


def _inputs(heads, n, d, b, group, vdtype, seed):
    packed, norms = workloads.make_random_packed(heads, n, d, b, seed=seed, device=DEV)
    wl = workloads.GQA_DECODE_128K.with_(d=d, batch=1, kv_heads=heads, group=group, T=n, seed=seed)
    q = workloads.make_queries(wl, DEV)
    s = workloads.make_signs(wl).to(DEV)
    g = torch.Generator(device=DEV).manual_seed(seed + 991)
    V = torch.randn((heads, n, d), generator=g, device=DEV).to(getattr(torch, vdtype))
    return packed, norms, q, s, V


def _check(q, packed, norms, V, out, scores, group, b, s):
    d = q.shape[1]
    heads = V.shape[0]
    Vh = V.cpu().double().numpy()
    vmax = np.abs(Vh).reshape(heads, -1).max(axis=1).repeat(group)[:, None]
    got = out.cpu().double().numpy()
    # 1. softmax and value sum of the GPU's own scores
    own = oracle.attention_from_scores(scores.cpu().double().numpy(), Vh, group)
    assert np.all(np.abs(got - own) <= ATTN_TOL * vmax), float((np.abs(got - own) / vmax).max())
    # 2. end to end, within the bound the score tolerance implies
    exp = oracle.attention(q.cpu().double().numpy(), packed.cpu().numpy(), norms.cpu().numpy(), Vh, group, b,
                           s.cpu().numpy())
    qn = np.linalg.norm(q.cpu().double().numpy(), axis=1)
    kmax = norms.cpu().double().numpy().max(axis=1).repeat(group)
    delta = 1e-4 * qn * kmax / math.sqrt(d)
    bound = (np.expm1(2 * delta)[:, None] + ATTN_TOL) * vmax
    assert np.all(np.abs(got - exp) <= bound), float((np.abs(got - exp) / bound).max())


@pytest.mark.parametrize("d,b,group,vdtype,n", [
    (128, 4, 4, "bfloat16", 5000), (128, 3, 1, "float16", 1025), (128, 2, 8, "bfloat16", 3000),
    (128, 4, 3, "float32", 777), (64, 3, 2, "bfloat16", 4097), (32, 2, 5, "float16", 300),
    (256, 2, 2, "float16", 2100), (512, 2, 8, "float16", 700),
])
def test_attention_parity(d, b, group, vdtype, n):
    heads = 3
    packed, norms, q, s, V = _inputs(heads, n, d, b, group, vdtype, seed=d + n + group)
    out, scores = axr.axr_attention(q, packed, norms, V, group, b, s)
    assert axr.axr_device_status() == 0
    _check(q, packed, norms, V, out, scores, group, b, s)


def test_attention_of_one_key_is_its_value_row():
    heads, d, b, group = 4, 128, 4, 4
    packed, norms, q, s, V = _inputs(heads, 1, d, b, group, "bfloat16", seed=3)
    out, _ = axr.axr_attention(q, packed, norms, V, group, b, s)
    want = V[:, 0].float().repeat_interleave(group, dim=0)
    assert torch.equal(out, want)


def test_attention_full_context_two_heads():
    """Two KV heads of the 128k-context GQA shape (bf16 values), compared whole."""
    wl = workloads.GQA_DECODE_128K
    heads = 2
    packed, norms, q, s, V = _inputs(heads, wl.T, wl.d, wl.b, wl.group, "bfloat16", seed=11)
    out, scores = axr.axr_attention(q, packed, norms, V, wl.group, wl.b, s)
    assert axr.axr_device_status() == 0
    _check(q, packed, norms, V, out, scores, wl.group, wl.b, s)


def test_caller_workspace_and_streams():
    """A workspace from the caller, on a side stream, gives the same output as the
    binding's own allocation on the default stream."""
    heads, n, d, b, group = 2, 3000, 128, 4, 4
    packed, norms, q, s, V = _inputs(heads, n, d, b, group, "bfloat16", seed=21)
    ref, _ = axr.axr_attention(q, packed, norms, V, group, b, s)
    ws = torch.full((axr.axr_attention_workspace_bytes(n, heads, group, d),), 0x7F, dtype=torch.uint8,
                    device=DEV)
    st = torch.cuda.Stream()
    st.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(st):
        out, _ = axr.axr_attention(q, packed, norms, V, group, b, s, workspace=ws, stream=st)
    st.synchronize()
    assert torch.equal(out, ref)
