"""Parity of the decode step (axr_append_scores) with the CPU oracle.

The step quantizes one new key per KV head into slot pos of a key cache and
scores every query head against keys 0 .. pos.  The oracle side is the plain
composition of its quantizer and its scores; the cache rows outside slot pos
must come back untouched.
"""
import numpy as np
import pytest
import torch

from lut_attention_b200 import axr, workloads
from parity import check_quantize, check_scores

pytestmark = pytest.mark.gpu
DEV = "cuda"


@pytest.fixture(autouse=True, scope="module")
def _libs(axr_lib, oracle_lib):
    return axr_lib


def _cache(heads, capacity, pos, d, b, dtype, seed):
    """A cache of `capacity` slots per head whose first pos slots hold quantized
    keys; the slots from pos on hold sentinel bytes and norms."""
    wl = workloads.MHA_DECODE_32K.with_(d=d, dtype=dtype, T=pos + 1, batch=1, kv_heads=heads, seed=seed)
    keys = workloads.make_keys(wl, DEV)                        # (heads, pos + 1, d)
    s = workloads.make_signs(wl).to(DEV)
    P = d * b // 8
    idx = torch.full((heads, capacity, P), 0xA5, dtype=torch.uint8, device=DEV)
    norms = torch.full((heads, capacity), -7.0, dtype=torch.float32, device=DEV)
    if pos > 0:
        for h in range(heads):
            axr.axr_quantize_keys(keys[h, :pos].contiguous(), b, s, idx=idx[h, :pos], norms=norms[h, :pos])
    return keys, s, idx, norms


@pytest.mark.parametrize("d,b,group,dtype", [
    (128, 4, 4, "bf16"), (128, 3, 1, "f16"), (128, 2, 8, "bf16"), (128, 4, 2, "f32"),
    (64, 3, 4, "bf16"), (256, 2, 2, "f16"), (512, 2, 8, "f16"), (8, 1, 3, "f32"),
    (256, 4, 4, "bf16"), (256, 3, 8, "f32"), (256, 1, 1, "f16"), (512, 4, 4, "bf16"), (512, 3, 2, "f16"),
    (512, 1, 5, "f32"),
])
def test_append_then_scores(d, b, group, dtype):
    heads, capacity, pos = 3, 704, 517          # 704 * P bytes: every head 16-byte aligned
    keys, s, idx, norms = _cache(heads, capacity, pos, d, b, dtype, seed=d + b + group)
    before_idx, before_norms = idx.clone(), norms.clone()
    wl = workloads.GQA_DECODE_128K.with_(d=d, dtype=dtype, batch=1, kv_heads=heads, group=group, T=pos + 1)
    q = workloads.make_queries(wl, DEV)
    k_new = keys[:, pos].contiguous()
    out = axr.axr_append_scores(k_new, q, idx, norms, pos, group, b, s)
    assert axr.axr_device_status() == 0
    assert out.shape == (heads * group, pos + 1)
    # the new keys: slot pos, exactly as the quantizer defines them
    rep = check_quantize(k_new, idx[:, pos], norms[:, pos], b, s)
    assert rep.ok(), rep
    # every other slot untouched
    keep = torch.ones(capacity, dtype=torch.bool, device=DEV)
    keep[pos] = False
    assert torch.equal(idx[:, keep], before_idx[:, keep])
    assert torch.equal(norms[:, keep], before_norms[:, keep])
    # scores against keys 0 .. pos from the cache's own codes
    assert check_scores(q, idx[:, :pos + 1].contiguous(), norms[:, :pos + 1].contiguous(), out, group, b, s) <= 1e-4


@pytest.mark.parametrize("d", [128, 256, 512])
@pytest.mark.parametrize("pos,capacity", [(0, 1), (0, 300), (299, 300), (128, 129), (255, 1000)])
def test_append_edges_of_the_cache(d, pos, capacity):
    """Empty cache (pos 0), the last slot, and positions on tile edges."""
    b, group, heads = 4, 4, 2
    keys, s, idx, norms = _cache(heads, capacity, pos, d, b, "bf16", seed=pos + capacity + d)
    wl = workloads.GQA_DECODE_128K.with_(d=d, batch=1, kv_heads=heads, group=group, T=pos + 1)
    q = workloads.make_queries(wl, DEV)
    out = axr.axr_append_scores(keys[:, pos].contiguous(), q, idx, norms, pos, group, b, s)
    assert axr.axr_device_status() == 0
    assert check_quantize(keys[:, pos], idx[:, pos], norms[:, pos], b, s).ok()
    assert check_scores(q, idx[:, :pos + 1].contiguous(), norms[:, :pos + 1].contiguous(), out, group, b, s) <= 1e-4


def test_decode_loop_builds_the_cache_key_by_key():
    """Eight decode steps from an empty cache: each appends one key per head and
    scores against everything so far; the final cache equals the oracle's codes of
    all eight keys, and each step's scores cover exactly the keys written so far."""
    d, b, group, heads, steps, capacity = 128, 3, 4, 4, 8, 16
    keys, s, idx, norms = _cache(heads, capacity, 0, d, b, "bf16", seed=77)
    wl = workloads.MHA_DECODE_32K.with_(d=d, dtype="bf16", T=steps, batch=1, kv_heads=heads, seed=78)
    seq = workloads.make_keys(wl, DEV)                           # (heads, steps, d)
    q = workloads.make_queries(workloads.GQA_DECODE_128K.with_(batch=1, kv_heads=heads, group=group), DEV)
    for pos in range(steps):
        out = axr.axr_append_scores(seq[:, pos].contiguous(), q, idx, norms, pos, group, b, s)
        assert out.shape == (heads * group, pos + 1)
        assert check_scores(q, idx[:, :pos + 1].contiguous(), norms[:, :pos + 1].contiguous(), out,
                            group, b, s) <= 1e-4
    assert axr.axr_device_status() == 0
    rep = check_quantize(seq.reshape(-1, d), idx[:, :steps].reshape(-1, d * b // 8),
                         norms[:, :steps].reshape(-1), b, s)
    assert rep.ok(), rep
    assert torch.all(idx[:, steps:] == 0xA5)


@pytest.mark.parametrize("d,launches", [(128, 1), (256, 1), (512, 1), (64, 2)])
def test_decode_step_launch_count(d, launches):
    """At d = 128, 256 and 512 the decode step is one launch of the tensor-core
    read kernel, which quantizes the new keys itself; below 128 it is the write
    kernel followed by the read kernel."""
    from torch.profiler import ProfilerActivity, profile

    b, group, heads, pos, capacity = 4, 4, 2, 200, 256
    keys, s, idx, norms = _cache(heads, capacity, pos, d, b, "bf16", seed=d)
    q = workloads.make_queries(workloads.GQA_DECODE_128K.with_(d=d, batch=1, kv_heads=heads, group=group), DEV)
    k_new = keys[:, pos].contiguous()
    axr.axr_append_scores(k_new, q, idx, norms, pos, group, b, s)
    torch.cuda.synchronize()
    with profile(activities=[ProfilerActivity.CUDA]) as prof:
        axr.axr_append_scores(k_new, q, idx, norms, pos, group, b, s)
        torch.cuda.synchronize()
    kernels = [e.name for e in prof.events() if e.device_type.name == "CUDA"]
    if not kernels:
        pytest.skip("the profiler recorded no kernels on this machine")
    ours = [k for k in kernels if "axr" in k]
    assert len(ours) == launches, ours
    if launches == 1:
        assert "scores_tc" in ours[0], ours


@pytest.mark.parametrize("d", [128, 256, 512])
def test_append_on_many_single_tile_heads(d):
    """Short caches (every head one tile): a stream rotates a head's queries and
    quantizes its new key in the same tile, for hundreds of heads in one launch.
    The key's sums of squares must not share scratch with the queries' maxima."""
    b, group, heads, pos, capacity = 4, 4, 300, 50, 64
    keys, s, idx, norms = _cache(heads, capacity, pos, d, b, "bf16", seed=d + 5)
    wl = workloads.GQA_DECODE_128K.with_(d=d, batch=1, kv_heads=heads, group=group, T=pos + 1, seed=d + 6)
    q = workloads.make_queries(wl, DEV)
    out = axr.axr_append_scores(keys[:, pos].contiguous(), q, idx, norms, pos, group, b, s)
    assert axr.axr_device_status() == 0
    assert check_quantize(keys[:, pos], idx[:, pos], norms[:, pos], b, s).ok(flip_fraction=None)
    assert check_scores(q, idx[:, :pos + 1].contiguous(), norms[:, :pos + 1].contiguous(), out, group, b, s) <= 1e-4
