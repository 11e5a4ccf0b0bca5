"""axr_attention_static: decode attention with the library's fixed scratch.

Collected last.  Two consecutive calls must each give exactly what
axr_attention gives with a caller workspace, and a shape whose partial sums do
not fit the fixed scratch must be refused before anything is enqueued.  The
test builds its own inputs, so it passes alone in a fresh process as well as
after the rest of the suite.
"""
import pytest
import torch

from lut_attention_b200 import axr, workloads

pytestmark = pytest.mark.gpu
DEV = "cuda"


def _inputs(heads, n, d, b, group, seed, vdtype=torch.bfloat16):
    packed, norms = workloads.make_random_packed(heads, n, d, b, seed=seed, device=DEV)
    wl = workloads.GQA_DECODE_128K.with_(d=d, batch=1, kv_heads=heads, group=group, T=n, seed=seed)
    q = workloads.make_queries(wl, DEV)
    s = workloads.make_signs(wl).to(DEV)
    g = torch.Generator(device=DEV).manual_seed(seed + 17)
    V = torch.randn((heads, n, d), generator=g, device=DEV).to(vdtype)
    return packed, norms, q, s, V


# (KV heads, keys, d, b, queries per KV head, value dtype): the padded group of
# 3 queries, a single query, eight queries, the narrow CUDA-core read (d = 32)
# and the widest head, with every value dtype; all fit the fixed scratch.
CASES = [
    (4, 9000, 128, 4, 4, torch.bfloat16),
    (3, 5000, 128, 3, 3, torch.float16),
    (2, 7001, 512, 2, 3, torch.float32),
    (5, 3000, 256, 4, 8, torch.bfloat16),
    (6, 4097, 32, 2, 1, torch.float16),
    (2, 130, 64, 1, 2, torch.float32),
]


@pytest.mark.parametrize("heads,n,d,b,group,vdtype", CASES)
def test_two_consecutive_calls_match_the_workspace_entry_point(axr_lib, heads, n, d, b, group, vdtype):
    packed, norms, q, s, V = _inputs(heads, n, d, b, group, seed=5 + n + d, vdtype=vdtype)
    ref_out, ref_scores = axr.axr_attention(q, packed, norms, V, group, b, s)
    for _ in range(2):
        scores = torch.full((heads * group, n), float("nan"), device=DEV)
        out = torch.full((heads * group, d), float("nan"), device=DEV)
        axr.axr_attention_static(q, packed, norms, V, group, b, s, scores, out)
        torch.cuda.synchronize()
        assert torch.equal(out, ref_out)
        assert torch.equal(scores, ref_scores)
    assert axr.axr_device_status() == 0


def test_shape_beyond_the_fixed_scratch_is_refused(axr_lib):
    # 4M keys x 4 KV heads x 4 queries at d = 128 need 4 * 4096 * 4 * 130 * 4 bytes > 16 MiB
    heads, n, d, b, group = 4, 1 << 22, 128, 2, 4
    assert axr.axr_attention_workspace_bytes(n, heads, group, d) > 16 << 20
    buf = torch.zeros(1 << 20, dtype=torch.uint8, device=DEV)
    p = buf.data_ptr()
    rc = axr_lib.axr_attention_static(p, axr.AXR_BF16, p, p, p, axr.AXR_BF16, n, heads, group, d, b, p, p, p,
                                      None)
    assert rc == axr.AXR_EUNSUPPORTED
    assert b"fixed scratch" in axr_lib.axr_last_error()
