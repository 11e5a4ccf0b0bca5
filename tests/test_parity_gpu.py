"""Parity of the CUDA path (called through the C ABI) with the CPU oracle.

Small cases are compared element by element; they span several CTAs and end in
a ragged tail.  The decode workloads run at full size and are compared on
sampled keys (first, last and seeded random keys of every head), which the
oracle computes one by one.  Tolerances are in tests/parity.py.
"""
import math

import numpy as np
import pytest
import torch

import oracle
from lut_attention_b200 import axr, workloads
from parity import check_quantize, check_scores, gpu_quantize, gpu_scores

pytestmark = pytest.mark.gpu

DIMS = (8, 16, 32, 64, 128, 256, 512)
DTYPES = ("f32", "f16", "bf16")
DEV = "cuda"


@pytest.fixture(autouse=True, scope="module")
def _libs(axr_lib, oracle_lib):
    return axr_lib


def _rows_for(d):
    # several CTAs of warp steps plus a ragged tail, oracle time ~ n * d^2
    return {8: 5001, 16: 5001, 32: 4001, 64: 3001, 128: 3001, 256: 1201, 512: 601}[d]


def _keys(d, dtype, n, seed):
    wl = workloads.MHA_DECODE_32K.with_(d=d, dtype=dtype, T=n, batch=1, kv_heads=1, seed=seed)
    return workloads.make_keys(wl, DEV).reshape(n, d), workloads.make_signs(wl).to(DEV)


def _assert_quantize(rep, what):
    assert rep.ok(), f"{what}: {rep}"


@pytest.mark.parametrize("dtype", DTYPES)
@pytest.mark.parametrize("b", [1, 2, 3, 4])
@pytest.mark.parametrize("d", DIMS)
def test_quantize_parity_grid(d, b, dtype):
    n = _rows_for(d)
    K, s = _keys(d, dtype, n, seed=1000 + d + b)
    idx, norms = gpu_quantize(K, b, s)
    assert idx.shape == (n, d * b // 8) and norms.shape == (n,)
    _assert_quantize(check_quantize(K, idx, norms, b, s), f"d={d} b={b} {dtype}")


@pytest.mark.parametrize("b", [1, 2, 3, 4])
@pytest.mark.parametrize("d", DIMS)
@pytest.mark.parametrize("group", [1, 4])
def test_scores_parity_random_packed(d, b, group):
    """The read kernel alone, on seeded random packed rows (every bit pattern is
    a valid index), so it is tested independently of the write kernel."""
    heads, n = 3, 2500
    packed, norms = workloads.make_random_packed(heads, n, d, b, seed=d * 10 + b, device=DEV)
    wl = workloads.GQA_DECODE_128K.with_(d=d, batch=1, kv_heads=heads, group=group, T=n)
    q = workloads.make_queries(wl, DEV)
    s = workloads.make_signs(wl).to(DEV)
    out = gpu_scores(q, packed, norms, group, b, s)
    assert out.shape == (heads * group, n)
    assert check_scores(q, packed, norms, out, group, b, s) <= 1e-4


@pytest.mark.parametrize("group", [1, 2, 3, 5, 8])
@pytest.mark.parametrize("qdtype", DTYPES)
def test_scores_parity_groups_and_query_dtypes(group, qdtype):
    d, b, heads, n = 128, 3, 2, 1500
    packed, norms = workloads.make_random_packed(heads, n, d, b, seed=77 + group, device=DEV)
    wl = workloads.GQA_DECODE_128K.with_(batch=1, kv_heads=heads, group=group, T=n, dtype=qdtype)
    q = workloads.make_queries(wl, DEV)
    s = workloads.make_signs(wl).to(DEV)
    out = gpu_scores(q, packed, norms, group, b, s)
    assert check_scores(q, packed, norms, out, group, b, s) <= 1e-4


@pytest.mark.parametrize("b", [2, 3, 4])
@pytest.mark.parametrize("heads,n,group", [(64, 3001, 4), (50, 100, 2), (3, 131, 8), (200, 77, 1),
                                           (4096, 100, 4), (3000, 64, 8)])
def test_scores_tile_ranges_cross_heads(heads, n, group, b):
    """d = 128 reads run on the tensor-core kernel, whose CTAs walk contiguous
    ranges of 128-key tiles: ranges cross KV heads (the query digits are rebuilt
    mid-range) and, for n < 128, every tile is a head of its own.  The last two
    shapes give each CTA about 28 and 21 such tiles, so every tile stream passes
    through more heads than the kernel keeps query scales for at once."""
    d = 128
    packed, norms = workloads.make_random_packed(heads, n, d, b, seed=heads + n + b, device=DEV)
    wl = workloads.GQA_DECODE_128K.with_(batch=1, kv_heads=heads, group=group, T=n)
    q = workloads.make_queries(wl, DEV)
    s = workloads.make_signs(wl).to(DEV)
    out = gpu_scores(q, packed, norms, group, b, s)
    assert check_scores(q, packed, norms, out, group, b, s) <= 1e-4


@pytest.mark.parametrize("d,b,heads,n,group", [
    (256, 2, 40, 300, 4), (256, 4, 200, 77, 8), (256, 3, 30, 1000, 1), (256, 1, 64, 129, 3),
    (512, 2, 40, 300, 4), (512, 4, 150, 77, 8), (512, 3, 20, 700, 2), (512, 1, 300, 64, 5),
])
def test_scores_wide_heads_cross_heads(d, b, heads, n, group):
    """d = 256 and 512 run on the tensor-core kernel as 2 and 4 subtiles per tile,
    with one B buffer per tile stream: a stream entering a new KV head waits for
    its products on the last head before writing the new query digits.  Many
    short heads make every CTA cross heads many times (n < 128: every tile a
    head of its own), for G up to 8 (one stream per CTA at d = 512)."""
    packed, norms = workloads.make_random_packed(heads, n, d, b, seed=heads + n + b + d, device=DEV)
    wl = workloads.GQA_DECODE_128K.with_(d=d, batch=1, kv_heads=heads, group=group, T=n)
    q = workloads.make_queries(wl, DEV)
    s = workloads.make_signs(wl).to(DEV)
    out = gpu_scores(q, packed, norms, group, b, s)
    assert check_scores(q, packed, norms, out, group, b, s) <= 1e-4


@pytest.mark.parametrize("d", [256, 512])
@pytest.mark.parametrize("dtype", ["bf16", "f16"])
@pytest.mark.parametrize("n", [1, 127, 129, 1000])
def test_quantize_wide_heads_tensor_core_tails(d, dtype, n):
    """The d = 256 / 512 tensor-core write on partial tiles (the TMA zero-fills the
    rows past n, the epilogue drops them).  Every code flip must lie inside the
    boundary window.  The in-window flip rate is capped at 1e-5 from n = 1000
    (2.6e5 and 5.1e5 coordinates, where the cap allows 2 and 5 flips); one or
    127 rows hold too few coordinates for a rate of 1e-5 to mean anything (the
    full-size tests check the rate on at least 2^20 rows)."""
    K, s = _keys(d, dtype, n, seed=9000 + d + n)
    for b in (2, 3):
        idx, norms = gpu_quantize(K, b, s)
        rep = check_quantize(K, idx, norms, b, s)
        cap = None if n < 1000 else 1e-5
        assert rep.ok(flip_fraction=cap), f"d={d} b={b} {dtype} n={n}: {rep}"


@pytest.mark.parametrize("offset", [0, 1, 2, 3])
def test_scores_norms_at_any_4_byte_offset(offset):
    """The tensor-core read kernel loads key norms by TMA from the 16-byte boundary
    at or below the norms pointer; a norms buffer that starts 4, 8 or 12 bytes past
    such a boundary must give the same scores."""
    d, b, heads, n, group = 128, 4, 5, 1000, 4
    packed, norms = workloads.make_random_packed(heads, n, d, b, seed=41 + offset, device=DEV)
    store = torch.zeros(heads * n + 4, dtype=torch.float32, device=DEV)
    shifted = store[offset:offset + heads * n].view(heads, n)
    shifted.copy_(norms)
    wl = workloads.GQA_DECODE_128K.with_(batch=1, kv_heads=heads, group=group, T=n)
    q = workloads.make_queries(wl, DEV)
    s = workloads.make_signs(wl).to(DEV)
    out = gpu_scores(q, packed, shifted, group, b, s)
    assert check_scores(q, packed, norms, out, group, b, s) <= 1e-4


def test_scores_group8_wide_head():
    d, b, heads, n, group = 512, 2, 1, 700, 8
    packed, norms = workloads.make_random_packed(heads, n, d, b, seed=5, device=DEV)
    wl = workloads.WIDE_D512.with_(batch=1, kv_heads=heads, group=group, T=n)
    q = workloads.make_queries(wl, DEV)
    s = workloads.make_signs(wl).to(DEV)
    out = gpu_scores(q, packed, norms, group, b, s)
    assert check_scores(q, packed, norms, out, group, b, s) <= 1e-4


@pytest.mark.parametrize("dtype", ["bf16", "f16"])
@pytest.mark.parametrize("n", [1, 5, 127, 128, 129, 255])
def test_quantize_tensor_core_partial_tiles(n, dtype):
    """d = 128 runs on the tensor-core kernel: tiles of 128 keys, the last one
    partly outside the tensor (loaded as zeros, never stored)."""
    K, s = _keys(128, dtype, n, seed=50 + n)
    idx, norms = gpu_quantize(K, 4, s)
    _assert_quantize(check_quantize(K, idx, norms, 4, s), f"n={n} {dtype}")


@pytest.mark.parametrize("b", [1, 2, 3, 4])
def test_quantize_tensor_core_many_tiles_per_cta(b):
    """Enough tiles that every CTA of the persistent grid runs several of them,
    wrapping the 4-stage load ring and both accumulators; every key checked."""
    n = 148 * 128 * 6 + 77
    K, s = _keys(128, "bf16", n, seed=60 + b)
    idx, norms = gpu_quantize(K, b, s)
    _assert_quantize(check_quantize(K, idx, norms, b, s), f"n={n} b={b}")


# ----------------------------------------------------------- whole pipeline --

def _sample_tokens(T, count, seed):
    rng = np.random.default_rng(seed)
    pick = {0, 1, T - 2, T - 1} | set(rng.integers(0, T, count).tolist())
    return torch.tensor(sorted(t for t in pick if 0 <= t < T), dtype=torch.long)


def _pipeline(wl, sample_per_head=None):
    K = workloads.make_keys(wl, DEV)                       # (heads, T, d)
    q = workloads.make_queries(wl, DEV)
    s = workloads.make_signs(wl).to(DEV)
    idx, norms = axr.axr_quantize_keys(K, wl.b, s)
    scores = axr.axr_scores(q, idx, norms, wl.group, wl.b, s)
    assert axr.axr_device_status() == 0
    if sample_per_head is None:
        tok = torch.arange(wl.T)
    else:
        tok = _sample_tokens(wl.T, sample_per_head, wl.seed)
    tok_d = tok.to(DEV)
    Ks, idxs, norms_s = K[:, tok_d], idx[:, tok_d], norms[:, tok_d]
    rep = check_quantize(Ks, idxs, norms_s, wl.b, s)
    _assert_quantize(rep, wl.describe())
    # read kernel on the library's own indices (keys it wrote), sampled tokens
    err = check_scores(q, idxs, norms_s, scores[:, tok_d], wl.group, wl.b, s)
    assert err <= 1e-4, f"{wl.describe()}: score error {err}"
    return rep, err


@pytest.mark.parametrize("name", [w.name for w in workloads.ALL])
def test_pipeline_small_all_recipes(name):
    wl = workloads.BY_NAME[name]
    small = wl.with_(batch=1, kv_heads=min(wl.kv_heads, 2), T=1537)
    _pipeline(small)


FULL = [(w.name, w.b) for w in workloads.ALL if w.name != "gqa_decode_128k"] + \
       [("gqa_decode_128k", b) for b in (2, 3, 4)]


@pytest.mark.parametrize("name,b", FULL)
def test_pipeline_full_size_sampled(name, b):
    wl = workloads.BY_NAME[name].with_(b=b)
    per_head = max(16, 4096 // wl.heads)
    rep, err = _pipeline(wl, sample_per_head=per_head)
    print(f"{wl.describe()}: flips={rep.flips}/{rep.coords} in-window={rep.in_window} "
          f"norm_rel={rep.max_norm_rel:.2e} score_err={err:.2e}")


# --------------------------------------------------------------- edge cases --

def test_zero_rows_is_a_noop():
    K = torch.zeros((0, 128), dtype=torch.bfloat16, device=DEV)
    s = torch.ones(128, dtype=torch.int8, device=DEV)
    idx = torch.full((4, 64), 0xAB, dtype=torch.uint8, device=DEV)
    norms = torch.full((4,), 7.0, device=DEV)
    axr.axr_quantize_keys(K, 4, s, idx=idx, norms=norms)
    torch.cuda.synchronize()
    assert torch.all(idx == 0xAB) and torch.all(norms == 7.0)
    out = torch.full((2, 0), 1.0, device=DEV)
    axr.axr_scores(torch.zeros((2, 128), device=DEV), torch.zeros((2, 0, 64), dtype=torch.uint8, device=DEV),
                   torch.zeros((2, 0), device=DEV), 1, 4, s, scores=out)


@pytest.mark.parametrize("b", [1, 2, 3, 4])
def test_zero_and_constant_keys(b):
    """Zero keys store norm 0 and index 2^(b-1)-1.  A constant key with all-plus
    signs rotates onto the first axis: every other rotated coordinate is exactly
    0, on the central boundary, and the kernel's exact Hadamard sum sends it to
    the lower index.  (The oracle's dense fp64 product leaves ~1e-17 residues
    there, inside the 1e-6 window, so those coordinates are compared through the
    window rule.)"""
    d = 128
    L = 1 << b
    K = torch.zeros((67, d), dtype=torch.float32, device=DEV)
    K[1::2] = 3.0
    s = torch.ones(d, dtype=torch.int8, device=DEV)
    idx, norms = gpu_quantize(K, b, s)
    rep = check_quantize(K, idx, norms, b, s)
    assert rep.ok(flip_fraction=None), f"constant keys b={b}: {rep}"
    codes = oracle.unpack(idx.cpu().numpy(), d, b)
    assert np.all(codes[0::2] == L // 2 - 1)
    assert np.all(norms[0::2].cpu().numpy() == 0)
    assert np.all(codes[1::2, 0] == L - 1) and np.all(codes[1::2, 1:] == L // 2 - 1)
    assert np.all(norms[1::2].cpu().numpy() == np.float32(np.sqrt(9.0 * d)))
    q = torch.randn((2, d), device=DEV)
    out = gpu_scores(q, idx[None], norms[None], 2, b, s)
    assert torch.all(out[:, 0::2] == 0)


def test_single_key_single_head():
    d, b = 64, 3
    K, s = _keys(d, "bf16", 1, seed=9)
    idx, norms = gpu_quantize(K, b, s)
    _assert_quantize(check_quantize(K, idx, norms, b, s), "n=1")
    q = torch.randn((1, d), device=DEV)
    out = gpu_scores(q, idx[None], norms[None], 1, b, s)
    assert check_scores(q, idx[None], norms[None], out, 1, b, s) <= 1e-4


def test_outputs_stay_inside_their_buffers():
    """Canary bytes around every output survive both kernels."""
    d, b, n, group = 128, 3, 1000, 4
    K, s = _keys(d, "bf16", n, seed=3)
    P = d * b // 8
    guard = 4096
    idx_buf = torch.full((guard + n * P + guard,), 0x5A, dtype=torch.uint8, device=DEV)
    norm_buf = torch.full((guard + n + guard,), -123.0, device=DEV)
    idx = idx_buf[guard:guard + n * P].view(n, P)
    norms = norm_buf[guard:guard + n]
    axr.axr_quantize_keys(K, b, s, idx=idx, norms=norms)
    q = torch.randn((group, d), device=DEV)
    sc_buf = torch.full((guard + group * n + guard,), -321.0, device=DEV)
    sc = sc_buf[guard:guard + group * n].view(group, n)
    axr.axr_scores(q, idx[None], norms[None], group, b, s, scores=sc)
    torch.cuda.synchronize()
    for buf, val in ((idx_buf, 0x5A), (norm_buf, -123.0), (sc_buf, -321.0)):
        assert torch.all(buf[:guard] == val) and torch.all(buf[-guard:] == val)


def test_device_argument_errors_do_not_launch():
    lib = axr.library()
    x = torch.zeros(1024, dtype=torch.uint8, device=DEV)
    p = x.data_ptr()
    assert lib.axr_quantize_keys(p + 4, 2, 8, 128, 4, p, p, p, None) == axr.AXR_EINVAL
    assert lib.axr_quantize_keys(p, 2, 8, 128, 4, p, p + 4, p, None) == axr.AXR_EINVAL
    assert lib.axr_scores(p, 2, p + 8, p, 8, 1, 1, 128, 4, p, p, None) == axr.AXR_EINVAL
    torch.cuda.synchronize()


def test_streams_are_respected():
    d, b, n = 128, 4, 20000
    K, s = _keys(d, "bf16", n, seed=4)
    st = torch.cuda.Stream()
    st.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(st):
        idx, norms = axr.axr_quantize_keys(K, b, s)
        out = axr.axr_scores(torch.randn((1, d), device=DEV), idx[None], norms[None], 1, b, s)
    st.synchronize()
    ref_idx, ref_norms = gpu_quantize(K, b, s)
    assert torch.equal(idx, ref_idx) and torch.equal(norms, ref_norms)
    assert torch.isfinite(out).all()
