"""Parity of the IsoQuant block-rotation path (axr_quantize_keys_block,
axr_scores_block) with the CPU oracle.

Tolerances are those of the Walsh-Hadamard path (tests/parity.py): codes
bit-exact except coordinates within 1e-6 of a decision point (such flips
counted, fewer than 1e-5 of all coordinates), norms within 1e-4, scores within
1e-4 of |q| |k| / sqrt(d).  The kernels compose each block's two quaternion
products in fp32, a relative error of a few 1e-7 on u: inside that window.
"""
import numpy as np
import pytest
import torch

import oracle
from lut_attention_b200 import axr, workloads
from parity import check_quantize, check_scores

pytestmark = pytest.mark.gpu

DIMS = (8, 16, 32, 64, 128, 256, 512)
DEV = "cuda"


@pytest.fixture(autouse=True, scope="module")
def _libs(axr_lib, oracle_lib):
    return axr_lib


def _rows_for(d):
    return {8: 5001, 16: 5001, 32: 4001, 64: 3001, 128: 3001, 256: 1201, 512: 601}[d]


def _setup(d, dtype, n, seed, fast=False, recipe_wl=workloads.MHA_DECODE_32K):
    wl = recipe_wl.with_(d=d, dtype=dtype, T=n, batch=1, kv_heads=1, seed=seed)
    K = workloads.make_keys(wl, DEV).reshape(n, d)
    quats = workloads.make_block_quats(wl, fast=fast)
    return K, quats.to(DEV), wl


def _gpu_quantize(K, b, quats):
    idx, norms = axr.axr_quantize_keys_block(K, b, quats)
    torch.cuda.synchronize()
    return idx, norms


@pytest.mark.parametrize("dtype", ("f32", "f16", "bf16"))
@pytest.mark.parametrize("b", [1, 2, 3, 4])
@pytest.mark.parametrize("d", DIMS)
def test_block_quantize_parity_grid(d, b, dtype):
    n = _rows_for(d)
    K, quats, _ = _setup(d, dtype, n, seed=2000 + d + b)
    idx, norms = _gpu_quantize(K, b, quats)
    assert idx.shape == (n, d * b // 8) and norms.shape == (n,)
    rep = check_quantize(K, idx, norms, b, None, quats=quats)
    assert rep.ok(), f"d={d} b={b} {dtype}: {rep}"


@pytest.mark.parametrize("d,b", [(128, 4), (128, 2), (256, 3), (512, 2), (32, 1)])
def test_block_quantize_fast_variant(d, b):
    """qR = 1 on every block (IsoQuant-Fast)."""
    n = _rows_for(d)
    K, quats, _ = _setup(d, "bf16", n, seed=3000 + d + b, fast=True)
    assert torch.equal(quats[:, 4:].cpu(), torch.tensor([[1.0, 0.0, 0.0, 0.0]]).repeat(d // 4, 1))
    idx, norms = _gpu_quantize(K, b, quats)
    rep = check_quantize(K, idx, norms, b, None, quats=quats)
    assert rep.ok(), f"d={d} b={b} fast: {rep}"


@pytest.mark.parametrize("d,b,group,qdtype", [
    (128, 4, 4, "bf16"), (128, 3, 1, "f32"), (128, 2, 8, "f16"), (128, 1, 3, "bf16"),
    (64, 4, 2, "f32"), (256, 2, 2, "f16"), (512, 3, 4, "bf16"), (8, 2, 1, "f32"), (16, 4, 5, "f16"),
])
def test_block_scores_parity(d, b, group, qdtype):
    """The read path on the library's own block-rotated codes (tensor-core kernel
    at d = 128, CUDA-core kernel otherwise) and on random packed rows."""
    heads, n = 3, 1100
    K, quats, wl = _setup(d, "bf16", heads * n, seed=4000 + d + b + group)
    idx, norms = _gpu_quantize(K, b, quats)
    idx, norms = idx.reshape(heads, n, -1), norms.reshape(heads, n)
    g = torch.Generator(device=DEV).manual_seed(d + group)
    q = torch.randn((heads * group, d), generator=g, device=DEV).to(getattr(torch, {
        "f32": "float32", "f16": "float16", "bf16": "bfloat16"}[qdtype]))
    scores = axr.axr_scores_block(q, idx, norms, group, b, quats)
    torch.cuda.synchronize()
    assert axr.axr_device_status() == 0
    err = check_scores(q, idx, norms, scores, group, b, None, quats=quats)
    assert err <= 1e-4, f"d={d} b={b} G={group}: score error {err}"
    packed, rn = workloads.make_random_packed(heads, n, d, b, seed=d + b, device=DEV)
    scores = axr.axr_scores_block(q, packed, rn, group, b, quats)
    torch.cuda.synchronize()
    err = check_scores(q, packed, rn, scores, group, b, None, quats=quats)
    assert err <= 1e-4, f"random packed d={d} b={b} G={group}: score error {err}"


def test_block_identity_rotation_matches_plain_quantization_of_unrotated_keys():
    """qL = qR = 1 on every block is the identity: the codes are those of the
    keys' own unit coordinates, computed here from the codebook on the host."""
    d, b, n = 128, 3, 2000
    K, _, _ = _setup(d, "f32", n, seed=5)
    quats = torch.tensor([[1.0, 0, 0, 0, 1.0, 0, 0, 0]], device=DEV).repeat(d // 4, 1)
    idx, norms = _gpu_quantize(K, b, quats)
    cent, bnd = axr.axr_make_codebook(d, b)
    Kh = K.double().cpu().numpy()
    u = Kh / np.linalg.norm(Kh, axis=1, keepdims=True)
    codes = (u[:, :, None] > bnd.astype(np.float64)[None, None, :]).sum(axis=2)
    got = oracle.unpack(idx.cpu().numpy(), d, b)
    assert (got != codes).mean() < 1e-5


def test_block_full_size_sampled():
    """gqa_decode_128k keys through the block rotation at full size (4.2 M rows,
    1 GB): sampled rows against the oracle, and the read kernel on them."""
    wl = workloads.GQA_DECODE_128K
    K = workloads.make_keys(wl, DEV)
    quats = workloads.make_block_quats(wl).to(DEV)
    idx, norms = axr.axr_quantize_keys_block(K, wl.b, quats)
    torch.cuda.synchronize()
    g = torch.Generator().manual_seed(77)
    rows = torch.randint(0, wl.T, (wl.heads, 64), generator=g)
    h_ix = torch.arange(wl.heads)[:, None].expand_as(rows)
    Ks = K[h_ix, rows].reshape(-1, wl.d)
    rep = check_quantize(Ks, idx[h_ix, rows].reshape(Ks.shape[0], -1), norms[h_ix, rows].reshape(-1), wl.b,
                         None, quats=quats)
    assert rep.ok(), str(rep)
    q = workloads.make_queries(wl, DEV)
    scores = axr.axr_scores_block(q, idx, norms, wl.group, wl.b, quats)
    torch.cuda.synchronize()
    hq = torch.arange(wl.heads * wl.group)
    s_rows = rows.repeat_interleave(wl.group, dim=0)
    err = check_scores(q, idx[h_ix, rows], norms[h_ix, rows], scores[hq[:, None], s_rows], wl.group, wl.b, None,
                       quats=quats)
    assert err <= 1e-4, f"score error {err}"
    del K, idx, norms, scores


def test_block_zero_rows_zero_keys_and_streams():
    d, b = 128, 4
    quats = workloads.make_block_quats(workloads.GQA_DECODE_128K).to(DEV)
    idx, norms = axr.axr_quantize_keys_block(torch.zeros((0, d), dtype=torch.bfloat16, device=DEV), b, quats)
    assert idx.numel() == 0 and norms.numel() == 0
    Z = torch.zeros((100, d), dtype=torch.bfloat16, device=DEV)
    idx, norms = _gpu_quantize(Z, b, quats)
    assert torch.all(norms == 0)
    assert torch.all(torch.from_numpy(oracle.unpack(idx.cpu().numpy(), d, b)) == (1 << (b - 1)) - 1)
    K, _, _ = _setup(d, "bf16", 3000, seed=8)
    ref_idx, ref_norms = _gpu_quantize(K, b, quats)
    st = torch.cuda.Stream()
    st.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(st):
        i2, n2 = axr.axr_quantize_keys_block(K, b, quats, stream=st)
    st.synchronize()
    assert torch.equal(i2, ref_idx) and torch.equal(n2, ref_norms)


def test_block_outputs_stay_inside_their_buffers():
    d, b, n = 64, 2, 777          # 16-byte packed rows: the interior slice stays aligned
    K, quats, _ = _setup(d, "f16", n, seed=9)
    P = d * b // 8
    idx = torch.full((n + 2, P), 0xAB, dtype=torch.uint8, device=DEV)
    norms = torch.full((n + 2,), -7.0, dtype=torch.float32, device=DEV)
    axr.axr_quantize_keys_block(K, b, quats, idx=idx[1:n + 1], norms=norms[1:n + 1])
    torch.cuda.synchronize()
    assert torch.all(idx[0] == 0xAB) and torch.all(idx[n + 1] == 0xAB)
    assert norms[0].item() == -7.0 and norms[n + 1].item() == -7.0
