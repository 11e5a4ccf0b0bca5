"""The write kernels' bucket tables (CPU only).

The tensor-core and block-rotation write kernels find a coordinate's code
without a search: g = u * g_scale + g_off, j = round(g), code = base[j] +
(g > tau[j]).  That is #{i : u > t_i} only if every unit bucket of g holds at
most one boundary t_i, base[j] counts the boundaries below bucket j, tau[j] is
the boundary inside it, and every |u| <= 1 lands inside the table.  These tests
build the host code that makes the tables, dump them for every supported
(d, b), and check them against the library's fp32 boundaries, including a
dense emulation of the kernels' fp32 arithmetic.
"""
import os
import shutil
import subprocess

import numpy as np
import pytest

from lut_attention_b200 import axr

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
CXX = shutil.which("g++") or shutil.which("c++")


@pytest.fixture(scope="module")
def tables(tmp_path_factory):
    if not CXX:
        pytest.skip("no C++ compiler")
    exe = tmp_path_factory.mktemp("bt") / "bucket_table_dump"
    csrc = os.path.join(ROOT, "lut_attention_b200", "csrc")
    cuda_inc = os.path.join(os.environ.get("CUDA_HOME", "/usr/local/cuda"), "include")
    subprocess.run([CXX, "-std=c++17", "-O1", "-I", os.path.join(ROOT, "include"), "-I", csrc, "-I", cuda_inc,
                    "-o", str(exe), os.path.join(ROOT, "tests", "native", "bucket_table_dump.cpp"),
                    os.path.join(csrc, "codebook.cpp")], check=True, capture_output=True)
    out = subprocess.run([str(exe)], check=True, capture_output=True, text=True).stdout.split("\n")
    res, i = {}, 0
    while i < len(out) and out[i]:
        _, d, b, nt, gs, go, margin = out[i].split()
        d, b, nt = int(d), int(b), int(nt)
        rows = [out[i + 1 + j].split() for j in range(nt)]
        tau = np.array([float.fromhex(r[0]) for r in rows])
        base = np.array([int(r[1]) for r in rows])
        res[(d, b)] = dict(nt=nt, g_scale=float.fromhex(gs), g_off=float.fromhex(go), margin=float.fromhex(margin),
                           tau=tau, base=base)
        i += 1 + nt
    return res


def test_every_shape_has_a_table(tables):
    assert sorted(tables) == [(d, b) for d in (8, 16, 32, 64, 128, 256, 512) for b in (1, 2, 3, 4)]


@pytest.mark.parametrize("d", [8, 16, 32, 64, 128, 256, 512])
@pytest.mark.parametrize("b", [1, 2, 3, 4])
def test_table_encodes_the_boundaries(tables, d, b):
    t = tables[(d, b)]
    _, bnd = axr.axr_make_codebook(d, b)
    # boundary positions in g as the host computes them: one fused multiply-add in
    # fp32 (the fp64 product of two fp32 values is exact, so one rounding at the end)
    tg = np.float32(bnd.astype(np.float64) * t["g_scale"] + t["g_off"]).astype(np.float64)
    j = np.floor(tg + 0.5).astype(int)
    # one boundary per bucket at most, each away from the bucket's edges
    assert len(set(j)) == len(j)
    assert np.all(np.abs(tg - np.floor(tg) - 0.5) >= t["margin"]) and t["margin"] >= 0.05
    # |u| <= 1 stays inside the table, with a bucket to spare on each side
    assert t["g_off"] - t["g_scale"] >= 1 and t["g_off"] + t["g_scale"] <= t["nt"] - 2
    for k in range(t["nt"]):
        inside = np.nonzero(j == k)[0]
        assert t["base"][k] == np.count_nonzero(tg < k - 0.5), (k, t["base"][k])
        if len(inside):
            assert t["tau"][k] == tg[inside[0]]
        else:
            assert np.isinf(t["tau"][k])


@pytest.mark.parametrize("d", [8, 128, 512])
@pytest.mark.parametrize("b", [1, 2, 3, 4])
def test_table_lookup_counts_boundaries(tables, d, b):
    """The kernels' fp32 steps (g by one fused multiply-add, j by the 1.5 * 2^23
    rounding, one compare) give #{i : u > t_i} for every unit coordinate u, except
    within the fp32 rounding of g around a boundary."""
    t = tables[(d, b)]
    _, bnd = axr.axr_make_codebook(d, b)
    rng = np.random.default_rng(d * 10 + b)
    u = np.concatenate([np.linspace(-1, 1, 200001), rng.normal(0, 1 / np.sqrt(d), 200000),
                        np.repeat(bnd.astype(np.float64), 64) + rng.normal(0, 1e-5, 64 * len(bnd))])
    u = np.clip(u, -1, 1).astype(np.float32)
    g = (u.astype(np.float64) * np.float64(np.float32(t["g_scale"])) + t["g_off"]).astype(np.float32)
    jj = ((g + np.float32(12582912.0)) - np.float32(12582912.0)).astype(np.int64)
    code = t["base"][jj] + (g.astype(np.float64) > t["tau"][jj])
    true = (u.astype(np.float64)[:, None] > bnd.astype(np.float64)[None, :]).sum(axis=1)
    near = np.min(np.abs(u.astype(np.float64)[:, None] - bnd.astype(np.float64)[None, :]), axis=1) < 1e-6
    assert np.all(code[~near] == true[~near])


@pytest.mark.parametrize("d", [128, 256, 512])
@pytest.mark.parametrize("b", [1, 2, 3, 4])
def test_packed_table_entries_count_boundaries(tables, d, b):
    """The tensor-core write kernel keeps one 32-bit word per bucket: the
    boundary the bucket holds in u units (2 if none) with its low 4 mantissa
    bits replaced by the base code.  It compares u with that word read as a
    float (the boundary moved by at most 15 ulp) through the sign bit of
    word - u, and takes the low b bits of word + that bit.  Emulated in fp32
    here, that is #{i : u > t_i} for every unit coordinate u outside 1e-6 of a
    boundary."""
    t = tables[(d, b)]
    _, bnd = axr.axr_make_codebook(d, b)
    nt = t["nt"]
    tau_u = np.array([bnd[t["base"][j]] if np.isfinite(t["tau"][j]) else 2.0 for j in range(nt)], np.float32)
    words = (tau_u.view(np.uint32) & np.uint32(0xFFFFFFF0)) | t["base"][:nt].astype(np.uint32)
    # every moved boundary stays within 2.3e-7 of the true one
    fin = tau_u < 2.0
    moved = words[fin].view(np.float32).astype(np.float64) - tau_u[fin].astype(np.float64)
    assert np.all(np.abs(moved) <= 2.3e-7)
    rng = np.random.default_rng(d * 10 + b + 7)
    u = np.concatenate([np.linspace(-1, 1, 200001), rng.normal(0, 1 / np.sqrt(d), 200000),
                        np.repeat(bnd.astype(np.float64), 64) + rng.normal(0, 1e-6, 64 * len(bnd)),
                        np.zeros(5), bnd.astype(np.float64)])
    u = np.clip(u, -1, 1).astype(np.float32)
    f = (u.astype(np.float64) * np.float64(np.float32(t["g_scale"])) + t["g_off"] + 12582912.0).astype(np.float32)
    j = f.view(np.uint32).astype(np.int64) - 0x4B400000
    assert j.min() >= 0 and j.max() < nt
    w = words[j]
    diff = w.view(np.float32) - u                       # fp32, exact in sign
    above = diff.view(np.uint32) >> np.uint32(31)
    assert np.array_equal(above == 1, u > w.view(np.float32))
    code = (w + above) & np.uint32((1 << b) - 1)
    true = (u.astype(np.float64)[:, None] > bnd.astype(np.float64)[None, :]).sum(axis=1)
    near = np.min(np.abs(u.astype(np.float64)[:, None] - bnd.astype(np.float64)[None, :]), axis=1) < 1e-6
    assert np.all(code[~near] == true[~near])
    assert np.all(code[u == 0] == (1 << (b - 1)) - 1)
