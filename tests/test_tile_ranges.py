"""The read kernels' split of the tiles over persistent CTAs (CPU only).

Each CTA scores a contiguous range of 128-key tiles; a range that crosses into
a new KV head pays for one more query rotation, charged as change_cost tiles.
The host code that computes the ranges (lut_read.cuh) is built with nvcc as
host code and its output checked: the ranges cover every tile once, in order,
and every CTA's cost (its tiles plus change_cost per head boundary inside its
range) is within one tile plus one change of the mean."""
import os
import shutil
import subprocess

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
NVCC = shutil.which("nvcc") or "/usr/local/cuda/bin/nvcc"

CASES = [  # total tiles, tiles per head, CTAs, change cost
    (32768, 1024, 148, 12), (65536, 512, 147, 6), (65536, 512, 147, 3), (2048, 256, 148, 12),
    (300, 1, 148, 12), (148, 1, 148, 12), (40, 8, 40, 12), (7, 7, 7, 12), (1000, 1000, 148, 12),
    (32768, 1024, 148, 0), (131072, 1024, 148, 12),
]


@pytest.fixture(scope="module")
def ranges(tmp_path_factory):
    if not os.path.exists(NVCC):
        pytest.skip("nvcc not found")
    exe = tmp_path_factory.mktemp("tr") / "tile_ranges_dump"
    csrc = os.path.join(ROOT, "lut_attention_b200", "csrc")
    subprocess.run([NVCC, "-std=c++17", "-O1", "-I", os.path.join(ROOT, "include"), "-I", csrc, "-o", str(exe),
                    os.path.join(ROOT, "tests", "native", "tile_ranges_dump.cu")], check=True, capture_output=True)
    args = [str(x) for c in CASES for x in c]
    out = subprocess.run([str(exe), *args], check=True, capture_output=True, text=True).stdout.strip().split("\n")
    return {c: [int(v) for v in line.split()] for c, line in zip(CASES, out)}


@pytest.mark.parametrize("case", CASES)
def test_ranges_cover_every_tile_in_order(ranges, case):
    total, tph, ctas, cc = case
    s = ranges[case]
    assert len(s) == ctas + 1 and s[0] == 0 and s[-1] == total
    assert all(a <= b for a, b in zip(s, s[1:]))


@pytest.mark.parametrize("case", CASES)
def test_every_cta_costs_about_the_same(ranges, case):
    total, tph, ctas, cc = case
    s = ranges[case]

    def cost(a, b):   # tiles plus one change per head boundary strictly inside (a, b)
        inside = len([t for t in range(a + 1, b) if t % tph == 0]) if b - a > 1 else 0
        return (b - a) + cc * inside

    total_cost = total + cc * (total // tph - 1)
    mean = total_cost / ctas
    costs = [cost(a, b) for a, b in zip(s, s[1:])]
    assert max(costs) <= mean + 1 + cc
    # the split charges exactly the boundaries the ranges cross
    assert sum(costs) + cc * len({c for c in s[1:-1] if c % tph == 0 and 0 < c < total}) == total_cost
