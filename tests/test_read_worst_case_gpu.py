"""The tensor-core read at the worst case of its fixed-point digits.

tests/digit_split.py bounds the score error of the digit split over all queries
and codes.  Here the read kernel runs the inputs that reach that bound:
  * every code on the centroid with the largest digit error, and the query
    q = +-D_0 e_0, whose rotation spreads evenly over all coordinates: the error
    must equal sqrt(d) times that centroid's digit error (the query digits are
    exact there), and stay inside the tolerance;
  * the same codes with queries whose largest rotated coordinate is M times the
    norm and whose other coordinates are all equal, for M across [1/sqrt(d), 1]:
    both the centroid digits and the query digits then err in one direction on
    every coordinate.
Scores are compared with the oracle on the same codes (no write path involved).
"""
import math

import numpy as np
import pytest
import torch

import digit_split
import oracle
from lut_attention_b200 import axr, workloads
from parity import check_scores, gpu_scores

pytestmark = pytest.mark.gpu
DEV = "cuda"


@pytest.fixture(autouse=True, scope="module")
def _libs(axr_lib, oracle_lib):
    return axr_lib


def _cache(heads, n, d, b, code, seed):
    codes = np.full((heads * n, d), code, dtype=np.uint8)
    packed = torch.from_numpy(oracle.pack(codes, b).reshape(heads, n, d * b // 8)).to(DEV)
    g = torch.Generator(device="cpu").manual_seed(seed)
    norms = torch.exp(torch.randn((heads, n), generator=g)).to(DEV)
    return packed, norms


@pytest.mark.parametrize("group", [1, 4])
@pytest.mark.parametrize("b", [2, 3, 4])
@pytest.mark.parametrize("d", [128, 256, 512])
def test_aligned_worst_case_reaches_the_predicted_error(d, b, group):
    heads, n = 3, 300
    cent, _ = axr.axr_make_codebook(d, b)
    i_star, predicted = digit_split.aligned_worst_case(cent, d)
    packed, norms = _cache(heads, n, d, b, i_star, seed=d + b)
    s = workloads.make_signs(workloads.GQA_DECODE_128K.with_(d=d)).to(DEV)
    q = torch.zeros((heads * group, d), dtype=torch.float32)
    rng = np.random.default_rng(d * 10 + b)
    for r in range(heads * group):
        q[r, 0] = float(s[0].item()) * float(rng.choice([-1.0, 1.0])) * float(np.exp(rng.normal()))
    q = q.to(DEV)
    out = gpu_scores(q, packed, norms, group, b, s)
    err = check_scores(q, packed, norms, out, group, b, s)
    assert err <= 1e-4
    # the kernel's digits are the ones restated in tests/digit_split.py
    assert abs(err - abs(predicted)) <= 2e-6, (err, predicted)


@pytest.mark.parametrize("b", [3, 4])
@pytest.mark.parametrize("d", [128, 512])
def test_worst_case_sweep_stays_inside_the_bound(d, b):
    heads, n, group = 2, 200, 4
    cent, _ = axr.axr_make_codebook(d, b)
    i_star, predicted = digit_split.aligned_worst_case(cent, d)
    bound, m_star = digit_split.worst_case_bound(cent, d)
    packed, norms = _cache(heads, n, d, b, i_star, seed=7 * d + b)
    s_cpu = workloads.make_signs(workloads.GQA_DECODE_128K.with_(d=d))
    s = s_cpu.to(DEV)
    R = oracle.rotation(d, s_cpu.numpy())
    sign = 1.0 if predicted >= 0 else -1.0
    Ms = sorted({1.0 / math.sqrt(d), 0.1, m_star, 0.5, 0.9, 1.0} | set(np.linspace(m_star * 0.8, m_star * 1.2, 7)))
    Ms = [m for m in Ms if 1.0 / math.sqrt(d) <= m <= 1.0]
    worst = 0.0
    for k in range(0, len(Ms), heads * group):
        batch = Ms[k:k + heads * group]
        qs = np.zeros((heads * group, d))
        for r, M in enumerate(batch):
            rest = math.sqrt(max(0.0, 1.0 - M * M) / (d - 1))
            qp = np.full(d, sign * rest)
            qp[1] = sign * M
            qs[r] = R.T @ qp * (1.0 + r)
        q = torch.from_numpy(qs).to(torch.float32).to(DEV)
        out = gpu_scores(q, packed, norms, group, b, s)
        worst = max(worst, check_scores(q, packed, norms, out, group, b, s))
    assert worst <= bound + 1e-6 and worst <= 1e-4, (worst, bound)
