"""Pins of the CPU oracle against what the pages and the mathematics fix.

Each test checks an oracle function against something other than the oracle
itself: a textbook construction or library routine (scipy's Hadamard matrix),
a closed form, numerical integration of the normal density, a published table,
brute force over every codeword on tiny inputs, or the pages' qualitative claims
(AXELRAM abstract: rotated unit-key coordinates concentrate to N(0, 1/d); the
codebook depends on d and b only; reading by table lookup needs no inverse
transform).  The 102.4x multiplication figure of the abstract stays unpinned.
"""
import math
import os

import numpy as np
import pytest
import scipy.integrate
import scipy.linalg
import torch

import oracle
from lut_attention_b200 import workloads

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")
DIMS = (8, 16, 32, 64, 128, 256, 512)


@pytest.fixture(autouse=True, scope="module")
def _built(oracle_lib):
    return oracle_lib


def _rng_signs(d, seed):
    rng = np.random.default_rng(seed)
    return (rng.integers(0, 2, d) * 2 - 1).astype(np.int8)


def _phi(x):
    return math.exp(-0.5 * x * x) / math.sqrt(2 * math.pi)


# ---------------------------------------------------------------- transform --

def test_hadamard_sylvester_recursion_and_scipy():
    assert np.array_equal(oracle.hadamard(2), np.array([[1, 1], [1, -1]], dtype=float))
    for d in (2, 4) + DIMS:
        H = oracle.hadamard(d)
        assert np.array_equal(H, scipy.linalg.hadamard(d).astype(float))
        assert np.array_equal(H @ H.T, d * np.eye(d))
        if d >= 4:
            h = oracle.hadamard(d // 2)
            assert np.array_equal(H, np.block([[h, h], [h, -h]]))


@pytest.mark.parametrize("d", DIMS)
def test_rotation_is_orthonormal_hadamard_times_signs(d):
    s = _rng_signs(d, d)
    R = oracle.rotation(d, s)
    expect = scipy.linalg.hadamard(d) * s[None, :] / math.sqrt(d)
    np.testing.assert_allclose(R, expect, rtol=0, atol=1e-15)
    np.testing.assert_allclose(R @ R.T, np.eye(d), rtol=0, atol=1e-12)
    x = np.random.default_rng(1).standard_normal((5, d))
    np.testing.assert_allclose(np.linalg.norm(x @ R.T, axis=1), np.linalg.norm(x, axis=1), rtol=1e-12)


def test_rotation_rejects_bad_signs():
    with pytest.raises(ValueError):
        oracle.rotation(8, np.array([1, -1, 0, 1, 1, 1, 1, 1], dtype=np.int8))


# ----------------------------------------------------------------- codebook --

def test_lloyd_max_one_bit_closed_form():
    c, _ = oracle.lloyd_max_std(1)
    r = math.sqrt(2 / math.pi)
    np.testing.assert_allclose(c, [-r, r], rtol=0, atol=1e-14)


@pytest.mark.parametrize("b", [1, 2, 3, 4])
def test_lloyd_max_conditions_by_quadrature(b):
    """Midpoint and centroid conditions, with the conditional means computed by
    adaptive quadrature of the normal density (not the oracle's erfc forms)."""
    c, iters = oracle.lloyd_max_std(b)
    L = 1 << b
    assert iters < 100000
    t = (c[:-1] + c[1:]) / 2
    edges = np.concatenate([[-np.inf], t, [np.inf]])
    for i in range(L):
        lo, hi = edges[i], edges[i + 1]
        mass = scipy.integrate.quad(_phi, lo, hi, epsabs=1e-15, epsrel=1e-13)[0]
        first = scipy.integrate.quad(lambda x: x * _phi(x), lo, hi, epsabs=1e-15, epsrel=1e-13)[0]
        assert abs(first / mass - c[i]) < 1e-10
    np.testing.assert_allclose(c, -c[::-1], rtol=0, atol=1e-13)


def _mse(c):
    t = (c[:-1] + c[1:]) / 2
    edges = np.concatenate([[-np.inf], t, [np.inf]])
    return sum(scipy.integrate.quad(lambda x, ci=ci: (x - ci) ** 2 * _phi(x), lo, hi,
                                    epsabs=1e-15, epsrel=1e-12)[0]
               for ci, lo, hi in zip(c, edges[:-1], edges[1:]))


def _classical_table():
    rows = {}
    with open(os.path.join(GOLDEN, "lloyd_max_classical.txt")) as f:
        for line in f:
            line = line.split("#")[0].split()
            if line:
                rows[int(line[0])] = (float(line[1]), [float(v) for v in line[2:]])
    return rows


@pytest.mark.parametrize("b", [1, 2, 3, 4])
def test_lloyd_max_matches_classical_table_and_is_a_minimum(b):
    c, _ = oracle.lloyd_max_std(b)
    mse_ref, pos_ref = _classical_table()[b]
    L = 1 << b
    np.testing.assert_allclose(c[L // 2:], pos_ref, rtol=0, atol=1e-3)
    m = _mse(c)
    assert abs(m - mse_ref) < 1e-3 * mse_ref + 1e-6
    # stationary: moving any centroid (with its boundaries) raises the distortion
    for i in range(L):
        for eps in (1e-3, -1e-3):
            cc = c.copy()
            cc[i] += eps
            if np.all(np.diff(cc) > 0):
                assert _mse(cc) > m


@pytest.mark.parametrize("d", DIMS)
@pytest.mark.parametrize("b", [1, 2, 3, 4])
def test_codebook_scaling_symmetry_and_boundaries(d, b):
    cent, bnd = oracle.codebook(d, b)
    c, _ = oracle.lloyd_max_std(b)
    L = 1 << b
    assert cent.dtype == np.float32 and cent.shape == (L,) and bnd.shape == (L - 1,)
    # N(0, 1/d) quantizer = N(0, 1) quantizer scaled by 1/sqrt(d), rounded to fp32
    np.testing.assert_allclose(cent.astype(np.float64), c / math.sqrt(d), rtol=1e-7, atol=0)
    assert np.array_equal(cent, -cent[::-1])
    assert np.all(np.diff(cent) > 0)
    mid = ((cent[:-1].astype(np.float64) + cent[1:].astype(np.float64)) / 2).astype(np.float32)
    assert np.array_equal(bnd, mid)
    assert bnd[L // 2 - 1] == 0.0


def test_codebook_is_data_independent():
    """The codebook is a function of (d, b) alone: repeated calls agree bit for bit."""
    a = oracle.codebook(128, 3)
    oracle.quantize(np.random.default_rng(0).standard_normal((16, 128)) * 1e3, 3, _rng_signs(128, 0))
    b = oracle.codebook(128, 3)
    assert np.array_equal(a[0], b[0]) and np.array_equal(a[1], b[1])


# ------------------------------------------------------------------ packing --

def test_packing_hand_worked_examples():
    with open(os.path.join(GOLDEN, "packing_examples.txt")) as f:
        for line in f:
            line = line.split("#")[0].strip()
            if not line:
                continue
            left, right = line.split("->")
            vals = [int(v) for v in left.split()]
            d, b, codes = vals[0], vals[1], np.array(vals[2:], dtype=np.uint8)[None, :]
            expect = np.array([int(x, 16) for x in right.split()], dtype=np.uint8)[None, :]
            assert np.array_equal(oracle.pack(codes, b), expect), (d, b)
            assert np.array_equal(oracle.unpack(expect, d, b), codes)


@pytest.mark.parametrize("d,b", [(8, 1), (16, 3), (128, 3), (128, 4), (512, 2)])
def test_pack_roundtrip_and_bit_positions(d, b):
    rng = np.random.default_rng(d * 10 + b)
    codes = rng.integers(0, 1 << b, (7, d)).astype(np.uint8)
    packed = oracle.pack(codes, b)
    assert packed.shape == (7, d * b // 8)
    assert np.array_equal(oracle.unpack(packed, d, b), codes)
    bits = np.unpackbits(packed, axis=1, bitorder="little")
    for j in range(d):
        for i in range(b):
            assert np.array_equal(bits[:, j * b + i], (codes[:, j] >> i) & 1)


# ------------------------------------------------------------ quantize path --

def test_rotated_unit_keys_have_unit_norm_and_variance_one_over_d():
    """AXELRAM abstract: after the transform each coordinate of a unit key is
    close to N(0, 1/d).  Checked on the first workload's 4096 keys."""
    wl = workloads.PR1_REF
    K = workloads.make_keys(wl).reshape(-1, wl.d).double().numpy()
    s = workloads.make_signs(wl).numpy()
    norms, U = oracle.rotate_unit(K, s)
    np.testing.assert_allclose((U * U).sum(axis=1), 1.0, rtol=0, atol=1e-6)
    np.testing.assert_allclose(norms, np.linalg.norm(K, axis=1), rtol=1e-7)
    n, d = U.shape
    var = (U * U).mean(axis=0) * d                    # per-coordinate variance x d
    se = math.sqrt(2.0 / n)
    assert np.all(np.abs(var - 1.0) < 5 * se)
    z = (U * math.sqrt(d)).ravel()
    assert abs(z.mean()) < 5 / math.sqrt(z.size)
    kurt = (z ** 4).mean() / (z ** 2).mean() ** 2
    assert abs(kurt - 3.0) < 0.1


@pytest.mark.parametrize("b", [1, 2, 3, 4])
def test_basis_vector_closed_form(b):
    """k = alpha e_m, q = beta e_m: every rotated coordinate is +-1/sqrt(d), so each
    lands on the centroid pair nearest to +-sigma, and the score is
    alpha * beta * c*(1) / sqrt(d), c*(1) that centroid in units of sigma."""
    d = 64
    s = _rng_signs(d, 3)
    cent, _ = oracle.codebook(d, b)
    sigma = 1 / math.sqrt(d)
    pos = cent[cent > 0].astype(np.float64)
    cstar = pos[np.argmin(np.abs(pos - sigma))] / sigma
    L = 1 << b
    for m, alpha, beta in [(0, 2.5, -1.5), (5, 0.75, 3.0), (63, 10.0, 0.125)]:
        K = np.zeros((1, d))
        K[0, m] = alpha
        packed, norms, _ = oracle.quantize(K, b, s)
        codes = oracle.unpack(packed, d, b)[0]
        H = scipy.linalg.hadamard(d)
        sgn = s[m] * H[:, m]
        expect_codes = np.where(sgn > 0, np.searchsorted(cent, sigma * cstar - 1e-9),
                                L - 1 - np.searchsorted(cent, sigma * cstar - 1e-9))
        assert np.array_equal(codes, expect_codes)
        assert norms[0] == np.float32(alpha)
        q = np.zeros((1, d))
        q[0, m] = beta
        sc = oracle.scores(q, packed[None], norms[None], 1, b, s)
        np.testing.assert_allclose(sc[0, 0], alpha * beta * cstar / math.sqrt(d), rtol=1e-6)


def test_zero_key():
    d, b = 32, 3
    packed, norms, _ = oracle.quantize(np.zeros((2, d)), b, _rng_signs(d, 1))
    assert np.all(norms == 0)
    assert np.all(oracle.unpack(packed, d, b) == (1 << (b - 1)) - 1)
    sc = oracle.scores(np.ones((1, d)), packed[None], norms[None], 1, b, _rng_signs(d, 1))
    assert np.all(sc == 0)


@pytest.mark.parametrize("b", [1, 2, 3])
def test_brute_force_nearest_codeword_d8(b):
    """d = 8: the oracle's per-coordinate indices give the codeword x in C^8 whose
    reconstruction norm * R^T x is nearest to k, over all L^8 codewords."""
    d = 8
    L = 1 << b
    cent, _ = oracle.codebook(d, b)
    rng = np.random.default_rng(100 + b)
    s = _rng_signs(d, 7 + b)
    R = scipy.linalg.hadamard(d) * s[None, :] / math.sqrt(d)
    K = rng.standard_normal((3, d)) * rng.lognormal(0, 1, (3, 1))
    packed, norms, _ = oracle.quantize(K, b, s)
    codes = oracle.unpack(packed, d, b)
    best = [np.inf] * K.shape[0]
    best_code = [None] * K.shape[0]
    for chunk in _codeword_chunks(L, d):
        unit = cent[chunk].astype(np.float64) @ R          # R^T x for every codeword x
        for r in range(K.shape[0]):
            dist = ((float(norms[r]) * unit - K[r]) ** 2).sum(axis=1)
            i = int(np.argmin(dist))
            if dist[i] < best[r]:
                best[r], best_code[r] = dist[i], chunk[i]
    for r in range(K.shape[0]):
        assert np.array_equal(codes[r], best_code[r])


def _codeword_chunks(L, d, chunk=1 << 18):
    total = L ** d
    digits = L ** np.arange(d - 1, -1, -1)
    for start in range(0, total, chunk):
        ids = np.arange(start, min(total, start + chunk))
        yield (ids[:, None] // digits[None, :]) % L


@pytest.mark.parametrize("b", [2, 4])
def test_quantization_mse_matches_lloyd_max(b):
    """On keys whose rotated coordinates are ~N(0, 1/d), the mean squared error per
    coordinate is the Lloyd-Max distortion times 1/d."""
    d, n = 512, 600
    K = np.random.default_rng(b).standard_normal((n, d))
    s = _rng_signs(d, b)
    packed, norms, _ = oracle.quantize(K, b, s)
    _, U = oracle.rotate_unit(K, s)
    cent, _ = oracle.codebook(d, b)
    recon = cent[oracle.unpack(packed, d, b)].astype(np.float64)
    mse = ((U - recon) ** 2).mean() * d
    ref = _classical_table()[b][0]
    assert abs(mse - ref) < 0.05 * ref


def test_margins_are_distances_to_decision_points():
    d, b = 64, 3
    K = np.random.default_rng(5).standard_normal((20, d))
    s = _rng_signs(d, 5)
    _, _, marg = oracle.quantize(K, b, s, margins=True)
    _, U = oracle.rotate_unit(K, s)
    cent, _ = oracle.codebook(d, b)
    mids = (cent[:-1].astype(np.float64) + cent[1:].astype(np.float64)) / 2
    expect = np.abs(U[:, :, None] - mids[None, None, :]).min(axis=2)
    np.testing.assert_allclose(marg, expect, rtol=0, atol=1e-15)


# ---------------------------------------------------------------- read path --

@pytest.mark.parametrize("d,b,group", [(8, 2, 1), (64, 3, 2), (128, 4, 4), (256, 1, 3)])
def test_lut_scores_equal_dequantized_dot(d, b, group):
    """Table lookup with the once-rotated query equals attention on dequantized,
    inverse-rotated keys (R is orthonormal), to rounding."""
    heads, n = 2, 9
    rng = np.random.default_rng(d + b)
    s = _rng_signs(d, d + b)
    K = rng.standard_normal((heads * n, d)) * rng.lognormal(0, 1, (heads * n, 1))
    packed, norms, _ = oracle.quantize(K, b, s)
    q = rng.standard_normal((heads * group, d))
    a = oracle.scores(q, packed.reshape(heads, n, -1), norms.reshape(heads, n), group, b, s)
    c = oracle.dequant_scores(q, packed.reshape(heads, n, -1), norms.reshape(heads, n), group, b, s)
    scale = np.linalg.norm(q, axis=1)[:, None] * np.repeat(norms.reshape(heads, n), group, axis=0)
    assert np.max(np.abs(a - c) / scale) < 1e-12


def test_scores_brute_force_d8():
    """d = 8 scores from an explicit dense rotation and the unpacked codes."""
    d, b, group, heads, n = 8, 3, 2, 2, 5
    rng = np.random.default_rng(11)
    s = _rng_signs(d, 11)
    codes = rng.integers(0, 1 << b, (heads * n, d)).astype(np.uint8)
    packed = oracle.pack(codes, b).reshape(heads, n, -1)
    norms = rng.lognormal(0, 1, (heads, n)).astype(np.float32)
    q = rng.standard_normal((heads * group, d))
    cent, _ = oracle.codebook(d, b)
    R = scipy.linalg.hadamard(d) * s[None, :] / math.sqrt(d)
    got = oracle.scores(q, packed, norms, group, b, s)
    for hq in range(heads * group):
        h = hq // group
        qr = R @ q[hq]
        for t in range(n):
            expect = norms[h, t] * np.dot(qr, cent[codes[h * n + t]].astype(np.float64)) / math.sqrt(d)
            assert abs(got[hq, t] - expect) < 1e-12 * (1 + abs(expect))


def test_oracle_is_not_imported_by_the_product():
    """The product package never imports the oracle (and vice versa)."""
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    pkg = os.path.join(root, "lut_attention_b200")
    for dirpath, _, files in os.walk(pkg):
        for f in files:
            if f.endswith((".py", ".cu", ".cuh", ".cpp", ".h")):
                text = open(os.path.join(dirpath, f)).read()
                assert "import oracle" not in text and "from oracle" not in text, f
                assert "oracle.c" not in text and "liboracle" not in text, f
    text = open(os.path.join(root, "oracle", "oracle.c")).read()
    assert "axr" not in text.replace("AXELRAM", "")
    assert "lut_attention_b200" not in open(os.path.join(root, "oracle", "__init__.py")).read()


def test_workloads_deterministic_and_shaped():
    wl = workloads.PR1_REF.with_(T=64)
    a = workloads.make_keys(wl)
    b = workloads.make_keys(wl)
    assert a.shape == (1, 64, 128) and a.dtype == torch.float32 and torch.equal(a, b)
    s = workloads.make_signs(wl)
    assert s.dtype == torch.int8 and set(s.tolist()) <= {-1, 1}
    for w in workloads.ALL:
        small = w.with_(T=8, batch=1)
        k = workloads.make_keys(small)
        assert k.shape == (small.heads, 8, w.d) and k.dtype == w.torch_dtype
        assert torch.isfinite(k.float()).all()
        q = workloads.make_queries(small)
        assert q.shape == (small.heads * w.group, w.d)


# ---------------------------------------------------------------- attention --

def test_attention_of_equal_scores_is_the_mean_value_row():
    """q = 0 gives every key the score 0, so the softmax is uniform."""
    d, b, heads, n, group = 16, 3, 2, 37, 2
    rng = np.random.default_rng(5)
    s = _rng_signs(d, 5)
    packed, norms, _ = oracle.quantize(rng.standard_normal((heads * n, d)), b, s)
    V = rng.standard_normal((heads, n, d))
    out = oracle.attention(np.zeros((heads * group, d)), packed.reshape(heads, n, -1), norms.reshape(heads, n),
                           V, group, b, s)
    for h in range(heads):
        for g in range(group):
            assert np.allclose(out[h * group + g], V[h].mean(axis=0), rtol=0, atol=1e-14)


def test_attention_single_key_returns_its_value_row():
    d, b = 8, 2
    s = _rng_signs(d, 6)
    packed, norms, _ = oracle.quantize(np.arange(1.0, d + 1.0)[None], b, s)
    V = np.arange(d, dtype=np.float64)[None, None] * 0.5
    out = oracle.attention(np.ones((3, d)), packed[None], norms[None], V, 3, b, s)
    assert np.array_equal(out, np.repeat(V[0], 3, axis=0))


def test_attention_brute_force_on_dequantized_keys():
    """Independent of the oracle's numpy path: scores on dequantized,
    inverse-rotated keys, then softmax and the weighted sum in plain loops."""
    d, b, heads, n, group = 8, 2, 2, 5, 2
    rng = np.random.default_rng(7)
    s = _rng_signs(d, 7)
    K = rng.standard_normal((heads * n, d)) * 3.0
    packed, norms, _ = oracle.quantize(K, b, s)
    packed, norms = packed.reshape(heads, n, -1), norms.reshape(heads, n)
    q = rng.standard_normal((heads * group, d))
    V = rng.standard_normal((heads, n, d))
    sd = oracle.dequant_scores(q, packed, norms, group, b, s)
    got = oracle.attention(q, packed, norms, V, group, b, s)
    for row in range(heads * group):
        h = row // group
        w = [math.exp(sd[row, t]) for t in range(n)]
        tot = sum(w)
        for j in range(d):
            exp_v = sum(w[t] * V[h, t, j] for t in range(n)) / tot
            assert abs(got[row, j] - exp_v) <= 1e-12 * (1.0 + abs(exp_v))


def test_attention_is_linear_in_values_and_shift_free_in_scores():
    rng = np.random.default_rng(8)
    s = rng.standard_normal((6, 40)) * 4.0
    V = rng.standard_normal((3, 40, 8))
    a = oracle.attention_from_scores(s, V, 2)
    assert np.allclose(oracle.attention_from_scores(s + 123.0, V, 2), a, rtol=1e-13, atol=1e-13)
    assert np.allclose(oracle.attention_from_scores(s, 2.5 * V - 1.0, 2), 2.5 * a - 1.0, rtol=1e-13, atol=1e-13)


# --------------------------------------------------- sign-pattern selection --
# AXELRAM abstract: a gradient-free, one-time choice of the sign pattern among
# candidates on a few calibration samples.  The criterion is the mean squared
# error of the quantized attention logits against the exact ones, per KV head;
# the choice minimises the worst head.

def _calibration(S, heads, n, d, group, seed, C):
    rng = np.random.default_rng(seed)
    K = rng.standard_normal((S, heads, n, d)) * rng.lognormal(0, 1, (S, heads, 1, 1))
    q = rng.standard_normal((S, heads * group, d))
    cand = (rng.integers(0, 2, (C, d)) * 2 - 1).astype(np.int8)
    return K, q, cand


@pytest.mark.parametrize("b", [1, 2, 3])
def test_sign_errors_brute_force_d8(b):
    """Every calibration key dequantized through an explicit dense rotation and
    a nearest-centroid search over all codewords, the logit error in loops."""
    S, heads, n, d, group, C = 2, 2, 5, 8, 2, 3
    K, q, cand = _calibration(S, heads, n, d, group, 30 + b, C)
    cent, _ = oracle.codebook(d, b)
    got = oracle.sign_errors(K, q, group, b, cand)
    assert got.shape == (C, heads)
    for c in range(C):
        R = scipy.linalg.hadamard(d) * cand[c][None, :].astype(float) / math.sqrt(d)
        for h in range(heads):
            tot = 0.0
            for s in range(S):
                for t in range(n):
                    k = K[s, h, t]
                    norm = float(np.float32(math.sqrt(sum(x * x for x in k))))   # stored in fp32
                    u = R @ k / math.sqrt(sum(x * x for x in k))
                    code = [min(range(len(cent)), key=lambda l: abs(u[j] - float(cent[l]))) for j in range(d)]
                    khat = R.T @ (norm * np.array([float(cent[l]) for l in code]))
                    for g in range(group):
                        qq = q[s, h * group + g]
                        e = (np.dot(qq, khat) - np.dot(qq, k)) / math.sqrt(d)
                        tot += e * e
            expect = tot / (S * n * group)
            assert abs(got[c, h] - expect) <= 1e-10 * expect


@pytest.mark.parametrize("b", [2, 4])
def test_sign_errors_planted_pattern_closed_form(b):
    """Keys k = a (D* . h_r), h_r a Walsh-Hadamard row, and queries along them:
    the pattern D* sends every key onto one rotated axis, u = e_r, which the
    codebook maps to the top centroid c_max and every other coordinate (u_j = 0,
    a tie with the central boundary) to the centroid c_0 just below zero.  A query
    along a key of the same row gets the logit times c_max, error |q| |k|
    (c_max - 1) / sqrt(d); along another row (exact logit 0) the error is
    |q| |k| c_0 / sqrt(d) (|k| as stored, in fp32, where the method uses it).  D* and -D* are the two worst candidates and never
    selected."""
    d, S, heads, n, group = 128, 2, 3, 4, 2
    rng = np.random.default_rng(40 + b)
    H = scipy.linalg.hadamard(d).astype(float)
    star = (rng.integers(0, 2, d) * 2 - 1).astype(np.int8)
    K = np.empty((S, heads, n, d))
    q = np.empty((S, heads * group, d))
    for s in range(S):
        for h in range(heads):
            for t in range(n):
                K[s, h, t] = 2.0 ** (h - t % 2) * star * H[rng.integers(0, d)]
            for g in range(group):
                q[s, h * group + g] = (g + 1) * 0.5 * K[s, h, 0]
    cand = np.concatenate([(rng.integers(0, 2, (6, d)) * 2 - 1).astype(np.int8), star[None], -star[None]])
    E = oracle.sign_errors(K, q, group, b, cand)
    cent = oracle.codebook(d, b)[0].astype(np.float64)
    c_max, c_0 = cent[-1], cent[(1 << b) // 2 - 1]
    for h in range(heads):
        expect = 0.0
        for s in range(S):
            k0 = K[s, h, 0] / np.linalg.norm(K[s, h, 0])
            for t in range(n):
                for g in range(group):
                    qn, kn = np.linalg.norm(q[s, h * group + g]), np.linalg.norm(K[s, h, t])
                    kn32 = float(np.float32(kn))                    # the stored norm
                    same = np.array_equal(K[s, h, t] / kn, k0)     # queries lie along key 0
                    e = qn * ((kn32 * c_max - kn) if same else kn32 * c_0) / math.sqrt(d)
                    expect += e * e
        expect /= S * n * group
        for c in (6, 7):
            assert abs(E[c, h] - expect) <= 1e-9 * expect
    worst = E.max(axis=1)
    assert worst[6] > 10 * worst[:6].max() and worst[7] > 10 * worst[:6].max()
    assert oracle.select_signs(E) < 6


def test_sign_errors_symmetries_and_scaling():
    """-D gives the same errors as D (the codebook is symmetric); doubling the
    keys or the queries multiplies every error by 4 exactly."""
    S, heads, n, d, group, C = 2, 2, 30, 64, 3, 3
    K, q, cand = _calibration(S, heads, n, d, group, 50, C)
    E = oracle.sign_errors(K, q, group, 3, cand)
    assert np.array_equal(oracle.sign_errors(K, q, group, 3, -cand), E)
    assert np.array_equal(oracle.sign_errors(2.0 * K, q, group, 3, cand), 4.0 * E)
    assert np.array_equal(oracle.sign_errors(K, 2.0 * q, group, 3, cand), 4.0 * E)


def test_sign_errors_are_means_over_samples_queries_and_keys():
    """Two samples of equal size average their errors; a group of identical
    query heads has the error of one; the order of the keys does not matter."""
    S, heads, n, d, group, C = 2, 3, 40, 32, 1, 4
    K, q, cand = _calibration(S, heads, n, d, group, 60, C)
    b = 2
    E = oracle.sign_errors(K, q, group, b, cand)
    E0 = oracle.sign_errors(K[:1], q[:1], group, b, cand)
    E1 = oracle.sign_errors(K[1:], q[1:], group, b, cand)
    np.testing.assert_allclose(E, 0.5 * (E0 + E1), rtol=1e-12)
    q3 = np.repeat(q, 3, axis=1)                       # query head h*3 + g repeats q[:, h]
    np.testing.assert_allclose(oracle.sign_errors(K, q3, 3, b, cand), E, rtol=1e-12)
    perm = np.random.default_rng(61).permutation(n)
    np.testing.assert_allclose(oracle.sign_errors(K[:, :, perm], q, group, b, cand), E, rtol=1e-12)


@pytest.mark.parametrize("b", [1, 2, 3, 4])
def test_sign_errors_match_lloyd_max_distortion(b):
    """Isotropic keys and queries with |q|^2 = d: each rotated coordinate is
    quantized with the Lloyd-Max error D_b / d of Max's table, so the logit error
    is about |q|^2 E|k|^2 D_b / d^2 = D_b (within 6%: sampling, and the unit-norm
    constraint couples the coordinates)."""
    mse = {}
    with open(os.path.join(GOLDEN, "lloyd_max_classical.txt")) as f:
        for line in f:
            if line.strip() and not line.startswith("#"):
                parts = line.split()
                mse[int(parts[0])] = float(parts[1])
    rng = np.random.default_rng(70 + b)
    d, n, group = 128, 3000, 8
    K = rng.standard_normal((1, 1, n, d))
    q = rng.standard_normal((1, group, d))
    q *= math.sqrt(d) / np.linalg.norm(q, axis=2, keepdims=True)
    cand = _rng_signs(d, 71)[None]
    E = oracle.sign_errors(K, q, group, b, cand)[0, 0]
    assert abs(E / mse[b] - 1.0) < 0.06, E / mse[b]


def test_select_signs_worst_head_and_lowest_index():
    E = np.array([[1.0, 5.0], [3.0, 3.0], [2.0, 4.0], [3.0, 2.5], [0.5, 3.0]])
    assert oracle.select_signs(E) == 1          # worst heads 5, 3, 4, 3, 3: the first 3
    assert oracle.select_signs(E[2:]) == 1
    S, heads, n, d, group = 1, 2, 20, 16, 2
    K, q, cand = _calibration(S, heads, n, d, group, 80, 3)
    dup = np.stack([cand[0], cand[1], cand[1], -cand[1], cand[2]])
    Ed = oracle.sign_errors(K, q, group, 2, dup)
    assert np.array_equal(Ed[1], Ed[2]) and np.array_equal(Ed[1], Ed[3])
    assert oracle.select_signs(Ed) != 2 and oracle.select_signs(Ed) != 3


# ------------------------------------------------------------ block rotation --
# IsoQuant abstract: each 4-element block is a quaternion v, rotated to
# qL v conj(qR) (IsoQuant-Full; qR = 1 is IsoQuant-Fast).

def _unit_quats(rng, m):
    z = rng.standard_normal((m, 2, 4))
    return (z / np.linalg.norm(z, axis=2, keepdims=True)).reshape(m, 8)


def _block_of(d, qL, qR):
    return oracle.block_rotation(d, np.concatenate([qL, qR])[None].repeat(d // 4, axis=0))[:4, :4]


def test_block_rotation_follows_hamilton_rules():
    """i, j, k multiply as i^2 = j^2 = k^2 = ijk = -1: left multiplication by i
    sends (1, i, j, k) to (i, -1, k, -j), and so on; right multiplication by
    conj(i) = -i sends them to (-i, 1, k, -j)."""
    one, i, j, k = np.eye(4)
    # columns = images of 1, i, j, k
    assert np.array_equal(_block_of(4, i, one), np.array([i, -one, k, -j]).T)
    assert np.array_equal(_block_of(4, j, one), np.array([j, -k, -one, i]).T)
    assert np.array_equal(_block_of(4, k, one), np.array([k, j, -i, -one]).T)
    assert np.array_equal(_block_of(4, one, i), np.array([-i, one, k, -j]).T)
    assert np.array_equal(_block_of(4, one, one), np.eye(4))


def test_block_rotation_is_orthonormal_and_block_diagonal():
    rng = np.random.default_rng(90)
    for d in (8, 32, 128, 512):
        quats = _unit_quats(rng, d // 4)
        R = oracle.block_rotation(d, quats)
        np.testing.assert_allclose(R @ R.T, np.eye(d), rtol=0, atol=1e-14)
        mask = np.kron(np.eye(d // 4), np.ones((4, 4)))
        assert np.all(R[mask == 0] == 0)


def test_block_rotation_isoclinic_and_conjugation_closed_forms():
    """Fast (qR = 1) turns every vector by the same angle: <v, a v> = a0 |v|^2.
    Full with qL = qR = a = cos(t/2) + sin(t/2) n fixes the real axis and turns
    the imaginary part about n by t (Rodrigues' formula)."""
    rng = np.random.default_rng(91)
    for _ in range(5):
        a = rng.standard_normal(4)
        a /= np.linalg.norm(a)
        T = _block_of(4, a, np.eye(4)[0])
        for _ in range(4):
            v = rng.standard_normal(4)
            assert abs(v @ T @ v - a[0] * (v @ v)) < 1e-13
        t = rng.uniform(0, np.pi)
        nvec = rng.standard_normal(3)
        nvec /= np.linalg.norm(nvec)
        a = np.concatenate([[math.cos(t / 2)], math.sin(t / 2) * nvec])
        T = _block_of(4, a, a)
        x = rng.standard_normal(3)
        rod = (x * math.cos(t) + np.cross(nvec, x) * math.sin(t) + nvec * (nvec @ x) * (1 - math.cos(t)))
        np.testing.assert_allclose(T @ np.concatenate([[2.5], x]), np.concatenate([[2.5], rod]), atol=1e-13)


@pytest.mark.parametrize("b", [1, 2, 3])
def test_block_quantize_and_scores_brute_force_d8(b):
    """d = 8 (two blocks): T built from the 4 x 4 left and right multiplication
    matrices, nearest codeword over all centroids, and the scores in loops."""
    d, n, heads, group = 8, 6, 2, 2
    rng = np.random.default_rng(100 + b)
    quats = _unit_quats(rng, 2)

    def left(a):
        return np.array([[a[0], -a[1], -a[2], -a[3]], [a[1], a[0], -a[3], a[2]],
                         [a[2], a[3], a[0], -a[1]], [a[3], -a[2], a[1], a[0]]])

    def right(c):     # v -> v c
        return np.array([[c[0], -c[1], -c[2], -c[3]], [c[1], c[0], c[3], -c[2]],
                         [c[2], -c[3], c[0], c[1]], [c[3], c[2], -c[1], c[0]]])

    T = np.zeros((d, d))
    for m in range(2):
        qL, qR = quats[m, :4], quats[m, 4:]
        T[4 * m:4 * m + 4, 4 * m:4 * m + 4] = right(qR * np.array([1, -1, -1, -1])) @ left(qL)
    K = rng.standard_normal((heads * n, d)) * 2.0
    packed, norms, _ = oracle.quantize_block(K, b, quats)
    cent, _ = oracle.codebook(d, b)
    codes = oracle.unpack(packed, d, b)
    for r in range(heads * n):
        nk = math.sqrt(sum(x * x for x in K[r]))
        assert norms[r] == np.float32(nk)
        u = T @ K[r] / float(np.float32(nk))
        for j in range(d):
            best = min(range(len(cent)), key=lambda l: abs(u[j] - float(cent[l])))
            assert codes[r, j] == best
    q = rng.standard_normal((heads * group, d))
    got = oracle.scores_block(q, packed.reshape(heads, n, -1), norms.reshape(heads, n), group, b, quats)
    for hq in range(heads * group):
        qr = T @ q[hq]
        for t in range(n):
            r = (hq // group) * n + t
            expect = norms[r] * sum(qr[j] * float(cent[codes[r, j]]) for j in range(d)) / math.sqrt(d)
            assert abs(got[hq, t] - expect) < 1e-12 * (1 + abs(expect))


@pytest.mark.parametrize("d,b", [(128, 4), (256, 2), (512, 3)])
def test_block_lut_scores_equal_dequantized_dot(d, b):
    """T is orthonormal, so reading through the once-rotated query equals the dot
    product with the dequantized, inverse-rotated key."""
    heads, n, group = 2, 7, 2
    rng = np.random.default_rng(d + b)
    quats = _unit_quats(rng, d // 4)
    K = rng.standard_normal((heads * n, d)) * rng.lognormal(0, 1, (heads * n, 1))
    packed, norms, _ = oracle.quantize_block(K, b, quats)
    q = rng.standard_normal((heads * group, d))
    a = oracle.scores_block(q, packed.reshape(heads, n, -1), norms.reshape(heads, n), group, b, quats)
    c = oracle.dequant_scores_block(q, packed.reshape(heads, n, -1), norms.reshape(heads, n), group, b, quats)
    scale = np.linalg.norm(q, axis=1)[:, None] * np.repeat(norms.reshape(heads, n), group, axis=0)
    assert np.max(np.abs(a - c) / scale) < 1e-12


@pytest.mark.parametrize("b", [2, 4])
def test_block_quantization_mse_matches_lloyd_max_on_isotropic_keys(b):
    """An orthonormal T keeps isotropic keys isotropic, so the coordinates of the
    rotated unit keys are ~N(0, 1/d) and quantize with Max's mean squared error
    D_b per unit variance (within 5%)."""
    mse = {}
    with open(os.path.join(GOLDEN, "lloyd_max_classical.txt")) as f:
        for line in f:
            if line.strip() and not line.startswith("#"):
                parts = line.split()
                mse[int(parts[0])] = float(parts[1])
    d, n = 128, 2000
    rng = np.random.default_rng(110 + b)
    quats = _unit_quats(rng, d // 4)
    K = rng.standard_normal((n, d))
    packed, norms, _ = oracle.quantize_block(K, b, quats)
    cent, _ = oracle.codebook(d, b)
    U = (oracle.block_rotation(d, quats) @ K.T).T / norms[:, None].astype(np.float64)
    err = np.mean((cent[oracle.unpack(packed, d, b)].astype(np.float64) - U) ** 2) * d
    assert abs(err / mse[b] - 1.0) < 0.05, err / mse[b]
