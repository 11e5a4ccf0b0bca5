"""The counting rules of the full-size parity report (CPU only).

Host logic: the chunk comparison of tests/full_parity.py is fed the oracle's own
outputs for a few hundred keys, then copies of them with one code changed, one
norm scaled and one score shifted, and must count exactly those changes.
"""
import math

import numpy as np

import full_parity
import oracle


def _chunk(seed=3, m=300, d=128, b=4, G=4):
    rng = np.random.default_rng(seed)
    K = rng.standard_normal((m, d)) * np.exp(0.5 * rng.standard_normal((m, 1)))
    s = np.where(rng.integers(0, 2, d) > 0, 1, -1).astype(np.int8)
    q = rng.standard_normal((G, d))
    idx, norms, marg = oracle.quantize(K, b, s, margins=True)
    sc = oracle.scores(q, idx[None], norms[None], G, b, s).astype(np.float32)
    return K, idx, norms, sc, q, s, marg


def test_oracle_against_itself_counts_nothing(oracle_lib):
    K, idx, norms, sc, q, s, marg = _chunk()
    r = full_parity._check_chunk(K, idx, norms, sc, q, 4, s)
    assert r["coords"] == K.size and r["flips"] == 0 and r["flips_outside_window"] == 0
    assert r["in_window"] == int((marg < full_parity.WINDOW).sum())
    assert r["max_norm_rel"] == 0.0 and r["bytes_mismatch_rows_without_flip"] == 0
    assert r["score_err"] < 1e-6 and r["e2e_score_err"] < 1e-6 and r["e2e_rows"] == K.shape[0]


def test_planted_changes_are_counted(oracle_lib):
    d, b, G = 128, 4, 4
    K, idx, norms, sc, q, s, marg = _chunk(d=d, b=b, G=G)
    codes = oracle.unpack(idx, d, b)
    # a code far from any boundary moved to its neighbour: a flip outside the window
    r0, j0 = np.unravel_index(np.argmax(marg), marg.shape)
    codes[r0, j0] = codes[r0, j0] + 1 if codes[r0, j0] < (1 << b) - 1 else codes[r0, j0] - 1
    bad_idx = oracle.pack(codes, b)
    bad_norms = norms.copy()
    bad_norms[7] *= 1.0 + 3e-4
    bad_sc = sc.copy()
    scale = np.linalg.norm(q[2]) * norms[11] / math.sqrt(d)
    bad_sc[2, 11] += np.float32(5e-4 * scale)
    r = full_parity._check_chunk(K, bad_idx, bad_norms, bad_sc, q, b, s)
    assert r["flips"] == 1 and r["flips_outside_window"] == 1
    assert 2.9e-4 < r["max_norm_rel"] < 3.1e-4
    assert r["score_err"] >= 4e-4       # the shifted score (and the moved code, scored on the library codes)
    assert r["e2e_rows"] == K.shape[0] - 1                       # the flipped row leaves the end-to-end check
    assert r["e2e_score_err"] >= 4e-4                             # the shifted score is seen end to end


def test_sample_tokens_hold_first_and_last():
    tok = full_parity.sample_tokens(65536, 8192, seed=5, h=3)
    assert tok[0] == 0 and tok[-1] == 65535 and len(tok) == 8192 + 2
    assert bool((tok[1:] > tok[:-1]).all())
