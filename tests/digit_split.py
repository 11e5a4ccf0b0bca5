"""The fixed-point split the tensor-core read kernel feeds its integer products,
restated in numpy from its definition, and the worst-case score error it allows.

AXELRAM (arXiv 2604.02638), abstract: scores are read by table lookup on the
stored indices.  The tensor-core read turns every looked-up centroid into two
signed 8-bit digits and every rotated query coordinate into three, so that the
table walk becomes an exact int32 contraction:
  * centroids: S_c = 127 / max|c|, v_i = round(c_i * 128 * S_c) (ties to even),
    hi_i = round(v_i / 128), lo_i = v_i - 128 hi_i; the kernel computes with
    c~_i = v_i / (128 S_c), so each centroid carries the error c~_i - c_i;
  * queries: with q'' the rotated query and S_q = 64 / max_j |q''_j|, the digits
    D0 + D1/128 + D2/128^2 represent q'' S_q to within 0.5 / 128^2, i.e. each
    coordinate to within 0.5 / (128^2 * 64) of max_j |q''_j|.

The score of a key is norm * sum_j q'_j c_j / sqrt(d) with q' = R q (||q'|| =
||q||), and the tolerance is 1e-4 ||q|| norm / sqrt(d).  Relative to that scale
the error is

    E = sum_j q'_j (c~_j - c_j) + sum_j (q~'_j - q'_j) c~_j,

and with M = max_j |q'_j| / ||q|| in [1/sqrt(d), 1]:

    |E| / ||q|| <= dc * (M + sqrt(d - 1) sqrt(1 - M^2)) + eq * M * d * max|c~|,

dc = max_i |c~_i - c_i|, eq = 0.5 / (128^2 * 64).  (sum_j |q'_j| is at most
M + sqrt(d-1) sqrt(1-M^2) for a unit vector whose largest entry is M.)  The
first term is largest when every code sits on the centroid with the largest
digit error and q' spreads evenly over the coordinates with that error's sign:
q' = +-||q|| (1, ..., 1) / sqrt(d), which is q = +-||q|| D_0 e_0.  Then every
query digit is exact and the error is exactly sqrt(d) * dc.
"""
from __future__ import annotations

import numpy as np

QUERY_DIGIT_ERR = 0.5 / (128.0 ** 2 * 64.0)


def centroid_digits(cent: np.ndarray):
    """(hi, lo, v, cmax) of the fp32 centroids: v = 128 hi + lo, |hi| <= 127."""
    cent = np.asarray(cent, dtype=np.float64)
    cmax = float(np.abs(cent).max())
    sc = 127.0 / cmax
    v = np.rint(cent * 128.0 * sc)            # numpy rounds ties to even
    hi = np.rint(v / 128.0)
    lo = v - 128.0 * hi
    return hi.astype(np.int64), lo.astype(np.int64), v.astype(np.int64), cmax


def represented_centroids(cent: np.ndarray) -> np.ndarray:
    """c~_i = v_i / (128 S_c): the centroids as the integer products see them."""
    _, _, v, cmax = centroid_digits(cent)
    return v / (128.0 * 127.0 / cmax)


def centroid_errors(cent: np.ndarray) -> np.ndarray:
    return represented_centroids(cent) - np.asarray(cent, dtype=np.float64)


def worst_case_bound(cent: np.ndarray, d: int, grid: int = 20001) -> tuple[float, float]:
    """(bound on |E| / ||q|| over all queries and codes, the M where it peaks)."""
    dc = float(np.abs(centroid_errors(cent)).max())
    ct = float(np.abs(represented_centroids(cent)).max())
    M = np.linspace(1.0 / np.sqrt(d), 1.0, grid)
    f = dc * (M + np.sqrt(d - 1.0) * np.sqrt(np.clip(1.0 - M * M, 0.0, None))) + QUERY_DIGIT_ERR * M * d * ct
    k = int(np.argmax(f))
    return float(f[k]), float(M[k])


def aligned_worst_case(cent: np.ndarray, d: int) -> tuple[int, float]:
    """(code i* with the largest digit error, the error sqrt(d) * (c~ - c)[i*]
    that all-i* rows give against q = sign * e_0 * D_0, in units of ||q|| ||k||
    / sqrt(d); its sign is the sign that query must carry)."""
    err = centroid_errors(cent)
    i = int(np.argmax(np.abs(err)))
    return i, float(np.sqrt(d) * err[i])
