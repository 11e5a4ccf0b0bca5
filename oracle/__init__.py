"""CPU oracle for the AXELRAM write path, read path, sign-pattern choice and block rotation: test infrastructure.

Only ``tests/``, ``__graft_entry__.smoke()`` and the CPU-baseline leg of
``bench.py`` may import this package.  The CUDA library never uses it, and it
imports nothing from the library.  The arithmetic lives in ``oracle.c`` (plain
C, fp64); this module compiles it with gcc and marshals numpy arrays into it.

Every function takes and returns numpy arrays on the host.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import threading

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "oracle.c")
_LIB_PATH = os.path.join(_HERE, "liboracle.so")
_lock = threading.Lock()
_lib = None


def build(force: bool = False) -> str:
    """Compile oracle.c into liboracle.so next to it (gcc, -O2, no fast-math)."""
    up_to_date = (
        os.path.exists(_LIB_PATH)
        and os.path.getmtime(_LIB_PATH) >= os.path.getmtime(_SRC)
    )
    if force or not up_to_date:
        tmp = f"{_LIB_PATH}.{os.getpid()}.tmp"
        subprocess.check_call(
            ["gcc", "-std=c11", "-O2", "-Wall", "-Wextra", "-shared", "-fPIC",
             "-o", tmp, _SRC, "-lm"]
        )
        os.replace(tmp, _LIB_PATH)
    return _LIB_PATH


def _load():
    global _lib
    with _lock:
        if _lib is not None:
            return _lib
        lib = ctypes.CDLL(build())
        P = ctypes.c_void_p
        i32, i64 = ctypes.c_int, ctypes.c_int64
        sig = {
            "oracle_hadamard": [i32, P],
            "oracle_rotation": [i32, P, P],
            "oracle_lloyd_max_std": [i32, P, P],
            "oracle_codebook": [i32, i32, P, P],
            "oracle_pack": [P, i64, i32, i32, P],
            "oracle_unpack": [P, i64, i32, i32, P],
            "oracle_rotate_unit": [P, i64, i32, P, P, P],
            "oracle_quantize": [P, i64, i32, i32, P, P, P, P],
            "oracle_scores": [P, P, P, i64, i32, i32, i32, i32, P, P],
            "oracle_dequant_scores": [P, P, P, i64, i32, i32, i32, i32, P, P],
            "oracle_block_rotation": [i32, P, P],
            "oracle_quantize_block": [P, i64, i32, i32, P, P, P, P],
            "oracle_scores_block": [P, P, P, i64, i32, i32, i32, i32, P, P],
            "oracle_dequant_scores_block": [P, P, P, i64, i32, i32, i32, i32, P, P],
        }
        for name, args in sig.items():
            fn = getattr(lib, name)
            fn.argtypes = args
            fn.restype = ctypes.c_int
        _lib = lib
        return lib


def _ptr(a: np.ndarray | None):
    return None if a is None else a.ctypes.data_as(ctypes.c_void_p)


def _check(rc: int, what: str) -> None:
    if rc != 0:
        raise ValueError(f"oracle: {what} rejected its arguments (rc={rc})")


def _signs(signs, d: int) -> np.ndarray:
    s = np.ascontiguousarray(np.asarray(signs), dtype=np.int8).reshape(-1)
    if s.shape[0] != d:
        raise ValueError(f"signs must have {d} entries, got {s.shape[0]}")
    return s


def hadamard(d: int) -> np.ndarray:
    """Sylvester-ordered Walsh-Hadamard matrix, entries +-1, shape (d, d)."""
    H = np.empty((d, d), dtype=np.float64)
    _check(_load().oracle_hadamard(d, _ptr(H)), "hadamard")
    return H


def rotation(d: int, signs) -> np.ndarray:
    """R = H diag(signs) / sqrt(d), shape (d, d)."""
    R = np.empty((d, d), dtype=np.float64)
    _check(_load().oracle_rotation(d, _ptr(_signs(signs, d)), _ptr(R)), "rotation")
    return R


def lloyd_max_std(b: int) -> tuple[np.ndarray, int]:
    """Lloyd-Max centroids of N(0,1), 2^b levels ascending (fp64), and iteration count."""
    c = np.empty(1 << b, dtype=np.float64)
    it = ctypes.c_int(0)
    _check(_load().oracle_lloyd_max_std(b, _ptr(c), ctypes.byref(it)), "lloyd_max_std")
    return c, it.value


def codebook(d: int, b: int) -> tuple[np.ndarray, np.ndarray]:
    """fp32 centroids (2^b, ascending) and fp32 decision boundaries (2^b - 1)."""
    L = 1 << b
    cent = np.empty(L, dtype=np.float32)
    bnd = np.empty(L - 1, dtype=np.float32)
    _check(_load().oracle_codebook(d, b, _ptr(cent), _ptr(bnd)), "codebook")
    return cent, bnd


def pack(codes: np.ndarray, b: int) -> np.ndarray:
    """(n, d) codes in [0, 2^b) -> (n, d*b/8) bytes, dense LSB-first bit stream."""
    codes = np.ascontiguousarray(codes, dtype=np.uint8)
    n, d = codes.shape
    out = np.empty((n, d * b // 8), dtype=np.uint8)
    _check(_load().oracle_pack(_ptr(codes), n, d, b, _ptr(out)), "pack")
    return out


def unpack(packed: np.ndarray, d: int, b: int) -> np.ndarray:
    """Inverse of :func:`pack`: (..., d*b/8) bytes -> (..., d) codes."""
    packed = np.ascontiguousarray(packed, dtype=np.uint8)
    lead = packed.shape[:-1]
    n = int(np.prod(lead)) if lead else 1
    out = np.empty(lead + (d,), dtype=np.uint8)
    _check(_load().oracle_unpack(_ptr(packed), n, d, b, _ptr(out)), "unpack")
    return out


def rotate_unit(K: np.ndarray, signs) -> tuple[np.ndarray, np.ndarray]:
    """fp32 norms (n,) and rotated unit keys U = R K / norm (n, d, fp64)."""
    K = np.ascontiguousarray(K, dtype=np.float64)
    n, d = K.shape
    norms = np.empty(n, dtype=np.float32)
    U = np.empty((n, d), dtype=np.float64)
    _check(_load().oracle_rotate_unit(_ptr(K), n, d, _ptr(_signs(signs, d)), _ptr(norms), _ptr(U)),
           "rotate_unit")
    return norms, U


def quantize(K: np.ndarray, b: int, signs, margins: bool = False):
    """Quantize-on-write of K (n, d).

    Returns ``(packed (n, d*b/8) uint8, norms (n,) fp32, margins)`` where
    ``margins`` is None unless requested, else (n, d) fp64 distances of every
    rotated unit coordinate to its nearest decision point.
    """
    K = np.ascontiguousarray(K, dtype=np.float64)
    n, d = K.shape
    packed = np.empty((n, d * b // 8), dtype=np.uint8)
    norms = np.empty(n, dtype=np.float32)
    marg = np.empty((n, d), dtype=np.float64) if margins else None
    _check(_load().oracle_quantize(_ptr(K), n, d, b, _ptr(_signs(signs, d)), _ptr(packed),
                                   _ptr(norms), _ptr(marg)), "quantize")
    return packed, norms, marg


def _read_args(q, packed, norms, group, b):
    q = np.ascontiguousarray(q, dtype=np.float64)
    hg, d = q.shape
    if hg % group:
        raise ValueError("q rows must be heads*group")
    heads = hg // group
    packed = np.ascontiguousarray(packed, dtype=np.uint8)
    norms = np.ascontiguousarray(norms, dtype=np.float32)
    if packed.ndim != 3 or packed.shape[0] != heads or packed.shape[2] != d * b // 8:
        raise ValueError(f"packed must be (heads, n, {d * b // 8})")
    n = packed.shape[1]
    if norms.shape != (heads, n):
        raise ValueError("norms must be (heads, n)")
    return q, packed, norms, heads, n, d


def scores(q, packed, norms, group: int, b: int, signs) -> np.ndarray:
    """LUT scores (heads*group, n), fp64: norm * sum_j (R q)_j c[idx_j] / sqrt(d)."""
    q, packed, norms, heads, n, d = _read_args(q, packed, norms, group, b)
    out = np.empty((heads * group, n), dtype=np.float64)
    _check(_load().oracle_scores(_ptr(q), _ptr(packed), _ptr(norms), n, heads, group, d, b,
                                 _ptr(_signs(signs, d)), _ptr(out)), "scores")
    return out


def dequant_scores(q, packed, norms, group: int, b: int, signs) -> np.ndarray:
    """Scores on dequantized, inverse-rotated keys: q . (norm R^T c[idx]) / sqrt(d)."""
    q, packed, norms, heads, n, d = _read_args(q, packed, norms, group, b)
    out = np.empty((heads * group, n), dtype=np.float64)
    _check(_load().oracle_dequant_scores(_ptr(q), _ptr(packed), _ptr(norms), n, heads, group, d,
                                         b, _ptr(_signs(signs, d)), _ptr(out)), "dequant_scores")
    return out


def attention_from_scores(s: np.ndarray, V: np.ndarray, group: int) -> np.ndarray:
    """Decode attention after the scores (fp64): for query head h*group + g,
    p = softmax(s[h*group + g, :]) over the n keys of KV head h, and the output
    is sum_t p_t V[h, t, :].  s: (heads*group, n); V: (heads, n, d) as stored.

    The pages define the scores only; softmax over a query's scores and the
    weighted sum of the value rows is the standard attention that consumes them.
    The values are read as given (not quantized).
    """
    s = np.asarray(s, dtype=np.float64)
    V = np.asarray(V, dtype=np.float64)
    heads, n, d = V.shape
    if s.shape != (heads * group, n):
        raise ValueError(f"scores must be ({heads * group}, {n})")
    m = s.max(axis=1, keepdims=True)
    p = np.exp(s - m)
    p /= p.sum(axis=1, keepdims=True)
    out = np.empty((heads * group, d), dtype=np.float64)
    for h in range(heads):
        out[h * group:(h + 1) * group] = p[h * group:(h + 1) * group] @ V[h]
    return out


def attention(q, packed, norms, V, group: int, b: int, signs) -> np.ndarray:
    """Decode attention on the quantized keys: softmax of the LUT scores
    (:func:`scores`) times the value rows, (heads*group, d) fp64."""
    return attention_from_scores(scores(q, packed, norms, group, b, signs), V, group)


def _quats(quats, d: int) -> np.ndarray:
    qs = np.ascontiguousarray(np.asarray(quats, dtype=np.float64))
    if qs.shape != (d // 4, 8):
        raise ValueError(f"quats must be ({d // 4}, 8): qL then qR of every 4-block")
    return qs


def block_rotation(d: int, quats) -> np.ndarray:
    """IsoQuant block rotation T (d, d): block m of coordinates 4m..4m+3 read as
    a quaternion v and mapped to qL v conj(qR), quats[m] = (qL, qR)."""
    R = np.empty((d, d), dtype=np.float64)
    _check(_load().oracle_block_rotation(d, _ptr(_quats(quats, d)), _ptr(R)), "block_rotation")
    return R


def quantize_block(K: np.ndarray, b: int, quats, margins: bool = False):
    """:func:`quantize` with the block rotation in place of H diag(signs)/sqrt(d)."""
    K = np.ascontiguousarray(K, dtype=np.float64)
    n, d = K.shape
    packed = np.empty((n, d * b // 8), dtype=np.uint8)
    norms = np.empty(n, dtype=np.float32)
    marg = np.empty((n, d), dtype=np.float64) if margins else None
    _check(_load().oracle_quantize_block(_ptr(K), n, d, b, _ptr(_quats(quats, d)), _ptr(packed), _ptr(norms),
                                         _ptr(marg)), "quantize_block")
    return packed, norms, marg


def scores_block(q, packed, norms, group: int, b: int, quats) -> np.ndarray:
    """:func:`scores` with the queries rotated by the block rotation."""
    q, packed, norms, heads, n, d = _read_args(q, packed, norms, group, b)
    out = np.empty((heads * group, n), dtype=np.float64)
    _check(_load().oracle_scores_block(_ptr(q), _ptr(packed), _ptr(norms), n, heads, group, d, b,
                                       _ptr(_quats(quats, d)), _ptr(out)), "scores_block")
    return out


def dequant_scores_block(q, packed, norms, group: int, b: int, quats) -> np.ndarray:
    """:func:`dequant_scores` with the block rotation."""
    q, packed, norms, heads, n, d = _read_args(q, packed, norms, group, b)
    out = np.empty((heads * group, n), dtype=np.float64)
    _check(_load().oracle_dequant_scores_block(_ptr(q), _ptr(packed), _ptr(norms), n, heads, group, d, b,
                                               _ptr(_quats(quats, d)), _ptr(out)), "dequant_scores_block")
    return out


def sign_errors(K, q, group: int, b: int, candidates) -> np.ndarray:
    """Calibration score error of each candidate sign pattern, (C, heads) fp64.

    AXELRAM abstract: the sign pattern D is chosen once, without gradients, from
    a set of candidates (200) on a few calibration samples (8), which removes the
    spikes that some patterns cause where key norms differ from head to head.  The
    pages rank candidates by perplexity, which needs a model; this criterion is the
    quantity the quantized cache perturbs, the attention logit.  For candidate
    D_c every calibration key is quantized with D_c (:func:`quantize`) and scored
    with D_c (:func:`scores`), and

        E[c, h] = mean over samples s, query heads g < group and keys t of
                  (score_c(q[s, h*group + g], k[s, h, t]) - q . k / sqrt(d))^2

    is its mean squared error against the exact logit.

    K: (samples, heads, n, d) keys; q: (samples, heads*group, d), the queries of
    each sample; candidates: (C, d) of +-1.
    """
    K = np.asarray(K, dtype=np.float64)
    if K.ndim != 4:
        raise ValueError("K must be (samples, heads, n, d)")
    S, heads, n, d = K.shape
    q = np.asarray(q, dtype=np.float64)
    if q.shape != (S, heads * group, d):
        raise ValueError(f"q must be ({S}, {heads * group}, {d})")
    cand = np.asarray(candidates)
    if cand.ndim != 2 or cand.shape[1] != d:
        raise ValueError(f"candidates must be (C, {d})")
    if n == 0:
        raise ValueError("no calibration keys")
    sq = np.zeros((cand.shape[0], heads), dtype=np.float64)
    for c in range(cand.shape[0]):
        for s in range(S):
            packed, norms, _ = quantize(K[s].reshape(heads * n, d), b, cand[c])
            approx = scores(q[s], packed.reshape(heads, n, -1), norms.reshape(heads, n), group, b, cand[c])
            for h in range(heads):
                rows = slice(h * group, (h + 1) * group)
                exact = q[s, rows] @ K[s, h].T / np.sqrt(d)
                diff = approx[rows] - exact
                sq[c, h] += np.sum(diff * diff)
    return sq / (S * group * n)


def select_signs(errors) -> int:
    """The candidate whose worst head has the smallest error: argmin over c of
    max over h of errors[c, h], the lowest index among equal values."""
    worst = np.asarray(errors, dtype=np.float64).max(axis=1)
    return int(np.argmin(worst))     # numpy returns the first of equal minima
