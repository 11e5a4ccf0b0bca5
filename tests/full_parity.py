"""Full-size parity of the write and read paths with the oracle, row by row.

The five decode workloads run at their full sizes through the C ABI, in the
launch configuration the benchmark times (one quantize call over every key of
the batch, one scores call over the whole cache).  Every key row (or, for the
two wide-head workloads, a seeded sample of at least 2^20 rows plus the first
and last row of every KV head) is then compared with the oracle on the host
cores, chunk by chunk in a thread pool (the oracle's C code runs without the
interpreter lock).

Per workload the report counts, over the compared coordinates:
  * in_window:   coordinates whose rotated unit value lies within 1e-6 of a
                 decision boundary (the oracle's fp64 margin);
  * flips:       codes that differ from the oracle's;
  * flips_outside_window: flips outside that window (must be 0);
  * max_norm_rel: worst |norm_gpu - norm_oracle| / norm_oracle;
  * score_err:   worst |s_gpu - s_oracle| / (||q|| ||k|| / sqrt(d)) with the
                 oracle scoring the library's own codes (the read path alone);
  * e2e_score_err: the same with the oracle scoring its own codes, over rows
                 without a flip (the whole path).

AXELRAM (arXiv 2604.02638), abstract: the codebook is fixed at design time and
each coordinate takes its nearest centroid, so the codes are a function of the
key alone; the bar is bit-exact codes outside the boundary window, flips inside
it fewer than 1e-5 of the coordinates, norms and scores within 1e-4.
"""
from __future__ import annotations

import math
import os
import time
from concurrent.futures import ThreadPoolExecutor
from dataclasses import asdict, dataclass, field

import numpy as np
import torch

import oracle
from lut_attention_b200 import axr, workloads
from parity import FLIP_FRACTION, NORM_RTOL, SCORE_TOL, WINDOW

# reports of this session, printed by the terminal summary hook in conftest.py
REPORTS: list = []

CHUNK_ROWS = 16384


@dataclass
class FullReport:
    workload: str
    b: int
    d: int
    group: int
    rows_total: int
    rows_checked: int
    coords: int = 0
    in_window: int = 0
    flips: int = 0
    flips_outside_window: int = 0
    bytes_mismatch_rows_without_flip: int = 0
    max_norm_rel: float = 0.0
    score_err: float = 0.0
    e2e_score_err: float = 0.0
    e2e_rows: int = 0
    host_seconds: float = 0.0
    host_threads: int = 0
    selection: str = ""
    notes: list = field(default_factory=list)

    @property
    def flip_fraction(self) -> float:
        return self.flips / self.coords if self.coords else 0.0

    def ok(self) -> bool:
        return (self.flips_outside_window == 0 and self.flips <= FLIP_FRACTION * self.coords
                and self.bytes_mismatch_rows_without_flip == 0 and self.max_norm_rel <= NORM_RTOL
                and self.score_err <= SCORE_TOL and self.e2e_score_err <= SCORE_TOL)

    def line(self) -> str:
        return (f"{self.workload} b={self.b}: rows {self.rows_checked}/{self.rows_total} ({self.selection}), "
                f"coords {self.coords}, in-window {self.in_window}, flips {self.flips} "
                f"({self.flip_fraction:.2e} of coords), flips outside window {self.flips_outside_window}, "
                f"max norm rel {self.max_norm_rel:.2e}, score err {self.score_err:.2e}, "
                f"e2e score err {self.e2e_score_err:.2e} over {self.e2e_rows} rows, "
                f"host {self.host_seconds:.0f} s on {self.host_threads} threads")

    def as_dict(self) -> dict:
        d = asdict(self)
        d["flip_fraction"] = self.flip_fraction
        d["ok"] = self.ok()
        return d


def host_threads() -> int:
    try:
        return max(1, len(os.sched_getaffinity(0)))
    except AttributeError:
        return os.cpu_count() or 1


def _check_chunk(K: np.ndarray, g_idx: np.ndarray, g_norms: np.ndarray, g_scores: np.ndarray,
                 qh: np.ndarray, b: int, s: np.ndarray) -> dict:
    """One chunk of one KV head: K (m, d) fp64, the library's codes (m, P), norms
    (m,) and scores (G, m) for those rows, and the head's G queries (G, d)."""
    m, d = K.shape
    G = qh.shape[0]
    o_idx, o_norms, marg = oracle.quantize(K, b, s, margins=True)
    oc = oracle.unpack(o_idx, d, b)
    gc = oracle.unpack(g_idx, d, b)
    flip = oc != gc
    rows_flip = flip.any(axis=1)
    on = o_norms.astype(np.float64)
    gn = g_norms.astype(np.float64)
    rel = np.where(on > 0, np.abs(gn - on) / np.where(on > 0, on, 1.0), np.abs(gn))
    # scores: the oracle on the library's codes (read path alone) and on its own (whole path)
    got = g_scores.astype(np.float64)
    scale = np.linalg.norm(qh, axis=1)[:, None] * gn[None, :] / math.sqrt(d)
    exp_lib = oracle.scores(qh, g_idx[None], g_norms[None].astype(np.float32), G, b, s)
    exp_own = oracle.scores(qh, o_idx[None], o_norms[None], G, b, s)
    nz = scale > 0
    if not np.all(got[~nz] == 0.0):
        raise AssertionError("a zero query or key must score exactly 0")
    err_lib = np.abs(got - exp_lib)[nz] / scale[nz]
    keep = nz & ~rows_flip[None, :]
    scale_own = np.linalg.norm(qh, axis=1)[:, None] * on[None, :] / math.sqrt(d)
    err_own = np.abs(got - exp_own)[keep] / np.where(scale_own[keep] > 0, scale_own[keep], 1.0)
    return {
        "coords": int(flip.size),
        "in_window": int((marg < WINDOW).sum()),
        "flips": int(flip.sum()),
        "flips_outside_window": int((flip & (marg >= WINDOW)).sum()),
        "bytes_mismatch_rows_without_flip": int(((o_idx != g_idx).any(axis=1) & ~rows_flip).sum()),
        "max_norm_rel": float(rel.max()) if rel.size else 0.0,
        "score_err": float(err_lib.max()) if err_lib.size else 0.0,
        "e2e_score_err": float(err_own.max()) if err_own.size else 0.0,
        "e2e_rows": int((~rows_flip).sum()),
    }


def sample_tokens(T: int, per_head: int, seed: int, h: int) -> torch.Tensor:
    """First, last and per_head other seeded tokens of one KV head (drawn without
    replacement), sorted and distinct."""
    g = torch.Generator(device="cpu").manual_seed(seed * 100_003 + h)
    pick = torch.randperm(T - 2, generator=g)[:per_head] + 1
    return torch.unique(torch.cat([pick, torch.tensor([0, T - 1])]))


def run(wl: workloads.Workload, device, min_rows: int | None = None) -> FullReport:
    """Quantize and score the whole workload on the GPU, then compare every row
    (min_rows None) or at least min_rows seeded rows plus each head's first and
    last row with the oracle."""
    K = workloads.make_keys(wl, device)                       # (heads, T, d)
    q = workloads.make_queries(wl, device)
    s_dev = workloads.make_signs(wl).to(device)
    idx, norms = axr.axr_quantize_keys(K, wl.b, s_dev)
    scores = axr.axr_scores(q, idx, norms, wl.group, wl.b, s_dev)
    torch.cuda.synchronize(device)
    status = axr.axr_device_status()
    if status != 0:
        raise AssertionError(f"{wl.name}: a bounded wait ran out in a tensor-core kernel (status {status})")
    s = workloads.make_signs(wl).numpy()
    qh_all = q.double().cpu().numpy()
    heads, T, d, G = wl.heads, wl.T, wl.d, wl.group
    if min_rows is None:
        per_head = None
        selection = "every row"
    else:
        per_head = -(-min_rows // heads)
        selection = f"seeded sample of {per_head} tokens per KV head plus its first and last"
    rep = FullReport(wl.name, wl.b, d, G, wl.rows, 0, selection=selection, host_threads=host_threads())
    t0 = time.perf_counter()
    keys = ("coords", "in_window", "flips", "flips_outside_window", "bytes_mismatch_rows_without_flip", "e2e_rows")
    with ThreadPoolExecutor(rep.host_threads) as pool:
        pending = []

        def drain(limit):
            while len(pending) > limit:
                r = pending.pop(0).result()
                for k in keys:
                    setattr(rep, k, getattr(rep, k) + r[k])
                for k in ("max_norm_rel", "score_err", "e2e_score_err"):
                    setattr(rep, k, max(getattr(rep, k), r[k]))

        for h in range(heads):
            qh = qh_all[h * G:(h + 1) * G]
            if per_head is None:
                spans = [torch.arange(a, min(T, a + CHUNK_ROWS)) for a in range(0, T, CHUNK_ROWS)]
            else:
                tok = sample_tokens(T, per_head, wl.seed, h)
                spans = list(torch.split(tok, CHUNK_ROWS))
            for tok in spans:
                td = tok.to(device)
                Kc = K[h].index_select(0, td).double().cpu().numpy()
                ic = idx[h].index_select(0, td).cpu().numpy()
                nc = norms[h].index_select(0, td).cpu().numpy()
                sc = scores[h * G:(h + 1) * G].index_select(1, td).cpu().numpy()
                rep.rows_checked += len(tok)
                pending.append(pool.submit(_check_chunk, Kc, ic, nc, sc, qh, wl.b, s))
                drain(2 * rep.host_threads)
        drain(0)
    rep.host_seconds = time.perf_counter() - t0
    del K, idx, norms, scores
    return rep
