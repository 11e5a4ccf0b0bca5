"""Comparison of the CUDA path (through the C ABI) with the CPU oracle.

Tolerances (stated with the method: bit-exact indices except within 1e-6 of a
decision boundary; norms and scores within 1e-4 of the natural scale):
  * indices: equal everywhere except coordinates whose rotated unit value lies
    within WINDOW = 1e-6 of a decision point (measured by the oracle in fp64);
    such flips are reported and must stay below 1e-5 of all coordinates;
  * norms: |norm_gpu - norm_oracle| <= 1e-4 * norm_oracle;
  * scores: |s_gpu - s_oracle| <= 1e-4 * ||q|| * ||k|| / sqrt(d).
"""
from __future__ import annotations

import math
from dataclasses import dataclass

import numpy as np
import torch

import oracle
from lut_attention_b200 import axr

WINDOW = 1e-6
FLIP_FRACTION = 1e-5
NORM_RTOL = 1e-4
SCORE_TOL = 1e-4


@dataclass
class QuantizeReport:
    coords: int
    flips: int
    flips_outside_window: int
    in_window: int
    max_norm_rel: float
    bytes_mismatch_rows_without_flip: int

    def ok(self, flip_fraction: float | None = FLIP_FRACTION) -> bool:
        """flip_fraction=None drops the cap on in-window flips (for degenerate
        inputs built to sit exactly on a boundary)."""
        return (self.flips_outside_window == 0
                and (flip_fraction is None or self.flips <= flip_fraction * self.coords)
                and self.max_norm_rel <= NORM_RTOL
                and self.bytes_mismatch_rows_without_flip == 0)


def to_f64(t: torch.Tensor) -> np.ndarray:
    return t.detach().to("cpu").to(torch.float64).numpy()


def check_quantize(K_rows: torch.Tensor, idx_rows: torch.Tensor, norms_rows: torch.Tensor,
                   b: int, signs: torch.Tensor | None, quats: torch.Tensor | None = None) -> QuantizeReport:
    """K_rows (m, d) inputs on any device, idx_rows / norms_rows the GPU outputs for
    those rows; compares with the oracle run on the same inputs (the block rotation
    of `quats` instead of the sign flip and Walsh-Hadamard transform if given)."""
    d = K_rows.shape[-1]
    Kh = to_f64(K_rows.reshape(-1, d))
    if quats is not None:
        o_idx, o_norms, marg = oracle.quantize_block(Kh, b, to_f64(quats), margins=True)
    else:
        o_idx, o_norms, marg = oracle.quantize(Kh, b, signs.cpu().numpy(), margins=True)
    g_idx = idx_rows.reshape(len(Kh), -1).cpu().numpy()
    g_norms = norms_rows.reshape(-1).cpu().numpy().astype(np.float64)
    oc = oracle.unpack(o_idx, d, b)
    gc = oracle.unpack(g_idx, d, b)
    flip = oc != gc
    rows_with_flip = flip.any(axis=1)
    bytes_bad = (o_idx != g_idx).any(axis=1) & ~rows_with_flip
    on = o_norms.astype(np.float64)
    rel = np.abs(g_norms - on) / np.where(on > 0, on, 1.0)
    rel = np.where(on > 0, rel, np.abs(g_norms))
    return QuantizeReport(
        coords=int(flip.size),
        flips=int(flip.sum()),
        flips_outside_window=int((flip & (marg >= WINDOW)).sum()),
        in_window=int((marg < WINDOW).sum()),
        max_norm_rel=float(rel.max()) if rel.size else 0.0,
        bytes_mismatch_rows_without_flip=int(bytes_bad.sum()),
    )


def check_scores(q: torch.Tensor, idx: torch.Tensor, norms: torch.Tensor, scores: torch.Tensor,
                 group: int, b: int, signs: torch.Tensor | None, quats: torch.Tensor | None = None) -> float:
    """Worst |s_gpu - s_oracle| / (||q|| ||k|| / sqrt(d)) over the given keys.
    idx (heads, m, P) / norms (heads, m) / scores (heads*group, m) on any device;
    queries rotated by the block rotation of `quats` if given."""
    d = q.shape[-1]
    qh = to_f64(q)
    if quats is not None:
        exp = oracle.scores_block(qh, idx.cpu().numpy(), norms.cpu().numpy(), group, b, to_f64(quats))
    else:
        exp = oracle.scores(qh, idx.cpu().numpy(), norms.cpu().numpy(), group, b, signs.cpu().numpy())
    got = scores.cpu().numpy().astype(np.float64)
    qn = np.linalg.norm(qh, axis=1)[:, None]
    kn = np.repeat(norms.cpu().numpy().astype(np.float64), group, axis=0)
    scale = qn * kn / math.sqrt(d)
    err = np.abs(got - exp)
    zero = scale == 0
    if zero.any():
        assert np.all(got[zero] == 0.0), "a zero query or key must score exactly 0"
    nz = ~zero
    return float((err[nz] / scale[nz]).max()) if nz.any() else 0.0


def gpu_quantize(K: torch.Tensor, b: int, signs: torch.Tensor):
    idx, norms = axr.axr_quantize_keys(K, b, signs)
    assert axr.axr_device_status() == 0, "a bounded wait ran out in a tensor-core kernel"
    return idx, norms


def gpu_scores(q, idx, norms, group, b, signs):
    out = axr.axr_scores(q, idx, norms, group, b, signs)
    assert axr.axr_device_status() == 0, "a bounded wait ran out in a tensor-core kernel"
    return out
