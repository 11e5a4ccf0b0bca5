"""Seeded synthetic inputs shaped like the AXELRAM decode workloads.

This module only draws random inputs.  It holds none of the method's arithmetic
(no rotation, codebook, quantization or scoring) so that the CUDA path and the
CPU oracle can both be fed from it without sharing any of the computation.

The pages evaluate on real models (Qwen2.5-3B, LLaMA-3.1-8B and others) that are
not available here; these recipes stand in for their key caches.  Every draw
comes from a ``torch.Generator`` seeded per workload, in a fixed order, so the
same (workload, device) always gives the same tensors.

Recipes (``LogNormal(m, s)`` means ``exp(m + s * N(0,1))``):

* ``row_lognormal``   K ~ N(0,1), each row times LogNormal(0, 0.5).
* ``channel_scaled``  K ~ N(0,1) times a per-(KV head, channel) LogNormal(0,1)
                      scale, fixed across batch and tokens; 4 distinct channels per
                      KV head (seeded choice) are further scaled by 20.  With
                      ``head_sigma`` > 0 every (batch, KV head) is also scaled by
                      LogNormal(0, head_sigma) (per-head norm heterogeneity).
* ``calibration``     calibration samples of one layer for choosing the sign
                      pattern (the batch holds the samples): ``channel_scaled``
                      keys whose KV-head scale LogNormal(0, head_sigma) belongs to
                      the head and is shared by every sample, plus a fixed offset
                      per KV head, ``key_bias`` times the head's channel scales
                      times a seeded N(0,1)^d vector, the same for all tokens and
                      samples.  Without a shared offset the distribution of the
                      keys is symmetric in every coordinate, and then every sign
                      pattern sees statistically the same keys.
* ``unit_uniform``    rows of N(0,1)^d, normalised, times a norm ~ U(lo, hi).
* ``student_t``       coordinates ~ Student-t(4) (a normal over the root of a
                      chi-square with 4 degrees of freedom / 4), rows renormalised
                      to a norm ~ U(lo, hi).

Queries are N(0,1) in the workload's dtype.  The sign pattern D is a seeded
+-1 int8 vector drawn on the CPU, one per workload (one per layer); the
candidates of a sign-pattern search are seeded +-1 rows, the first of them
that default pattern.  A block rotation takes seeded unit quaternions, two per
4-element block (one for the fast variant).
"""
from __future__ import annotations

import dataclasses
from dataclasses import dataclass

import torch

_DTYPES = {"f32": torch.float32, "f16": torch.float16, "bf16": torch.bfloat16}


@dataclass(frozen=True)
class Workload:
    name: str
    batch: int          # B
    kv_heads: int       # H (KV heads per batch element)
    group: int          # G (query heads per KV head)
    d: int              # head dimension
    b: int              # bits per coordinate
    T: int              # keys per (batch, KV head): the context length
    dtype: str          # "f32" | "f16" | "bf16" for keys and queries
    seed: int
    recipe: str
    head_sigma: float = 0.0
    norm_lo: float = 0.0
    norm_hi: float = 0.0
    key_bias: float = 0.0

    @property
    def heads(self) -> int:
        """KV heads with the batch folded in: B * H."""
        return self.batch * self.kv_heads

    @property
    def rows(self) -> int:
        """Quantized key rows: B * H * T."""
        return self.heads * self.T

    @property
    def torch_dtype(self) -> torch.dtype:
        return _DTYPES[self.dtype]

    def with_(self, **kw) -> "Workload":
        return dataclasses.replace(self, **kw)

    def describe(self) -> str:
        return (f"{self.name}: B={self.batch} Hkv={self.kv_heads} G={self.group} d={self.d} "
                f"b={self.b} T={self.T} {self.dtype}")


# The five decode workloads of the benchmark description.
PR1_REF = Workload("pr1_ref", 1, 1, 1, 128, 4, 4096, "f32", 1, "row_lognormal")
MHA_DECODE_32K = Workload("mha_decode_32k", 8, 32, 1, 128, 3, 32768, "bf16", 2, "channel_scaled")
GQA_DECODE_128K = Workload("gqa_decode_128k", 4, 8, 4, 128, 4, 131072, "bf16", 3, "channel_scaled",
                           head_sigma=1.5)
WRITE_2E24 = Workload("write_2e24", 1, 1, 1, 128, 4, 1 << 24, "bf16", 4, "unit_uniform",
                      norm_lo=0.1, norm_hi=50.0)
WIDE_D256 = Workload("wide_heads_d256", 16, 8, 2, 256, 2, 65536, "f16", 5, "student_t",
                     norm_lo=1.0, norm_hi=10.0)
WIDE_D512 = WIDE_D256.with_(name="wide_heads_d512", d=512)
# Sign-pattern search of one layer of the GQA shape: 8 calibration samples (the
# batch) of 2048 tokens, 200 candidates.
GQA_SIGN_CALIBRATION = Workload("gqa_sign_calibration", 8, 8, 4, 128, 4, 2048, "bf16", 6, "calibration",
                                head_sigma=1.5, key_bias=1.0)
SIGN_CANDIDATES = 200

ALL = (PR1_REF, MHA_DECODE_32K, GQA_DECODE_128K, WRITE_2E24, WIDE_D256, WIDE_D512)
BY_NAME = {w.name: w for w in ALL}


def make_signs(wl: Workload) -> torch.Tensor:
    """Seeded sign pattern D in {+1, -1}^d, int8, on the CPU."""
    g = torch.Generator(device="cpu").manual_seed(1_000_003 * wl.seed + wl.d)
    return (torch.randint(0, 2, (wl.d,), generator=g, dtype=torch.int8) * 2 - 1).to(torch.int8)


def make_sign_candidates(wl: Workload, count: int) -> torch.Tensor:
    """Seeded candidate sign patterns (count, d), int8 +-1, on the CPU; row 0 is
    the workload's own pattern (:func:`make_signs`)."""
    g = torch.Generator(device="cpu").manual_seed(2_000_029 * wl.seed + wl.d + count)
    c = (torch.randint(0, 2, (count, wl.d), generator=g, dtype=torch.int8) * 2 - 1).to(torch.int8)
    if count:
        c[0] = make_signs(wl)
    return c


def make_block_quats(wl: Workload, fast: bool = False) -> torch.Tensor:
    """Seeded unit quaternions for a block rotation, (d/4, 8) fp32 on the CPU:
    per 4-element block qL then qR, each (w, x, y, z) uniform on the unit sphere
    (a normalised N(0, I_4) draw).  fast: qR = (1, 0, 0, 0) on every block."""
    g = torch.Generator(device="cpu").manual_seed(3_000_017 * wl.seed + wl.d)
    z = torch.randn((wl.d // 4, 2, 4), generator=g, dtype=torch.float64)
    z = z / z.norm(dim=2, keepdim=True)
    if fast:
        z[:, 1] = torch.tensor([1.0, 0.0, 0.0, 0.0], dtype=torch.float64)
    return z.reshape(wl.d // 4, 8).to(torch.float32)


def make_queries(wl: Workload, device="cpu") -> torch.Tensor:
    """Queries (B*H*G, d) ~ N(0,1) in the workload dtype."""
    g = torch.Generator(device=device).manual_seed(7_919 * wl.seed + 17)
    q = torch.randn((wl.heads * wl.group, wl.d), generator=g, device=device, dtype=torch.float32)
    return q.to(wl.torch_dtype)


def _lognormal(shape, sigma, g, device):
    return torch.exp(sigma * torch.randn(shape, generator=g, device=device, dtype=torch.float32))


def make_keys(wl: Workload, device="cpu", chunk_rows: int = 1 << 20) -> torch.Tensor:
    """Keys (B*H, T, d) in the workload dtype, drawn by the workload's recipe.

    Rows are drawn in chunks of ``chunk_rows`` (a fixed split, so the result does
    not depend on memory) to bound the fp32 temporaries of the large workloads.
    """
    g = torch.Generator(device=device).manual_seed(104_729 * wl.seed + 1)
    d, heads, T = wl.d, wl.heads, wl.T
    out = torch.empty((heads, T, d), dtype=wl.torch_dtype, device=device)
    flat = out.view(heads * T, d)

    if wl.recipe == "channel_scaled":
        chan = _lognormal((wl.kv_heads, d), 1.0, g, device)
        for h in range(wl.kv_heads):
            pick = torch.randperm(d, generator=g, device=device)[:4]
            chan[h, pick] *= 20.0
        head = (_lognormal((heads,), wl.head_sigma, g, device) if wl.head_sigma > 0
                else torch.ones(heads, device=device))
        scale = chan.repeat(wl.batch, 1) * head[:, None]            # (B*H, d)
        for h in range(heads):
            for t0 in range(0, T, chunk_rows):
                t1 = min(T, t0 + chunk_rows)
                z = torch.randn((t1 - t0, d), generator=g, device=device, dtype=torch.float32)
                out[h, t0:t1] = (z * scale[h]).to(wl.torch_dtype)
        return out

    if wl.recipe == "calibration":
        chan = _lognormal((wl.kv_heads, d), 1.0, g, device)
        for h in range(wl.kv_heads):
            pick = torch.randperm(d, generator=g, device=device)[:4]
            chan[h, pick] *= 20.0
        head = (_lognormal((wl.kv_heads,), wl.head_sigma, g, device) if wl.head_sigma > 0
                else torch.ones(wl.kv_heads, device=device))
        bias = wl.key_bias * torch.randn((wl.kv_heads, d), generator=g, device=device, dtype=torch.float32)
        for s in range(wl.batch):
            for h in range(wl.kv_heads):
                for t0 in range(0, T, chunk_rows):
                    t1 = min(T, t0 + chunk_rows)
                    z = torch.randn((t1 - t0, d), generator=g, device=device, dtype=torch.float32)
                    out[s * wl.kv_heads + h, t0:t1] = ((z + bias[h]) * chan[h] * head[h]).to(wl.torch_dtype)
        return out

    rows = heads * T
    for r0 in range(0, rows, chunk_rows):
        r1 = min(rows, r0 + chunk_rows)
        m = r1 - r0
        if wl.recipe == "row_lognormal":
            z = torch.randn((m, d), generator=g, device=device, dtype=torch.float32)
            x = z * _lognormal((m, 1), 0.5, g, device)
        elif wl.recipe == "unit_uniform":
            z = torch.randn((m, d), generator=g, device=device, dtype=torch.float32)
            r = wl.norm_lo + (wl.norm_hi - wl.norm_lo) * torch.rand(
                (m, 1), generator=g, device=device, dtype=torch.float32)
            x = z / z.norm(dim=1, keepdim=True) * r
        elif wl.recipe == "student_t":
            z = torch.randn((m, d), generator=g, device=device, dtype=torch.float32)
            chi2 = torch.zeros((m, d), device=device, dtype=torch.float32)
            for _ in range(4):
                w = torch.randn((m, d), generator=g, device=device, dtype=torch.float32)
                chi2 += w * w
            x = z / torch.sqrt(chi2 / 4.0)
            r = wl.norm_lo + (wl.norm_hi - wl.norm_lo) * torch.rand(
                (m, 1), generator=g, device=device, dtype=torch.float32)
            x = x / x.norm(dim=1, keepdim=True) * r
        else:
            raise ValueError(f"unknown recipe {wl.recipe!r}")
        flat[r0:r1] = x.to(wl.torch_dtype)
    return out


def make_random_packed(heads: int, n: int, d: int, b: int, seed: int, device="cpu"):
    """Seeded random packed index rows (heads, n, d*b/8) uint8 and norms (heads, n) fp32.

    Every b-bit pattern is a valid index, so uniform random bytes are valid packed
    rows for any b; this drives the read path independently of the write path.
    """
    g = torch.Generator(device=device).manual_seed(15_485_863 * seed + 5)
    P = d * b // 8
    packed = torch.randint(0, 256, (heads, n, P), generator=g, device=device, dtype=torch.int32)
    norms = _lognormal((heads, n), 1.0, g, device)
    return packed.to(torch.uint8), norms
