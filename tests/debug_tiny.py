"""Every entry point of the C ABI on tiny shapes, checked against the oracle.

Run as a script so that the library it loads can be chosen per process:

    AXR_DEBUG=1 python tests/debug_tiny.py            # libaxr_debug.so: bounds checks on
    python tests/debug_tiny.py                        # libaxr.so
    AXR_DEBUG=1 python tests/debug_tiny.py --slack 4  # every span 4 bytes short

Without --slack, every call must match the oracle (codes bit-exact outside the
boundary window, norms and scores within 1e-4, attention within the bound the
score tolerance implies, sign-choice errors within 1e-4 relative) and leave the
device status at 0: in the debug build no load or store fell outside the
buffers the call describes.

With --slack N (debug build only) every buffer span the checks allow is N bytes
shorter than the buffer: the last accesses of each buffer count as outside, so
every call must record status bit 16 and leave the last bytes of its outputs
as they were (their stores were skipped).  No access leaves its real buffer.

Prints one line per case and exits non-zero on the first failure.
"""
from __future__ import annotations

import argparse
import math
import os
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, HERE)
sys.path.insert(0, os.path.dirname(HERE))

import numpy as np  # noqa: E402
import torch  # noqa: E402

import oracle  # noqa: E402
from lut_attention_b200 import axr, workloads  # noqa: E402
from parity import check_quantize, check_scores  # noqa: E402

DEV = "cuda"
BOUNDS = 16
TINY_N = (1, 3, 31, 33)
ATTN_TOL = 2e-5


def _keys(d, n, heads, dtype, seed):
    wl = workloads.MHA_DECODE_32K.with_(d=d, dtype=dtype, T=n, batch=1, kv_heads=heads, seed=seed)
    return workloads.make_keys(wl, DEV), workloads.make_signs(wl).to(DEV)


def _queries(d, heads, group, seed, dtype=torch.float32):
    g = torch.Generator(device=DEV).manual_seed(seed)
    return torch.randn((heads * group, d), generator=g, device=DEV).to(dtype)


class Runner:
    def __init__(self, slack: int):
        self.slack = slack
        self.cases = 0

    def status(self, what: str) -> None:
        st = axr.axr_device_status()
        if self.slack:
            assert st & BOUNDS, f"{what}: the shortened spans recorded no bounds bit (status {st})"
        else:
            assert st == 0, f"{what}: device status {st}"
        self.cases += 1
        print(f"ok  {what}" + (f" (status {st})" if self.slack else ""), flush=True)

    # -- write and read -------------------------------------------------------
    def quantize_and_scores(self, d, b, n, group, dtype):
        heads = 2
        K, s = _keys(d, n, heads, dtype, seed=d * 7 + n + b)
        P = d * b // 8
        idx = torch.full((heads, n, P), 0x5A, dtype=torch.uint8, device=DEV)
        norms = torch.full((heads, n), -1.0, dtype=torch.float32, device=DEV)
        axr.axr_quantize_keys(K.reshape(-1, d), b, s, idx=idx.view(-1, P), norms=norms.view(-1))
        if self.slack:
            torch.cuda.synchronize()
            tail = idx.view(-1)[-min(self.slack, idx.numel()):]
            assert torch.all(tail == 0x5A), "quantize wrote into the withheld bytes of idx"
            assert norms.view(-1)[-1].item() == -1.0 or self.slack < 4, "quantize wrote the withheld norm"
        else:
            rep = check_quantize(K.reshape(-1, d), idx.view(-1, P), norms.view(-1), b, s)
            assert rep.ok(flip_fraction=None if n * heads * d < 10 ** 5 else 1e-5), rep
        self.status(f"quantize d={d} b={b} n={n} {dtype}")
        q = _queries(d, heads, group, seed=n + d)
        sc = torch.full((heads * group, n), -3.0, dtype=torch.float32, device=DEV)
        axr.axr_scores(q, idx, norms, group, b, s, scores=sc)
        if self.slack:
            torch.cuda.synchronize()
            assert sc.view(-1)[-1].item() == -3.0, "scores wrote the withheld score"
        else:
            err = check_scores(q, idx, norms, sc, group, b, s)
            assert err <= 1e-4, f"score error {err}"
        self.status(f"scores d={d} b={b} n={n} G={group}")

    def append(self, d, b, n, group, dtype):
        heads, pos = 2, n - 1
        capacity = (n + 2 + 15) // 16 * 16      # every head's slice of the cache 16-byte aligned
        K, s = _keys(d, n, heads, dtype, seed=d * 11 + n)
        P = d * b // 8
        idx = torch.full((heads, capacity, P), 0xA5, dtype=torch.uint8, device=DEV)
        norms = torch.full((heads, capacity), -7.0, dtype=torch.float32, device=DEV)
        if pos > 0:
            for h in range(heads):
                axr.axr_quantize_keys(K[h, :pos].contiguous(), b, s, idx=idx[h, :pos], norms=norms[h, :pos])
        torch.cuda.synchronize()
        axr.axr_device_status()
        before_i, before_n = idx.clone(), norms.clone()
        q = _queries(d, heads, group, seed=3 * n + d)
        out = axr.axr_append_scores(K[:, pos].contiguous(), q, idx, norms, pos, group, b, s)
        torch.cuda.synchronize()
        keep = torch.ones(capacity, dtype=torch.bool, device=DEV)
        keep[pos] = False
        assert torch.equal(idx[:, keep], before_i[:, keep]), "append touched another slot"
        assert torch.equal(norms[:, keep], before_n[:, keep]), "append touched another norm"
        if not self.slack:
            rep = check_quantize(K[:, pos], idx[:, pos], norms[:, pos], b, s)
            assert rep.ok(flip_fraction=None), rep
            err = check_scores(q, idx[:, :pos + 1].contiguous(), norms[:, :pos + 1].contiguous(), out, group, b, s)
            assert err <= 1e-4, f"decode step score error {err}"
        self.status(f"append d={d} b={b} pos={pos} G={group}")

    # -- attention ------------------------------------------------------------
    def attention(self, d, b, n, group, vdtype, static):
        heads = 2
        packed, norms = workloads.make_random_packed(heads, n, d, b, seed=d + n, device=DEV)
        wl = workloads.GQA_DECODE_128K.with_(d=d, batch=1, kv_heads=heads, group=group, T=n, seed=n)
        q = workloads.make_queries(wl, DEV)
        s = workloads.make_signs(wl).to(DEV)
        g = torch.Generator(device=DEV).manual_seed(d * n)
        V = torch.randn((heads, n, d), generator=g, device=DEV).to(getattr(torch, vdtype))
        sc = torch.full((heads * group, n), -5.0, dtype=torch.float32, device=DEV)
        out = torch.full((heads * group, d), -9.0, dtype=torch.float32, device=DEV)
        if static:
            axr.axr_attention_static(q, packed, norms, V, group, b, s, sc, out)
        else:
            axr.axr_attention(q, packed, norms, V, group, b, s, scores=sc, out=out)
        torch.cuda.synchronize()
        name = "attention_static" if static else "attention"
        if self.slack:
            assert out.view(-1)[-1].item() == -9.0, f"{name} wrote the withheld output"
        else:
            Vh = V.cpu().double().numpy()
            vmax = np.abs(Vh).reshape(heads, -1).max(axis=1).repeat(group)[:, None]
            got = out.cpu().double().numpy()
            own = oracle.attention_from_scores(sc.cpu().double().numpy(), Vh, group)
            assert np.all(np.abs(got - own) <= ATTN_TOL * vmax), float((np.abs(got - own) / vmax).max())
            assert check_scores(q, packed, norms, sc, group, b, s) <= 1e-4
            exp = oracle.attention(q.cpu().double().numpy(), packed.cpu().numpy(), norms.cpu().numpy(), Vh,
                                   group, b, s.cpu().numpy())
            qn = np.linalg.norm(q.cpu().double().numpy(), axis=1)
            kmax = norms.cpu().double().numpy().max(axis=1).repeat(group)
            bound = (np.expm1(2e-4 * qn * kmax / math.sqrt(d))[:, None] + ATTN_TOL) * vmax
            assert np.all(np.abs(got - exp) <= bound), float((np.abs(got - exp) / bound).max())
        self.status(f"{name} d={d} b={b} n={n} G={group} {vdtype}")

    # -- sign choice ----------------------------------------------------------
    def select_signs(self, d, b, n, group):
        S, H, C = 1, 2, 3
        wl = workloads.GQA_SIGN_CALIBRATION.with_(batch=S, kv_heads=H, group=group, d=d, b=b, T=n, dtype="f32",
                                                  seed=d + n)
        K = workloads.make_keys(wl).reshape(S, H, n, d)
        q = workloads.make_queries(wl).float().reshape(S, H * group, d)
        cand = workloads.make_sign_candidates(wl, C)
        errors = torch.full((C, H), -2.0, dtype=torch.float32, device=DEV)
        best = torch.full((1,), -77, dtype=torch.int32, device=DEV)
        axr.axr_select_signs(K.to(DEV), q.to(DEV), group, b, cand.to(DEV), errors=errors, best=best)
        torch.cuda.synchronize()
        if self.slack:
            assert errors.view(-1)[-1].item() == -2.0, "select_signs wrote the withheld error"
            if self.slack >= 4:
                assert best.item() == -77, "select_signs wrote the withheld choice"
        else:
            exp = oracle.sign_errors(K.double().numpy(), q.double().numpy(), group, b, cand.numpy())
            np.testing.assert_allclose(errors.cpu().double().numpy(), exp, rtol=1e-4, atol=0)
            worst = exp.max(axis=1)
            assert worst[int(best.item())] <= worst.min() * (1 + 1e-4)
        self.status(f"select_signs d={d} b={b} n={n} G={group}")

    # -- block rotation -------------------------------------------------------
    def block(self, d, b, n, group, dtype):
        wl = workloads.MHA_DECODE_32K.with_(d=d, dtype=dtype, T=n, batch=1, kv_heads=1, seed=d + 5 * n)
        K = workloads.make_keys(wl, DEV).reshape(n, d)
        quats = workloads.make_block_quats(wl).to(DEV)
        P = d * b // 8
        idx = torch.full((n, P), 0x3C, dtype=torch.uint8, device=DEV)
        norms = torch.full((n,), -4.0, dtype=torch.float32, device=DEV)
        axr.axr_quantize_keys_block(K, b, quats, idx=idx, norms=norms)
        torch.cuda.synchronize()
        if self.slack:
            assert norms[-1].item() == -4.0, "block quantize wrote the withheld norm"
        else:
            rep = check_quantize(K, idx, norms, b, None, quats=quats)
            assert rep.ok(flip_fraction=None), rep
        self.status(f"quantize_block d={d} b={b} n={n} {dtype}")
        q = _queries(d, 1, group, seed=d + n + 1)
        sc = torch.full((group, n), -6.0, dtype=torch.float32, device=DEV)
        axr.axr_scores_block(q, idx[None], norms[None], group, b, quats, scores=sc)
        torch.cuda.synchronize()
        if self.slack:
            assert sc.view(-1)[-1].item() == -6.0, "block scores wrote the withheld score"
        else:
            assert check_scores(q, idx[None], norms[None], sc, group, b, None, quats=quats) <= 1e-4
        self.status(f"scores_block d={d} b={b} n={n} G={group}")


def run(slack: int) -> int:
    torch.manual_seed(0)
    oracle.build()
    debug = axr.axr_debug_build()
    print(f"library: {os.path.basename(axr.LIB_PATH)} (debug build: {debug}), span slack {slack}", flush=True)
    if slack:
        assert debug, "--slack needs the debug build (AXR_DEBUG=1)"
    if debug:
        axr.axr_debug_set_span_slack(slack)
    r = Runner(slack)
    for n in TINY_N:
        # CUDA-core kernels (d = 8; attention needs d >= 32)
        r.quantize_and_scores(8, 3, n, 3, "f32")
        r.append(8, 2, n, 2, "f32")
        r.select_signs(8, 2, n, 2)
        r.block(8, 4, n, 2, "f32")
        r.attention(32, 2, n, 3, "float32", static=False)
        r.attention(32, 2, n, 3, "float16", static=True)
    for n in (1, 3, 33, 129):
        # tensor-core kernels: 128-, 256- and 512-wide heads
        for d, b, group in ((128, 4, 4), (128, 3, 8), (256, 2, 2), (512, 4, 5)):
            r.quantize_and_scores(d, b, n, group, "bf16")
            r.append(d, b, n, group, "bf16")
        r.block(128, 2, n, 4, "bf16")
        r.attention(128, 4, n, 4, "bfloat16", static=True)
    if debug:
        axr.axr_debug_set_span_slack(0)
    print(f"all {r.cases} cases passed", flush=True)
    return 0


def main() -> int:
    ap = argparse.ArgumentParser(description=__doc__, formatter_class=argparse.RawDescriptionHelpFormatter)
    ap.add_argument("--slack", type=int, default=0)
    args = ap.parse_args()
    if not torch.cuda.is_available():
        print("no CUDA device", file=sys.stderr)
        return 2
    return run(args.slack)


if __name__ == "__main__":
    sys.exit(main())
