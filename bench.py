"""Benchmark of the AXELRAM hot path on B200: quantize-on-write + LUT score-on-read.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl axr|reference]
                    [--workload gqa_decode_128k] [--b 4]

One step is one pass of the whole path over one batch of the workload: every key
of the batch is quantized (sign flip, Walsh-Hadamard, norm, Lloyd-Max indices,
packing) and every query head is scored against every key of its KV head by
table lookup on the packed indices.  The read kernel scores the cache written one
step earlier (two cache buffers, same keys), so neither kernel finds the other's
output in L2; every input is larger than the 126 MB L2.

Multi-GPU: one process per GPU (torchrun).  The batch is sharded: every rank runs
its own batch of the workload (weak scaling), with no collective on the data
path; the only collectives are the barrier and the max-over-ranks of the time.

Prints ONE JSON line on rank 0.  ``value`` is LUT attention scores per second for
the whole job; keys quantized per second and each kernel's HBM throughput are
reported beside it.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import math
import os
import statistics
import sys
import threading
import time

import torch
import torch.distributed as dist

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

from lut_attention_b200 import axr, workloads  # noqa: E402

NOMINAL_HBM_GBS = 8000.0          # B200 HBM3e nominal figure the targets are quoted against
FALLBACK_HBM_GBS = 6650.0         # earlier measurement on this machine, used only without a measured file
L2_BYTES = 126 * 2 ** 20


def log(*a):
    print(*a, file=sys.stderr, flush=True)


# ------------------------------------------------------------------ helpers --

def dist_env():
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return world, rank, local


def shard_workload(wl: workloads.Workload, rank: int, world: int) -> workloads.Workload:
    """Weak scaling: rank r runs batch elements [r*B, (r+1)*B) of a global batch
    of world*B, i.e. the workload with its own seed.  Rank 0 keeps the base seed."""
    return wl.with_(seed=wl.seed + 7919 * rank)


def algorithmic_bytes(wl: workloads.Workload, elem_bytes: int) -> dict:
    """Bytes each kernel must move per launch (one step of the workload).

    write: key row in (d * elem) + packed row out (d*b/8) + norm out (4) per key;
    read:  packed row (d*b/8) + norm (4) in + G scores out (4G) per key row,
           plus the queries (B*H*G*d*elem) and the sign vector (d) once per call.
    """
    P = wl.d * wl.b // 8
    rows = wl.rows
    write = rows * (wl.d * elem_bytes + P + 4)
    read = rows * (P + 4 + 4 * wl.group) + wl.heads * wl.group * wl.d * elem_bytes + wl.d
    return {"write": write, "read": read, "write_per_key": wl.d * elem_bytes + P + 4,
            "read_per_row": P + 4 + 4 * wl.group}


def measured_peak():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            return float(json.load(f)["hbm_gbs"]), "measured"
    except Exception:
        return FALLBACK_HBM_GBS, "fallback"


def kernel_source_hash(name: str) -> str:
    with open(os.path.join(ROOT, "lut_attention_b200", "csrc", name), "rb") as f:
        return hashlib.sha256(f.read()).hexdigest()[:16]


def max_over_ranks(values, world: int, device) -> list:
    """Element-wise maximum of per-rank timings (ms) over all ranks: the job is as
    slow as its slowest rank.  Every rank must call it, in the same order."""
    t = torch.tensor(values, dtype=torch.float64, device=device)
    if world > 1:
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return t.tolist()


def job_scores_per_s(wl: workloads.Workload, world: int, ms_per_step: float) -> float:
    """Whole-job throughput: every rank scores its own batch each step."""
    return wl.heads * wl.group * wl.T * world / (ms_per_step * 1e-3)


def kernel_file(kind: str, wl: workloads.Workload) -> str:
    """Source file of the kernel the library runs for this workload (api.cu takes the
    tensor-core kernels at d = 128, 256 and 512, for the write path with bf16/f16 keys;
    the read path at d = 128 has a kernel of its own; AXR_READ_KERNEL=cuda_core sends
    every read to the CUDA-core kernel)."""
    tc_width = wl.d in (128, 256, 512)
    if kind == "quantize_keys":
        return "quantize_keys_tc.cu" if tc_width and wl.dtype in ("bf16", "f16") else "quantize_keys.cu"
    if os.environ.get("AXR_READ_KERNEL") == "cuda_core":
        return "scores.cu"
    if wl.d == 128:
        return "scores_tc128.cu"
    return "scores_tc.cu" if tc_width else "scores.cu"


def profiled_traffic(kernel_file: str, workload: str, b: int):
    """DRAM bytes per launch from the committed ncu summary, when that summary was
    taken on the current kernel source (its hash line matches); else None."""
    path = os.path.join(ROOT, "profiles", "traffic.txt")
    if not os.path.exists(path):
        return None
    want = kernel_source_hash(kernel_file)
    with open(path) as f:
        for line in f:
            parts = line.split("#")[0].split()
            if len(parts) == 5 and parts[0] == kernel_file and parts[1] == workload \
                    and parts[2] == f"b={b}" and parts[3] == want:
                return int(float(parts[4]))
    return None


class ClockSampler:
    """Samples SM clock and clock-event reasons through NVML while running."""

    REASONS = {
        "sw_power_cap": 0x4, "hw_slowdown": 0x8, "sw_thermal_slowdown": 0x20,
        "hw_thermal_slowdown": 0x40, "hw_power_brake_slowdown": 0x80,
    }

    def __init__(self, device_index: int, period_s: float = 0.005):
        self.period = period_s
        self.samples = []
        self.max_mhz = None
        self._stop = threading.Event()
        self._busy = threading.Event()
        self._thread = None
        try:
            import pynvml
            pynvml.nvmlInit()
            uuid = None
            try:
                uuid = torch.cuda.get_device_properties(device_index).uuid
            except Exception:
                pass
            handle = None
            if uuid is not None:
                s = str(uuid)
                s = s if s.startswith("GPU-") else "GPU-" + s
                try:
                    handle = pynvml.nvmlDeviceGetHandleByUUID(s.encode())
                except Exception:
                    handle = None
            if handle is None:
                vis = os.environ.get("CUDA_VISIBLE_DEVICES", "")
                idx = int(vis.split(",")[device_index]) if vis and vis.split(",")[0].isdigit() else device_index
                handle = pynvml.nvmlDeviceGetHandleByIndex(idx)
            self._nvml, self._h = pynvml, handle
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(handle, pynvml.NVML_CLOCK_SM)
        except Exception as e:  # no NVML: report no clocks rather than guess
            log(f"clock sampling unavailable: {e}")
            self._nvml = None

    def _run(self):
        nv = self._nvml
        while not self._stop.is_set():
            if self._busy.is_set():
                try:
                    mhz = nv.nvmlDeviceGetClockInfo(self._h, nv.NVML_CLOCK_SM)
                    get = getattr(nv, "nvmlDeviceGetCurrentClocksEventReasons", None) or \
                        nv.nvmlDeviceGetCurrentClocksThrottleReasons
                    reasons = get(self._h)
                    self.samples.append((mhz, reasons))
                except Exception:
                    pass
            time.sleep(self.period)

    def start(self):
        if self._nvml is not None:
            self._thread = threading.Thread(target=self._run, daemon=True)
            self._thread.start()

    def busy(self, on: bool):
        (self._busy.set if on else self._busy.clear)()

    def stop(self):
        self._stop.set()
        if self._thread:
            self._thread.join()

    def mark(self) -> int:
        """Index of the next sample, to summarise a later window on its own."""
        return len(self.samples)

    def summary(self, start: int = 0, stop: int | None = None):
        window = self.samples[start:stop]
        if not window:
            return {"sm_mhz": None, "sm_max_mhz": self.max_mhz, "reasons": [], "samples": 0}
        mhz = statistics.median(s[0] for s in window)
        active = set()
        for _, r in window:
            for name, bit in self.REASONS.items():
                if r & bit:
                    active.add(name)
        return {"sm_mhz": mhz, "sm_max_mhz": self.max_mhz, "reasons": sorted(active),
                "samples": len(window)}


# ----------------------------------------------------------------- the step --

def timed_steps(path, stream, steps: int, barrier):
    """K steps between CUDA events on the launching stream, with a barrier and a
    synchronize on both sides: (elapsed ms, mean write ms, mean read ms).  Each
    kernel is also bracketed by its own events."""
    ev = [[torch.cuda.Event(enable_timing=True) for _ in range(3)] for _ in range(steps)]
    start = torch.cuda.Event(enable_timing=True)
    end = torch.cuda.Event(enable_timing=True)
    barrier()
    start.record(stream)
    for i in range(steps):
        ev[i][0].record(stream)
        path.quantize(i % 2)
        ev[i][1].record(stream)
        path.score((i + 1) % 2)
        ev[i][2].record(stream)
    end.record(stream)
    barrier()
    elapsed_ms = start.elapsed_time(end)
    t_write = sum(e[0].elapsed_time(e[1]) for e in ev) / steps
    t_read = sum(e[1].elapsed_time(e[2]) for e in ev) / steps
    return elapsed_ms, t_write, t_read


class Path:
    """Device buffers and the two kernels of one step."""

    def __init__(self, wl: workloads.Workload, device):
        self.wl = wl
        self.K = workloads.make_keys(wl, device)                 # (heads, T, d)
        self.q = workloads.make_queries(wl, device)
        self.signs = workloads.make_signs(wl).to(device)
        P = wl.d * wl.b // 8
        self.idx = [torch.empty((wl.heads, wl.T, P), dtype=torch.uint8, device=device) for _ in range(2)]
        self.norms = [torch.empty((wl.heads, wl.T), dtype=torch.float32, device=device) for _ in range(2)]
        self.scores = torch.empty((wl.heads * wl.group, wl.T), dtype=torch.float32, device=device)
        for i in range(2):
            self.quantize(i)

    def quantize(self, i):
        axr.axr_quantize_keys(self.K, self.wl.b, self.signs, idx=self.idx[i], norms=self.norms[i])

    def score(self, i):
        axr.axr_scores(self.q, self.idx[i], self.norms[i], self.wl.group, self.wl.b, self.signs,
                       scores=self.scores)


def run_decode_step(path: Path, steps: int) -> dict:
    """The decode step the cache serves: append one key per KV head at the last
    slot (pos = T - 1) and score every query head against all T keys
    (axr_append_scores), timed against scoring the same T keys alone."""
    wl = path.wl
    k_new = path.K[:, -1].contiguous()
    pos = wl.T - 1

    def append():
        axr.axr_append_scores(k_new, path.q, path.idx[0], path.norms[0], pos, wl.group, wl.b, path.signs,
                              scores=path.scores)

    def time_ms(fn):
        for _ in range(3):
            fn()
        torch.cuda.synchronize()
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record()
        for _ in range(steps):
            fn()
        b.record()
        torch.cuda.synchronize()
        return a.elapsed_time(b) / steps

    t_step = time_ms(append)
    t_scores = time_ms(lambda: path.score(0))
    return {"ms": t_step, "scores_only_ms": t_scores, "context": wl.T,
            "queries": wl.heads * wl.group, "keys_appended": wl.heads}


def run_attention(path: Path, steps: int) -> dict:
    """Decode attention on the cache (axr_attention: scores, then the softmax of
    every query head's scores and the weighted sum of bf16 value rows)."""
    wl = path.wl
    g = torch.Generator(device=path.K.device).manual_seed(4242)
    V = torch.randn((wl.heads, wl.T, wl.d), generator=g, device=path.K.device).to(torch.bfloat16)
    ws = torch.empty(axr.axr_attention_workspace_bytes(wl.T, wl.heads, wl.group, wl.d), dtype=torch.uint8,
                     device=path.K.device)
    out = torch.empty((wl.heads * wl.group, wl.d), dtype=torch.float32, device=path.K.device)

    def step():
        axr.axr_attention(path.q, path.idx[0], path.norms[0], V, wl.group, wl.b, path.signs, scores=path.scores,
                          workspace=ws, out=out)

    for _ in range(3):
        step()
    torch.cuda.synchronize()
    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    a.record()
    for _ in range(steps):
        step()
    b.record()
    torch.cuda.synchronize()
    ms = a.elapsed_time(b) / steps
    # per key: packed row + norm + scores written and read back + bf16 value row
    per_key = wl.d * wl.b // 8 + 4 + 8 * wl.group + 2 * wl.d
    byts = wl.rows * per_key
    del V, ws
    return {"ms": ms, "algo_bytes": byts, "gbs": byts / (ms * 1e-3) / 1e9, "bytes_per_key": per_key,
            "value_dtype": "bf16", "launches": 3}


# fp32 lanes of one B200 SM and its maximum SM clock: the ALU roofline of the
# CUDA-core sign-choice kernel is 148 SMs x 128 lanes x 1.965 GHz (one op per
# lane per cycle, an FMA counted as one op)
ALU_LANES_PER_SM = 128
SM_MAX_GHZ = 1.965


def sign_select_ops_per_key(wl: workloads.Workload) -> int:
    """Arithmetic that scoring one calibration key against one candidate needs:
    the Walsh-Hadamard butterflies (d log2 d), the squared norm and the
    normalisation (2d), a b-step binary search (d b compares), the residual (d),
    the projection on G rotated queries (G d FMAs), and scaling and squaring
    each of the G logit errors (2G)."""
    d = wl.d
    return d * (d.bit_length() - 1) + 2 * d + d * wl.b + d + wl.group * d + 2 * wl.group


def run_sign_select(device, steps: int) -> dict:
    """The one-time sign-pattern choice of one layer of the GQA shape: 200
    candidates on 8 calibration samples of 2048 tokens (axr_select_signs: the
    error kernel and the argmin)."""
    wl = workloads.GQA_SIGN_CALIBRATION
    K = workloads.make_keys(wl, device).reshape(wl.batch, wl.kv_heads, wl.T, wl.d)
    q = workloads.make_queries(wl, device).reshape(wl.batch, wl.kv_heads * wl.group, wl.d)
    C = workloads.SIGN_CANDIDATES
    cand = workloads.make_sign_candidates(wl, C).to(device)
    errors = torch.empty((C, wl.kv_heads), dtype=torch.float32, device=device)
    best = torch.empty(1, dtype=torch.int32, device=device)

    def step():
        axr.axr_select_signs(K, q, wl.group, wl.b, cand, errors=errors, best=best)

    for _ in range(3):
        step()
    torch.cuda.synchronize()
    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    a.record()
    for _ in range(steps):
        step()
    b.record()
    torch.cuda.synchronize()
    ms = a.elapsed_time(b) / steps
    key_cands = wl.rows * C
    ops = key_cands * sign_select_ops_per_key(wl)
    peak = torch.cuda.get_device_properties(device).multi_processor_count * ALU_LANES_PER_SM * SM_MAX_GHZ * 1e9
    out = {"ms": ms, "candidates": C, "samples": wl.batch, "kv_heads": wl.kv_heads, "tokens": wl.T,
           "chosen": int(best.item()), "key_candidates_per_s": key_cands / (ms * 1e-3),
           "roofline": {"bound": "alu", "kernel": "sign_errors", "source": "sign_select.cu",
                        "ops_per_key_candidate": sign_select_ops_per_key(wl),
                        "achieved": ops / (ms * 1e-3) / 1e12, "peak": peak / 1e12, "unit": "Tops/s",
                        "peak_kind": "nominal: SMs x 128 fp32 lanes x 1.965 GHz",
                        "frac": ops / (ms * 1e-3) / peak},
           "launches": 2}
    del K, q, cand, errors, best
    return out


BLOCK_GRID_DIMS = (128, 256, 512)
BLOCK_GRID_BITS = (2, 3, 4)
BLOCK_GRID_DTYPES = ("f16", "f32")


def run_block_grid(device, steps: int) -> dict:
    """Quantize-on-write with the IsoQuant block rotation against the sign flip and
    Walsh-Hadamard transform, on the 18 settings d x b x key dtype of the IsoQuant
    comparison: 2^28 bytes of keys per setting (larger than L2), rows N(0,1)^d
    normalised and scaled by U(0.1, 50).  Times each write call with CUDA events
    (average of `steps` after 3 warm-up calls) and its algorithmic HBM rate."""
    rows = []
    peak, _ = measured_peak()
    for dt in BLOCK_GRID_DTYPES:
        for d in BLOCK_GRID_DIMS:
            esize = 2 if dt == "f16" else 4
            n = (1 << 28) // (d * esize)
            wl = workloads.WRITE_2E24.with_(d=d, T=n, dtype=dt, seed=40 + d)
            K = workloads.make_keys(wl, device).reshape(n, d)
            signs = workloads.make_signs(wl).to(device)
            quats = workloads.make_block_quats(wl).to(device)
            for b in BLOCK_GRID_BITS:
                P = d * b // 8
                idx = torch.empty((n, P), dtype=torch.uint8, device=device)
                norms = torch.empty(n, dtype=torch.float32, device=device)

                def time_ms(fn):
                    for _ in range(3):
                        fn()
                    torch.cuda.synchronize()
                    a, e = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
                    a.record()
                    for _ in range(steps):
                        fn()
                    e.record()
                    torch.cuda.synchronize()
                    return a.elapsed_time(e) / steps

                t_h = time_ms(lambda: axr.axr_quantize_keys(K, b, signs, idx=idx, norms=norms))
                t_b = time_ms(lambda: axr.axr_quantize_keys_block(K, b, quats, idx=idx, norms=norms))
                byts = n * (d * esize + P + 4)
                rows.append({"d": d, "b": b, "dtype": dt, "keys": n, "hadamard_ms": t_h, "block_ms": t_b,
                             "hadamard_gbs": byts / (t_h * 1e-3) / 1e9, "block_gbs": byts / (t_b * 1e-3) / 1e9,
                             "block_frac_of_measured": byts / (t_b * 1e-3) / 1e9 / peak,
                             "block_speedup": t_h / t_b})
                del idx, norms
            del K
    sp = [r["block_speedup"] for r in rows]
    return {"settings": rows, "mean_block_speedup": sum(sp) / len(sp),
            "bytes_per_key": "d * key bytes + d*b/8 + 4", "peak_gbs": peak}


def run_cpu_baseline(wl: workloads.Workload, target_s: float):
    """The oracle, as it stands (single thread), on a bounded sample of the
    workload: consecutive chunks of keys of one KV head (drawn by the workload's
    recipe on the host), each quantized and scored against that head's G query
    heads, until about ``target_s`` seconds of work.  Returns scores/s and a
    description of the sample."""
    import oracle

    oracle.build()
    chunk = min(1 << 14, wl.T)
    one = wl.with_(batch=1, T=min(wl.T, 1 << 20))
    q = workloads.make_queries(one, "cpu").double().numpy()          # (H*G, d)
    s = workloads.make_signs(wl).numpy()
    keys = workloads.make_keys(one, "cpu")                            # (H, T', d)
    done, busy = 0, 0.0
    for h in range(keys.shape[0]):
        qh = q[h * wl.group:(h + 1) * wl.group]
        for t0 in range(0, keys.shape[1], chunk):
            if busy >= target_s:
                break
            Kd = keys[h, t0:t0 + chunk].double().numpy()
            start = time.perf_counter()
            packed, norms, _ = oracle.quantize(Kd, wl.b, s)
            oracle.scores(qh, packed[None], norms[None], wl.group, wl.b, s)
            busy += time.perf_counter() - start
            done += Kd.shape[0]
    rate = wl.group * done / busy
    single = {
        "value": rate, "unit": "scores/s", "cores": 1,
        "sample": (f"{done} keys of {wl.name} (b={wl.b}, batch element 0, head by head, chunks of "
                   f"{chunk}): quantized and scored against their {wl.group} query heads by the fp64 "
                   f"oracle; {busy:.1f} s on one host thread"),
    }
    # the same oracle in one process per host core (up to POOL_MAX), about 24 s of
    # CPU work in total, each process on the first chunk of KV head 0
    n = min(host_cores(), POOL_MAX)
    if n <= 1:
        return rate, dict(single, kind="oracle")
    per = max(1.0, 24.0 / n)
    Kd = keys[0, :chunk].double().numpy()
    rate_n, wall = pooled_oracle_rate(n, Kd, q[:wl.group], s, wl, per, chunk)
    return rate_n, {
        "value": rate_n, "unit": "scores/s", "cores": n, "kind": "oracle",
        "sample": (f"{n} processes (spawned, one thread each), each quantizing and scoring the first "
                   f"{Kd.shape[0]} keys of KV head 0 of {wl.name} (b={wl.b}) against its {wl.group} query "
                   f"heads with the fp64 oracle for {per:.1f} s; rate = all scores / {wall:.2f} s"),
        "single_thread": single,
    }


POOL_MAX = 32


def host_cores() -> int:
    try:
        return len(os.sched_getaffinity(0))
    except AttributeError:
        return os.cpu_count() or 1


def pooled_oracle_rate(n, K, q, s, wl, per_worker_s, chunk):
    """The oracle in n spawned processes at once (oracle/pool.py), each busy for
    about per_worker_s seconds: total scores / the longest busy time."""
    import multiprocessing as mp

    from oracle import pool as opool

    ctx = mp.get_context("spawn")
    with ctx.Pool(n, initializer=opool.init, initargs=(K, q, s, wl.b, wl.group)) as pl:
        res = pl.starmap(opool.run_for, [(per_worker_s, chunk)] * n)
    wall = max(r[1] for r in res)
    return sum(r[0] for r in res) / wall, wall


def reference_arm(args, wl, world, rank):
    """--impl reference: the CPU oracle on this machine's host cores, same metric."""
    if rank != 0:
        return
    import oracle

    oracle.build()
    per_step_s = max(0.5, min(5.0, 150.0 / max(1, args.steps + args.warmup)))
    K = workloads.make_keys(wl.with_(batch=1, kv_heads=1, T=min(wl.T, 1 << 16)), "cpu")[0].double().numpy()
    q = workloads.make_queries(wl.with_(batch=1, kv_heads=1), "cpu").double().numpy()
    s = workloads.make_signs(wl).numpy()

    def step(S):
        packed, norms, _ = oracle.quantize(K[:S], wl.b, s)
        oracle.scores(q, packed[None], norms[None], wl.group, wl.b, s)

    t0 = time.perf_counter()
    step(128)
    dt = time.perf_counter() - t0
    S = int(min(K.shape[0], max(64, 128 * per_step_s / max(dt, 1e-6))))
    n = min(host_cores(), POOL_MAX)
    if n > 1:
        # one spawned process per host core (up to POOL_MAX), each a step of S keys
        import multiprocessing as mp

        from oracle import pool as opool

        with mp.get_context("spawn").Pool(n, initializer=opool.init,
                                          initargs=(K, q[:wl.group], s, wl.b, wl.group)) as pl:
            for _ in range(args.warmup):
                pl.map(opool.step, [S] * n)
            t0 = time.perf_counter()
            for _ in range(args.steps):
                pl.map(opool.step, [S] * n)
            el = time.perf_counter() - t0
    else:
        for _ in range(args.warmup):
            step(S)
        t0 = time.perf_counter()
        for _ in range(args.steps):
            step(S)
        el = time.perf_counter() - t0
    rate = wl.group * S * n * args.steps / el
    sample = (f"each step: first {S} keys of KV head 0 of {wl.name} (b={wl.b}) quantized and scored "
              f"against its {wl.group} query heads by the fp64 oracle, in each of {n} host processes "
              f"(one thread each)")
    line = {
        "impl": "reference", "metric": "lut_attention_scores_per_s", "value": rate, "unit": "scores/s",
        "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": el / args.steps * 1e3, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": config_dict(wl, world),
        "cpu_baseline": {"value": rate, "unit": "scores/s", "cores": n, "kind": "oracle", "sample": sample},
        "e2e": {"value": rate, "unit": "scores/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


def config_dict(wl, world):
    return {
        "workload": wl.name, "batch": wl.batch, "kv_heads": wl.kv_heads, "group": wl.group,
        "d": wl.d, "b": wl.b, "context": wl.T, "key_dtype": wl.dtype,
        "global_batch": wl.batch * world, "parallelism": f"shard{world}" if world > 1 else "single",
        "l2": "inputs larger than L2 (126 MB); read kernel scores the cache written one step earlier",
        "read_kernel": "cuda_core" if os.environ.get("AXR_READ_KERNEL") == "cuda_core" else "auto",
    }


def main():
    ap = argparse.ArgumentParser(description=__doc__, formatter_class=argparse.RawDescriptionHelpFormatter)
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=2000)
    ap.add_argument("--warmup", type=int, default=20)
    ap.add_argument("--impl", choices=["axr", "reference"], default="axr")
    ap.add_argument("--workload", default="gqa_decode_128k", choices=sorted(workloads.BY_NAME))
    ap.add_argument("--b", type=int, default=None, help="bits per coordinate (default: the workload's)")
    ap.add_argument("--read-kernel", choices=["auto", "cuda_core"], default="auto",
                    help="cuda_core: run every read on the CUDA-core kernel (sets AXR_READ_KERNEL before the "
                         "library loads), to compare it with the tensor-core read on the same workload")
    ap.add_argument("--tokens", type=int, default=None,
                    help="keys per KV head instead of the workload's context: a reduced case for profiler "
                         "captures (its line is not the workload's figure and carries no profiled traffic)")
    ap.add_argument("--e2e-steps", type=int, default=10)
    ap.add_argument("--sustain-seconds", type=float, default=1.5,
                    help="length of the extra window of steps timed after the K steps (0: none)")
    ap.add_argument("--cpu-baseline-seconds", type=float, default=12.0)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-legs", action="store_true",
                    help="skip the legs after the step (decode step, attention, sign choice, block-rotation grid)")
    args = ap.parse_args()
    args.warmup = max(args.warmup, 3)

    if args.read_kernel == "cuda_core":
        os.environ["AXR_READ_KERNEL"] = "cuda_core"
    world, rank, local = dist_env()
    base = workloads.BY_NAME[args.workload]
    if args.b is not None:
        base = base.with_(b=args.b)
    if args.tokens is not None:
        base = base.with_(T=args.tokens)

    if args.impl == "reference":
        reference_arm(args, base, world, rank)
        return

    torch.cuda.set_device(local)
    device = torch.device("cuda", local)
    if world > 1:
        from datetime import timedelta
        dist.init_process_group("nccl", timeout=timedelta(seconds=120), device_id=device)
    wl = shard_workload(base, rank, world)
    elem = torch.tensor([], dtype=wl.torch_dtype).element_size()
    algo = algorithmic_bytes(wl, elem)

    # cpu baseline first (rank 0, N=1): the host is idle while the GPU runs later
    cpu_baseline = None
    if world == 1 and rank == 0 and not args.no_cpu_baseline:
        _, cpu_baseline = run_cpu_baseline(wl, args.cpu_baseline_seconds)

    path = Path(wl, device)
    stream = torch.cuda.current_stream(device)
    clocks = ClockSampler(local)
    clocks.start()

    def barrier():
        if world > 1:
            dist.barrier()
        torch.cuda.synchronize(device)

    clocks.busy(True)
    for i in range(args.warmup):
        path.quantize(i % 2)
        path.score((i + 1) % 2)
    barrier()

    barrier()
    mark0 = clocks.mark()
    elapsed_ms, t_write, t_read = timed_steps(path, stream, args.steps, barrier)
    clock_window = clocks.summary(mark0)
    elapsed_ms, t_write, t_read = max_over_ranks([elapsed_ms, t_write, t_read], world, device)
    ms_per_step = elapsed_ms / args.steps

    # a longer window of the same steps (at least --sustain-seconds), so that the
    # power-capped clock the kernels settle at is measured even for a short run;
    # every rank runs the same number of steps
    sus_steps = max(1, math.ceil(args.sustain_seconds * 1e3 / max(ms_per_step, 1e-3)))
    sus_steps = int(max_over_ranks([float(sus_steps)], world, device)[0])
    sustained = None
    if args.sustain_seconds > 0:
        barrier()
        mark1 = clocks.mark()
        s_el, s_w, s_r = timed_steps(path, stream, sus_steps, barrier)
        s_clocks = clocks.summary(mark1)
        s_el, s_w, s_r = max_over_ranks([s_el, s_w, s_r], world, device)
        sustained = {"steps": sus_steps, "seconds": s_el * 1e-3, "ms_per_step": s_el / sus_steps,
                     "write_ms": s_w, "read_ms": s_r, "clocks": s_clocks}
    clocks.busy(False)

    # end to end through the public API with host buffers
    e2e = run_e2e(wl, path, device, args.e2e_steps, world)
    decode_step = attention = sign_select = block_rotation = None
    if not args.no_legs:
        decode_step = run_decode_step(path, 200)
        attention = run_attention(path, 100)
        sign_select = run_sign_select(device, 5)
        block_rotation = run_block_grid(device, 10)
    clocks.stop()

    if rank != 0:
        if world > 1:
            dist.destroy_process_group()
        return

    keys_per_step = wl.rows * world
    peak, peak_kind = measured_peak()
    write_gbs = algo["write"] / (t_write * 1e-3) / 1e9
    read_gbs = algo["read"] / (t_read * 1e-3) / 1e9
    kernels = {
        "quantize_keys": {"ms": t_write, "algo_bytes": algo["write"], "gbs": write_gbs,
                          "frac_of_measured": write_gbs / peak, "frac_of_8tbs": write_gbs / NOMINAL_HBM_GBS,
                          "keys_per_s": wl.rows / (t_write * 1e-3),
                          "bytes_per_key": algo["write_per_key"]},
        "scores": {"ms": t_read, "algo_bytes": algo["read"], "gbs": read_gbs,
                   "frac_of_measured": read_gbs / peak, "frac_of_8tbs": read_gbs / NOMINAL_HBM_GBS,
                   "scores_per_s": wl.heads * wl.group * wl.T / (t_read * 1e-3),
                   "bytes_per_row": algo["read_per_row"]},
    }
    dominant = "quantize_keys" if t_write >= t_read else "scores"

    def roofline(kind):
        k = kernels[kind]
        src = kernel_file(kind, wl)
        return {"bound": "hbm", "kernel": kind, "source": src, "achieved": k["gbs"], "peak": peak,
                "peak_kind": peak_kind, "unit": "GB/s", "frac": k["gbs"] / peak,
                "frac_of_8tbs": k["gbs"] / NOMINAL_HBM_GBS,
                "traffic": None if args.tokens is not None else profiled_traffic(src, wl.name, wl.b)}

    if sustained is not None:
        mhz = sustained["clocks"].get("sm_mhz")
        top = sustained["clocks"].get("sm_max_mhz") or mhz
        for kind, key, byts in (("quantize_keys", "write", algo["write"]), ("scores", "read", algo["read"])):
            ms = sustained[f"{key}_ms"]
            gbs = byts / (ms * 1e-3) / 1e9
            sustained[key] = {"ms": ms, "gbs": gbs, "frac_of_measured": gbs / peak,
                              "frac_of_8tbs": gbs / NOMINAL_HBM_GBS,
                              # the time at the median clock scaled to the maximum clock
                              "ms_at_max_clock": ms * mhz / top if mhz and top else None}
        sustained["value"] = job_scores_per_s(wl, world, sustained["ms_per_step"])
    line = {
        "metric": "lut_attention_scores_per_s",
        "value": job_scores_per_s(wl, world, ms_per_step),
        "unit": "scores/s",
        "n_gpus": world,
        "steps": args.steps,
        "warmup": args.warmup,
        "ms_per_step": ms_per_step,
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": "f32",
        "data": "synthetic",
        "config": config_dict(wl, world),
        "keys_per_s": keys_per_step / (ms_per_step * 1e-3),
        "kernels": kernels,
        "roofline": roofline(dominant),
        "roofline_write": roofline("quantize_keys"),
        "roofline_read": roofline("scores"),
        "gpu_launches": 2 * args.steps,
        "clocks": clock_window,
        "sustained": sustained,
        "e2e": e2e,
        "decode_step": decode_step,
        "attention": attention,
        "sign_select": sign_select,
        "block_rotation": block_rotation,
        "cpu_baseline": cpu_baseline,
    }
    print(json.dumps(line), flush=True)
    del path
    if world > 1:
        dist.destroy_process_group()


def run_e2e(wl, path, device, steps, world):
    """Same metric through the public API, inputs starting in pinned host memory:
    per step H2D of the keys and queries, both kernels, D2H of the scores."""
    K_host = path.K.cpu().pin_memory()
    q_host = path.q.cpu().pin_memory()
    out_host = torch.empty(path.scores.shape, dtype=torch.float32).pin_memory()
    K_dev = torch.empty_like(path.K)
    q_dev = torch.empty_like(path.q)
    stream = torch.cuda.current_stream(device)
    h2d = K_host.numel() * K_host.element_size() + q_host.numel() * q_host.element_size()
    d2h = out_host.numel() * 4

    def step():
        K_dev.copy_(K_host, non_blocking=True)
        q_dev.copy_(q_host, non_blocking=True)
        idx, norms = axr.axr_quantize_keys(K_dev, wl.b, path.signs, idx=path.idx[0], norms=path.norms[0])
        axr.axr_scores(q_dev, idx, norms, wl.group, wl.b, path.signs, scores=path.scores)
        out_host.copy_(path.scores, non_blocking=True)

    step()
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize(device)
    a = torch.cuda.Event(enable_timing=True)
    b = torch.cuda.Event(enable_timing=True)
    a.record(stream)
    for _ in range(steps):
        step()
    b.record(stream)
    torch.cuda.synchronize(device)
    ms = max_over_ranks([a.elapsed_time(b) / steps], world, device)[0]
    return {"value": job_scores_per_s(wl, world, ms), "unit": "scores/s",
            "ms_per_step": ms, "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h}


if __name__ == "__main__":
    main()
