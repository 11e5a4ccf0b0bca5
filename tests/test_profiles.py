"""The committed profile summaries match the kernels they describe (CPU only).

bench.py reports `roofline.traffic` from profiles/traffic.txt only when the
line's source hash equals the current kernel source.  These tests fail when a
kernel of the default bench workload changes without its DRAM bytes being
captured again (or carried over with a stated reason), and when a profile
summary names a kernel source that does not exist.
"""
import os
import re

import bench
from lut_attention_b200 import workloads

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def test_default_workload_kernels_have_current_traffic():
    wl = workloads.GQA_DECODE_128K
    for kind in ("quantize_keys", "scores"):
        src = bench.kernel_file(kind, wl)
        traffic = bench.profiled_traffic(src, wl.name, wl.b)
        assert traffic is not None, f"profiles/traffic.txt has no line for the current {src}"
        # the captured bytes are close to the algorithmic bytes of one launch
        # (writes still in L2 at the end of a launch are not counted)
        per_row = (2 * wl.d + wl.d * wl.b // 8 + 4) if kind == "quantize_keys" else (wl.d * wl.b // 8 + 4 + 4 * wl.group)
        algorithmic = wl.rows * per_row
        assert 0.85 * algorithmic <= traffic <= 1.02 * algorithmic, (src, traffic, algorithmic)


def test_kernel_files_follow_the_library_dispatch():
    assert bench.kernel_file("quantize_keys", workloads.GQA_DECODE_128K) == "quantize_keys_tc.cu"
    assert bench.kernel_file("scores", workloads.GQA_DECODE_128K) == "scores_tc.cu"
    assert bench.kernel_file("quantize_keys", workloads.WIDE_D512) == "quantize_keys_tc.cu"
    assert bench.kernel_file("scores", workloads.WIDE_D256) == "scores_tc.cu"
    assert bench.kernel_file("quantize_keys", workloads.PR1_REF) == "quantize_keys.cu"     # fp32 keys


def test_profile_summaries_name_existing_sources_and_commands():
    csrc = os.path.join(ROOT, "lut_attention_b200", "csrc")
    for name in os.listdir(os.path.join(ROOT, "profiles")):
        text = open(os.path.join(ROOT, "profiles", name)).read()
        for src in set(re.findall(r"\b([a-z_]+\.cu)\b", text)):
            assert os.path.exists(os.path.join(csrc, src)), (name, src)
        if name.endswith(".md"):
            assert "--clock-control none" in text, f"{name}: the ncu command is missing or locks clocks"
