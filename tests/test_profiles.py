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


def test_traffic_lines_carry_the_hash_they_were_captured_on():
    """Every line of profiles/traffic.txt names the source hash listed on its
    `# captured:` line: a line is never relabelled to a later source."""
    text = open(os.path.join(ROOT, "profiles", "traffic.txt")).read()
    cap = [ln for ln in text.splitlines() if ln.startswith("# captured:")]
    assert len(cap) == 1, "traffic.txt needs exactly one '# captured:' line"
    words = cap[0].split(":", 1)[1].split()
    captured = dict(zip(words[0::2], words[1::2]))
    lines = [ln.split() for ln in text.splitlines() if ln.strip() and not ln.startswith("#")]
    assert lines
    for parts in lines:
        assert len(parts) == 5, parts
        assert parts[0] in captured and parts[3] == captured[parts[0]], parts


def test_kernel_files_follow_the_library_dispatch():
    assert bench.kernel_file("quantize_keys", workloads.GQA_DECODE_128K) == "quantize_keys_tc.cu"
    assert bench.kernel_file("scores", workloads.GQA_DECODE_128K) == "scores_tc128.cu"
    assert bench.kernel_file("quantize_keys", workloads.WIDE_D512) == "quantize_keys_tc.cu"
    assert bench.kernel_file("scores", workloads.WIDE_D256) == "scores_tc.cu"
    assert bench.kernel_file("quantize_keys", workloads.PR1_REF) == "quantize_keys.cu"     # fp32 keys


def test_profile_summaries_name_existing_sources_and_commands():
    csrc = os.path.join(ROOT, "lut_attention_b200", "csrc")
    for name in os.listdir(os.path.join(ROOT, "profiles")):
        text = open(os.path.join(ROOT, "profiles", name)).read()
        for src in set(re.findall(r"\b([a-z_]+\.cu)\b", text)):
            assert os.path.exists(os.path.join(csrc, src)), (name, src)
        if name.endswith(".md") and "ncu" in text:
            for cmd in re.findall(r"^\s*ncu --.*$", text, flags=re.M):
                assert "--clock-control none" in cmd, f"{name}: an ncu command locks clocks"
            assert re.search(r"^\s*ncu --.*$", text, flags=re.M), f"{name}: the ncu command is missing"


def test_full_size_parity_report_is_of_the_current_kernels():
    """profiles/parity_full_size.md (the every-row comparison with the oracle) was
    produced by the current write and read kernel sources."""
    text = open(os.path.join(ROOT, "profiles", "parity_full_size.md")).read()
    line = [ln for ln in text.splitlines() if ln.startswith("sources: ")]
    assert len(line) == 1
    words = line[0].split()[1:]
    recorded = dict(zip(words[0::2], words[1::2]))
    assert set(recorded) == {"quantize_keys_tc.cu", "quantize_keys.cu", "scores_tc128.cu", "scores_tc.cu"}
    for src, h in recorded.items():
        assert bench.kernel_source_hash(src) == h, f"{src} changed since the full-size parity run"
