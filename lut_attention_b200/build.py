"""Build libaxr.so in-tree with nvcc for sm_100a.

    python -m lut_attention_b200.build [--force] [--ptxas-verbose] [--debug]

Each source compiles to an object under ``_build/`` (in parallel), then nvcc
links them into ``lut_attention_b200/libaxr.so`` with the CUDA runtime linked
statically, so the library does not depend on which libcudart PyTorch loads.

``--debug`` builds ``lut_attention_b200/libaxr_debug.so`` from the same sources
with ``-DAXR_DEBUG`` (objects under ``_build/debug/``): every kernel then
checks its plain global loads and stores against the buffers the call
describes and records status bit 16 instead of making one that falls outside.
The binding loads it instead of libaxr.so when ``AXR_DEBUG=1`` is set.
"""
from __future__ import annotations

import argparse
import os
import shutil
import subprocess
import sys
from concurrent.futures import ThreadPoolExecutor

PKG = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(PKG)
CSRC = os.path.join(PKG, "csrc")
INCLUDE = os.path.join(ROOT, "include")
BUILD_DIR = os.path.join(ROOT, "_build")
LIB_PATH = os.path.join(PKG, "libaxr.so")
DEBUG_LIB_PATH = os.path.join(PKG, "libaxr_debug.so")

SOURCES = ["api.cu", "attention.cu", "codebook.cpp", "quantize_keys.cu", "quantize_keys_block.cu",
           "quantize_keys_tc.cu", "scores.cu", "scores_tc.cu", "scores_tc128.cu", "sign_select.cu"]
HEADERS = [os.path.join(INCLUDE, "axr.h")] + [
    os.path.join(CSRC, f) for f in os.listdir(CSRC) if f.endswith((".cuh", ".h"))
]

ARCH = ["-gencode", "arch=compute_100a,code=sm_100a"]
COMMON = ["-O3", "-std=c++17", "-lineinfo", "-Xcompiler", "-fPIC,-Wall", "-I", INCLUDE, "-I", CSRC]


def nvcc() -> str:
    path = shutil.which("nvcc") or "/usr/local/cuda/bin/nvcc"
    if not os.path.exists(path):
        raise RuntimeError("nvcc not found: the CUDA toolkit is required to build libaxr")
    return path


def _stale(target: str, deps: list[str]) -> bool:
    if not os.path.exists(target):
        return True
    t = os.path.getmtime(target)
    return any(os.path.getmtime(d) > t for d in deps)


def build(force: bool = False, ptxas_verbose: bool = False, jobs: int | None = None, debug: bool = False) -> str:
    build_dir = os.path.join(BUILD_DIR, "debug") if debug else BUILD_DIR
    lib_path = DEBUG_LIB_PATH if debug else LIB_PATH
    os.makedirs(build_dir, exist_ok=True)
    cc = nvcc()
    objs, cmds = [], []
    for src in SOURCES:
        src_path = os.path.join(CSRC, src)
        obj = os.path.join(build_dir, os.path.splitext(src)[0] + ".o")
        objs.append(obj)
        if force or _stale(obj, [src_path] + HEADERS):
            flags = list(COMMON) + ARCH + (["-DAXR_DEBUG"] if debug else [])
            if ptxas_verbose and src.endswith(".cu"):
                flags += ["-Xptxas", "-v"]
            cmds.append([cc, *flags, "-c", src_path, "-o", obj])

    def run(cmd):
        r = subprocess.run(cmd, capture_output=True, text=True)
        return cmd, r

    failed = []
    with ThreadPoolExecutor(max_workers=jobs or min(8, os.cpu_count() or 1)) as ex:
        for cmd, r in ex.map(run, cmds):
            out = (r.stdout + r.stderr).strip()
            if out and (ptxas_verbose or r.returncode != 0):
                print(out, file=sys.stderr)
            if r.returncode != 0:
                failed.append(os.path.basename(cmd[-3]))
    if failed:
        raise RuntimeError(f"nvcc failed on: {', '.join(failed)}")

    if force or cmds or _stale(lib_path, objs):
        tmp = f"{lib_path}.{os.getpid()}.tmp"
        subprocess.check_call([cc, "-shared", *ARCH, "-o", tmp, *objs, "-cudart", "static"])
        os.replace(tmp, lib_path)
    return lib_path


def main() -> None:
    ap = argparse.ArgumentParser(description=__doc__)
    ap.add_argument("--force", action="store_true")
    ap.add_argument("--ptxas-verbose", action="store_true")
    ap.add_argument("--debug", action="store_true", help="build libaxr_debug.so (-DAXR_DEBUG)")
    args = ap.parse_args()
    print(build(force=args.force, ptxas_verbose=args.ptxas_verbose, debug=args.debug))


if __name__ == "__main__":
    main()
