"""The debug build (libaxr_debug.so, -DAXR_DEBUG) on the GPU.

In that build every kernel checks each plain global load and store against
the buffer the call's arguments describe and records status bit 16 instead of
making one that falls outside.  Two runs of tests/debug_tiny.py, each in a
process of its own (the binding loads one library per process):
  * every entry point on tiny shapes (n = 1, 3, 31, 33 at d = 8 and 32; n = 1,
    3, 33, 129 on the tensor-core kernels at d = 128, 256, 512) against the
    oracle, with device status 0: no access left its buffer;
  * the same calls with every span 4 bytes short: each records bit 16 and
    leaves the last bytes of its outputs untouched, so the checks do fire
    (no access leaves the real buffers: they are 4 bytes longer than the spans).
The tiny cases also run here, in this process, on the release library.
"""
import os
import subprocess
import sys

import pytest

import debug_tiny
from lut_attention_b200 import axr, build

pytestmark = pytest.mark.gpu
HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(HERE)


@pytest.fixture(scope="module")
def debug_lib():
    if not os.path.exists(build.DEBUG_LIB_PATH):
        build.build(debug=True)
    return build.DEBUG_LIB_PATH


def _run(args, timeout=900):
    env = dict(os.environ, AXR_DEBUG="1")
    r = subprocess.run([sys.executable, os.path.join(HERE, "debug_tiny.py"), *args], cwd=ROOT, env=env,
                       capture_output=True, text=True, timeout=timeout)
    out = r.stdout + r.stderr
    assert r.returncode == 0, out[-4000:]
    return out


def test_debug_build_tiny_shapes_match_the_oracle_with_status_0(debug_lib):
    out = _run([])
    assert "debug build: True" in out and "cases passed" in out, out[-2000:]


def test_debug_build_checks_fire_on_shortened_spans(debug_lib):
    out = _run(["--slack", "4"])
    assert "span slack 4" in out and "cases passed" in out, out[-2000:]


def test_tiny_shapes_on_the_release_library(axr_lib, oracle_lib):
    assert not axr.axr_debug_build() or axr.DEBUG
    assert debug_tiny.run(0) == 0
