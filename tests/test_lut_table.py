"""The read kernels' per-lane lookup table (CPU only).

lut_read.cuh builds, in shared memory, a table replicated for the 32 lanes of a
warp: entry (field, lane) at field * 256 + lane * EB holds the hi digits of the
C codes of the field (code i = bits B i .. B i + B - 1 of the field), then their
lo digits.  C = 2 codes per field at b = 3, 4 and 4 at b = 1, 2.  At b = 3 the
table is indexed by a whole byte r: the entries at r * 256 read the field from
bits 0..5 of r, those at r * 256 + 128 from bits 2..7.  The table builder is
compiled with nvcc as host code and run with the thread counts of the kernels;
its bytes must equal this definition, and nothing outside the table is written.
"""
import os
import shutil
import subprocess

import numpy as np
import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
NVCC = shutil.which("nvcc") or "/usr/local/cuda/bin/nvcc"
THREADS = (512, 384, 352, 17)     # the d = 128 kernel at G <= 4 and G <= 8, a wide kernel's workers, and odd

HI = np.array([7 * i - 50 for i in range(16)], dtype=np.int64).astype(np.int8)
LO = np.array([100 + i for i in range(16)], dtype=np.int64).astype(np.int8)


@pytest.fixture(scope="module")
def exe(tmp_path_factory):
    if not os.path.exists(NVCC):
        pytest.skip("nvcc not found")
    out = tmp_path_factory.mktemp("lut") / "lut_table_dump"
    csrc = os.path.join(ROOT, "lut_attention_b200", "csrc")
    subprocess.run([NVCC, "-std=c++17", "-O1", "-I", os.path.join(ROOT, "include"), "-I", csrc, "-o", str(out),
                    os.path.join(ROOT, "tests", "native", "lut_table_dump.cu")], check=True, capture_output=True)
    return str(out)


def expected(b: int) -> np.ndarray:
    c = 2 if b >= 3 else 4
    eb = 2 * c
    tab = np.zeros(65536, dtype=np.uint8)

    def entry(field):
        codes = [(field >> (b * i)) & ((1 << b) - 1) for i in range(c)]
        return np.array([HI[k] for k in codes] + [LO[k] for k in codes], dtype=np.int8).view(np.uint8)

    if b == 3:
        for r in range(256):
            for lane in range(32):
                tab[r * 256 + lane * eb: r * 256 + (lane + 1) * eb] = entry(r & 63)
                tab[r * 256 + 128 + lane * eb: r * 256 + 128 + (lane + 1) * eb] = entry(r >> 2)
    else:
        for field in range(1 << (c * b)):
            for lane in range(32):
                tab[field * 256 + lane * eb: field * 256 + (lane + 1) * eb] = entry(field)
    return tab


@pytest.mark.parametrize("nthreads", THREADS)
def test_table_matches_its_definition(exe, nthreads):
    lines = subprocess.run([exe, str(nthreads)], check=True, capture_output=True, text=True).stdout.split()
    assert len(lines) == 4
    for b, line in zip((1, 2, 3, 4), lines):
        got = np.frombuffer(bytes.fromhex(line), dtype=np.uint8)
        assert got.size == 65536
        want = expected(b)
        bad = np.flatnonzero(got != want)
        assert bad.size == 0, f"b={b}, {nthreads} threads: {bad.size} bytes differ, first at {bad[:4]}"


def test_definition_is_not_vacuous():
    # the test digits are distinct, so a swapped hi/lo byte or a wrong code order shows
    assert len(set(HI.tolist()) | set(LO.tolist())) == 32
    # b = 4: field 0x21 holds codes 1 (bits 0..3) then 2 (bits 4..7)
    e = expected(4)[0x21 * 256: 0x21 * 256 + 4].view(np.int8)
    assert e.tolist() == [HI[1], HI[2], LO[1], LO[2]]
    # b = 3, second table: byte 0b10110100 holds the field 0b101101 (bits 2..7)
    r = 0b10110100
    e = expected(3)[r * 256 + 128: r * 256 + 132].view(np.int8)
    assert e.tolist() == [HI[0b101], HI[0b101], LO[0b101], LO[0b101]]
