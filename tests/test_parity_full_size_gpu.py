"""Full-size parity of the whole path with the oracle, on every workload.

Each workload runs at its full size in the benchmark's launch configuration,
and every key row is compared with the oracle (at least 2^20 seeded rows plus
each KV head's first and last for the two wide-head workloads, where the oracle's
dense d x d rotation makes every row too slow).  The boundary-window counts of
each workload are printed in the terminal summary of the run, and written as
JSON lines to the file named by the AXR_PARITY_REPORT environment variable when
it is set.  Counting rules and tolerances: tests/full_parity.py.
"""
import json
import os

import pytest
import torch

import full_parity
from lut_attention_b200 import workloads

pytestmark = pytest.mark.gpu

WIDE_SAMPLE_ROWS = 1 << 20

CASES = [("pr1_ref", 4), ("mha_decode_32k", 3), ("gqa_decode_128k", 2), ("gqa_decode_128k", 3),
         ("gqa_decode_128k", 4), ("write_2e24", 4), ("wide_heads_d256", 2), ("wide_heads_d512", 2)]


@pytest.fixture(autouse=True, scope="module")
def _libs(axr_lib, oracle_lib):
    return axr_lib


@pytest.mark.parametrize("name,b", CASES)
def test_full_size_parity(name, b):
    wl = workloads.BY_NAME[name].with_(b=b)
    sample = WIDE_SAMPLE_ROWS if name.startswith("wide_heads") else None
    rep = full_parity.run(wl, torch.device("cuda", 0), min_rows=sample)
    torch.cuda.empty_cache()
    full_parity.REPORTS.append(rep.line())
    out = os.environ.get("AXR_PARITY_REPORT")
    if out:
        with open(out, "a") as f:
            f.write(json.dumps(rep.as_dict()) + "\n")
    if sample is None:
        assert rep.rows_checked == wl.rows
    else:
        assert rep.rows_checked >= sample
    assert rep.ok(), rep.line()
