"""lut_attention_b200: AXELRAM-style quantize-on-write and LUT score-on-read on B200.

The product is ``libaxr.so`` (C ABI in ``include/axr.h``; CUDA kernels for
sm_100a under ``csrc/``).  ``axr`` is its thin Python binding and
``workloads`` draws the seeded synthetic inputs.  Importing the package does not
load the library; the first call does, and raises if it has not been built.
"""
from .axr import (  # noqa: F401
    AxrError,
    axr_append_scores,
    axr_attention,
    axr_attention_static,
    axr_attention_workspace_bytes,
    axr_debug_build,
    axr_debug_set_span_slack,
    axr_device_status,
    axr_make_codebook,
    axr_quantize_keys,
    axr_quantize_keys_block,
    axr_scores,
    axr_scores_block,
    axr_select_signs,
    library,
    packed_row_bytes,
)

__all__ = [
    "AxrError",
    "axr_append_scores",
    "axr_attention",
    "axr_attention_static",
    "axr_attention_workspace_bytes",
    "axr_debug_build",
    "axr_debug_set_span_slack",
    "axr_device_status",
    "axr_make_codebook",
    "axr_quantize_keys",
    "axr_quantize_keys_block",
    "axr_scores",
    "axr_scores_block",
    "axr_select_signs",
    "library",
    "packed_row_bytes",
]
