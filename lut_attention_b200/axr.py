"""Python binding of libaxr (the C ABI in include/axr.h): argument marshalling only.

Every computation runs in libaxr's CUDA kernels.  This module checks tensor
shapes, allocates outputs when the caller gives none, passes raw device
pointers and the current CUDA stream, and turns status codes into exceptions.
There is no CPU path: without the built library or a CUDA device the calls raise.
"""
from __future__ import annotations

import ctypes
import os
import threading

import numpy as np
import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
# AXR_DEBUG=1 selects the debug build (device-side bounds checks, status bit 16)
DEBUG = os.environ.get("AXR_DEBUG", "") == "1"
LIB_PATH = os.path.join(_HERE, "libaxr_debug.so" if DEBUG else "libaxr.so")

AXR_OK, AXR_EINVAL, AXR_EUNSUPPORTED, AXR_ECUDA = 0, -1, -2, -3
AXR_F32, AXR_F16, AXR_BF16 = 0, 1, 2
_DTYPE_CODE = {torch.float32: AXR_F32, torch.float16: AXR_F16, torch.bfloat16: AXR_BF16}

# every symbol include/axr.h declares, with its ctypes signature
_P, _I32, _I64 = ctypes.c_void_p, ctypes.c_int, ctypes.c_int64
SIGNATURES = {
    "axr_make_codebook": (_I32, [_I32, _I32, _P, _P]),
    "axr_quantize_keys": (_I32, [_P, _I32, _I64, _I32, _I32, _P, _P, _P, _P]),
    "axr_scores": (_I32, [_P, _I32, _P, _P, _I64, _I32, _I32, _I32, _I32, _P, _P, _P]),
    "axr_append_scores": (_I32, [_P, _I32, _P, _I32, _P, _P, _I64, _I64, _I32, _I32, _I32, _I32, _P, _P, _P]),
    "axr_attention_workspace_bytes": (_I32, [_I64, _I32, _I32, _I32, _P]),
    "axr_attention": (_I32, [_P, _I32, _P, _P, _P, _I32, _I64, _I32, _I32, _I32, _I32, _P, _P, _P, _I64, _P, _P]),
    "axr_attention_static": (_I32, [_P, _I32, _P, _P, _P, _I32, _I64, _I32, _I32, _I32, _I32, _P, _P, _P, _P]),
    "axr_quantize_keys_block": (_I32, [_P, _I32, _I64, _I32, _I32, _P, _P, _P, _P]),
    "axr_scores_block": (_I32, [_P, _I32, _P, _P, _I64, _I32, _I32, _I32, _I32, _P, _P, _P]),
    "axr_select_signs": (_I32, [_P, _I32, _P, _I32, _I64, _I32, _I32, _I32, _I32, _I32, _P, _I32, _P, _P, _P]),
    "axr_status_string": (ctypes.c_char_p, [_I32]),
    "axr_last_error": (ctypes.c_char_p, []),
    "axr_version": (_I32, []),
    "axr_device_status": (_I32, [_I32, _P]),
    "axr_debug_build": (_I32, []),
    "axr_debug_set_span_slack": (_I32, [_I64]),
}

_lock = threading.Lock()
_lib = None


class AxrError(RuntimeError):
    def __init__(self, status: int, where: str, detail: str):
        super().__init__(f"{where}: status {status} ({detail})")
        self.status = status


def library() -> ctypes.CDLL:
    """Load libaxr.so (built in-tree by ``python -m lut_attention_b200.build``)."""
    global _lib
    with _lock:
        if _lib is None:
            if not os.path.exists(LIB_PATH):
                raise RuntimeError(
                    f"{os.path.basename(LIB_PATH)} is missing at {LIB_PATH}: build it with "
                    f"`python -m lut_attention_b200.build{' --debug' if DEBUG else ''}` (needs nvcc)")
            lib = ctypes.CDLL(LIB_PATH)
            for name, (res, args) in SIGNATURES.items():
                fn = getattr(lib, name)
                fn.restype = res
                fn.argtypes = args
            _lib = lib
        return _lib


def _raise(rc: int, where: str) -> None:
    if rc != AXR_OK:
        lib = library()
        detail = lib.axr_last_error().decode() or lib.axr_status_string(rc).decode()
        raise AxrError(rc, where, detail)


def _stream_handle(stream, device=None) -> int:
    if stream is None:
        stream = torch.cuda.current_stream(device)
    return int(stream.cuda_stream) if hasattr(stream, "cuda_stream") else int(stream)


def _call(name: str, device: torch.device, stream, *args) -> None:
    """Call libaxr's `name` with the tensors' device current (the library checks its
    pointers against, and launches on, the current device), on `stream` or that
    device's current stream; a status other than AXR_OK raises."""
    with torch.cuda.device(device):
        rc = getattr(library(), name)(*args, _stream_handle(stream, device))
    _raise(rc, name)


def _require_cuda(t: torch.Tensor, name: str) -> None:
    if not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor (libaxr has no CPU path)")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")


def _check_signs(signs: torch.Tensor, d: int) -> None:
    """The sign pattern D: int8, one entry per coordinate (the kernels read d of them)."""
    if signs.dtype != torch.int8:
        raise ValueError("signs must be int8")
    if signs.numel() != d:
        raise ValueError(f"signs must have d={d} entries, got {signs.numel()}")


def _check_read_operands(idx: torch.Tensor, norms: torch.Tensor) -> None:
    """Packed codes are bytes and key norms fp32: the kernels read n*P bytes and
    4*n bytes through these pointers, whatever dtype the tensor carries."""
    if idx.dtype != torch.uint8 or norms.dtype != torch.float32:
        raise ValueError("idx must be uint8 and norms float32")


def axr_make_codebook(d: int, b: int) -> tuple[np.ndarray, np.ndarray]:
    """fp32 centroids (2^b, ascending) and boundaries (2^b - 1) for (d, b)."""
    L = 1 << b if 0 < b < 31 else 1
    cent = np.zeros(max(L, 1), dtype=np.float32)
    bnd = np.zeros(max(L - 1, 1), dtype=np.float32)
    rc = library().axr_make_codebook(d, b, cent.ctypes.data_as(_P), bnd.ctypes.data_as(_P))
    _raise(rc, "axr_make_codebook")
    return cent[:L], bnd[:L - 1]


def packed_row_bytes(d: int, b: int) -> int:
    return d * b // 8


def axr_quantize_keys(K: torch.Tensor, b: int, signs: torch.Tensor,
                      idx: torch.Tensor | None = None, norms: torch.Tensor | None = None,
                      stream=None) -> tuple[torch.Tensor, torch.Tensor]:
    """Quantize-on-write of keys K (..., d) -> (idx (..., d*b/8) uint8, norms (...) fp32)."""
    _require_cuda(K, "K")
    _require_cuda(signs, "signs")
    if K.dtype not in _DTYPE_CODE:
        raise ValueError(f"K dtype {K.dtype} not supported")
    d = K.shape[-1]
    _check_signs(signs, d)
    lead = K.shape[:-1]
    n = K.numel() // d if d else 0
    P = packed_row_bytes(d, b)
    if idx is None:
        idx = torch.empty(lead + (P,), dtype=torch.uint8, device=K.device)
    if norms is None:
        norms = torch.empty(lead, dtype=torch.float32, device=K.device)
    _require_cuda(idx, "idx")
    _require_cuda(norms, "norms")
    _check_read_operands(idx, norms)
    if idx.numel() < n * P or norms.numel() < n:
        raise ValueError("idx/norms too small")
    _call("axr_quantize_keys", K.device, stream,
          K.data_ptr(), _DTYPE_CODE[K.dtype], n, d, b, signs.data_ptr(), idx.data_ptr(), norms.data_ptr())
    return idx, norms


def axr_scores(q: torch.Tensor, idx: torch.Tensor, norms: torch.Tensor, group: int, b: int,
               signs: torch.Tensor, scores: torch.Tensor | None = None,
               stream=None) -> torch.Tensor:
    """LUT scores (heads*group, n) fp32 of queries q (heads*group, d) against packed
    keys idx (heads, n, d*b/8) with norms (heads, n)."""
    for t, name in ((q, "q"), (idx, "idx"), (norms, "norms"), (signs, "signs")):
        _require_cuda(t, name)
    if q.dtype not in _DTYPE_CODE:
        raise ValueError(f"q dtype {q.dtype} not supported")
    _check_read_operands(idx, norms)
    hg, d = q.shape
    _check_signs(signs, d)
    if group < 1 or hg % group:
        raise ValueError("q must have heads*group rows")
    heads = hg // group
    if idx.dim() != 3 or idx.shape[0] != heads or idx.shape[2] != packed_row_bytes(d, b):
        raise ValueError(f"idx must be (heads={heads}, n, {packed_row_bytes(d, b)})")
    n = idx.shape[1]
    if tuple(norms.shape) != (heads, n):
        raise ValueError(f"norms must be ({heads}, {n})")
    if scores is None:
        scores = torch.empty((hg, n), dtype=torch.float32, device=q.device)
    _require_cuda(scores, "scores")
    if scores.numel() < hg * n or scores.dtype != torch.float32:
        raise ValueError("scores must be float32 with (heads*group)*n elements")
    _call("axr_scores", q.device, stream,
          q.data_ptr(), _DTYPE_CODE[q.dtype], idx.data_ptr(), norms.data_ptr(), n, heads, group, d, b,
          signs.data_ptr(), scores.data_ptr())
    return scores


def _check_quats(quats: torch.Tensor, d: int) -> None:
    _require_cuda(quats, "quats")
    if quats.dtype != torch.float32 or tuple(quats.shape) != (d // 4, 8) or not quats.is_contiguous():
        raise ValueError(f"quats must be a contiguous ({d // 4}, 8) float32 tensor: qL then qR per 4-block")


def axr_quantize_keys_block(K: torch.Tensor, b: int, quats: torch.Tensor, idx: torch.Tensor | None = None,
                            norms: torch.Tensor | None = None, stream=None) -> tuple[torch.Tensor, torch.Tensor]:
    """Quantize-on-write of keys K (..., d) with the IsoQuant block rotation given
    by quats (d/4, 8) -> (idx (..., d*b/8) uint8, norms (...) fp32)."""
    _require_cuda(K, "K")
    if K.dtype not in _DTYPE_CODE:
        raise ValueError(f"K dtype {K.dtype} not supported")
    d = K.shape[-1]
    _check_quats(quats, d)
    lead = K.shape[:-1]
    n = K.numel() // d if d else 0
    P = packed_row_bytes(d, b)
    if idx is None:
        idx = torch.empty(lead + (P,), dtype=torch.uint8, device=K.device)
    if norms is None:
        norms = torch.empty(lead, dtype=torch.float32, device=K.device)
    _require_cuda(idx, "idx")
    _require_cuda(norms, "norms")
    _check_read_operands(idx, norms)
    if idx.numel() < n * P or norms.numel() < n:
        raise ValueError("idx/norms too small")
    _call("axr_quantize_keys_block", K.device, stream,
          K.data_ptr(), _DTYPE_CODE[K.dtype], n, d, b, quats.data_ptr(), idx.data_ptr(), norms.data_ptr())
    return idx, norms


def axr_scores_block(q: torch.Tensor, idx: torch.Tensor, norms: torch.Tensor, group: int, b: int,
                     quats: torch.Tensor, scores: torch.Tensor | None = None, stream=None) -> torch.Tensor:
    """LUT scores (heads*group, n) fp32 of queries q (heads*group, d) against keys
    written by :func:`axr_quantize_keys_block` with the same quats."""
    for t, name in ((q, "q"), (idx, "idx"), (norms, "norms")):
        _require_cuda(t, name)
    if q.dtype not in _DTYPE_CODE:
        raise ValueError(f"q dtype {q.dtype} not supported")
    _check_read_operands(idx, norms)
    hg, d = q.shape
    _check_quats(quats, d)
    if group < 1 or hg % group:
        raise ValueError("q must have heads*group rows")
    heads = hg // group
    if idx.dim() != 3 or idx.shape[0] != heads or idx.shape[2] != packed_row_bytes(d, b):
        raise ValueError(f"idx must be (heads={heads}, n, {packed_row_bytes(d, b)})")
    n = idx.shape[1]
    if tuple(norms.shape) != (heads, n):
        raise ValueError(f"norms must be ({heads}, {n})")
    if scores is None:
        scores = torch.empty((hg, n), dtype=torch.float32, device=q.device)
    _require_cuda(scores, "scores")
    if scores.numel() < hg * n or scores.dtype != torch.float32:
        raise ValueError("scores must be float32 with (heads*group)*n elements")
    _call("axr_scores_block", q.device, stream,
          q.data_ptr(), _DTYPE_CODE[q.dtype], idx.data_ptr(), norms.data_ptr(), n, heads, group, d, b,
          quats.data_ptr(), scores.data_ptr())
    return scores


def axr_append_scores(k_new: torch.Tensor, q: torch.Tensor, idx: torch.Tensor, norms: torch.Tensor, pos: int,
                      group: int, b: int, signs: torch.Tensor, scores: torch.Tensor | None = None,
                      stream=None) -> torch.Tensor:
    """One decode step on a key cache: quantize the new key of every KV head
    (k_new (heads, d)) into slot ``pos`` of idx (heads, capacity, d*b/8) and norms
    (heads, capacity), then score the query heads q (heads*group, d) against keys
    0 .. pos.  Returns scores (heads*group, pos+1) fp32."""
    for t, name in ((k_new, "k_new"), (q, "q"), (idx, "idx"), (norms, "norms"), (signs, "signs")):
        _require_cuda(t, name)
    if k_new.dtype not in _DTYPE_CODE or q.dtype not in _DTYPE_CODE:
        raise ValueError("k_new and q must be float32, float16 or bfloat16")
    _check_read_operands(idx, norms)
    heads, d = k_new.shape
    _check_signs(signs, d)
    hg, dq = q.shape
    if dq != d or group < 1 or hg != heads * group:
        raise ValueError(f"q must be ({heads}*{group}, {d})")
    if idx.dim() != 3 or idx.shape[0] != heads or idx.shape[2] != packed_row_bytes(d, b):
        raise ValueError(f"idx must be (heads={heads}, capacity, {packed_row_bytes(d, b)})")
    capacity = idx.shape[1]
    if tuple(norms.shape) != (heads, capacity):
        raise ValueError(f"norms must be ({heads}, {capacity})")
    if not 0 <= pos < capacity:
        raise ValueError(f"pos={pos} is outside the cache [0, {capacity})")
    if scores is None:
        scores = torch.empty((hg, pos + 1), dtype=torch.float32, device=q.device)
    _require_cuda(scores, "scores")
    if scores.numel() < hg * (pos + 1) or scores.dtype != torch.float32:
        raise ValueError("scores must be float32 with (heads*group)*(pos+1) elements")
    _call("axr_append_scores", k_new.device, stream,
          k_new.data_ptr(), _DTYPE_CODE[k_new.dtype], q.data_ptr(), _DTYPE_CODE[q.dtype], idx.data_ptr(),
          norms.data_ptr(), capacity, pos, heads, group, d, b, signs.data_ptr(), scores.data_ptr())
    return scores


def axr_attention_workspace_bytes(n: int, heads: int, group: int, d: int) -> int:
    """Scratch bytes axr_attention needs for this shape."""
    out = ctypes.c_int64(0)
    _raise(library().axr_attention_workspace_bytes(n, heads, group, d, ctypes.byref(out)),
           "axr_attention_workspace_bytes")
    return out.value


def axr_attention(q: torch.Tensor, idx: torch.Tensor, norms: torch.Tensor, V: torch.Tensor, group: int, b: int,
                  signs: torch.Tensor, scores: torch.Tensor | None = None, workspace: torch.Tensor | None = None,
                  out: torch.Tensor | None = None, stream=None) -> tuple[torch.Tensor, torch.Tensor]:
    """Decode attention on packed keys idx (heads, n, d*b/8) with norms (heads, n)
    and values V (heads, n, d): returns (out (heads*group, d) fp32, scores
    (heads*group, n) fp32).  A workspace is allocated when none is given."""
    for t, name in ((q, "q"), (idx, "idx"), (norms, "norms"), (V, "V"), (signs, "signs")):
        _require_cuda(t, name)
    if q.dtype not in _DTYPE_CODE or V.dtype not in _DTYPE_CODE:
        raise ValueError("q and V must be float32, float16 or bfloat16")
    _check_read_operands(idx, norms)
    hg, d = q.shape
    _check_signs(signs, d)
    if group < 1 or hg % group:
        raise ValueError("q must have heads*group rows")
    heads = hg // group
    if idx.dim() != 3 or idx.shape[0] != heads or idx.shape[2] != packed_row_bytes(d, b):
        raise ValueError(f"idx must be (heads={heads}, n, {packed_row_bytes(d, b)})")
    n = idx.shape[1]
    if tuple(norms.shape) != (heads, n) or tuple(V.shape) != (heads, n, d):
        raise ValueError(f"norms must be ({heads}, {n}) and V ({heads}, {n}, {d})")
    if scores is None:
        scores = torch.empty((hg, n), dtype=torch.float32, device=q.device)
    if out is None:
        out = torch.empty((hg, d), dtype=torch.float32, device=q.device)
    need = axr_attention_workspace_bytes(n, heads, group, d)
    if workspace is None:
        workspace = torch.empty(max(need, 16), dtype=torch.uint8, device=q.device)
    for t, name in ((scores, "scores"), (out, "out"), (workspace, "workspace")):
        _require_cuda(t, name)
    if scores.numel() < hg * n or out.numel() < hg * d or scores.dtype != torch.float32 \
            or out.dtype != torch.float32:
        raise ValueError("scores and out must be float32 and large enough")
    ws_bytes = workspace.numel() * workspace.element_size()
    _call("axr_attention", q.device, stream,
          q.data_ptr(), _DTYPE_CODE[q.dtype], idx.data_ptr(), norms.data_ptr(), V.data_ptr(),
          _DTYPE_CODE[V.dtype], n, heads, group, d, b, signs.data_ptr(), scores.data_ptr(),
          workspace.data_ptr(), ws_bytes, out.data_ptr())
    return out, scores


def axr_attention_static(q: torch.Tensor, idx: torch.Tensor, norms: torch.Tensor, V: torch.Tensor, group: int,
                         b: int, signs: torch.Tensor, scores: torch.Tensor, out: torch.Tensor,
                         stream=None) -> tuple[torch.Tensor, torch.Tensor]:
    """axr_attention with the library's fixed scratch instead of a workspace.
    scores (heads*group, n) and out (heads*group, d), fp32, come from the caller:
    this call allocates nothing.  Calls on one device must not overlap."""
    for t, name in ((q, "q"), (idx, "idx"), (norms, "norms"), (V, "V"), (signs, "signs"), (scores, "scores"),
                    (out, "out")):
        _require_cuda(t, name)
    if q.dtype not in _DTYPE_CODE or V.dtype not in _DTYPE_CODE:
        raise ValueError("q and V must be float32, float16 or bfloat16")
    _check_read_operands(idx, norms)
    hg, d = q.shape
    _check_signs(signs, d)
    if group < 1 or hg % group:
        raise ValueError("q must have heads*group rows")
    heads = hg // group
    if idx.dim() != 3 or idx.shape[0] != heads or idx.shape[2] != packed_row_bytes(d, b):
        raise ValueError(f"idx must be (heads={heads}, n, {packed_row_bytes(d, b)})")
    n = idx.shape[1]
    if tuple(norms.shape) != (heads, n) or tuple(V.shape) != (heads, n, d):
        raise ValueError(f"norms must be ({heads}, {n}) and V ({heads}, {n}, {d})")
    if scores.dtype != torch.float32 or out.dtype != torch.float32 or scores.numel() < hg * n \
            or out.numel() < hg * d:
        raise ValueError("scores and out must be float32 and large enough")
    _call("axr_attention_static", q.device, stream,
          q.data_ptr(), _DTYPE_CODE[q.dtype], idx.data_ptr(), norms.data_ptr(), V.data_ptr(),
          _DTYPE_CODE[V.dtype], n, heads, group, d, b, signs.data_ptr(), scores.data_ptr(), out.data_ptr())
    return out, scores


def axr_select_signs(K: torch.Tensor, q: torch.Tensor, group: int, b: int, candidates: torch.Tensor,
                     errors: torch.Tensor | None = None, best: torch.Tensor | None = None,
                     stream=None) -> tuple[torch.Tensor, torch.Tensor]:
    """Sign-pattern choice on calibration keys K (samples, heads, n, d) and
    queries q (samples, heads*group, d) among candidates (C, d) int8: returns
    (errors (C, heads) fp32, the logit error of each candidate per KV head;
    best, a one-element int32 tensor holding the chosen candidate's index)."""
    for t, name in ((K, "K"), (q, "q"), (candidates, "candidates")):
        _require_cuda(t, name)
    if K.dtype not in _DTYPE_CODE or q.dtype not in _DTYPE_CODE:
        raise ValueError("K and q must be float32, float16 or bfloat16")
    if candidates.dtype != torch.int8 or candidates.dim() != 2:
        raise ValueError("candidates must be a (C, d) int8 tensor")
    if K.dim() != 4:
        raise ValueError("K must be (samples, heads, n, d)")
    samples, heads, n, d = K.shape
    if tuple(q.shape) != (samples, heads * group, d):
        raise ValueError(f"q must be ({samples}, {heads * group}, {d})")
    C = candidates.shape[0]
    if candidates.shape[1] != d:
        raise ValueError(f"candidates must have {d} columns")
    if not (K.is_contiguous() and q.is_contiguous() and candidates.is_contiguous()):
        raise ValueError("K, q and candidates must be contiguous")
    if errors is None:
        errors = torch.empty((C, heads), dtype=torch.float32, device=K.device)
    if best is None:
        best = torch.empty(1, dtype=torch.int32, device=K.device)
    for t, name in ((errors, "errors"), (best, "best")):
        _require_cuda(t, name)
    if errors.dtype != torch.float32 or errors.numel() < C * heads or best.dtype != torch.int32:
        raise ValueError("errors must be float32 with C*heads elements, best int32")
    _call("axr_select_signs", K.device, stream,
          K.data_ptr(), _DTYPE_CODE[K.dtype], q.data_ptr(), _DTYPE_CODE[q.dtype], n, samples, heads, group, d,
          b, candidates.data_ptr(), C, errors.data_ptr(), best.data_ptr())
    return errors, best


def axr_device_status(clear: bool = True) -> int:
    """Bits recorded on the device (0 = none): 1, 2, 4 a bounded wait that ran out
    in a tensor-core kernel, 8 a read kernel whose stages did not fit, 16 (debug
    build only) a load or store outside its buffer, skipped."""
    out = ctypes.c_uint(0)
    _raise(library().axr_device_status(1 if clear else 0, ctypes.byref(out)), "axr_device_status")
    return out.value


def axr_debug_build() -> bool:
    """True when the loaded library is the debug build (libaxr_debug.so)."""
    return bool(library().axr_debug_build())


def axr_debug_set_span_slack(nbytes: int) -> None:
    """Debug build: shorten every buffer span the bounds checks allow by nbytes
    (0 restores them); raises in the release build."""
    _raise(library().axr_debug_set_span_slack(int(nbytes)), "axr_debug_set_span_slack")
