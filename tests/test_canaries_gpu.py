"""Outputs stay inside their buffers: every output of the decode step, decode
attention (with a caller workspace and with the fixed scratch) and the
sign-pattern choice is a view into a larger buffer whose guard bytes on both
sides hold a sentinel; after the call the guards must be intact.  Covers the
CUDA-core and the tensor-core kernels (fused decode step at d = 128, 256, 512;
two launches at d = 64)."""
import pytest
import torch

from lut_attention_b200 import axr, workloads

pytestmark = pytest.mark.gpu
DEV = "cuda"
GUARD = 4096      # elements on each side; keeps every interior view 16-byte aligned


@pytest.fixture(autouse=True, scope="module")
def _libs(axr_lib):
    return axr_lib


def guarded(n, dtype, fill):
    buf = torch.full((GUARD + n + GUARD,), fill, dtype=dtype, device=DEV)
    return buf, buf[GUARD:GUARD + n]


def intact(buf, fill):
    return bool(torch.all(buf[:GUARD] == fill)) and bool(torch.all(buf[-GUARD:] == fill))


@pytest.mark.parametrize("d,b,group,pos,capacity", [
    (128, 4, 4, 300, 301), (128, 3, 8, 0, 1), (256, 2, 2, 129, 200), (512, 4, 5, 127, 128),
    (512, 1, 1, 0, 7), (64, 3, 3, 99, 100),
])
def test_decode_step_outputs_stay_inside(d, b, group, pos, capacity):
    heads, P = 3, d * b // 8
    wl = workloads.MHA_DECODE_32K.with_(d=d, dtype="bf16", T=pos + 1, batch=1, kv_heads=heads, seed=d + pos)
    K = workloads.make_keys(wl, DEV)
    s = workloads.make_signs(wl).to(DEV)
    ibuf, iv = guarded(heads * capacity * P, torch.uint8, 0x6B)
    nbuf, nv = guarded(heads * capacity, torch.float32, -11.0)
    idx, norms = iv.view(heads, capacity, P), nv.view(heads, capacity)
    for h in range(heads):
        if pos:
            axr.axr_quantize_keys(K[h, :pos].contiguous(), b, s, idx=idx[h, :pos], norms=norms[h, :pos])
    q = torch.randn((heads * group, d), device=DEV)
    sbuf, sv = guarded(heads * group * (pos + 1), torch.float32, -13.0)
    axr.axr_append_scores(K[:, pos].contiguous(), q, idx, norms, pos, group, b, s, scores=sv)
    torch.cuda.synchronize()
    assert axr.axr_device_status() == 0
    assert intact(ibuf, 0x6B) and intact(nbuf, -11.0) and intact(sbuf, -13.0)
    # slots after pos were never written
    assert torch.all(idx[:, pos + 1:] == 0x6B) and torch.all(norms[:, pos + 1:] == -11.0)
    assert torch.isfinite(sv).all()


@pytest.mark.parametrize("d,b,group,n,vdtype", [
    (128, 4, 4, 5000, torch.bfloat16), (32, 2, 3, 77, torch.float32), (256, 2, 2, 1000, torch.float16),
    (512, 3, 8, 300, torch.bfloat16),
])
@pytest.mark.parametrize("static", [False, True])
def test_attention_outputs_stay_inside(d, b, group, n, vdtype, static):
    heads = 2
    packed, norms = workloads.make_random_packed(heads, n, d, b, seed=d + n, device=DEV)
    q = torch.randn((heads * group, d), device=DEV)
    s = workloads.make_signs(workloads.GQA_DECODE_128K.with_(d=d)).to(DEV)
    V = torch.randn((heads, n, d), device=DEV).to(vdtype)
    sbuf, sv = guarded(heads * group * n, torch.float32, -17.0)
    obuf, ov = guarded(heads * group * d, torch.float32, -19.0)
    scores, out = sv.view(heads * group, n), ov.view(heads * group, d)
    if static:
        axr.axr_attention_static(q, packed, norms, V, group, b, s, scores, out)
        wbuf = None
    else:
        need = axr.axr_attention_workspace_bytes(n, heads, group, d)
        wbuf, wv = guarded(need, torch.uint8, 0x2D)
        axr.axr_attention(q, packed, norms, V, group, b, s, scores=scores, workspace=wv, out=out)
    torch.cuda.synchronize()
    assert axr.axr_device_status() == 0
    assert intact(sbuf, -17.0) and intact(obuf, -19.0)
    assert wbuf is None or intact(wbuf, 0x2D)
    assert torch.isfinite(out).all()


@pytest.mark.parametrize("d,b,G,n,C", [(128, 4, 4, 300, 6), (8, 1, 1, 50, 4), (512, 3, 2, 40, 3)])
def test_sign_choice_outputs_stay_inside(d, b, G, n, C):
    S, H = 2, 3
    wl = workloads.GQA_SIGN_CALIBRATION.with_(batch=S, kv_heads=H, group=G, d=d, b=b, T=n, dtype="bf16", seed=d)
    K = workloads.make_keys(wl).reshape(S, H, n, d).to(DEV)
    q = workloads.make_queries(wl).reshape(S, H * G, d).to(DEV)
    cand = workloads.make_sign_candidates(wl, C).to(DEV)
    ebuf, ev = guarded(C * H, torch.float32, -23.0)
    bbuf, bv = guarded(1, torch.int32, -29)
    axr.axr_select_signs(K, q, G, b, cand, errors=ev.view(C, H), best=bv)
    torch.cuda.synchronize()
    assert intact(ebuf, -23.0) and intact(bbuf, -29)
    assert 0 <= int(bv.item()) < C and torch.isfinite(ev).all()
