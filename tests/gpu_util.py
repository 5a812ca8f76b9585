"""Shared helpers for the GPU parity tests: seeded inputs, the CUDA path
through the C ABI, and the comparison bars."""
import math

import numpy as np
import pytest
import torch

import mmsp_inputs as mi

needs_gpu = pytest.mark.skipif(not torch.cuda.is_available(), reason="needs a CUDA GPU")

# Bars (attention): fp32 O within max-abs 1e-2 and mean-abs 1e-3 of the fp64
# oracle, LSE within 1e-3 absolute; bf16 O within 1 bf16 ulp of RNE(fp32 O).
O_MAX_ABS = 1e-2
O_MEAN_ABS = 1e-3
LSE_MAX_ABS = 1e-3


def lib():
    import long_context_multimodal_b200 as m

    return m


def shard_rows(x, N, P, inverse=False):
    """Permute the rows of a [N, ...] CUDA tensor through mmsp_shard."""
    m = lib()
    out = torch.empty_like(x)
    row_bytes = x.numel() // N * x.element_size() if N else 16
    m.mmsp_shard(None, None, N, P, src=x, dst=out, row_bytes=row_bytes, inverse=inverse)
    return out


def run_forward(q, k, v, P, causal=1, step_begin=0, step_end=None, flags=None, scale=None,
                o_acc=None, lse=None, doc_start=None):
    """q, k, v: rank-local CUDA bf16 [N, H, d]. Returns (o_acc fp32, lse, o_out bf16)."""
    m = lib()
    N, hq, d = q.shape
    hkv = k.shape[1]
    if step_end is None:
        step_end = P
    if flags is None:
        flags = m.MMSP_FINALIZE
    if scale is None:
        scale = 1.0 / math.sqrt(d)
    if o_acc is None:
        o_acc = torch.full((N, hq, d), float("nan"), device=q.device, dtype=torch.float32)
    if lse is None:
        lse = torch.full((N, hq), float("nan"), device=q.device, dtype=torch.float32)
    o_out = torch.full((N, hq, d), float("nan"), device=q.device, dtype=torch.bfloat16)
    m.mmsp_attn_fwd(q, k, v, N, P, hq, hkv, d, scale, causal, step_begin, step_end, o_acc, lse,
                    o_out if flags & m.MMSP_FINALIZE else None, flags, doc_start=doc_start)
    m.mmsp_device_status()
    return o_acc, lse, o_out


def inputs(N, hq, hkv, d, seed, seg=None, with_dout=False):
    """Seeded global-order inputs on the GPU plus the segment table."""
    if seg is None:
        seg = mi.random_segments(N, seed + 17)
    vis = mi.token_kinds(*seg) == mi.VISUAL
    q, k, v, do = mi.make_tensors(N, hq, hkv, d, seed, vis, device="cuda", with_dout=with_dout)
    return seg, q, k, v, do


def compare_attention(o, lse, o_ref, lse_ref, what=""):
    o = np.asarray(o, np.float64)
    lse = np.asarray(lse, np.float64)
    err = np.abs(o - o_ref)
    lerr = np.abs(lse - lse_ref)
    assert np.isfinite(o).all() and np.isfinite(lse).all(), what + ": non-finite output"
    assert err.max() <= O_MAX_ABS, f"{what}: O max-abs {err.max():.3e}"
    assert err.mean() <= O_MEAN_ABS, f"{what}: O mean-abs {err.mean():.3e}"
    assert lerr.max() <= LSE_MAX_ABS, f"{what}: LSE max-abs {lerr.max():.3e}"
    return float(err.max()), float(err.mean()), float(lerr.max())


def check_bf16_rounding(o_out, o_acc):
    """bf16 output = round-to-nearest-even of the fp32 output (1 ulp slack)."""
    ref = o_acc.to(torch.bfloat16)
    a = o_out.view(torch.int16).to(torch.int32)
    b = ref.view(torch.int16).to(torch.int32)
    assert int((a - b).abs().max()) <= 1


# Gradient bars (a reading; none is stated for the backward): per tensor,
# max|g - g_ref| / max(1, max|g_ref|) <= 1e-2 and mean|g - g_ref| / mean|g_ref|
# <= 1e-2, on the fp32/bf16 outputs against the fp64 oracle.
G_MAX_REL = 1e-2
G_MEAN_REL = 1e-2


def compare_grad(g, g_ref, what):
    g = np.asarray(g, np.float64)
    g_ref = np.asarray(g_ref, np.float64)
    assert np.isfinite(g).all(), what + ": non-finite"
    err = np.abs(g - g_ref)
    mx = err.max() / max(1.0, np.abs(g_ref).max())
    mn = err.mean() / max(np.abs(g_ref).mean(), 1e-30)
    assert mx <= G_MAX_REL, f"{what}: max rel {mx:.3e}"
    assert mn <= G_MEAN_REL, f"{what}: mean rel {mn:.3e}"
    return float(mx), float(mn)


def run_backward(ql, kl, vl, o_out, dol, lse, P, causal=1, fp32_dq=False, doc_start=None):
    """Rank-local inputs; returns (dq bf16, dk bf16, dv bf16, dq fp32 or None)."""
    m = lib()
    N, hq, d = ql.shape
    hkv = kl.shape[1]
    ws_bytes = m.mmsp_bwd_workspace_bytes(N, P, hq, d)
    ws = torch.empty(ws_bytes, dtype=torch.uint8, device=ql.device)
    dq = torch.full_like(ql, float("nan"))
    dk = torch.full_like(kl, float("nan"))
    dv = torch.full_like(vl, float("nan"))
    dq32 = torch.full((N, hq, d), float("nan"), device=ql.device) if fp32_dq else None
    m.mmsp_attn_bwd(ql, kl, vl, o_out, dol, lse, N, P, hq, hkv, d, 1.0 / math.sqrt(d), causal, dq, dk, dv, dq32,
                    ws, ws_bytes, doc_start=doc_start)
    m.mmsp_device_status()
    return dq, dk, dv, dq32
