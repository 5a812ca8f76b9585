"""Backward of the ring attention on the GPU (C ABI) against the fp64
oracle: whole gradients at small sizes (ragged chunks, GQA ratios, one
rank, non-causal) and the stages called separately. The full workload sizes
are in test_gpu_full_size.py."""
import math

import pytest
import torch

from oracle import attention as A
from gpu_util import (compare_attention, compare_grad, inputs, lib, needs_gpu, run_backward, run_forward,
                      shard_rows)

pytestmark = [pytest.mark.gpu, needs_gpu]


def _fwd_bwd(q, k, v, do, P, causal=1, fp32_dq=False):
    N = q.shape[0]
    ql, kl, vl, dol = (shard_rows(x, N, P) for x in (q, k, v, do))
    o_acc, lse, o_out = run_forward(ql, kl, vl, P, causal=causal)
    dq, dk, dv, dq32 = run_backward(ql, kl, vl, o_out, dol, lse, P, causal=causal, fp32_dq=fp32_dq)
    back = lambda x: shard_rows(x, N, P, inverse=True)
    out = {"O": back(o_acc), "LSE": back(lse), "dQ": back(dq), "dK": back(dk), "dV": back(dv)}
    if dq32 is not None:
        out["dQ32"] = back(dq32)
    return out


CASES = [
    # N, P, Hq, Hkv
    (1024, 2, 2, 1),
    (1200, 3, 4, 2),   # C = 200: ragged key and query tiles
    (600, 1, 2, 2),    # one rank
    (144, 2, 7, 1),    # C = 36: chunk shorter than a tile
    (2048, 8, 28, 4),  # C = 128, GQA 7:1
    (2560, 4, 3, 1),   # C = 320
]


@pytest.mark.parametrize("N,P,hq,hkv", CASES)
def test_backward_matches_oracle_whole_gradients(N, P, hq, hkv):
    d = 128
    _, q, k, v, do = inputs(N, hq, hkv, d, seed=3 * N + P, with_dout=True)
    out = _fwd_bwd(q, k, v, do, P, fp32_dq=True)
    ref = A.causal_attention_bwd(*(x.float().cpu().numpy() for x in (q, k, v, do)))
    compare_attention(out["O"].cpu().numpy(), out["LSE"].cpu().numpy(), ref["O"], ref["LSE"], "fwd")
    for name in ("dQ", "dK", "dV"):
        compare_grad(out[name].float().cpu().numpy(), ref[name], f"{name} N={N} P={P}")
    compare_grad(out["dQ32"].cpu().numpy(), ref["dQ"], "dQ fp32")
    # bf16 dQ is the RNE rounding of the fp32 accumulator
    assert torch.equal(out["dQ"].view(torch.int16), out["dQ32"].to(torch.bfloat16).view(torch.int16))


def test_backward_non_causal():
    N, P, hq, hkv, d = 512, 2, 2, 1, 128
    _, q, k, v, do = inputs(N, hq, hkv, d, seed=77, with_dout=True)
    out = _fwd_bwd(q, k, v, do, P, causal=0)
    tq, tk, tv = (x.double().cpu().requires_grad_(True) for x in (q, k, v))
    G = hq // hkv
    o = torch.nn.functional.scaled_dot_product_attention(
        tq.transpose(0, 1), tk.repeat_interleave(G, 1).transpose(0, 1),
        tv.repeat_interleave(G, 1).transpose(0, 1)).transpose(0, 1)
    o.backward(do.double().cpu())
    for name, ref in (("dQ", tq.grad), ("dK", tk.grad), ("dV", tv.grad)):
        compare_grad(out[name].float().cpu().numpy(), ref.numpy(), name + " non-causal")


def test_backward_stages_match_the_single_call():
    """prepare + dQ + dK/dV called separately (dQ first) give what
    mmsp_attn_bwd gives."""
    m = lib()
    N, P, hq, hkv, d = 1200, 3, 4, 2, 128
    _, q, k, v, do = inputs(N, hq, hkv, d, seed=5, with_dout=True)
    ql, kl, vl, dol = (shard_rows(x, N, P) for x in (q, k, v, do))
    _, lse, o = run_forward(ql, kl, vl, P)
    dq, dk, dv, _ = run_backward(ql, kl, vl, o, dol, lse, P)
    wsb = m.mmsp_bwd_workspace_bytes(N, P, hq, d)
    ws = torch.empty(wsb, dtype=torch.uint8, device="cuda")
    dq2, dk2, dv2 = (torch.full_like(x, float("nan")) for x in (ql, kl, vl))
    sc = 1 / math.sqrt(d)
    m.mmsp_attn_bwd_prepare(o, dol, lse, N, P, hq, d, ws, wsb)
    m.mmsp_attn_bwd_dq(ql, kl, vl, dol, N, P, hq, hkv, d, sc, 1, dq2, None, ws, wsb)
    m.mmsp_attn_bwd_dkdv(ql, kl, vl, dol, N, P, hq, hkv, d, sc, 1, dk2, dv2, ws, wsb)
    m.mmsp_device_status()
    for a, b in ((dq, dq2), (dk, dk2), (dv, dv2)):
        assert torch.equal(a.view(torch.int16), b.view(torch.int16))
