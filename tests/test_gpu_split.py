"""The ring split across GPUs, run on one GPU: the calls each GPU of a split
ring makes for its range of virtual ranks (mmsp_attn_fwd and the backward
stages with rank_begin/rank_end) are issued one range after another on the
same buffers. Every output element is computed by exactly one range, with
the same work items as the whole-ring call, so the result must equal the
whole ring bit for bit and the fp64 oracle within the attention bars.
(Several GPUs are not available here; the exchange between them is tested
on CPU with gloo ranks in test_split_gloo.py.)"""
import math

import numpy as np
import pytest
import torch

from oracle import attention as A
from gpu_util import (compare_attention, compare_grad, inputs, lib, needs_gpu, run_backward, run_forward,
                      shard_rows)

pytestmark = [pytest.mark.gpu, needs_gpu]


def _same_bits(a, b, what):
    assert torch.equal(a.contiguous().view(torch.int16 if a.element_size() == 2 else torch.int32),
                       b.contiguous().view(torch.int16 if b.element_size() == 2 else torch.int32)), what


@pytest.mark.parametrize("N,P,hq,hkv,world,docs", [
    (2400, 4, 28, 4, 2, False),   # C = 300: ragged tiles
    (2048, 8, 4, 2, 4, False),    # C = 128
    (4096, 8, 7, 1, 8, False),    # one virtual rank per GPU
    (3000, 6, 4, 4, 3, True),     # packed documents
])
def test_ranges_one_after_another_equal_the_whole_ring(N, P, hq, hkv, world, docs):
    from long_context_multimodal_b200 import split

    m = lib()
    d = 128
    C = N // (2 * P)
    _, q, k, v, do = inputs(N, hq, hkv, d, seed=N + P, with_dout=True)
    ds = None
    ds_host = None
    if docs:
        doc_len = np.array([700, 1, 333, 966, 1000], np.int32)
        ds = torch.empty(N, dtype=torch.int32, device="cuda")
        m.mmsp_doc_starts(doc_len, N, ds)
        ds_host = A.document_starts(doc_len)
    ql, kl, vl, dol = (shard_rows(x, N, P) for x in (q, k, v, do))
    scale = 1.0 / math.sqrt(d)
    # whole ring
    o32, lse, o = run_forward(ql, kl, vl, P, doc_start=ds)
    dq, dk, dv, _ = run_backward(ql, kl, vl, o, dol, lse, P, doc_start=ds)
    # the ranges of a `world`-GPU split, one after another
    ranges = [split.owned_ranks(P, world, g, C) for g in range(world)]
    lse2 = torch.full_like(lse, float("nan"))
    o2 = torch.full_like(o, float("nan"))
    o32b = torch.full_like(o32, float("nan"))
    for rr in ranges:
        m.mmsp_attn_fwd(ql, kl, vl, N, P, hq, hkv, d, scale, 1, 0, P, o32b, lse2, o2, m.MMSP_FINALIZE,
                        doc_start=ds, rank_begin=rr.begin, rank_end=rr.end)
    m.mmsp_device_status()
    _same_bits(lse2, lse, "LSE")
    _same_bits(o2, o, "O bf16")
    _same_bits(o32b, o32, "O fp32")
    wsb = m.mmsp_bwd_workspace_bytes(N, P, hq, d)
    ws = torch.full((wsb,), 255, dtype=torch.uint8, device="cuda")
    dq2, dk2, dv2 = (torch.full_like(x, float("nan")) for x in (ql, kl, vl))
    for rr in ranges:
        m.mmsp_attn_bwd_prepare(o, dol, lse, N, P, hq, d, ws, wsb, rank_begin=rr.begin, rank_end=rr.end)
    for rr in reversed(ranges):
        m.mmsp_attn_bwd_dkdv(ql, kl, vl, dol, N, P, hq, hkv, d, scale, 1, dk2, dv2, ws, wsb, doc_start=ds,
                             rank_begin=rr.begin, rank_end=rr.end)
        m.mmsp_attn_bwd_dq(ql, kl, vl, dol, N, P, hq, hkv, d, scale, 1, dq2, None, ws, wsb, doc_start=ds,
                           rank_begin=rr.begin, rank_end=rr.end)
    m.mmsp_device_status()
    _same_bits(dq2, dq, "dQ")
    _same_bits(dk2, dk, "dK")
    _same_bits(dv2, dv, "dV")
    # and the oracle, in global order
    ref = A.causal_attention_bwd(q.float().cpu().numpy(), k.float().cpu().numpy(), v.float().cpu().numpy(),
                                 do.float().cpu().numpy(), doc_start=ds_host)
    og = shard_rows(o32b, N, P, inverse=True).cpu().numpy()
    lg = shard_rows(lse2, N, P, inverse=True).cpu().numpy()
    compare_attention(og, lg, ref["O"], ref["LSE"], f"split forward N={N} world={world}")
    for name, t in (("dQ", dq2), ("dK", dk2), ("dV", dv2)):
        g = shard_rows(t, N, P, inverse=True).float().cpu().numpy()
        compare_grad(g, ref[name], f"split {name} N={N} world={world}")
