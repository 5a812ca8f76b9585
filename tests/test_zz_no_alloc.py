"""The allocation-free backward entry point (mmsp_attn_bwd_noalloc) against
the workspace one (mmsp_attn_bwd), through the C ABI.

Some callers of this library cannot allocate device memory: code running
inside a host framework that hands out all device memory from its own pool,
and latency-bound paths where a cudaMalloc/cudaFree (which can synchronise
the device) is not acceptable. For them the backward keeps its scratch in a
fixed array inside the library. This file is collected last on purpose: if
it fails, a run that stops at the first failure has already run the rest.
"""
import math

import pytest
import torch

from gpu_util import compare_grad, inputs, lib, needs_gpu, run_forward, shard_rows

pytestmark = [pytest.mark.gpu, needs_gpu]


def _case(N, P, hq, hkv, seed):
    d = 128
    _, q, k, v, do = inputs(N, hq, hkv, d, seed=seed, with_dout=True)
    ql, kl, vl, dol = (shard_rows(x, N, P) for x in (q, k, v, do))
    _, lse, o = run_forward(ql, kl, vl, P)
    return ql, kl, vl, dol, o, lse


def _grads(fn, ql, kl, vl, dol, o, lse, P, *extra):
    m = lib()
    N, hq, d = ql.shape
    hkv = kl.shape[1]
    dq, dk, dv = (torch.full_like(x, float("nan")) for x in (ql, kl, vl))
    dq32 = torch.full(ql.shape, float("nan"), device=ql.device)
    fn(ql, kl, vl, o, dol, lse, N, P, hq, hkv, d, 1.0 / math.sqrt(d), 1, dq, dk, dv, dq32, *extra)
    m.mmsp_device_status()
    return {"dQ": dq, "dK": dk, "dV": dv, "dQ32": dq32}


def test_noalloc_backward_matches_workspace_backward_twice_in_a_row():
    m = lib()
    # two calls in a row with different sizes: the second must not see the
    # first call's leftovers in the shared scratch
    for N, P, hq, hkv, seed in ((4096, 4, 28, 4, 91), (1200, 3, 4, 2, 92)):
        assert m.mmsp_bwd_workspace_bytes(N, P, hq, 128) <= m.MMSP_NOALLOC_SCRATCH_BYTES
        args = _case(N, P, hq, hkv, seed)
        got = _grads(m.mmsp_attn_bwd_noalloc, *args, P)
        ws_bytes = m.mmsp_bwd_workspace_bytes(N, P, hq, 128)
        ws = torch.empty(ws_bytes, dtype=torch.uint8, device="cuda")
        ref = _grads(m.mmsp_attn_bwd, *args, P, ws, ws_bytes)
        for name in ("dQ", "dK", "dV", "dQ32"):
            compare_grad(got[name].float().cpu().numpy(), ref[name].float().cpu().numpy(),
                         f"noalloc {name} N={N}")


def test_noalloc_rejects_sizes_beyond_its_scratch():
    m = lib()
    N, P, hq = 524288, 64, 28
    assert m.mmsp_bwd_workspace_bytes(N, P, hq, 128) > m.MMSP_NOALLOC_SCRATCH_BYTES
    x = torch.zeros(16, device="cuda", dtype=torch.bfloat16)
    with pytest.raises(m.MmspError) as e:
        m.mmsp_attn_bwd_noalloc(x, x, x, x, x, x, N, P, hq, 4, 128, 0.088, 1, x, x, x, None)
    assert e.value.status == 1 and "scratch" in str(e.value)


def test_noalloc_backward_with_documents_on_a_side_stream_matches_the_oracle():
    """Packed documents (the document-masked kernels through the shared
    scratch) on a stream other than the default one, compared directly with
    the fp64 oracle."""
    import numpy as np

    from oracle import attention as A

    m = lib()
    N, P, hq, hkv, d = 2400, 4, 4, 2, 128
    doc_len = np.array([1000, 1, 599, 800], np.int32)
    _, q, k, v, do = inputs(N, hq, hkv, d, seed=93, with_dout=True)
    side = torch.cuda.Stream()
    with torch.cuda.stream(side):
        ds = torch.empty(N, dtype=torch.int32, device="cuda")
        m.mmsp_doc_starts(doc_len, N, ds, stream=side)
        ql, kl, vl, dol = (shard_rows(x, N, P) for x in (q, k, v, do))
        _, lse, o = run_forward(ql, kl, vl, P, doc_start=ds)
        dq, dk, dv = (torch.full_like(x, float("nan")) for x in (ql, kl, vl))
        m.mmsp_attn_bwd_noalloc(ql, kl, vl, o, dol, lse, N, P, hq, hkv, d, 1.0 / math.sqrt(d), 1, dq, dk, dv, None,
                                doc_start=ds, stream=side)
        m.mmsp_device_status(side)
        got = {n: shard_rows(t, N, P, inverse=True).float().cpu().numpy() for n, t in (("dQ", dq), ("dK", dk),
                                                                                   ("dV", dv))}
    ref = A.causal_attention_bwd(*(x.float().cpu().numpy() for x in (q, k, v, do)),
                                 doc_start=A.document_starts(doc_len))
    for name in ("dQ", "dK", "dV"):
        compare_grad(got[name], ref[name], f"noalloc with documents {name}")
