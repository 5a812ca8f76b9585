"""Document-masked (packed) causal attention on the GPU (C ABI) against the
fp64 oracle: mmsp_doc_starts bit-exact, forward and backward with documents
that do not line up with tiles or chunks, the degenerate layouts (one
document, one token per document), accumulation over ring-step ranges, and a
sampled check on a 64K-token packed buffer of videos."""
import math

import numpy as np
import pytest
import torch

import mmsp_inputs as mi
from oracle import attention as A
from gpu_util import (compare_attention, compare_grad, lib, needs_gpu, run_backward, run_forward, shard_rows)

pytestmark = [pytest.mark.gpu, needs_gpu]


def _doc_start_dev(doc_len, N):
    m = lib()
    ds = torch.full((max(N, 1),), -7, dtype=torch.int32, device="cuda")
    m.mmsp_doc_starts(doc_len, N, ds)
    torch.cuda.synchronize()
    return ds[:N]


def _tensors(N, hq, hkv, d, seed, doc_len=None, seg=None, with_dout=False):
    if seg is None:
        seg = mi.random_segments(N, seed + 17)
    vis = mi.token_kinds(*seg) == mi.VISUAL
    q, k, v, do = mi.make_tensors(N, hq, hkv, d, seed, vis, device="cuda", with_dout=with_dout)
    return q, k, v, do


def _cpu(*xs):
    return [x.float().cpu().numpy() for x in xs]


@pytest.mark.parametrize("N,seed,max_len", [(1, 1, 5), (777, 2, 40), (4096, 3, 700), (20000, 4, 3000)])
def test_doc_starts_bit_exact(N, seed, max_len):
    doc_len = mi.random_segments(N, seed, max_len=max_len)[0]
    got = _doc_start_dev(doc_len, N).cpu().numpy()
    np.testing.assert_array_equal(got, A.document_starts(doc_len))


def test_doc_starts_rejects_bad_tables():
    m = lib()
    ds = torch.zeros(16, dtype=torch.int32, device="cuda")
    for bad in ([4, 4, 4], [8, 0, 8], [17]):
        with pytest.raises(m.MmspError) as e:
            m.mmsp_doc_starts(bad, 16, ds)
        assert e.value.status == 1
    with pytest.raises(m.MmspError):
        m.mmsp_doc_starts(np.ones(m.MMSP_MAX_SEGMENTS + 1, np.int32), m.MMSP_MAX_SEGMENTS + 1,
                          torch.zeros(m.MMSP_MAX_SEGMENTS + 1, dtype=torch.int32, device="cuda"))
    m.mmsp_doc_starts([], 0, ds)  # N = 0: nothing to do


def test_doc_start_needs_causal():
    m = lib()
    N, P, H, d = 256, 2, 2, 64
    x = torch.zeros((N, H, d), dtype=torch.bfloat16, device="cuda")
    ds = torch.zeros(N, dtype=torch.int32, device="cuda")
    lse = torch.zeros((N, H), device="cuda")
    with pytest.raises(m.MmspError) as e:
        m.mmsp_attn_fwd(x, x, x, N, P, H, H, d, 0.125, 0, 0, P, None, lse, None, 0, doc_start=ds)
    assert e.value.status == 1


FWD_CASES = [
    # N, P, Hq, Hkv, d, document layout
    (1200, 3, 4, 2, 128, "random:300"),   # C = 200, many boundaries inside tiles
    (2048, 4, 2, 1, 64, "random:9"),      # many tiny documents (several per tile)
    (4608, 2, 2, 2, 128, "videos"),       # C = 1152, video documents of 576-token frames
    (144, 2, 7, 1, 128, "random:20"),     # C = 36: chunk shorter than a tile
    (3000, 5, 4, 4, 64, "random:1100"),   # documents spanning several chunks
]


def _layout(kind, N, seed):
    if kind == "videos":
        doc_len, sl, sk = mi.packed_documents(N, seed, max_frames=3, text_max=200)
        return doc_len, (sl, sk)
    mx = int(kind.split(":")[1])
    return mi.random_segments(N, seed + 5, max_len=mx)[0], None


@pytest.mark.parametrize("N,P,hq,hkv,d,kind", FWD_CASES)
def test_forward_documents_match_oracle(N, P, hq, hkv, d, kind):
    seed = 11 * N + P
    doc_len, seg = _layout(kind, N, seed)
    q, k, v, _ = _tensors(N, hq, hkv, d, seed, seg=seg)
    ds = _doc_start_dev(doc_len, N)
    ql, kl, vl = (shard_rows(x, N, P) for x in (q, k, v))
    o_acc, lse, o_out = run_forward(ql, kl, vl, P, doc_start=ds)
    o = shard_rows(o_acc, N, P, inverse=True).cpu().numpy()
    l = shard_rows(lse, N, P, inverse=True).cpu().numpy()
    O, L = A.causal_attention(*_cpu(q, k, v), doc_start=A.document_starts(doc_len))
    compare_attention(o, l, O, L, f"doc fwd N={N} P={P} {kind}")


def test_forward_documents_accumulate_over_step_ranges():
    """Ring steps [0, 2) then [2, P) with MMSP_ACCUMULATE equal the oracle."""
    m = lib()
    N, P, hq, hkv, d = 2400, 4, 4, 2, 128
    doc_len = mi.random_segments(N, 91, max_len=500)[0]
    q, k, v, _ = _tensors(N, hq, hkv, d, 91)
    ds = _doc_start_dev(doc_len, N)
    ql, kl, vl = (shard_rows(x, N, P) for x in (q, k, v))
    o_acc, lse, _ = run_forward(ql, kl, vl, P, step_begin=0, step_end=2, flags=0, doc_start=ds)
    o_acc, lse, _ = run_forward(ql, kl, vl, P, step_begin=2, step_end=P, flags=m.MMSP_ACCUMULATE,
                                o_acc=o_acc, lse=lse, doc_start=ds)
    o = shard_rows(o_acc, N, P, inverse=True).cpu().numpy()
    l = shard_rows(lse, N, P, inverse=True).cpu().numpy()
    O, L = A.causal_attention(*_cpu(q, k, v), doc_start=A.document_starts(doc_len))
    compare_attention(o, l, O, L, "doc fwd accumulate")


def test_one_document_matches_the_plain_path():
    """doc_start all zero selects the document kernels but masks nothing. The
    document forward raises the running max only past a 2^8 margin and
    corrects the dominant term of O; the plain forward raises it at every
    increase. So the two forwards differ only by the bf16 rounding of P: both
    match the oracle, and their LSEs agree to 1e-5. Given the same forward
    outputs, the document backward is bit-identical to the plain backward."""
    N, P, hq, hkv, d = 2560, 4, 4, 2, 128
    q, k, v, do = _tensors(N, hq, hkv, d, 5, with_dout=True)
    ds = _doc_start_dev([N], N)
    ql, kl, vl, dol = (shard_rows(x, N, P) for x in (q, k, v, do))
    a = run_forward(ql, kl, vl, P)
    b = run_forward(ql, kl, vl, P, doc_start=ds)
    back = lambda x: shard_rows(x, N, P, inverse=True).float().cpu().numpy()
    o_ref, lse_ref = A.causal_attention(*_cpu(q, k, v))
    compare_attention(back(a[0]), back(a[1]), o_ref, lse_ref, "plain path")
    compare_attention(back(b[0]), back(b[1]), o_ref, lse_ref, "one document")
    assert float((a[1] - b[1]).abs().max()) <= 1e-5
    ga = run_backward(ql, kl, vl, a[2], dol, a[1], P, fp32_dq=True)
    gb = run_backward(ql, kl, vl, a[2], dol, a[1], P, fp32_dq=True, doc_start=ds)
    for x, y in zip(ga, gb):
        assert torch.equal(x, y)


def test_one_token_per_document_closed_form():
    """Every token its own document: P = 1 on the diagonal only, so O = v
    (up to the fp32 rounding of the row max inside exp2), LSE = scale * q.k,
    dV = sum of dO over the kv group, dQ = dK = 0 up to the rounding of D
    against dP."""
    N, P, hq, hkv, d = 1024, 2, 4, 2, 128
    q, k, v, do = _tensors(N, hq, hkv, d, 8, with_dout=True)
    ds = _doc_start_dev(np.ones(N, np.int32), N)
    ql, kl, vl, dol = (shard_rows(x, N, P) for x in (q, k, v, do))
    o_acc, lse, o_out = run_forward(ql, kl, vl, P, doc_start=ds)
    back = lambda x: shard_rows(x, N, P, inverse=True)
    g = hq // hkv
    vrep = v.float().repeat_interleave(g, dim=1)
    assert ((back(o_acc) - vrep).abs() <= 2 ** -20 * vrep.abs()).all()
    s = (q.float() * k.float().repeat_interleave(g, dim=1)).sum(-1) / math.sqrt(d)
    assert (back(lse) - s).abs().max().item() < 1e-3
    dq, dk, dv, _ = run_backward(ql, kl, vl, o_out, dol, lse, P, doc_start=ds)
    dv_ref = do.float().view(N, hkv, g, d).sum(2)
    assert (back(dv).float() - dv_ref).abs().max().item() <= 2 ** -7 * dv_ref.abs().max().item()
    assert back(dq).float().abs().max().item() < 2e-2
    assert back(dk).float().abs().max().item() < 2e-2


BWD_CASES = [
    (1200, 3, 4, 2, "random:300"),
    (2048, 4, 2, 1, "random:9"),
    (4608, 2, 2, 2, "videos"),
    (144, 2, 7, 1, "random:20"),
    (3000, 5, 4, 4, "random:1100"),
]


@pytest.mark.parametrize("N,P,hq,hkv,kind", BWD_CASES)
def test_backward_documents_match_oracle(N, P, hq, hkv, kind):
    d = 128
    seed = 13 * N + P
    doc_len, seg = _layout(kind, N, seed)
    q, k, v, do = _tensors(N, hq, hkv, d, seed, seg=seg, with_dout=True)
    ds = _doc_start_dev(doc_len, N)
    ql, kl, vl, dol = (shard_rows(x, N, P) for x in (q, k, v, do))
    o_acc, lse, o_out = run_forward(ql, kl, vl, P, doc_start=ds)
    dq, dk, dv, dq32 = run_backward(ql, kl, vl, o_out, dol, lse, P, fp32_dq=True, doc_start=ds)
    back = lambda x: shard_rows(x, N, P, inverse=True).float().cpu().numpy()
    ref = A.causal_attention_bwd(*_cpu(q, k, v, do), doc_start=A.document_starts(doc_len))
    compare_attention(back(o_acc), back(lse), ref["O"], ref["LSE"], "doc fwd")
    compare_grad(back(dq), ref["dQ"], f"doc dQ N={N}")
    compare_grad(back(dq32), ref["dQ"], f"doc dQ32 N={N}")
    compare_grad(back(dk), ref["dK"], f"doc dK N={N}")
    compare_grad(back(dv), ref["dV"], f"doc dV N={N}")


def test_packed_videos_64k_sampled():
    """A 65,536-token buffer of packed videos (P = 8, Hq = 28, Hkv = 4, d =
    128): sampled O/LSE and dQ rows, and dK/dV of the last keys, against the
    oracle with the same document starts."""
    N, P, hq, hkv, d = 65536, 8, 28, 4, 128
    doc_len, sl, sk = mi.packed_documents(N, 44)
    q, k, v, do = _tensors(N, hq, hkv, d, 44, seg=(sl, sk), with_dout=True)
    ds = _doc_start_dev(doc_len, N)
    ds_host = A.document_starts(doc_len)
    np.testing.assert_array_equal(ds.cpu().numpy(), ds_host)
    ql, kl, vl, dol = (shard_rows(x, N, P) for x in (q, k, v, do))
    o_acc, lse, o_out = run_forward(ql, kl, vl, P, doc_start=ds)
    dq, dk, dv, _ = run_backward(ql, kl, vl, o_out, dol, lse, P, doc_start=ds)
    back = lambda x: shard_rows(x, N, P, inverse=True)
    C = N // (2 * P)
    rows = mi.sample_rows(N, C, 96, seed=45)
    starts = np.cumsum(np.concatenate([[0], doc_len[:-1]]))
    rows = np.unique(np.concatenate([rows, starts[1:9], starts[1:9] - 1]))
    qc, kc, vc, doc = _cpu(q, k, v, do)
    r = A.attention_bwd_rows(qc[rows], kc, vc, doc[rows], rows, doc_start=ds_host)
    compare_attention(back(o_acc)[rows].cpu().numpy(), back(lse)[rows].cpu().numpy(), r["O"], r["LSE"],
                      "64k doc rows")
    compare_grad(back(dq)[rows].float().cpu().numpy(), r["dQ"], "64k doc dQ rows")
    keys = np.arange(N - 300, N, 7)
    j0 = int(keys.min())
    kk = A.attention_bwd_keys(qc[j0:], kc, vc, doc[j0:], keys, doc_start=ds_host)
    compare_grad(back(dk)[keys].float().cpu().numpy(), kk["dK"], "64k doc dK keys")
    compare_grad(back(dv)[keys].float().cpu().numpy(), kk["dV"], "64k doc dV keys")
