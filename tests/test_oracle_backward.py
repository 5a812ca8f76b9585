"""Pins for the fp64 backward oracle (CPU only): finite differences, a
library autograd cross-check and closed-form gradient sums."""
import math

import numpy as np
import pytest
import torch

from oracle import attention as A


def _inputs(N, hq, hkv, d, seed):
    rng = np.random.default_rng(seed)
    q = rng.standard_normal((N, hq, d))
    k = rng.standard_normal((N, hkv, d)) * 1.5
    v = rng.standard_normal((N, hkv, d))
    do = rng.standard_normal((N, hq, d))
    return q, k, v, do


def test_finite_differences():
    """L = sum(dO * O): central differences in fp64 at N <= 64, d = 8."""
    N, hq, hkv, d = 12, 4, 2, 8
    q, k, v, do = _inputs(N, hq, hkv, d, 7)
    g = A.causal_attention_bwd(q, k, v, do)

    def loss(q_, k_, v_):
        O, _ = A.causal_attention(q_, k_, v_)
        return float((O * do).sum())

    eps = 1e-6
    rng = np.random.default_rng(0)
    for name, x, grad in [("q", q, g["dQ"]), ("k", k, g["dK"]), ("v", v, g["dV"])]:
        for _ in range(12):
            idx = tuple(int(rng.integers(0, s)) for s in x.shape)
            xp, xm = x.copy(), x.copy()
            xp[idx] += eps
            xm[idx] -= eps
            args_p = {"q": (xp, k, v), "k": (q, xp, v), "v": (q, k, xp)}[name]
            args_m = {"q": (xm, k, v), "k": (q, xm, v), "v": (q, k, xm)}[name]
            fd = (loss(*args_p) - loss(*args_m)) / (2 * eps)
            assert abs(fd - grad[idx]) < 1e-6, (name, idx, fd, grad[idx])


@pytest.mark.parametrize("N,hq,hkv,d", [(40, 4, 4, 8), (77, 6, 2, 16)])
def test_matches_torch_autograd_fp64(N, hq, hkv, d):
    q, k, v, do = _inputs(N, hq, hkv, d, N)
    g = A.causal_attention_bwd(q, k, v, do, block=16)
    tq, tk, tv = (torch.tensor(x, requires_grad=True) for x in (q, k, v))
    G = hq // hkv
    out = torch.nn.functional.scaled_dot_product_attention(
        tq.transpose(0, 1), tk.repeat_interleave(G, 1).transpose(0, 1),
        tv.repeat_interleave(G, 1).transpose(0, 1), is_causal=True).transpose(0, 1)
    out.backward(torch.tensor(do))
    np.testing.assert_allclose(g["O"], out.detach().numpy(), atol=1e-12)
    np.testing.assert_allclose(g["dQ"], tq.grad.numpy(), atol=1e-11)
    np.testing.assert_allclose(g["dK"], tk.grad.numpy(), atol=1e-11)
    np.testing.assert_allclose(g["dV"], tv.grad.numpy(), atol=1e-11)


def test_closed_form_gradient_sums():
    """sum_j dV_j (per kv head) = sum_i sum_{h in group} dO_i,h and
    sum_j dK_j = 0, because each row of dS sums to zero."""
    N, hq, hkv, d = 64, 6, 2, 8
    q, k, v, do = _inputs(N, hq, hkv, d, 11)
    g = A.causal_attention_bwd(q, k, v, do, block=16)
    G = hq // hkv
    for kh in range(hkv):
        np.testing.assert_allclose(g["dV"][:, kh].sum(0),
                                   do[:, kh * G:(kh + 1) * G].sum((0, 1)), atol=1e-10)
        np.testing.assert_allclose(g["dK"][:, kh].sum(0), 0.0, atol=1e-10)


def test_rows_and_keys_variants_equal_full():
    N, hq, hkv, d = 90, 4, 2, 8
    q, k, v, do = _inputs(N, hq, hkv, d, 3)
    g = A.causal_attention_bwd(q, k, v, do, block=32)
    rows = np.array([0, 5, 44, 89])
    r = A.attention_bwd_rows(q[rows], k, v, do[rows], rows, block=2)
    np.testing.assert_allclose(r["dQ"], g["dQ"][rows], atol=1e-12)
    np.testing.assert_allclose(r["LSE"], g["LSE"][rows], atol=1e-12)
    keys = np.array([60, 61, 75, 89])
    kk = A.attention_bwd_keys(q[60:], k, v, do[60:], keys, block=7)
    np.testing.assert_allclose(kk["dK"], g["dK"][keys], atol=1e-12)
    np.testing.assert_allclose(kk["dV"], g["dV"][keys], atol=1e-12)


def test_document_mask_backward_equals_separate_documents():
    lengths = [9, 20, 1, 14]
    N = sum(lengths)
    q, k, v, do = _inputs(N, 4, 2, 8, 21)
    ds = np.concatenate([[sum(lengths[:i])] * L for i, L in enumerate(lengths)]).astype(np.int64)
    g = A.causal_attention_bwd(q, k, v, do, block=8, doc_start=ds)
    pos = 0
    for L in lengths:
        sl = slice(pos, pos + L)
        gd = A.causal_attention_bwd(q[sl], k[sl], v[sl], do[sl])
        for name in ("O", "dQ", "dK", "dV"):
            np.testing.assert_allclose(g[name][sl], gd[name], atol=1e-12)
        pos += L


def test_document_sampled_helpers_agree_with_whole_backward():
    """attention_bwd_rows / attention_bwd_keys with documents equal the
    whole-sequence backward (itself pinned to per-document attention)."""
    lengths = [30, 5, 1, 40, 24]
    N = sum(lengths)
    q, k, v, do = _inputs(N, 4, 2, 8, 23)
    ds = A.document_starts(lengths)
    g = A.causal_attention_bwd(q, k, v, do, block=16, doc_start=ds)
    rows = np.array([0, 29, 30, 35, 36, 50, 99])
    r = A.attention_bwd_rows(q[rows], k, v, do[rows], rows, block=3, doc_start=ds)
    np.testing.assert_allclose(r["dQ"], g["dQ"][rows], atol=1e-12)
    np.testing.assert_allclose(r["O"], g["O"][rows], atol=1e-12)
    np.testing.assert_allclose(r["LSE"], g["LSE"][rows], atol=1e-12)
    keys = np.array([70, 75, 76, 99])
    kk = A.attention_bwd_keys(q[70:], k, v, do[70:], keys, block=9, doc_start=ds)
    np.testing.assert_allclose(kk["dK"], g["dK"][keys], atol=1e-12)
    np.testing.assert_allclose(kk["dV"], g["dV"][keys], atol=1e-12)


@pytest.mark.parametrize("lengths,hq,hkv,d", [([9, 20, 1, 14], 4, 2, 8), ([1, 1, 40, 3, 19], 6, 3, 16)])
def test_document_mask_matches_torch_sdpa_autograd_fp64(lengths, hq, hkv, d):
    """Library cross-check of the document-masked forward and backward:
    torch scaled_dot_product_attention with an explicit boolean mask
    (doc_start[i] <= j <= i) and autograd, in fp64 on CPU."""
    N = sum(lengths)
    q, k, v, do = _inputs(N, hq, hkv, d, 31 + N)
    ds = A.document_starts(lengths)
    g = A.causal_attention_bwd(q, k, v, do, block=8, doc_start=ds)
    tq, tk, tv = (torch.tensor(x, requires_grad=True) for x in (q, k, v))
    G = hq // hkv
    i = torch.arange(N)[:, None]
    j = torch.arange(N)[None, :]
    mask = (j <= i) & (j >= torch.as_tensor(ds)[:, None])
    out = torch.nn.functional.scaled_dot_product_attention(
        tq.transpose(0, 1), tk.repeat_interleave(G, 1).transpose(0, 1),
        tv.repeat_interleave(G, 1).transpose(0, 1), attn_mask=mask).transpose(0, 1)
    out.backward(torch.tensor(do))
    np.testing.assert_allclose(g["O"], out.detach().numpy(), atol=1e-12)
    np.testing.assert_allclose(g["dQ"], tq.grad.numpy(), atol=1e-11)
    np.testing.assert_allclose(g["dK"], tk.grad.numpy(), atol=1e-11)
    np.testing.assert_allclose(g["dV"], tv.grad.numpy(), atol=1e-11)
