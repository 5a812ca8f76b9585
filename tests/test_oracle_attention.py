"""Pins for the fp64 forward oracle (CPU only): a hand-worked example, closed
forms, special cases and a library cross-check."""
import math

import numpy as np
import pytest
import torch

from conftest import load_golden
from oracle import attention as A


def _hand_inputs():
    g = load_golden("attention_hand.txt")
    N, hq, hkv = 3, 4, 2
    q = np.zeros((N, hq, 1))
    for h in range(hq):
        q[:, h, 0] = g["q_heads"][h]
    k = np.zeros((N, hkv, 1))
    v = np.zeros((N, hkv, 1))
    k[:, 0, 0], v[:, 0, 0] = g["k_head0"], g["v_head0"]
    k[:, 1, 0], v[:, 1, 0] = g["k_head1"], g["v_head1"]
    return g, q, k, v


def test_hand_worked_example():
    g, q, k, v = _hand_inputs()
    O, L = A.causal_attention(q, k, v)
    for h in range(4):
        np.testing.assert_allclose(O[:, h, 0], g[f"O_head{h}"], rtol=0, atol=1e-12)
        np.testing.assert_allclose(L[:, h], g[f"LSE_head{h}"], rtol=0, atol=1e-12)


def test_hand_worked_example_rows():
    g, q, k, v = _hand_inputs()
    O, L = A.attention_rows(q[[2, 0]], k, v, [2, 0])
    np.testing.assert_allclose(O[0, 1, 0], g["O_head1"][2], atol=1e-12)
    np.testing.assert_allclose(L[1, 3], g["LSE_head3"][0], atol=1e-12)


def test_single_visible_key():
    rng = np.random.default_rng(1)
    q, k, v = rng.standard_normal((3, 8, 2, 16)).astype(np.float64)
    O, L = A.causal_attention(q, k, v)
    np.testing.assert_array_equal(O[0], v[0])  # row 0 sees only key 0
    s00 = (q[0] * k[0]).sum(-1) / 4.0
    np.testing.assert_allclose(L[0], s00, atol=1e-15)


def test_equal_scores_give_prefix_mean():
    rng = np.random.default_rng(2)
    N, d = 50, 8
    q = rng.standard_normal((N, 2, d))
    k = np.tile(rng.standard_normal((1, 1, d)), (N, 1, 1))  # all keys equal
    v = rng.standard_normal((N, 1, d))
    O, L = A.causal_attention(q, k, v, block=16)
    for i in range(N):
        for h in range(2):
            np.testing.assert_allclose(O[i, h], v[: i + 1, 0].mean(0), atol=1e-12)
            s = float(q[i, h] @ k[0, 0]) / math.sqrt(d)
            np.testing.assert_allclose(L[i, h], s + math.log(i + 1), atol=1e-12)


def test_softmax_rows_sum_to_one():
    rng = np.random.default_rng(3)
    N, d = 40, 8
    q = rng.standard_normal((N, 1, d)) * 3
    k = rng.standard_normal((N, 1, d)) * 3
    v = np.ones((N, 1, d))
    O, L = A.causal_attention(q, k, v)
    # with v = 1 the output is the row sum of the softmax weights
    np.testing.assert_allclose(O, 1.0, atol=1e-12)


@pytest.mark.parametrize("N,hq,hkv,d", [(37, 4, 4, 16), (96, 6, 2, 8), (130, 7, 1, 32)])
def test_matches_torch_sdpa_fp64(N, hq, hkv, d):
    """Library cross-check: torch scaled_dot_product_attention(is_causal) in
    fp64 on CPU, with kv heads repeated in contiguous groups."""
    g = torch.Generator().manual_seed(N)
    q = torch.randn(N, hq, d, generator=g, dtype=torch.float64)
    k = torch.randn(N, hkv, d, generator=g, dtype=torch.float64) * 2
    v = torch.randn(N, hkv, d, generator=g, dtype=torch.float64)
    O, L = A.causal_attention(q.numpy(), k.numpy(), v.numpy(), block=32)
    G = hq // hkv
    kr = k.repeat_interleave(G, dim=1)
    vr = v.repeat_interleave(G, dim=1)
    ref = torch.nn.functional.scaled_dot_product_attention(
        q.transpose(0, 1), kr.transpose(0, 1), vr.transpose(0, 1), is_causal=True)
    np.testing.assert_allclose(O, ref.transpose(0, 1).numpy(), atol=1e-12)
    # LSE against torch.logsumexp over the masked score matrix
    s = torch.einsum("ihd,jhd->hij", q, kr) / math.sqrt(d)
    mask = torch.ones(N, N, dtype=torch.bool).tril()
    lse = torch.logsumexp(s.masked_fill(~mask, float("-inf")), dim=-1).T
    np.testing.assert_allclose(L, lse.numpy(), atol=1e-12)


def test_rows_equal_full():
    rng = np.random.default_rng(5)
    N = 300
    q = rng.standard_normal((N, 4, 16))
    k = rng.standard_normal((N, 2, 16))
    v = rng.standard_normal((N, 2, 16))
    O, L = A.causal_attention(q, k, v, block=64)
    rows = np.array([0, 1, 63, 64, 150, 299])
    Or, Lr = A.attention_rows(q[rows], k, v, rows, block=4)
    np.testing.assert_allclose(Or, O[rows], atol=1e-12)
    np.testing.assert_allclose(Lr, L[rows], atol=1e-12)


def test_gqa_mapping_is_contiguous_groups():
    assert [A.kv_head(h, 28, 4) for h in range(28)] == [h // 7 for h in range(28)]
    assert [A.kv_head(h, 4, 4) for h in range(4)] == [0, 1, 2, 3]


def _doc_start(lengths):
    out = []
    pos = 0
    for L in lengths:
        out += [pos] * L
        pos += L
    return np.asarray(out, np.int64)


def test_document_starts_by_hand():
    """Worked by hand from the definition (first position of each token's
    document)."""
    np.testing.assert_array_equal(A.document_starts([3, 1, 2]), [0, 0, 0, 3, 4, 4])
    np.testing.assert_array_equal(A.document_starts([1, 1, 1]), [0, 1, 2])
    np.testing.assert_array_equal(A.document_starts([5]), [0] * 5)
    assert A.document_starts([]).size == 0
    with pytest.raises(ValueError):
        A.document_starts([2, 0, 1])
    np.testing.assert_array_equal(A.document_starts([7, 1, 30]), _doc_start([7, 1, 30]))


def test_document_mask_equals_separate_documents():
    """Packed sequence with attention reset at document boundaries = plain
    causal attention of each document on its own (brute force)."""
    rng = np.random.default_rng(12)
    lengths = [7, 1, 30, 12, 50]
    N = sum(lengths)
    q = rng.standard_normal((N, 4, 8))
    k = rng.standard_normal((N, 2, 8)) * 2
    v = rng.standard_normal((N, 2, 8))
    ds = _doc_start(lengths)
    O, L = A.causal_attention(q, k, v, block=16, doc_start=ds)
    pos = 0
    for Ln in lengths:
        sl = slice(pos, pos + Ln)
        Od, Ld = A.causal_attention(q[sl], k[sl], v[sl])
        np.testing.assert_allclose(O[sl], Od, atol=1e-12)
        np.testing.assert_allclose(L[sl], Ld, atol=1e-12)
        pos += Ln
    # sampled rows agree with the whole-sequence version
    rows = np.array([0, 6, 7, 8, 37, 38, 99])
    Or, Lr = A.attention_rows(q[rows], k, v, rows, block=3, doc_start=ds)
    np.testing.assert_allclose(Or, O[rows], atol=1e-12)
    np.testing.assert_allclose(Lr, L[rows], atol=1e-12)


def test_single_document_is_plain_causal():
    rng = np.random.default_rng(13)
    q, k, v = rng.standard_normal((3, 40, 2, 8))
    O, L = A.causal_attention(q, k, v, doc_start=np.zeros(40, np.int64))
    O2, L2 = A.causal_attention(q, k, v)
    np.testing.assert_array_equal(O, O2)
    np.testing.assert_array_equal(L, L2)
