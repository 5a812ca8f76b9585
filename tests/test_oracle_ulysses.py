"""Pins of the Ulysses all-to-all oracle (oracle/ulysses.py) against what the
pages and the mathematics fix, independently of how the oracle is written:
where every element must land (traced by its coordinates), the inverse
property, the send/receive buffers against the collective, and the property
2-D MM-SP relies on -- attention of each rank's head group over the whole
sequence equals those heads of the full attention (GQA head groups
included)."""
import math

import numpy as np
import pytest

from oracle import attention as A
from oracle import ulysses as U


def _coded(P_u, S, H, d):
    """Rank i's [S, H, d] with every element encoding (rank, s, h, e)."""
    return [np.array([[[((i * 1000 + s) * 100 + h) * 10 + e for e in range(d)] for h in range(H)]
                      for s in range(S)], dtype=np.int64) for i in range(P_u)]


@pytest.mark.parametrize("P_u,S,H", [(1, 3, 4), (2, 5, 4), (4, 3, 8), (2, 1, 2), (4, 6, 28)])
def test_every_element_lands_where_the_transpose_puts_it(P_u, S, H):
    d = 3
    ys = U.seq_to_heads(_coded(P_u, S, H, d))
    hl = H // P_u
    for j, y in enumerate(ys):
        assert y.shape == (P_u * S, hl, d)
        for t in range(P_u * S):
            for hh in range(hl):
                for e in range(d):
                    # position t of the group's sequence is token t % S of rank t // S;
                    # local head hh of rank j is global head j * hl + hh
                    assert y[t, hh, e] == (((t // S) * 1000 + t % S) * 100 + j * hl + hh) * 10 + e


@pytest.mark.parametrize("P_u,S,H", [(1, 4, 2), (2, 7, 4), (4, 2, 8), (8, 3, 8)])
def test_inverse_all_to_all_returns_every_rank_its_input(P_u, S, H):
    xs = _coded(P_u, S, H, 2)
    back = U.heads_to_seq(U.seq_to_heads(xs))
    for a, b in zip(xs, back):
        assert np.array_equal(a, b)


def test_send_and_receive_buffers_implement_the_collective():
    """Block j of rank i's packed buffer arrives as block i at rank j
    (an all-to-all of equal blocks); the received blocks, read in order,
    are the forward result, and unpacking the inverse's received blocks
    gives the rank's tokens back."""
    P_u, S, H, d = 4, 5, 8, 3
    xs = _coded(P_u, S, H, d)
    sent = [U.pack(x, P_u) for x in xs]
    received = [np.stack([sent[i][j] for i in range(P_u)]) for j in range(P_u)]
    ys = U.seq_to_heads(xs)
    for j in range(P_u):
        assert np.array_equal(received[j].reshape(P_u * S, H // P_u, d), ys[j])
    # inverse: rank j sends its [P_u*S, Hl] as P_u sequence blocks; rank i
    # receives block i of every rank and unpacks
    back_recv = [np.stack([ys[j].reshape(P_u, S, H // P_u, d)[i] for j in range(P_u)]) for i in range(P_u)]
    for i in range(P_u):
        assert np.array_equal(U.unpack(back_recv[i], P_u), xs[i])
    for x in xs:
        assert np.array_equal(U.unpack(U.pack(x, P_u), P_u), x)


@pytest.mark.parametrize("P_u,hq,hkv", [(2, 4, 2), (4, 8, 4), (2, 28, 4), (4, 28, 4)])
def test_head_sharded_attention_equals_the_full_attention_heads(P_u, hq, hkv):
    """What Ulysses relies on: after the transpose every rank holds the whole
    sequence for H/P_u query heads and the matching Hkv/P_u kv heads, and
    its attention equals those heads of the full attention."""
    rng = np.random.default_rng(3)
    S, d = 12, 8
    N = P_u * S
    q, k, v = rng.normal(size=(N, hq, d)), rng.normal(size=(N, hkv, d)), rng.normal(size=(N, hkv, d))
    O, L = A.causal_attention(q, k, v)
    split = lambda x: [x[i * S:(i + 1) * S] for i in range(P_u)]
    qs, ks, vs = (U.seq_to_heads(split(x)) for x in (q, k, v))
    hl = hq // P_u
    for j in range(P_u):
        o, l = A.causal_attention(qs[j], ks[j], vs[j], scale=1 / math.sqrt(d))
        np.testing.assert_allclose(o, O[:, j * hl:(j + 1) * hl], atol=1e-12)
        np.testing.assert_allclose(l, L[:, j * hl:(j + 1) * hl], atol=1e-12)
    # and the inverse transpose puts every rank's output rows back
    outs = U.heads_to_seq([A.causal_attention(qs[j], ks[j], vs[j])[0] for j in range(P_u)])
    np.testing.assert_allclose(np.concatenate(outs), O, atol=1e-12)


def test_planted_mistakes_are_caught():
    """A transpose that interleaves heads (h -> h % P_u groups) instead of
    contiguous groups breaks GQA: the coordinate trace catches it."""
    P_u, S, H, d = 2, 3, 4, 1
    xs = _coded(P_u, S, H, d)
    wrong = [np.concatenate([x[:, j::P_u] for x in xs]) for j in range(P_u)]
    right = U.seq_to_heads(xs)
    assert not all(np.array_equal(a, b) for a, b in zip(wrong, right))
