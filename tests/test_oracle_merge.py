"""Pins for the oracle's log-sum-exp merge and ring simulation (CPU only)."""
import numpy as np
import pytest

from conftest import load_golden
from oracle import attention as A
from oracle import merge as M

NINF = -np.inf


def test_hand_worked_merge():
    g = load_golden("merge_hand.txt")
    o, l = M.lse_merge(np.array(g["o_a"]), np.array(g["lse_a"][0]),
                       np.array(g["o_b"]), np.array(g["lse_b"][0]))
    np.testing.assert_allclose(o, g["o_out"], atol=1e-14)
    np.testing.assert_allclose(l, g["lse_out"][0], atol=1e-14)


def test_empty_partial_is_identity_and_both_empty_is_empty():
    rng = np.random.default_rng(0)
    o = rng.standard_normal((5, 8))
    l = rng.standard_normal(5)
    z = np.zeros((5, 8))
    e = np.full(5, NINF)
    for args in [(o, l, z, e), (z, e, o, l)]:
        oo, ll = M.lse_merge(*args)
        np.testing.assert_array_equal(oo, o)
        np.testing.assert_array_equal(ll, l)
    oo, ll = M.lse_merge(z, e, z, e)
    assert np.all(oo == 0) and np.all(ll == NINF) and not np.any(np.isnan(oo))


def test_commutative_and_associative():
    rng = np.random.default_rng(1)
    parts = [(rng.standard_normal((7, 16)), rng.standard_normal(7) * 5) for _ in range(3)]
    (a, la), (b, lb), (c, lc) = parts
    o1, l1 = M.lse_merge(a, la, b, lb)
    o2, l2 = M.lse_merge(b, lb, a, la)
    np.testing.assert_allclose(o1, o2, atol=1e-12)
    np.testing.assert_allclose(l1, l2, atol=1e-12)
    x, lx = M.lse_merge(*M.lse_merge(a, la, b, lb), c, lc)
    y, ly = M.lse_merge(a, la, *M.lse_merge(b, lb, c, lc))
    np.testing.assert_allclose(x, y, atol=1e-12)
    np.testing.assert_allclose(lx, ly, atol=1e-12)


def test_merge_of_disjoint_blocks_equals_attention_over_union():
    """LSE(union) = logaddexp(LSE_a, LSE_b) (numpy's routine) and the merged
    output equals the definition over the union of the two key sets."""
    rng = np.random.default_rng(2)
    R, J, d = 9, 30, 8
    q = rng.standard_normal((R, d))
    k = rng.standard_normal((J, d)) * 2
    v = rng.standard_normal((J, d))
    qpos = np.full(R, J)  # every key visible
    kpos = np.arange(J)
    perm = rng.permutation(J)
    ia, ib = np.sort(perm[:11]), np.sort(perm[11:])
    oa, la = M.block_attention(q, qpos, k[ia], v[ia], kpos[ia], 0.25)
    ob, lb = M.block_attention(q, qpos, k[ib], v[ib], kpos[ib], 0.25)
    o, l = M.lse_merge(oa, la, ob, lb)
    np.testing.assert_allclose(l, np.logaddexp(la, lb), atol=1e-12)
    s = q @ k.T * 0.25
    w = np.exp(s - s.max(1, keepdims=True))
    np.testing.assert_allclose(o, (w / w.sum(1, keepdims=True)) @ v, atol=1e-12)


@pytest.mark.parametrize("N,P", [(8, 1), (8, 2), (8, 4), (24, 3), (24, 6), (24, 12),
                                 (64, 4), (96, 16)])
def test_ring_equals_unsharded_attention(N, P):
    """Brute force: the ring over P virtual ranks, merged, equals the plain
    definition of causal attention."""
    rng = np.random.default_rng(N * 100 + P)
    q = rng.standard_normal((N, 4, 8))
    k = rng.standard_normal((N, 2, 8)) * 2
    v = rng.standard_normal((N, 2, 8))
    O, L, pairs = M.ring_attention(q, k, v, P)
    Or, Lr = A.causal_attention(q, k, v)
    np.testing.assert_allclose(O, Or, atol=1e-12)
    np.testing.assert_allclose(L, Lr, atol=1e-12)


@pytest.mark.parametrize("N,P", [(24, 3), (64, 4), (96, 8)])
def test_ring_steps_have_two_full_blocks_after_step_zero(N, P):
    """Per step s >= 1 each rank sees exactly two full C x C blocks (2C^2
    visible pairs); step 0 sees one full and two diagonal blocks."""
    C = N // (2 * P)
    rng = np.random.default_rng(0)
    q = rng.standard_normal((N, 1, 4))
    _, _, pairs = M.ring_attention(q, q, q, P)
    assert np.all(pairs[:, 0] == C * C + C * (C + 1))
    if P > 1:
        assert np.all(pairs[:, 1:] == 2 * C * C)
    assert np.all(pairs.sum(axis=1) == C * (2 * P * C + 1))


def test_ring_step_partials_merge_to_full_and_follow_ring_order():
    """The per-step partials merged over all steps equal the definition, and
    step s gives rank r exactly the keys of rank (r - s) mod P."""
    N, P = 48, 4
    C = N // (2 * P)
    rng = np.random.default_rng(9)
    q = rng.standard_normal((N, 2, 8))
    k = rng.standard_normal((N, 1, 8))
    v = rng.standard_normal((N, 1, 8))
    Ol, Ll = None, None
    for s in range(P):
        o, l = M.ring_step_partials(q, k, v, P, s)
        if Ol is None:
            Ol, Ll = o, l
        else:
            Ol, Ll = M.lse_merge(Ol, Ll, o, l)
        # rank 1 at step 1 holds rank 0's K/V (chunks 0 and 2P-1); its chunk-0
        # queries (global chunk 1) see all of chunk 0 and nothing of chunk 2P-1
        if s == 1:
            r = 1
            rows = slice(r * 2 * C, r * 2 * C + C)
            g0 = np.arange(0, C)
            ref_o, ref_l = M.block_attention(q[C:2 * C, 0], np.arange(C, 2 * C), k[g0, 0], v[g0, 0], g0,
                                             1 / np.sqrt(8))
            np.testing.assert_allclose(o[rows, 0], ref_o, atol=1e-12)
            np.testing.assert_allclose(l[rows, 0], ref_l, atol=1e-12)
    from oracle import sharder
    l2g = sharder.shard_maps([N], [0], N, P)["local2global"]
    Og = sharder.permute_rows(Ol, l2g, inverse=True)
    Or, Lr = A.causal_attention(q, k, v)
    np.testing.assert_allclose(Og, Or, atol=1e-12)
