"""Log-sum-exp merge and a ring simulation over P virtual ranks (oracle; test
infrastructure only).

The merge replaces the combine in "LongVILA Guide" (aifetchly), section
"Implementation", ``LongVILAMultiModalAttention.forward``: that sketch adds
softmax(block) @ V of every ring step into one accumulator, i.e. it sums
blocks that were each normalised on their own, which is not attention over
the union of the blocks. The reading taken: each step yields (O_s, LSE_s),
normalised over that step's visible keys, and two such partial results over
disjoint key sets combine as

    m   = max(LSE_a, LSE_b)
    LSE = m + ln(exp(LSE_a - m) + exp(LSE_b - m))
    O   = exp(LSE_a - LSE) O_a + exp(LSE_b - LSE) O_b

with (O, LSE) = (0, -inf) when both inputs are empty.

The ring order follows the same page: ``LongVILAParallelContext`` (section
"Identify Ring Neighbors") gives each rank a previous and a next ring rank,
and the ring loop sends the current K/V block to the next rank and receives
the following one from the previous rank, P steps in all (Ring-SP paragraph
of section "MM-SP Mechanics": P-1 shifts). So at step s rank r holds the
K/V block that rank (r - s) mod P started with.
"""
from __future__ import annotations

import math

import numpy as np

from . import sharder

NEG_INF = -np.inf


def lse_merge(o_a, lse_a, o_b, lse_b):
    """Merge two partial results. o_*: [..., d], lse_*: [...] (fp64)."""
    o_a = np.asarray(o_a, np.float64)
    o_b = np.asarray(o_b, np.float64)
    lse_a = np.asarray(lse_a, np.float64)
    lse_b = np.asarray(lse_b, np.float64)
    m = np.maximum(lse_a, lse_b)
    empty = m == NEG_INF
    m_safe = np.where(empty, 0.0, m)
    with np.errstate(divide="ignore"):
        lse = m_safe + np.log(np.exp(lse_a - m_safe) + np.exp(lse_b - m_safe))
    lse = np.where(empty, NEG_INF, lse)
    lse_safe = np.where(empty, 0.0, lse)
    wa = np.where(empty, 0.0, np.exp(lse_a - lse_safe))
    wb = np.where(empty, 0.0, np.exp(lse_b - lse_safe))
    o = wa[..., None] * o_a + wb[..., None] * o_b
    return o, lse


def block_attention(qb, qpos, kb, vb, kpos, scale):
    """Attention of query rows (one head) over one K/V block, normalised over
    that block's visible keys only (kpos <= qpos). Empty rows: (0, -inf)."""
    s = (qb @ kb.T) * scale
    visible = kpos[None, :] <= qpos[:, None]
    s = np.where(visible, s, NEG_INF)
    m = s.max(axis=1) if s.shape[1] > 0 else np.full(len(qpos), NEG_INF)
    empty = m == NEG_INF
    m_safe = np.where(empty, 0.0, m)
    with np.errstate(divide="ignore"):
        lse = m_safe + np.log(np.exp(s - m_safe[:, None]).sum(axis=1))
    lse = np.where(empty, NEG_INF, lse)
    p = np.exp(s - np.where(empty, 0.0, lse)[:, None])
    p = np.where(visible, p, 0.0)
    return p @ vb, lse


def ring_attention(q, k, v, P: int, scale=None):
    """Simulate the ring over P virtual ranks on zigzag shards and merge the
    per-step partials with ``lse_merge``. Returns (O, LSE) in global order,
    plus the per-rank, per-step count of visible (q, k) pairs (for balance
    checks) as an int array [P, P]."""
    q = np.asarray(q, np.float64)
    k = np.asarray(k, np.float64)
    v = np.asarray(v, np.float64)
    N, hq, d = q.shape
    hkv = k.shape[1]
    if scale is None:
        scale = 1.0 / math.sqrt(d)
    maps = sharder.shard_maps([N], [0], N, P)
    l2g = maps["local2global"]
    C2 = N // P
    ql = sharder.permute_rows(q, l2g)
    kl = sharder.permute_rows(k, l2g)
    vl = sharder.permute_rows(v, l2g)
    pos = l2g.astype(np.int64)

    O = np.zeros((P, C2, hq, d))
    L = np.full((P, C2, hq), NEG_INF)
    pairs = np.zeros((P, P), np.int64)
    # each rank starts with its own K/V block
    cur = [(kl[r * C2:(r + 1) * C2], vl[r * C2:(r + 1) * C2], pos[r * C2:(r + 1) * C2])
           for r in range(P)]
    for step in range(P):
        for r in range(P):
            kb, vb, kpos = cur[r]
            qpos = pos[r * C2:(r + 1) * C2]
            pairs[r, step] = int((kpos[None, :] <= qpos[:, None]).sum())
            for h in range(hq):
                kh = (h * hkv) // hq
                ob, lb = block_attention(ql[r * C2:(r + 1) * C2, h], qpos,
                                         kb[:, kh], vb[:, kh], kpos, scale)
                O[r, :, h], L[r, :, h] = lse_merge(O[r, :, h], L[r, :, h], ob, lb)
        # receive from the previous ring rank
        cur = [cur[(r - 1) % P] for r in range(P)]
    Og = sharder.permute_rows(O.reshape(N, hq, d), l2g, inverse=True)
    Lg = sharder.permute_rows(L.reshape(N, hq), l2g, inverse=True)
    return Og, Lg, pairs


def ring_step_partials(q, k, v, P: int, step: int, scale=None):
    """Partial (O, LSE) of every virtual rank at one ring step, in rank-local
    order [N, Hq, d] / [N, Hq]: rank r's queries against the K/V block it
    holds after `step` receives from its previous ring rank."""
    q = np.asarray(q, np.float64)
    k = np.asarray(k, np.float64)
    v = np.asarray(v, np.float64)
    N, hq, d = q.shape
    hkv = k.shape[1]
    if scale is None:
        scale = 1.0 / math.sqrt(d)
    maps = sharder.shard_maps([N], [0], N, P)
    l2g = maps["local2global"]
    C2 = N // P
    ql = sharder.permute_rows(q, l2g)
    kl = sharder.permute_rows(k, l2g)
    vl = sharder.permute_rows(v, l2g)
    pos = l2g.astype(np.int64)
    cur = [(kl[r * C2:(r + 1) * C2], vl[r * C2:(r + 1) * C2], pos[r * C2:(r + 1) * C2]) for r in range(P)]
    for _ in range(step):
        cur = [cur[(r - 1) % P] for r in range(P)]
    O = np.zeros((N, hq, d))
    L = np.full((N, hq), NEG_INF)
    for r in range(P):
        kb, vb, kpos = cur[r]
        sl = slice(r * C2, (r + 1) * C2)
        for h in range(hq):
            kh = (h * hkv) // hq
            O[sl, h], L[sl, h] = block_attention(ql[sl, h], pos[sl], kb[:, kh], vb[:, kh], kpos, scale)
    return O, L
