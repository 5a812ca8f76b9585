"""Pins of the frame-aligned, modality-balanced encoder shard oracle
(oracle/frames.py): a hand-worked table (tests/golden/frames_hand.txt), and
the properties the reading fixes, checked directly on the maps: a
permutation; every frame whole, on one rank, in consecutive rows in order;
every rank's visual tokens within one frame of the even share V/P (so whole
576-token frames per rank differ by at most one) and text tokens balanced
to within one; sequence order kept inside each rank; the re-shard map equals
the encoder map composed with the zigzag map. A planted mistake (splitting
frames token by token) is caught."""
import os

import numpy as np
import pytest

import mmsp_inputs as mi
from oracle import frames as F
from oracle import sharder

GOLDEN = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden", "frames_hand.txt")


def _golden():
    vals = {}
    for line in open(GOLDEN):
        if line.startswith("#") or ":" not in line:
            continue
        k, v = line.split(":", 1)
        vals[k.strip()] = [int(x) for x in v.split()]
    return vals


def test_hand_worked_table():
    g = _golden()
    enc, counts = F.frame_plan(g["seg_len"], g["seg_kind"], g["P"][0])
    assert enc.tolist() == g["global2enc"]
    assert counts.reshape(-1).tolist() == g["enc_counts"]


def _check_properties(seg_len, seg_kind, P, enc, counts):
    seg_len = np.asarray(seg_len)
    seg_kind = np.asarray(seg_kind)
    N = int(seg_len.sum())
    assert sorted(enc.tolist()) == list(range(N)), "not a permutation"
    kinds = np.repeat(seg_kind, seg_len)
    ends = np.cumsum(counts.sum(1))
    rank_of_row = np.searchsorted(ends, enc, side="right")
    starts = np.concatenate([[0], np.cumsum(seg_len)[:-1]])
    frame_lens = [int(L) for L, k in zip(seg_len, seg_kind) if k == 1]
    for s0, L, k in zip(starts, seg_len, seg_kind):
        rows = enc[s0:s0 + L]
        if k == 1:   # a frame: one rank, consecutive rows, in order
            assert len(set(rank_of_row[s0:s0 + L].tolist())) == 1
            assert np.array_equal(rows, rows[0] + np.arange(L))
    for e in range(P):
        mine = np.nonzero(rank_of_row == e)[0]           # global tokens of rank e, ascending
        r = enc[mine]
        vis = mine[kinds[mine] == 1]
        txt = mine[kinds[mine] == 0]
        assert counts[e, 0] == len(vis) and counts[e, 1] == len(txt)
        # rows: visual tokens first, each group in sequence order
        assert np.array_equal(np.sort(r), np.concatenate([enc[vis], enc[txt]]))
        assert np.all(np.diff(enc[vis]) == 1) and np.all(np.diff(enc[txt]) == 1)
    if frame_lens:
        # a rank starts at the first frame at or after its share e*V/P, so
        # its visual tokens are within one (longest) frame of V/P
        V = sum(frame_lens)
        assert (np.abs(counts[:, 0] - V / P) < max(frame_lens)).all()
    assert counts[:, 1].max() - counts[:, 1].min() <= 1


@pytest.mark.parametrize("seed,N,P", [(1, 600, 3), (2, 2048, 8), (3, 4096, 4), (4, 1200, 6), (5, 4096, 1)])
def test_properties_on_random_tables(seed, N, P):
    seg_len, seg_kind = mi.random_segments(N, seed)
    enc, counts = F.frame_plan(seg_len, seg_kind, P)
    _check_properties(seg_len, seg_kind, P, enc, counts)


def test_properties_on_the_workload_layouts():
    for name in ("n4k", "n32k"):
        w = mi.WORKLOADS[name]
        seg_len, seg_kind = mi.workload_layout(w)
        enc, counts = F.frame_plan(seg_len, seg_kind, w.P)
        _check_properties(seg_len, seg_kind, w.P, enc, counts)
        # 576-token frames: whole frames per rank differ by at most one
        assert (counts[:, 0] % mi.FRAME_TOKENS == 0).all()
        assert counts[:, 0].max() - counts[:, 0].min() <= mi.FRAME_TOKENS


def test_reshard_map_composes_with_the_zigzag_map():
    seg_len, seg_kind = mi.random_segments(1200, 9)
    out = F.shard_frames(seg_len, seg_kind, 1200, 3)
    l2g = sharder.shard_maps(seg_len, seg_kind, 1200, 3)["local2global"]
    for l in range(1200):
        assert out["local2enc"][l] == out["global2enc"][l2g[l]]


def test_only_text_or_only_frames():
    enc, counts = F.frame_plan([10], [0], 4)
    assert enc.tolist() == list(range(10)) and counts[:, 0].tolist() == [0] * 4
    enc, counts = F.frame_plan([4, 4, 4, 4], [1, 1, 1, 1], 2)
    assert enc.tolist() == list(range(16)) and counts[:, 1].tolist() == [0, 0]


def test_planted_mistake_splitting_frames_is_caught():
    """Assigning visual tokens one by one (floor(P * v / V) per token) splits
    a frame across ranks; the frame check must fail."""
    g = _golden()
    seg_len, seg_kind, P = g["seg_len"], g["seg_kind"], g["P"][0]
    kinds = np.repeat(seg_kind, seg_len)
    V, T = int((kinds == 1).sum()), int((kinds == 0).sum())
    owner = np.zeros(len(kinds), int)
    owner[kinds == 1] = (P * np.arange(V)) // V
    owner[kinds == 0] = (P * np.arange(T)) // T
    counts = np.array([[(owner[kinds == 1] == e).sum(), (owner[kinds == 0] == e).sum()] for e in range(P)])
    base = np.concatenate([[0], np.cumsum(counts.sum(1))[:-1]])
    enc = np.zeros(len(kinds), int)
    nv, nt = base.copy(), base + counts[:, 0]
    for t in range(len(kinds)):
        e = owner[t]
        if kinds[t] == 1:
            enc[t] = nv[e]; nv[e] += 1
        else:
            enc[t] = nt[e]; nt[e] += 1
    with pytest.raises(AssertionError):
        _check_properties(seg_len, seg_kind, P, enc, counts)
