"""Pins for the oracle sharder and the input layout generator (CPU only)."""
import numpy as np
import pytest

from conftest import load_golden
from oracle import sharder
import mmsp_inputs as mi


def _ints(x):
    return np.asarray(x, dtype=np.int64)


def test_hand_worked_case_a():
    g = load_golden("zigzag_small.txt")
    N, P = int(g["A_N"][0]), int(g["A_P"][0])
    m = sharder.shard_maps([N], [0], N, P)
    assert np.array_equal(m["local2global"], _ints(g["A_local2global"]))
    assert np.array_equal(m["global2local"], _ints(g["A_global2local"]))


def test_hand_worked_case_b_with_segments():
    g = load_golden("zigzag_small.txt")
    N, P = int(g["B_N"][0]), int(g["B_P"][0])
    m = sharder.shard_maps(_ints(g["B_seg_len"]), _ints(g["B_seg_kind"]), N, P)
    assert np.array_equal(m["local2global"], _ints(g["B_local2global"]))
    assert np.array_equal(m["global2local"], _ints(g["B_global2local"]))
    assert np.array_equal(m["modality_local"], _ints(g["B_modality_local"]))
    assert np.array_equal(m["segid_local"], _ints(g["B_segid_local"]))
    assert np.array_equal(m["rank_counts"].reshape(-1), _ints(g["B_rank_counts"]))


@pytest.mark.parametrize("N,P", [(16, 1), (16, 2), (48, 4), (60, 5), (256, 8), (1024, 16)])
def test_every_token_exactly_once(N, P):
    sl, sk = mi.random_segments(N, seed=N + P, max_len=37)
    m = sharder.shard_maps(sl, sk, N, P)
    l2g = m["local2global"].astype(np.int64)
    # a permutation: every global position appears once
    assert np.array_equal(np.sort(l2g), np.arange(N))
    # the inverse composes to identity both ways
    g2l = m["global2local"].astype(np.int64)
    assert np.array_equal(g2l[l2g], np.arange(N))
    assert np.array_equal(l2g[g2l], np.arange(N))
    # per-rank counts cover all tokens; totals agree with the layout
    rc = m["rank_counts"]
    assert rc.sum() == N
    assert np.all(rc.sum(axis=1) == N // P)
    kinds = mi.token_kinds(sl, sk)
    assert rc[:, 1].sum() == int((kinds == 1).sum())
    # modality of each local slot is the kind of its global token
    assert np.array_equal(m["modality_local"], kinds[l2g])


def test_zigzag_balance_closed_form():
    """Each rank's visible causal pairs = C(2PC+1); total N(N+1)/2 (derived
    from the zigzag reading: chunks r and 2P-1-r together see 2P-1 full
    chunks plus two diagonal chunks)."""
    for N, P in [(64, 4), (96, 3), (200, 5), (512, 8)]:
        C = N // (2 * P)
        m = sharder.shard_maps([N], [0], N, P)
        pos = m["local2global"].astype(np.int64).reshape(P, 2 * C)
        per_rank = []
        for r in range(P):
            q = pos[r]
            per_rank.append(int(sum(int(x) + 1 for x in q)))  # row i sees i+1 keys
        assert all(x == C * (2 * P * C + 1) for x in per_rank)
        assert sum(per_rank) == N * (N + 1) // 2


def test_rejects_bad_sizes():
    with pytest.raises(ValueError):
        sharder.shard_maps([10], [0], 10, 3)
    with pytest.raises(ValueError):
        sharder.shard_maps([5, 4], [0, 1], 8, 2)


def test_permute_rows_roundtrip():
    N, P = 40, 4
    x = np.arange(N * 3).reshape(N, 3)
    m = sharder.shard_maps([N], [0], N, P)
    y = sharder.permute_rows(x, m["local2global"])
    assert np.array_equal(y[:, 0] // 3, m["local2global"])
    assert np.array_equal(sharder.permute_rows(y, m["local2global"], inverse=True), x)


def test_layout_frame_tokens_match_pages():
    # "LongVILA Guide", section "Problem", item 1: 3,600 frames at 576 tokens
    # per frame give 2,073,600 visual tokens.
    sl, sk = mi.make_layout(3600, 0, 0, seed=0)
    assert int(sl.sum()) == 2073600 and np.all(sk == mi.VISUAL)


@pytest.mark.parametrize("name", list(mi.WORKLOADS))
def test_workload_layouts(name):
    w = mi.WORKLOADS[name]
    sl, sk = mi.workload_layout(w)
    assert int(sl.sum()) == w.N
    assert w.N % (2 * w.P) == 0
    assert int((sk == mi.VISUAL).sum()) == w.frames
    assert int((sk == mi.TEXT).sum()) == w.text_segments
    assert int(sl[sk == mi.TEXT].sum()) == w.text_tokens
    assert np.all(sl >= 1)
    assert sk[0] == mi.TEXT  # the sequence opens with text


@pytest.mark.parametrize("N,seed", [(1000, 5), (4608, 3), (65536, 44), (7, 1)])
def test_packed_documents_recipe(N, seed):
    """The packed-video input recipe: documents of (prompt text, whole
    576-token frames, answer text), cut at N; the segment table covers the
    same tokens and only the last document may hold a partial frame."""
    doc_len, seg_len, seg_kind = mi.packed_documents(N, seed)
    assert int(doc_len.sum()) == N and int(seg_len.sum()) == N
    assert (doc_len >= 1).all() and (seg_len >= 1).all()
    kinds = mi.token_kinds(seg_len, seg_kind)
    starts = np.concatenate([[0], np.cumsum(doc_len)[:-1]])
    for i, (s0, L) in enumerate(zip(starts, doc_len)):
        k = kinds[s0:s0 + L]
        assert k[0] == mi.TEXT  # every document opens with its prompt
        if i < len(doc_len) - 1:
            # frames are whole inside complete documents
            vis = np.flatnonzero(np.diff(np.concatenate([[0], k.astype(np.int8), [0]])))
            runs = vis[1::2] - vis[0::2]
            assert (runs % mi.FRAME_TOKENS == 0).all()
