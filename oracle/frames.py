"""Frame-aligned, modality-balanced encoder shard and its re-shard into the
zigzag attention layout (oracle; test infrastructure only).

Source: "LongVILA Guide" (aifetchly), section "Problem": modality-switching
boundaries leave one rank with pure text and another with dense visual
patches, and the ranks then stall in the collectives. Reading (the pages
give no algorithm): before attention, the per-token work that depends on
the modality (the vision tower and projector for frames, the embedding for
text) is spread so that every rank gets a contiguous block of WHOLE frames
holding its share of the visual tokens, and its share of the text tokens:

  * a frame (one visual segment of the table) is never split: frame f goes
    to encoder rank floor(P * V_f / V), V_f = visual tokens before frame f,
    V = all visual tokens (contiguous blocks; every rank's visual tokens
    within one frame of the even share V/P);
  * text token number t (counting text tokens only, in sequence order) goes
    to rank floor(P * t / T), T = all text tokens;
  * the encoder layout concatenates the ranks in order; rank e's block is
    its frames' tokens in sequence order followed by its text tokens in
    sequence order.

The maps: global2enc[g] = the encoder-layout row of global token g, and
local2enc[l] = global2enc[local2global[l]] (the row a zigzag rank-local
slot reads when the encoder's output is re-sharded for attention);
enc_counts[e] = (visual tokens, text tokens) of encoder rank e.

Plain loops over tokens and segments, easy to check by eye.
"""
from __future__ import annotations

import numpy as np

from . import sharder


def frame_plan(seg_len, seg_kind, P: int):
    """Per global token: (encoder rank, row in the encoder layout).
    Returns (global2enc [N] int32, enc_counts [P, 2] int32)."""
    seg_len = [int(x) for x in seg_len]
    seg_kind = [int(x) for x in seg_kind]
    V = sum(L for L, k in zip(seg_len, seg_kind) if k == 1)
    T = sum(L for L, k in zip(seg_len, seg_kind) if k == 0)
    # owner rank of every token
    owner = []
    kind_of = []
    v_before = 0
    t_index = 0
    for L, k in zip(seg_len, seg_kind):
        if k == 1:
            e = (P * v_before) // V
            for _ in range(L):
                owner.append(e)
                kind_of.append(1)
            v_before += L
        else:
            for _ in range(L):
                owner.append((P * t_index) // T)
                kind_of.append(0)
                t_index += 1
    N = len(owner)
    counts = [[0, 0] for _ in range(P)]
    for g in range(N):
        counts[owner[g]][0 if kind_of[g] == 1 else 1] += 1
    base = [0] * P
    for e in range(1, P):
        base[e] = base[e - 1] + counts[e - 1][0] + counts[e - 1][1]
    # rows: each rank's visual tokens in order, then its text tokens in order
    next_vis = [base[e] for e in range(P)]
    next_txt = [base[e] + counts[e][0] for e in range(P)]
    global2enc = [0] * N
    for g in range(N):
        e = owner[g]
        if kind_of[g] == 1:
            global2enc[g] = next_vis[e]
            next_vis[e] += 1
        else:
            global2enc[g] = next_txt[e]
            next_txt[e] += 1
    return np.asarray(global2enc, np.int32), np.asarray(counts, np.int32)


def shard_frames(seg_len, seg_kind, N: int, P: int):
    """All outputs of the frame shard: global2enc, local2enc (through the
    zigzag local2global of sharder.shard_maps) and enc_counts."""
    global2enc, counts = frame_plan(seg_len, seg_kind, P)
    if len(global2enc) != N:
        raise ValueError("segment lengths must sum to N")
    l2g = sharder.shard_maps(seg_len, seg_kind, N, P)["local2global"]
    local2enc = np.asarray([global2enc[l2g[l]] for l in range(N)], np.int32)
    return {"global2enc": global2enc, "local2enc": local2enc, "enc_counts": counts}
