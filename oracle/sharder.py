"""Naive zigzag sharder (oracle; test infrastructure only).

Follows "LongVILA Guide" (aifetchly), section "Multi-Modal Sequence
Parallelism (MM-SP) Mechanics", Ring-SP paragraph (each rank holds N/P
tokens of the sequence), and class ``LongVILAMultiModalAttention`` docstring
(local length = total length / number of ranks). The zigzag assignment is a
reading (the pages only say the sequence is split along its length): split
[0, N) into 2P equal chunks of C = N/(2P) tokens; virtual rank r owns chunk
r followed by chunk 2P-1-r, in that local order.

Written with plain Python loops on purpose: easy to check by eye, no
vectorised index tricks.
"""
from __future__ import annotations

import numpy as np


def zigzag_chunks(P: int, r: int):
    """The two global chunk indices rank r owns, in its local order."""
    return (r, 2 * P - 1 - r)


def shard_maps(seg_len, seg_kind, N: int, P: int):
    """All index outputs of the shard step.

    Returns a dict of numpy arrays:
      local2global [N] int32 -- global position of local slot r*2C + t
      global2local [N] int32 -- the inverse permutation
      modality_local [N] uint8 -- kind (0 text, 1 visual) of each local slot
      segid_local [N] int32 -- index into the segment table of each local slot
      rank_counts [P, 2] int32 -- per rank: number of text, visual tokens
    """
    if N % (2 * P) != 0:
        raise ValueError("N must be divisible by 2P")
    seg_len = [int(x) for x in seg_len]
    seg_kind = [int(x) for x in seg_kind]
    if sum(seg_len) != N:
        raise ValueError("segment lengths must sum to N")
    C = N // (2 * P)

    # token -> segment, by walking the table in sequence order
    seg_of_token = []
    for s, L in enumerate(seg_len):
        for _ in range(L):
            seg_of_token.append(s)

    local2global = [0] * N
    for r in range(P):
        first, second = zigzag_chunks(P, r)
        for t in range(2 * C):
            if t < C:
                g = first * C + t
            else:
                g = second * C + (t - C)
            local2global[r * 2 * C + t] = g

    global2local = [0] * N
    for loc in range(N):
        global2local[local2global[loc]] = loc

    modality_local = [0] * N
    segid_local = [0] * N
    rank_counts = [[0, 0] for _ in range(P)]
    for loc in range(N):
        s = seg_of_token[local2global[loc]]
        segid_local[loc] = s
        modality_local[loc] = seg_kind[s]
        rank_counts[loc // (2 * C)][seg_kind[s]] += 1

    return {
        "local2global": np.asarray(local2global, np.int32),
        "global2local": np.asarray(global2local, np.int32),
        "modality_local": np.asarray(modality_local, np.uint8),
        "segid_local": np.asarray(segid_local, np.int32),
        "rank_counts": np.asarray(rank_counts, np.int32),
    }


def permute_rows(x, local2global, inverse: bool = False):
    """Gather rows of x into rank-local order (dst[l] = src[local2global[l]]),
    or scatter them back when inverse (dst[local2global[l]] = src[l])."""
    x = np.asarray(x)
    out = np.empty_like(x)
    if not inverse:
        for loc in range(len(local2global)):
            out[loc] = x[local2global[loc]]
    else:
        for loc in range(len(local2global)):
            out[local2global[loc]] = x[loc]
    return out
