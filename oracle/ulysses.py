"""Ulysses sequence <-> head all-to-all of 2-D MM-SP, by its definition
(oracle; test infrastructure only).

Source: "LongVILA Guide" (aifetchly), section "Multi-Modal Sequence
Parallelism (MM-SP) Mechanics": Ulysses turns the sequence-sharded
(B, N/P, H, D) into the head-sharded (B, N, H/P, D) with one all_to_all and
turns it back with the inverse all_to_all; MM-SP runs Ulysses over P_u GPUs
of a node and Ring attention over P_r node groups, P = P_u x P_r. Section
"Implementation", class UlyssesAllToAll: each rank splits its tensor into
world_size contiguous pieces along the scatter dimension and sends piece j
to rank j; each rank concatenates the pieces it receives along the gather
dimension, in the order of the sending ranks; the backward does the same
with the two dimensions swapped.

Here a rank's tensor is [S, H, d] (B = 1). Every function works on plain
Python lists of the P_u ranks' arrays; nothing is shared with the CUDA path.
"""
from __future__ import annotations

import numpy as np


def seq_to_heads(xs):
    """Forward all-to-all over the P_u ranks of one Ulysses group.

    xs[i]: rank i's [S, H, d] (its S consecutive tokens, every head).
    Returns ys with ys[j]: [P_u * S, H / P_u, d] -- every rank's tokens in
    rank order, heads [j * H/P_u, (j + 1) * H/P_u)."""
    P_u = len(xs)
    H = xs[0].shape[1]
    if H % P_u:
        raise ValueError("the head count must be a multiple of the group size")
    hl = H // P_u
    ys = []
    for j in range(P_u):                 # receiving rank
        pieces = [xs[i][:, j * hl:(j + 1) * hl] for i in range(P_u)]   # piece j of every sender, sender order
        ys.append(np.concatenate(pieces, axis=0))
    return ys


def heads_to_seq(ys):
    """Inverse all-to-all: ys[j] [P_u * S, Hl, d] -> xs[i] [S, P_u * Hl, d]
    (rank i's tokens, every head; heads of rank j's group at j * Hl)."""
    P_u = len(ys)
    if ys[0].shape[0] % P_u:
        raise ValueError("the sequence length must be a multiple of the group size")
    S = ys[0].shape[0] // P_u
    xs = []
    for i in range(P_u):                 # receiving rank
        pieces = [ys[j][i * S:(i + 1) * S] for j in range(P_u)]          # piece i of every sender, sender order
        xs.append(np.concatenate(pieces, axis=1))
    return xs


def pack(x, P_u):
    """One rank's send buffer of the forward all-to-all: [S, H, d] ->
    [P_u, S, H / P_u, d], block j = the head group bound for rank j."""
    S, H = x.shape[0], x.shape[1]
    hl = H // P_u
    out = np.empty((P_u, S, hl) + x.shape[2:], dtype=x.dtype)
    for j in range(P_u):
        out[j] = x[:, j * hl:(j + 1) * hl]
    return out


def unpack(y, P_u):
    """One rank's receive buffer of the inverse all-to-all back to its
    tokens: [P_u, S, Hl, d] (block i from rank i = the heads of rank i's
    group) -> [S, P_u * Hl, d]."""
    hl = y.shape[2]
    out = np.empty((y.shape[1], P_u * hl) + y.shape[3:], dtype=y.dtype)
    for i in range(P_u):
        out[:, i * hl:(i + 1) * hl] = y[i]
    return out
