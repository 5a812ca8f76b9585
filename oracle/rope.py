"""Rotary position embedding (RoPE) with a large base, by its definition, in
fp64 (oracle; test infrastructure only).

Source: "LongVILA Guide" (aifetchly), the three-stage curriculum, Stage 2
"Context Scaling and RoPE Extension" (the RoPE base frequency theta is raised
from 10,000 to 10,000,000 before long-context training), and section
"Distributed Training Configuration" (the launcher passes a RoPE base of
10,000,000). The pages name RoPE but print no formula; this is the standard
rotary embedding (Su et al., RoFormer): for a head vector x of even length
d and i in [0, d/2), the pair (a_i, b_i) is rotated by the angle
pos * theta^(-2i/d):

    a_i' = a_i cos(phi_i) - b_i sin(phi_i)
    b_i' = a_i sin(phi_i) + b_i cos(phi_i),   phi_i = pos * theta^(-2i/d)

Pairing (a reading; the pages do not say): "half" pairs element i with
element i + d/2 (the layout of the Llama-family backbones LongVILA builds
on), "interleaved" pairs elements 2i and 2i+1 (the RoFormer paper's
layout). Both are provided.

Position (a reading): the token's global position in the packed sequence;
with document starts given, the position within its document
(pos = g - doc_start[g]), i.e. positions restart with every packed sample
like the attention mask does.

The fused operation on the hot path is the shard gather of Q and K with RoPE
applied on the way (``shard_rope``) and, for the gradients, the transposed
rotation (angle -phi) applied while scattering back to global order.

Written as plain loops over the pairs with fp64 numpy arrays.
"""
from __future__ import annotations

import numpy as np

from . import sharder


def inv_freq(d: int, theta: float):
    """theta^(-2i/d) for i in [0, d/2), fp64."""
    return np.array([theta ** (-2.0 * i / d) for i in range(d // 2)], dtype=np.float64)


def positions(N: int, doc_start=None):
    """Position of each global token: g, or g - doc_start[g]."""
    g = np.arange(N, dtype=np.int64)
    if doc_start is None:
        return g
    return g - np.asarray(doc_start, np.int64)


def pair_index(d: int, interleaved: bool):
    """(first, second) element index of each of the d/2 rotated pairs."""
    if interleaved:
        return [2 * i for i in range(d // 2)], [2 * i + 1 for i in range(d // 2)]
    return [i for i in range(d // 2)], [i + d // 2 for i in range(d // 2)]


def rope(x, pos, theta: float = 1e7, interleaved: bool = False, inverse: bool = False):
    """Rotate every head vector of x [N, H, d] by its token's position.

    inverse=True applies the transpose (angle -phi), which undoes the
    rotation and is the gradient map dL/dx = R^T dL/dx'."""
    x = np.asarray(x, dtype=np.float64)
    N, H, d = x.shape
    if d % 2:
        raise ValueError("d must be even")
    pos = np.asarray(pos, dtype=np.float64)
    f = inv_freq(d, theta)
    sign = -1.0 if inverse else 1.0
    first, second = pair_index(d, interleaved)
    out = np.empty_like(x)
    for i in range(d // 2):
        phi = sign * pos * f[i]                     # [N]
        c = np.cos(phi)[:, None]
        s = np.sin(phi)[:, None]
        a = x[:, :, first[i]]
        b = x[:, :, second[i]]
        out[:, :, first[i]] = a * c - b * s
        out[:, :, second[i]] = a * s + b * c
    return out


def _local2global(N: int, P: int):
    return sharder.shard_maps([N], [0], N, P)["local2global"] if N else np.zeros(0, np.int32)


def shard_rope(x_global, N: int, P: int, theta: float = 1e7, interleaved: bool = False, doc_start=None):
    """Rank-local rows of RoPE(x): row l holds the rotated global row
    local2global(l) (the shard gather with the rotation fused)."""
    rot = rope(x_global, positions(N, doc_start), theta, interleaved)
    return sharder.permute_rows(rot, _local2global(N, P))


def unshard_rope_grad(g_local, N: int, P: int, theta: float = 1e7, interleaved: bool = False, doc_start=None):
    """Global-order gradient with respect to the un-rotated rows: scatter the
    rank-local gradient rows back and apply the transposed rotation."""
    g = sharder.permute_rows(np.asarray(g_local, np.float64), _local2global(N, P), inverse=True)
    return rope(g, positions(N, doc_start), theta, interleaved, inverse=True)
