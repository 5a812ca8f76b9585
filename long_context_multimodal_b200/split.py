"""The ring split across GPUs: each GPU owns a contiguous range of the P
virtual ranks and runs the attention calls for that range only.

Source: "LongVILA Guide" (aifetchly), section "Multi-Modal Sequence
Parallelism (MM-SP) Mechanics", Ring-SP paragraph (each of P ranks holds N/P
tokens; K/V blocks travel around the ring so every rank sees every block)
and the double-buffering paragraph (the transfer of the next block overlaps
the attention on the current one); section "Implementation",
LongVILAMultiModalAttention.forward (the per-rank ring loop with P2P
exchange of K and V between ring neighbours).

On B200 + NVSwitch every GPU reaches every peer at full bandwidth, and the
whole K/V of a 1M-token sequence is 2 GiB (about 3 ms of NVLink traffic
against seconds of attention), so instead of P-1 neighbour shifts the K/V
blocks are all-gathered once (one NCCL collective) and each GPU then runs
its ranks' whole ring from local HBM in one persistent launch. The
backward's key-owner stage needs every rank's queries, output gradients and
prepared (LSE, D) rows; these are all-gathered the same way, so no gradient
is reduced across GPUs: every GPU writes dQ of its own queries and dK, dV of
its own keys.

Every tensor keeps its full rank-local [P][2C][H][d] shape on every GPU;
GPU g fills and owns rows [rb*2C, re*2C) of its ranks [rb, re). The
collectives are plain torch.distributed calls (NCCL on GPUs, gloo in the
CPU tests); the kernels are the C ABI calls of libmmsp.so, reached through
`ops` (the binding module by default) so that the exchange bookkeeping can
be exercised on CPU with stand-ins.
"""
from __future__ import annotations

from dataclasses import dataclass

import torch
import torch.distributed as dist


@dataclass(frozen=True)
class RankRange:
    """The virtual ranks [begin, end) one GPU owns and their rank-local rows."""

    begin: int
    end: int
    C: int  # zigzag chunk length N / (2P)

    @property
    def rows(self) -> slice:
        return slice(self.begin * 2 * self.C, self.end * 2 * self.C)


def owned_ranks(P: int, world: int, rank: int, C: int) -> RankRange:
    """Contiguous, equal blocks of P / world virtual ranks per GPU. Zigzag
    gives every virtual rank the same causal work, so equal blocks balance
    the GPUs."""
    if world < 1 or P % world:
        raise ValueError(f"P ({P}) must be a multiple of the number of GPUs ({world})")
    if not 0 <= rank < world:
        raise ValueError(f"rank {rank} out of range for {world} GPUs")
    n = P // world
    return RankRange(rank * n, (rank + 1) * n, C)


def all_gather_rows(full, rr: RankRange, group=None):
    """Fill every GPU's copy of a rank-local [P*2C, ...] tensor from the GPU
    that owns each block of rows (one all-gather; the owned rows are
    copied out first so that the collective never reads what it writes)."""
    own = full[rr.rows].contiguous()
    dist.all_gather_into_tensor(full, own, group=group)
    return full


def workspace_slabs(ws_flat, P: int, Hq: int, C: int):
    """The two per-rank arrays of the backward workspace (LSE*log2(e) and D)
    as [P * Hq * 2 * Cp] fp32 views, in the rank-major layout the library
    documents for mmsp_attn_bwd (array B starts half-way into the buffer)."""
    Cp = (C + 127) // 128 * 128
    n = P * Hq * 2 * Cp
    f = ws_flat.view(torch.float32)
    half = f.numel() // 2
    return f[:n], f[half:half + n]


def forward(ops, ql, kl, vl, N, P, Hq, Hkv, d, scale, lse, o_out, rr: RankRange, group=None, o_acc=None,
            doc_start=None, stream=None):
    """Forward of this GPU's ranks: gather every rank's K, V, then one launch
    over the ring for ranks [rr.begin, rr.end)."""
    all_gather_rows(kl, rr, group)
    all_gather_rows(vl, rr, group)
    ops.mmsp_attn_fwd(ql, kl, vl, N, P, Hq, Hkv, d, scale, 1, 0, P, o_acc, lse, o_out, ops.MMSP_FINALIZE,
                      doc_start=doc_start, stream=stream, rank_begin=rr.begin, rank_end=rr.end)


def backward(ops, ql, kl, vl, ol, dol, lse, N, P, Hq, Hkv, d, scale, dql, dkl, dvl, ws, ws_bytes, rr: RankRange,
             group=None, doc_start=None, stream=None):
    """Backward of this GPU's ranks (K, V already gathered by `forward`):
    prepare the (LSE, D) rows of the owned ranks, gather every rank's Q, dO
    and prepared rows, then dQ of the owned queries and dK, dV of the owned
    keys."""
    ops.mmsp_attn_bwd_prepare(ol, dol, lse, N, P, Hq, d, ws, ws_bytes, stream=stream, rank_begin=rr.begin,
                              rank_end=rr.end)
    C = N // (2 * P)
    Cp = (C + 127) // 128 * 128
    slab = Hq * 2 * Cp
    for arr in workspace_slabs(ws, P, Hq, C):
        own = arr[rr.begin * slab:rr.end * slab].contiguous()
        dist.all_gather_into_tensor(arr, own, group=group)
    all_gather_rows(ql, rr, group)
    all_gather_rows(dol, rr, group)
    ops.mmsp_attn_bwd_dq(ql, kl, vl, dol, N, P, Hq, Hkv, d, scale, 1, dql, None, ws, ws_bytes, doc_start=doc_start,
                         stream=stream, rank_begin=rr.begin, rank_end=rr.end)
    ops.mmsp_attn_bwd_dkdv(ql, kl, vl, dol, N, P, Hq, Hkv, d, scale, 1, dkl, dvl, ws, ws_bytes,
                           doc_start=doc_start, stream=stream, rank_begin=rr.begin, rank_end=rr.end)
