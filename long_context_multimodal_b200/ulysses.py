"""The Ulysses level of 2-D MM-SP: the sequence <-> head all-to-all among the
P_u GPUs of an NVLink domain.

Source: "LongVILA Guide" (aifetchly), section "Multi-Modal Sequence
Parallelism (MM-SP) Mechanics" (P = P_u x P_r; Ulysses all-to-all inside
the node, the ring across P_r node groups) and section "Implementation",
UlyssesAllToAll (forward: heads scattered, sequence gathered; backward: the
reverse all-to-all).

seq_to_heads: this GPU's [S, H, d] tokens -> [P_u * S, H / P_u, d], the
group's whole sequence for this GPU's head group (pack kernel, then one
all_to_all_single: the packed blocks are in destination order and the
received blocks land in source order, which is the head-sharded layout).
heads_to_seq: the inverse (one all_to_all_single of the head-sharded tensor
as it is, then the unpack kernel). Each is the other's backward. After
seq_to_heads of Q, K and V, the ring level runs mmsp_attn_fwd on H / P_u
query heads and Hkv / P_u kv heads: contiguous head groups keep the GQA
mapping (query head h reads kv head floor(h * Hkv / Hq)) within a group as
long as P_u divides Hkv.

The transposes are the C ABI call mmsp_ulysses_transpose, reached through
`ops` (the binding module by default) so that the collective's bookkeeping
can run on CPU with stand-ins; the all-to-all is torch.distributed (NCCL on
GPUs: plain peer transfers, no multicast).
"""
from __future__ import annotations

import torch
import torch.distributed as dist


def _ops(ops):
    if ops is None:
        import long_context_multimodal_b200 as ops
    return ops


def seq_to_heads(x, group=None, ops=None, stream=None):
    """[S, H, d] on each of the group's P_u ranks -> [P_u * S, H / P_u, d]."""
    ops = _ops(ops)
    P_u = dist.get_world_size(group)
    S, H = x.shape[0], x.shape[1]
    if H % P_u:
        raise ValueError(f"H ({H}) must be a multiple of the Ulysses group size ({P_u})")
    row_bytes = x[0, 0].numel() * x.element_size()
    packed = torch.empty((P_u, S, H // P_u) + tuple(x.shape[2:]), dtype=x.dtype, device=x.device)
    ops.mmsp_ulysses_transpose(x, packed, S, H, P_u, row_bytes, unpack=False, stream=stream)
    out = torch.empty_like(packed)
    dist.all_to_all_single(out, packed, group=group)
    return out.view((P_u * S, H // P_u) + tuple(x.shape[2:]))


def heads_to_seq(y, group=None, ops=None, stream=None):
    """[P_u * S, Hl, d] head-sharded -> [S, P_u * Hl, d] on each rank."""
    ops = _ops(ops)
    P_u = dist.get_world_size(group)
    if y.shape[0] % P_u:
        raise ValueError(f"sequence length ({y.shape[0]}) must be a multiple of the group size ({P_u})")
    S, hl = y.shape[0] // P_u, y.shape[1]
    recv = torch.empty_like(y)
    dist.all_to_all_single(recv, y.contiguous(), group=group)
    out = torch.empty((S, P_u * hl) + tuple(y.shape[2:]), dtype=y.dtype, device=y.device)
    row_bytes = y[0, 0].numel() * y.element_size()
    ops.mmsp_ulysses_transpose(recv, out, S, P_u * hl, P_u, row_bytes, unpack=True, stream=stream)
    return out
