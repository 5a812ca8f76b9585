"""The Ulysses sequence <-> head transpose (mmsp_ulysses_transpose) on the GPU:
bit-exact against the oracle's pack/unpack, and 2-D MM-SP (P = P_u x P_r)
emulated on one GPU -- every emulated GPU's tokens packed by the kernel, the
all-to-all within each Ulysses group done by block copies, ring attention
(forward and backward) per head group over the P_r ring ranks, and the
inverse transpose by the kernel -- against the fp64 oracle."""
import math

import numpy as np
import pytest
import torch

from oracle import attention as A
from oracle import ulysses as U
from gpu_util import compare_attention, compare_grad, inputs, lib, needs_gpu, run_backward, run_forward, shard_rows

pytestmark = [pytest.mark.gpu, needs_gpu]


@pytest.mark.parametrize("S,H,P_u,width,dtype", [
    (0, 4, 2, 128, torch.bfloat16),
    (1, 4, 4, 128, torch.bfloat16),
    (1000, 28, 4, 128, torch.bfloat16),
    (777, 28, 7, 128, torch.bfloat16),
    (513, 8, 1, 64, torch.bfloat16),
    (300, 4, 2, 128, torch.float32),
    (64, 6, 3, 8, torch.float32),     # 32-byte rows
])
def test_pack_and_unpack_match_the_oracle(S, H, P_u, width, dtype):
    m = lib()
    g = torch.Generator(device="cuda").manual_seed(S + H)
    x = torch.randn((S, H, width), device="cuda", generator=g).to(dtype)
    packed = torch.full((P_u, S, H // P_u, width), float("nan"), device="cuda", dtype=dtype)
    rb = width * x.element_size()
    m.mmsp_ulysses_transpose(x, packed, S, H, P_u, rb)
    back = torch.full_like(x, float("nan"))
    m.mmsp_ulysses_transpose(packed, back, S, H, P_u, rb, unpack=True)
    m.mmsp_device_status()
    bits = torch.int16 if dtype == torch.bfloat16 else torch.int32
    ref = U.pack(x.cpu().view(bits).numpy(), P_u)  # the oracle moves the raw bit patterns
    assert torch.equal(packed.cpu().view(bits), torch.from_numpy(ref))
    assert torch.equal(back.view(bits), x.view(bits))


def _emulate_2d(fn_per_group, tensors, heads, N, P_r, P_u):
    """tensors: rank-local (P_r-ring zigzag order) [N, H, width] CUDA tensors
    with heads[i] heads each. Split every ring rank's 2C tokens over P_u
    emulated GPUs, pack with the kernel, do the group all-to-all by block
    copies, and hand fn_per_group(j, head-sharded tensors) the ring's
    rank-local tensors of head group j ([N, H/P_u, width] each). Returns the
    per-group results."""
    m = lib()
    C2 = N // P_r
    S = C2 // P_u
    grouped = []
    for t, H in zip(tensors, heads):
        width = t.shape[2]
        rb = width * t.element_size()
        hl = H // P_u
        out = torch.empty((P_u, N, hl, width), dtype=t.dtype, device=t.device)  # [group j][ring rows]
        for r in range(P_r):
            packs = []
            for u in range(P_u):
                x = t[r * C2 + u * S:r * C2 + (u + 1) * S].contiguous()
                p = torch.empty((P_u, S, hl, width), dtype=t.dtype, device=t.device)
                m.mmsp_ulysses_transpose(x, p, S, H, P_u, rb)
                packs.append(p)
            for j in range(P_u):          # receiver (r, j): block j of every sender u, in sender order
                for u in range(P_u):
                    out[j, r * C2 + u * S:r * C2 + (u + 1) * S] = packs[u][j]
        grouped.append(out)
    return [fn_per_group(j, *[gt[j].contiguous() for gt in grouped]) for j in range(P_u)]


def _unemulate_2d(per_group, H, N, P_r, P_u):
    """Inverse: per_group[j] [N, H/P_u, width] (ring rank-local order) ->
    [N, H, width]: every emulated GPU (r, u) receives block u of each group's
    rows of ring rank r, and the kernel unpacks them."""
    m = lib()
    C2 = N // P_r
    S = C2 // P_u
    t0 = per_group[0]
    hl, width = t0.shape[1], t0.shape[2]
    rb = width * t0.element_size()
    out = torch.empty((N, H, width), dtype=t0.dtype, device=t0.device)
    for r in range(P_r):
        for u in range(P_u):
            recv = torch.stack([per_group[j][r * C2 + u * S:r * C2 + (u + 1) * S] for j in range(P_u)]).contiguous()
            dst = torch.empty((S, H, width), dtype=t0.dtype, device=t0.device)
            m.mmsp_ulysses_transpose(recv, dst, S, H, P_u, rb, unpack=True)
            out[r * C2 + u * S:r * C2 + (u + 1) * S] = dst
    return out


@pytest.mark.parametrize("N,P_r,P_u,hq,hkv", [(4096, 4, 2, 28, 4), (2048, 2, 4, 28, 4), (3072, 3, 4, 8, 4)])
def test_2d_mmsp_emulated_on_one_gpu_matches_the_oracle(N, P_r, P_u, hq, hkv):
    m = lib()
    d = 128
    _, q, k, v, do = inputs(N, hq, hkv, d, seed=N + P_u, with_dout=True)
    ql, kl, vl, dol = (shard_rows(x, N, P_r) for x in (q, k, v, do))
    res = {}

    def per_group(j, qj, kj, vj, doj):
        o32, lse, o = run_forward(qj, kj, vj, P_r)
        dq, dk, dv, _ = run_backward(qj, kj, vj, o, doj, lse, P_r)
        res[j] = lse
        return o32, dq, dk, dv

    outs = _emulate_2d(per_group, [ql, kl, vl, dol], [hq, hkv, hkv, hq], N, P_r, P_u)
    m.mmsp_device_status()
    o = _unemulate_2d([x[0] for x in outs], hq, N, P_r, P_u)
    dq = _unemulate_2d([x[1] for x in outs], hq, N, P_r, P_u)
    dk = _unemulate_2d([x[2] for x in outs], hkv, N, P_r, P_u)
    dv = _unemulate_2d([x[3] for x in outs], hkv, N, P_r, P_u)
    m.mmsp_device_status()
    ref = A.causal_attention_bwd(q.float().cpu().numpy(), k.float().cpu().numpy(), v.float().cpu().numpy(),
                                 do.float().cpu().numpy())
    hl = hq // P_u
    lse = torch.cat([res[j] for j in range(P_u)], dim=1)  # [N, hq] in head-group order
    og = shard_rows(o, N, P_r, inverse=True).cpu().numpy()
    lg = shard_rows(lse.contiguous(), N, P_r, inverse=True).cpu().numpy()
    compare_attention(og, lg, ref["O"], ref["LSE"], f"2-D MM-SP forward P_u={P_u} P_r={P_r}")
    assert hl * P_u == hq
    for name, t in (("dQ", dq), ("dK", dk), ("dV", dv)):
        g = shard_rows(t, N, P_r, inverse=True).float().cpu().numpy()
        compare_grad(g, ref[name], f"2-D MM-SP {name} P_u={P_u} P_r={P_r}")
