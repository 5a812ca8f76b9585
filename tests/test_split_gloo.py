"""The ring split across GPUs (long_context_multimodal_b200.split) on two
gloo ranks on CPU: the exchange bookkeeping of the forward and the backward.

The kernels are replaced by stand-ins that compute, in fp64 from the
definitions (oracle), exactly what each C ABI call computes for a range of
virtual ranks, reading only what the CUDA kernel reads: the forward reads
every rank's K/V, prepare writes the owned ranks' (LSE*log2(e), D) slabs of
the rank-major workspace, dQ reads the owned queries and every K/V, dK/dV
reads every rank's Q, dO and workspace slabs. Rows a GPU has not received
stay NaN, so a missing exchange fails the comparison with the oracle.
"""
import math
import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

from oracle import attention as A
from oracle import sharder

N, P, HQ, HKV, D = 256, 4, 4, 2, 8
LOG2E = 1.4426950408889634


class OracleOps:
    """Stand-ins for the library calls the split uses (CPU, fp64)."""

    MMSP_FINALIZE = 2

    def __init__(self, l2g):
        self.l2g = np.asarray(l2g, np.int64)
        self.g2l = np.argsort(self.l2g)

    def _global(self, x):
        return x.double().numpy()[self.g2l]

    def _rows(self, P_, rank_begin, rank_end):
        C = N // (2 * P_)
        return np.arange(rank_begin * 2 * C, rank_end * 2 * C)

    def mmsp_attn_fwd(self, ql, kl, vl, N_, P_, Hq, Hkv, d, scale, causal, sb, se, o_acc, lse, o_out, flags,
                      doc_start=None, stream=None, rank_begin=0, rank_end=None):
        loc = self._rows(P_, rank_begin, rank_end)
        rows = self.l2g[loc]
        o, l = A.attention_rows(ql.double().numpy()[loc], self._global(kl), self._global(vl), rows, scale)
        lse[loc] = torch.from_numpy(l).float()
        o_out[loc] = torch.from_numpy(o).float()

    def mmsp_attn_bwd_prepare(self, ol, dol, lse, N_, P_, Hq, d, ws, ws_bytes, stream=None, rank_begin=0,
                              rank_end=None):
        from long_context_multimodal_b200 import split

        C = N_ // (2 * P_)
        Cp = (C + 127) // 128 * 128
        lse2, dd = split.workspace_slabs(ws, P_, Hq, C)
        for r in range(rank_begin, rank_end):
            for h in range(Hq):
                for c in range(2):
                    base = ((r * Hq + h) * 2 + c) * Cp
                    loc = r * 2 * C + c * C + np.arange(C)
                    lse2[base:base + C] = lse[loc, h] * LOG2E
                    dd[base:base + C] = (ol[loc, h].double() * dol[loc, h].double()).sum(-1).float()
                    lse2[base + C:base + Cp] = math.inf
                    dd[base + C:base + Cp] = 0.0

    def _ws_rows(self, ws, P_, Hq, loc):
        """(LSE*log2(e), D) [len(loc), Hq] from the workspace at local rows."""
        from long_context_multimodal_b200 import split

        C = N // (2 * P_)
        Cp = (C + 127) // 128 * 128
        lse2, dd = split.workspace_slabs(ws, P_, Hq, C)
        r, rem = loc // (2 * C), loc % (2 * C)
        c, t = rem // C, rem % C
        idx = ((r[:, None] * Hq + np.arange(Hq)[None, :]) * 2 + c[:, None]) * Cp + t[:, None]
        return lse2.double().numpy()[idx], dd.double().numpy()[idx]

    def _grads(self, ql, kl, vl, dol, ws, P_, Hq, Hkv, scale, qloc):
        """dS for queries at local rows qloc against every key (global order),
        from the workspace's LSE and D (as the kernels do)."""
        G = Hq // Hkv
        rows = self.l2g[qloc]
        lse2, dvec = self._ws_rows(ws, P_, Hq, qloc)
        k, v = self._global(kl), self._global(vl)
        q, do = ql.double().numpy()[qloc], dol.double().numpy()[qloc]
        out = []
        for h in range(Hq):
            kh = h // G
            s = q[:, h] @ k[:, kh].T * scale
            p = np.exp2(s * LOG2E - lse2[:, h:h + 1])
            p[np.arange(N)[None, :] > rows[:, None]] = 0.0
            ds = p * (do[:, h] @ v[:, kh].T - dvec[:, h:h + 1])
            out.append((p, ds))
        return out

    def mmsp_attn_bwd_dq(self, ql, kl, vl, dol, N_, P_, Hq, Hkv, d, scale, causal, dql, dq32, ws, ws_bytes,
                         doc_start=None, stream=None, rank_begin=0, rank_end=None):
        loc = self._rows(P_, rank_begin, rank_end)
        k = self._global(kl)
        G = Hq // Hkv
        for h, (_, ds) in enumerate(self._grads(ql, kl, vl, dol, ws, P_, Hq, Hkv, scale, loc)):
            dql[loc, h] = torch.from_numpy(scale * ds @ k[:, h // G]).float()

    def mmsp_attn_bwd_dkdv(self, ql, kl, vl, dol, N_, P_, Hq, Hkv, d, scale, causal, dkl, dvl, ws, ws_bytes,
                           doc_start=None, stream=None, rank_begin=0, rank_end=None):
        kloc = self._rows(P_, rank_begin, rank_end)
        kglob = self.l2g[kloc]
        allq = np.arange(N)
        q, do = ql.double().numpy(), dol.double().numpy()
        G = Hq // Hkv
        dk = np.zeros((len(kloc), Hkv, D))
        dv = np.zeros((len(kloc), Hkv, D))
        for h, (p, ds) in enumerate(self._grads(ql, kl, vl, dol, ws, P_, Hq, Hkv, scale, allq)):
            kh = h // G
            dv[:, kh] += p[:, kglob].T @ do[:, h]
            dk[:, kh] += scale * ds[:, kglob].T @ q[:, h]
        dkl[kloc] = torch.from_numpy(dk).float()
        dvl[kloc] = torch.from_numpy(dv).float()


def _inputs():
    g = torch.Generator().manual_seed(5)
    q, k, v, do = (torch.randn(N, h, D, generator=g) for h in (HQ, HKV, HKV, HQ))
    maps = sharder.shard_maps(np.array([N]), np.array([0]), N, P)
    return q, k, v, do, maps["local2global"]


def _worker(rank, world, port, out):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        from long_context_multimodal_b200 import split

        q, k, v, do, l2g = _inputs()
        C = N // (2 * P)
        rr = split.owned_ranks(P, world, rank, C)
        nan = lambda *s: torch.full(s, float("nan"))
        # every buffer full-size; only the owned rows hold this GPU's data
        ql, kl, vl, dol = nan(N, HQ, D), nan(N, HKV, D), nan(N, HKV, D), nan(N, HQ, D)
        for full, src in ((ql, q), (kl, k), (vl, v), (dol, do)):
            full[rr.rows] = src[l2g][rr.rows]
        ops = OracleOps(l2g)
        lse, o = nan(N, HQ), nan(N, HQ, D)
        scale = 1 / math.sqrt(D)
        split.forward(ops, ql, kl, vl, N, P, HQ, HKV, D, scale, lse, o, rr)
        Cp = (C + 127) // 128 * 128
        ws_bytes = 2 * P * HQ * 2 * Cp * 4
        ws = torch.full((ws_bytes,), 255, dtype=torch.uint8)  # NaN bit patterns
        dq, dk, dv = nan(N, HQ, D), nan(N, HKV, D), nan(N, HKV, D)
        split.backward(ops, ql, kl, vl, o, dol, lse, N, P, HQ, HKV, D, scale, dq, dk, dv, ws, ws_bytes, rr)
        res = {name: t[rr.rows].clone() for name, t in
               (("O", o), ("LSE", lse), ("dQ", dq), ("dK", dk), ("dV", dv))}
        res["rows"] = (rr.rows.start, rr.rows.stop)
        out[rank] = res
    finally:
        dist.destroy_process_group()


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


@pytest.mark.parametrize("world", [2])
def test_split_ring_over_gloo_matches_the_oracle(world):
    out = mp.Manager().dict()
    mp.spawn(_worker, args=(world, _free_port(), out), nprocs=world, join=True)
    q, k, v, do, l2g = _inputs()
    ref = A.causal_attention_bwd(q.numpy(), k.numpy(), v.numpy(), do.numpy())
    covered = np.zeros(N, bool)
    for rank in range(world):
        got = out[rank]
        a, b = got["rows"]
        covered[a:b] = True
        g = l2g[a:b]
        for name in ("O", "LSE", "dQ", "dK", "dV"):
            x = got[name].double().numpy()
            assert np.isfinite(x).all(), f"rank {rank} {name}: rows missing after the exchange"
            np.testing.assert_allclose(x, ref[name][g], atol=1e-5, rtol=1e-5, err_msg=f"rank {rank} {name}")
    assert covered.all()


def test_owned_ranks_partition_the_ring_evenly():
    from long_context_multimodal_b200 import split

    for P_, world in ((64, 8), (64, 1), (128, 4), (8, 2)):
        C = 16
        rs = [split.owned_ranks(P_, world, g, C) for g in range(world)]
        assert rs[0].begin == 0 and rs[-1].end == P_
        assert all(a.end == b.begin for a, b in zip(rs, rs[1:]))
        assert len({r.end - r.begin for r in rs}) == 1
        # zigzag: every virtual rank has the same number of visible causal
        # pairs, so equal blocks of ranks carry equal work
        n = P_ * 2 * C
        l2g = sharder.shard_maps(np.array([n]), np.array([0]), n, P_)["local2global"]
        per_gpu = [int((l2g[r.rows] + 1).sum()) for r in rs]
        assert len(set(per_gpu)) == 1
    with pytest.raises(ValueError):
        split.owned_ranks(6, 4, 0, 16)
