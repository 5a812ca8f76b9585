"""The Ulysses all-to-all (long_context_multimodal_b200.ulysses) on 2 and 4
gloo ranks on CPU: the collective's bookkeeping against the oracle's
definition, the inverse, and the adjoint property that makes each the
other's backward. The transpose kernel is replaced by a stand-in built from
the oracle's pack/unpack (the kernel itself is checked on the GPU in
test_gpu_ulysses.py)."""
import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

from oracle import ulysses as U

S, H, D = 6, 8, 4


class OracleOps:
    @staticmethod
    def mmsp_ulysses_transpose(src, dst, S_, H_, P_u, row_bytes, unpack=False, stream=None):
        x = src.numpy()
        if unpack:
            y = U.unpack(x.reshape((P_u, S_, H_ // P_u) + x.shape[-1:]), P_u)
        else:
            y = U.pack(x.reshape((S_, H_) + x.shape[-1:]), P_u)
        dst.copy_(torch.from_numpy(np.ascontiguousarray(y)).reshape(dst.shape))


def _inputs(world):
    g = torch.Generator().manual_seed(7)
    xs = [torch.randn(S, H, D, generator=g) for _ in range(world)]
    ys = [torch.randn(world * S, H // world, D, generator=g) for _ in range(world)]
    return xs, ys


def _worker(rank, world, port, out):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        from long_context_multimodal_b200 import ulysses

        xs, ys = _inputs(world)
        fwd = ulysses.seq_to_heads(xs[rank], ops=OracleOps)
        back = ulysses.heads_to_seq(fwd, ops=OracleOps)
        inv = ulysses.heads_to_seq(ys[rank], ops=OracleOps)
        # <seq_to_heads(x), y> summed over ranks, and <x, heads_to_seq(y)>
        ip = torch.tensor([float((fwd.double() * ys[rank].double()).sum()),
                           float((xs[rank].double() * inv.double()).sum())], dtype=torch.float64)
        dist.all_reduce(ip)
        out[rank] = {"fwd": fwd.clone(), "back": back.clone(), "ip": ip.clone()}
    finally:
        dist.destroy_process_group()


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


@pytest.mark.parametrize("world", [2, 4])
def test_ulysses_all_to_all_over_gloo(world):
    out = mp.Manager().dict()
    mp.spawn(_worker, args=(world, _free_port(), out), nprocs=world, join=True)
    xs, _ = _inputs(world)
    ref = U.seq_to_heads([x.numpy() for x in xs])
    for r in range(world):
        assert np.array_equal(out[r]["fwd"].numpy(), ref[r]), f"rank {r}: head-sharded layout"
        assert torch.equal(out[r]["back"], xs[r]), f"rank {r}: inverse"
        a, b = out[r]["ip"].tolist()
        # the transpose is a permutation: its adjoint (the backward) is the inverse
        assert abs(a - b) <= 1e-9 * max(1.0, abs(a))
