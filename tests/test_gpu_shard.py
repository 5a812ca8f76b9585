"""Shard step on the GPU through the C ABI, bit-exact against the oracle."""
import numpy as np
import pytest
import torch

import mmsp_inputs as mi
from oracle import sharder
from gpu_util import lib, needs_gpu

pytestmark = [pytest.mark.gpu, needs_gpu]


def _maps(seg_len, seg_kind, N, P):
    m = lib()
    dev = "cuda"
    out = {
        "local2global": torch.full((N,), -7, dtype=torch.int32, device=dev),
        "global2local": torch.full((N,), -7, dtype=torch.int32, device=dev),
        "modality_local": torch.full((N,), 9, dtype=torch.uint8, device=dev),
        "segid_local": torch.full((N,), -7, dtype=torch.int32, device=dev),
        "rank_counts": torch.full((P, 2), -7, dtype=torch.int32, device=dev),
    }
    m.mmsp_shard(seg_len, seg_kind, N, P, out["local2global"], out["global2local"], out["modality_local"],
                 out["segid_local"], out["rank_counts"])
    m.mmsp_device_status()
    return {k: v.cpu().numpy() for k, v in out.items()}


def _assert_maps_equal(got, ref):
    for key in ref:
        assert got[key].dtype == ref[key].dtype, key
        assert np.array_equal(got[key], ref[key]), key


@pytest.mark.parametrize("name", list(mi.WORKLOADS))
def test_workload_maps_bit_exact(name):
    w = mi.WORKLOADS[name]
    sl, sk = mi.workload_layout(w)
    _assert_maps_equal(_maps(sl, sk, w.N, w.P), sharder.shard_maps(sl, sk, w.N, w.P))


@pytest.mark.parametrize("N,P,maxlen", [(2, 1, 1), (8, 4, 1), (12, 3, 5), (1000, 5, 37), (4096, 64, 3),
                                        (30000, 15, 20), (65536, 128, 600)])
def test_random_segment_maps_bit_exact(N, P, maxlen):
    sl, sk = mi.random_segments(N, seed=N + P, max_len=maxlen)
    assert len(sl) <= 4096
    _assert_maps_equal(_maps(sl, sk, N, P), sharder.shard_maps(sl, sk, N, P))


def test_segment_table_at_capacity():
    N, P = 8192, 4
    sl = np.full(4096, 2, np.int32)
    sk = (np.arange(4096) % 2).astype(np.uint8)
    _assert_maps_equal(_maps(sl, sk, N, P), sharder.shard_maps(sl, sk, N, P))


@pytest.mark.parametrize("N,P,row_bytes", [(4096, 4, 512), (1200, 3, 7168), (2, 1, 16), (65536, 32, 1024), (600, 1, 8), (1200, 3, 112), (144, 2, 28)])
def test_row_permute_bit_exact_and_inverse(N, P, row_bytes):
    m = lib()
    g = torch.Generator(device="cuda").manual_seed(N)
    src = torch.randint(0, 256, (N, row_bytes), generator=g, dtype=torch.uint8, device="cuda")
    dst = torch.empty_like(src)
    m.mmsp_shard(None, None, N, P, src=src, dst=dst, row_bytes=row_bytes)
    back = torch.empty_like(src)
    m.mmsp_shard(None, None, N, P, src=dst, dst=back, row_bytes=row_bytes, inverse=True)
    m.mmsp_device_status()
    l2g = torch.as_tensor(sharder.shard_maps([N], [0], N, P)["local2global"].astype(np.int64), device="cuda")
    assert torch.equal(dst, src[l2g])
    assert torch.equal(back, src)


def test_full_size_row_permute_of_queries():
    """n1m: Q rows (28 heads x 128 x bf16 = 7168 bytes) gathered and scattered back."""
    w = mi.WORKLOADS["n1m"]
    m = lib()
    g = torch.Generator(device="cuda").manual_seed(5)
    q = torch.randn((w.N, w.hq, w.d), generator=g, device="cuda").to(torch.bfloat16)
    ql = torch.empty_like(q)
    m.mmsp_shard(None, None, w.N, w.P, src=q, dst=ql, row_bytes=w.hq * w.d * 2)
    back = torch.empty_like(q)
    m.mmsp_shard(None, None, w.N, w.P, src=ql, dst=back, row_bytes=w.hq * w.d * 2, inverse=True)
    m.mmsp_device_status()
    assert torch.equal(back.view(torch.int16), q.view(torch.int16))
    C = w.C
    # spot rows: local slot r*2C + t holds global r*C + t (t < C) or (2P-1-r)*C + t - C
    for r in (0, 1, w.P - 1):
        for t in (0, C - 1, C, 2 * C - 1):
            gpos = r * C + t if t < C else (2 * w.P - 1 - r) * C + (t - C)
            assert torch.equal(ql[r * 2 * C + t].view(torch.int16), q[gpos].view(torch.int16))
