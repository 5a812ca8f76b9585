"""The frame-aligned, modality-balanced encoder shard (mmsp_shard_frames) and
the indexed re-shard (mmsp_gather_rows) on the GPU: maps bit-exact against
the oracle (oracle/frames.py) for every workload layout and random tables,
and the round trip global -> encoder layout -> zigzag layout equal to the
zigzag gather of mmsp_shard, bit for bit."""
import numpy as np
import pytest
import torch

import mmsp_inputs as mi
from oracle import frames as F
from gpu_util import lib, needs_gpu, shard_rows

pytestmark = [pytest.mark.gpu, needs_gpu]


def _maps(seg_len, seg_kind, N, P):
    m = lib()
    g2e = torch.full((N,), -1, dtype=torch.int32, device="cuda")
    l2e = torch.full((N,), -1, dtype=torch.int32, device="cuda")
    cnt = torch.full((P, 2), -1, dtype=torch.int32, device="cuda")
    m.mmsp_shard_frames(seg_len, seg_kind, N, P, g2e, l2e, cnt)
    m.mmsp_device_status()
    return g2e, l2e, cnt


@pytest.mark.parametrize("name", ["n4k", "n32k", "n128k", "n512k", "n1m"])
def test_maps_match_the_oracle_on_the_workloads(name):
    w = mi.WORKLOADS[name]
    seg_len, seg_kind = mi.workload_layout(w)
    g2e, l2e, cnt = _maps(seg_len, seg_kind, w.N, w.P)
    ref = F.shard_frames(seg_len, seg_kind, w.N, w.P)
    assert np.array_equal(g2e.cpu().numpy(), ref["global2enc"])
    assert np.array_equal(l2e.cpu().numpy(), ref["local2enc"])
    assert np.array_equal(cnt.cpu().numpy(), ref["enc_counts"])


@pytest.mark.parametrize("seed,N,P", [(1, 600, 3), (2, 2048, 8), (3, 4096, 4), (4, 1200, 6), (5, 4096, 1),
                                      (6, 65536, 16)])
def test_maps_match_the_oracle_on_random_tables(seed, N, P):
    seg_len, seg_kind = mi.random_segments(N, seed)
    g2e, l2e, cnt = _maps(seg_len, seg_kind, N, P)
    ref = F.shard_frames(seg_len, seg_kind, N, P)
    for got, key in ((g2e, "global2enc"), (l2e, "local2enc"), (cnt, "enc_counts")):
        assert np.array_equal(got.cpu().numpy(), ref[key]), key


def test_reshard_round_trip_equals_the_zigzag_gather():
    m = lib()
    w = mi.WORKLOADS["n32k"]
    seg_len, seg_kind = mi.workload_layout(w)
    q, _, _, _ = mi.workload_tensors(w, device="cuda", with_dout=False)
    N, P = w.N, w.P
    g2e, l2e, _ = _maps(seg_len, seg_kind, N, P)
    rb = q[0].numel() * q.element_size()
    enc = torch.full_like(q, float("nan"))
    m.mmsp_gather_rows(q, enc, g2e, N, rb, scatter=True)        # encoder layout: enc[g2e[g]] = q[g]
    zig = torch.full_like(q, float("nan"))
    m.mmsp_gather_rows(enc, zig, l2e, N, rb)                    # attention layout: zig[l] = enc[l2e[l]]
    back = torch.full_like(q, float("nan"))
    m.mmsp_gather_rows(zig, back, l2e, N, rb, scatter=True)     # the gradient path back
    m.mmsp_device_status()
    ref = shard_rows(q, N, P)
    assert torch.equal(zig.view(torch.int16), ref.view(torch.int16))
    assert torch.equal(back.view(torch.int16), enc.view(torch.int16))
    e_np = enc.view(torch.int16).cpu().numpy()
    q_np = q.view(torch.int16).cpu().numpy()
    assert np.array_equal(e_np[g2e.cpu().numpy()], q_np)


def test_out_of_range_index_is_skipped_and_reported():
    m = lib()
    src = torch.arange(64 * 8, dtype=torch.float32, device="cuda").view(64, 8)
    dst = torch.zeros_like(src)
    idx = torch.arange(64, dtype=torch.int32, device="cuda").flip(0).contiguous()
    idx[5] = 64
    idx[9] = -3
    m.mmsp_gather_rows(src, dst, idx, 64, 32)
    with pytest.raises(m.MmspError) as e:
        m.mmsp_device_status()
    assert e.value.status == 1 and "out of range" in str(e.value)
    ok = torch.ones(64, dtype=torch.bool)
    ok[5] = ok[9] = False
    ref = src.flip(0)
    assert torch.equal(dst[ok.cuda()], ref[ok.cuda()])
    assert bool((dst[5] == 0).all()) and bool((dst[9] == 0).all())
    m.mmsp_device_status()  # the report was cleared
