"""Ring-blockwise causal attention forward on the GPU (C ABI) against the
fp64 oracle: whole outputs at small sizes (several tiles, ragged chunk
tails, every GQA ratio used), per-ring-step partials, the unfused
step-by-step path with the standalone merge. The full workload sizes are in
test_gpu_full_size.py."""
import math

import numpy as np
import pytest
import torch

import mmsp_inputs as mi
from oracle import attention as A
from oracle import merge as M
from gpu_util import (check_bf16_rounding, compare_attention, inputs, lib, needs_gpu, run_forward,
                      shard_rows)

pytestmark = [pytest.mark.gpu, needs_gpu]


def _path(q, k, v, P, causal=1):
    """global-order inputs -> shard -> attention over the whole ring -> global order."""
    N = q.shape[0]
    ql, kl, vl = (shard_rows(x, N, P) for x in (q, k, v))
    o_acc, lse, o_out = run_forward(ql, kl, vl, P, causal=causal)
    check_bf16_rounding(o_out, o_acc)
    return (shard_rows(o_acc, N, P, inverse=True), shard_rows(lse, N, P, inverse=True),
            shard_rows(o_out, N, P, inverse=True))


CASES = [
    # N, P, Hq, Hkv, d
    (4096, 4, 4, 4, 64),     # the n4k workload shape
    (1200, 3, 4, 2, 128),    # C = 200: ragged tiles and row blocks
    (600, 1, 2, 1, 128),     # one rank
    (144, 2, 7, 1, 128),     # C = 36: chunk shorter than a tile
    (2048, 8, 28, 4, 128),   # C = 128: exact tiles, GQA 7:1
    (1536, 2, 2, 2, 64),     # C = 384: three tiles, a half-empty row block
    (2560, 4, 3, 1, 128),    # C = 320
]


@pytest.mark.parametrize("N,P,hq,hkv,d", CASES)
def test_forward_matches_oracle_whole_output(N, P, hq, hkv, d):
    seg, q, k, v, _ = inputs(N, hq, hkv, d, seed=N + 7 * P + d)
    o, lse, _ = _path(q, k, v, P)
    o_ref, lse_ref = A.causal_attention(q.float().cpu().numpy(), k.float().cpu().numpy(),
                                        v.float().cpu().numpy())
    compare_attention(o.cpu().numpy(), lse.cpu().numpy(), o_ref, lse_ref, f"N={N} P={P}")


def test_n4k_workload_whole_output():
    w = mi.WORKLOADS["n4k"]
    q, k, v, _ = mi.workload_tensors(w, device="cuda")
    o, lse, o_out = _path(q, k, v, w.P)
    o_ref, lse_ref = A.causal_attention(q.float().cpu().numpy(), k.float().cpu().numpy(),
                                        v.float().cpu().numpy())
    compare_attention(o.cpu().numpy(), lse.cpu().numpy(), o_ref, lse_ref, "n4k")


def test_non_causal_whole_output():
    N, P, hq, hkv, d = 1024, 2, 4, 4, 128
    _, q, k, v, _ = inputs(N, hq, hkv, d, seed=11)
    o, lse, _ = _path(q, k, v, P, causal=0)
    qn, kn, vn = (x.double().cpu().numpy() for x in (q, k, v))
    o_ref = np.zeros((N, hq, d))
    lse_ref = np.zeros((N, hq))
    allpos = np.arange(N)
    for h in range(hq):
        o_ref[:, h], lse_ref[:, h] = M.block_attention(qn[:, h], np.full(N, N), kn[:, h], vn[:, h], allpos,
                                                       1 / math.sqrt(d))
    compare_attention(o.cpu().numpy(), lse.cpu().numpy(), o_ref, lse_ref, "non-causal")


def test_each_ring_step_partial_and_unfused_merge_path():
    """Step s alone gives every rank its partial over the K/V of rank
    (r - s) mod P (empty rows: LSE -inf, O 0); merging the steps with the
    standalone mmsp_lse_merge, or with MMSP_ACCUMULATE, gives the whole
    attention."""
    m = lib()
    N, P, hq, hkv, d = 1024, 4, 4, 2, 128
    _, q, k, v, _ = inputs(N, hq, hkv, d, seed=23)
    ql, kl, vl = (shard_rows(x, N, P) for x in (q, k, v))
    qn, kn, vn = (x.double().cpu().numpy() for x in (q, k, v))
    run_o = run_l = None
    acc_o = torch.empty((N, hq, d), device="cuda")
    acc_l = torch.empty((N, hq), device="cuda")
    for s in range(P):
        o_s, l_s, _ = run_forward(ql, kl, vl, P, step_begin=s, step_end=s + 1, flags=0)
        ref_o, ref_l = M.ring_step_partials(qn, kn, vn, P, s)
        lo = l_s.cpu().numpy()
        oo = o_s.cpu().numpy()
        empty = np.isneginf(ref_l)
        assert np.array_equal(np.isneginf(lo), empty), f"step {s}: empty rows differ"
        assert np.all(oo[empty] == 0)
        fin = ~empty
        compare_attention(oo[fin], lo[fin], ref_o[fin], ref_l[fin], f"step {s}")
        if run_o is None:
            run_o, run_l = o_s.clone(), l_s.clone()
        else:
            m.mmsp_lse_merge(run_o, run_l, o_s, l_s, run_o, run_l, N, hq, d)
        flags = (m.MMSP_ACCUMULATE if s > 0 else 0) | (m.MMSP_FINALIZE if s == P - 1 else 0)
        _, _, o_out = run_forward(ql, kl, vl, P, step_begin=s, step_end=s + 1, flags=flags, o_acc=acc_o,
                                  lse=acc_l)
    m.mmsp_device_status()
    check_bf16_rounding(o_out, acc_o)
    o_ref, lse_ref = A.causal_attention(q.float().cpu().numpy(), k.float().cpu().numpy(),
                                        v.float().cpu().numpy())
    for name, oo, ll in (("merge kernel", run_o, run_l), ("accumulate", acc_o, acc_l)):
        og = shard_rows(oo, N, P, inverse=True).cpu().numpy()
        lg = shard_rows(ll, N, P, inverse=True).cpu().numpy()
        compare_attention(og, lg, o_ref, lse_ref, name)


def test_empty_sequence_is_a_noop():
    m = lib()
    x = torch.zeros(64, device="cuda", dtype=torch.bfloat16)
    l = torch.zeros(64, device="cuda")
    m.mmsp_attn_fwd(x, x, x, 0, 4, 4, 4, 64, 0.125, 1, 0, 4, None, l, None, 0)
    m.mmsp_device_status()
