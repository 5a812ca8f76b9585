"""Parity at the full workload sizes, in the configuration the benchmark
times (whole ring, all P virtual ranks in one forward launch and the three
backward stages), against the fp64 oracle:

* n32k: the whole forward output (every row and head);
* n128k, n512k, n1m: O, LSE and dQ at 4096 seeded random query rows (every
  head) plus the forced rows 0, N-1 and every zigzag chunk start; dK and dV
  of one kv head (a different one per workload) at 1024 seeded keys drawn
  from the last 4096 positions (the oracle needs every row after the first
  sampled key in full, with the query heads of that kv head, so the keys
  sit near the end), together with O, LSE and dQ of those last rows for
  those query heads; and the closed-form gradient sums over the whole
  sequence, which pin every key of every kv head.

The inputs are the workload's own (mmsp_inputs.workload_tensors, drawn on
the GPU); the oracle receives copies of the sampled rows and of K, V.
Bars: O max-abs 1e-2 and mean-abs 1e-3 (fp32 O), LSE 1e-3 absolute, bf16 O
within 1 ulp of RNE(fp32 O); gradients per tensor max-rel 1e-2 and
mean-rel 1e-2.
"""
import numpy as np
import pytest
import torch

import mmsp_inputs as mi
from oracle import attention as A
from gpu_util import check_bf16_rounding, compare_attention, compare_grad, needs_gpu, run_backward, run_forward, shard_rows

pytestmark = [pytest.mark.gpu, needs_gpu]

N_ROWS = 4096      # seeded random query rows (every head), plus the forced rows
N_KEYS = 1024      # seeded keys for dK/dV ...
KEY_WINDOW = 4096  # ... drawn from the last KEY_WINDOW positions


def _closed_forms(dk, dv, do, hkv):
    """sum_j dV_j = sum_i sum_{h in group} dO_i,h and sum_j dK_j = 0 (each row
    of dS sums to zero), within twice the bf16 rounding of the outputs."""
    N, hq, d = do.shape
    G = hq // hkv
    sdv = dv.double().sum(0)
    sdo = do.double().view(N, hkv, G, d).sum((0, 2))
    assert bool(((sdv - sdo).abs() <= 2.0 ** -8 * dv.double().abs().sum(0) + 1e-6).all()), "sum dV != sum dO"
    sdk = dk.double().sum(0)
    assert bool((sdk.abs() <= 2.0 ** -8 * dk.double().abs().sum(0) + 1e-6).all()), "sum dK != 0"


def test_n32k_whole_forward_output():
    w = mi.WORKLOADS["n32k"]
    q, k, v, _ = mi.workload_tensors(w, device="cuda", with_dout=False)
    N, P = w.N, w.P
    ql, kl, vl = (shard_rows(x, N, P) for x in (q, k, v))
    o_acc, lse, o_out = run_forward(ql, kl, vl, P)
    check_bf16_rounding(o_out, o_acc)
    o = shard_rows(o_acc, N, P, inverse=True).cpu().numpy()
    l = shard_rows(lse, N, P, inverse=True).cpu().numpy()
    del ql, kl, vl, o_acc, lse, o_out
    qc, kc, vc = (x.float().cpu().numpy() for x in (q, k, v))
    del q, k, v
    torch.cuda.empty_cache()
    ref = A.attention_rows(qc, kc, vc, np.arange(N))
    compare_attention(o, l, ref[0], ref[1], f"n32k whole output ({N} rows x {w.hq} heads)")


@pytest.mark.parametrize("name", ["n128k", "n512k", "n1m"],
                         ids=[f"{n}-{N_ROWS}rows-{N_KEYS}keys" for n in ("n128k", "n512k", "n1m")])
def test_full_size_sampled_parity(name):
    w = mi.WORKLOADS[name]
    N, P = w.N, w.P
    q, k, v, do = mi.workload_tensors(w, device="cuda", with_dout=True)
    ql, kl, vl, dol = (shard_rows(x, N, P) for x in (q, k, v, do))
    o_acc, lse, o_out = run_forward(ql, kl, vl, P)
    check_bf16_rounding(o_out, o_acc)
    dq, dk, dv, _ = run_backward(ql, kl, vl, o_out, dol, lse, P)
    del ql, kl, vl, dol, o_out
    back = lambda x: shard_rows(x, N, P, inverse=True)
    O, LSE, dQ, dK, dV = back(o_acc), back(lse), back(dq), back(dk), back(dv)
    del o_acc, lse, dq, dk, dv
    _closed_forms(dK, dV, do, w.hkv)
    rows = mi.sample_rows(N, w.C, N_ROWS, 3000 + w.index)
    assert len(rows) >= N_ROWS + 2
    keys = mi.sample_keys(N, KEY_WINDOW, N_KEYS, 4000 + w.index)
    j0 = int(keys.min())
    kvh = w.index % w.hkv
    heads = [h for h in range(w.hq) if A.kv_head(h, w.hq, w.hkv) == kvh]
    ridx = torch.as_tensor(rows, device="cuda")
    kidx = torch.as_tensor(keys, device="cuda")
    got = {"O": O[ridx].cpu().numpy(), "LSE": LSE[ridx].cpu().numpy(), "dQ": dQ[ridx].float().cpu().numpy(),
           "dK": dK[kidx].float().cpu().numpy(), "dV": dV[kidx].float().cpu().numpy(),
           "O_tail": O[j0:].cpu().numpy(), "LSE_tail": LSE[j0:].cpu().numpy(),
           "dQ_tail": dQ[j0:].float().cpu().numpy()}
    qr, dor = q[ridx].float().cpu().numpy(), do[ridx].float().cpu().numpy()
    qt, dot = q[j0:].float().cpu().numpy(), do[j0:].float().cpu().numpy()
    kc, vc = k.float().cpu().numpy(), v.float().cpu().numpy()
    del q, k, v, do, O, LSE, dQ, dK, dV
    torch.cuda.empty_cache()
    ref = A.attention_bwd_rows(qr, kc, vc, dor, rows)
    compare_attention(got["O"], got["LSE"], ref["O"], ref["LSE"], f"{name} fwd at {len(rows)} rows")
    compare_grad(got["dQ"], ref["dQ"], f"{name} dQ at {len(rows)} rows")
    refk = A.attention_bwd_keys(qt, kc, vc, dot, keys, kv_heads=[kvh])
    compare_grad(got["dK"][:, kvh], refk["dK"][:, kvh], f"{name} dK at {len(keys)} keys, kv head {kvh}")
    compare_grad(got["dV"][:, kvh], refk["dV"][:, kvh], f"{name} dV at {len(keys)} keys, kv head {kvh}")
    compare_attention(got["O_tail"][:, heads], got["LSE_tail"][:, heads], refk["O_tail"][:, heads],
                      refk["LSE_tail"][:, heads], f"{name} fwd last {N - j0} rows")
    compare_grad(got["dQ_tail"][:, heads], refk["dQ_tail"][:, heads], f"{name} dQ last {N - j0} rows")
