"""A seeded sweep of random small shapes through the C ABI against the fp64
oracle: ragged chunk lengths (chunks shorter than a tile, a tile and a few
rows, several tiles), 1 to 6 virtual ranks, GQA ratios 1 to 7, and random
packed-document layouts on some of the cases. The forward (O, LSE) runs on
every case and the backward (dQ, dK, dV) on the d = 128 ones, each compared
element by element with the oracle at the same tolerances as the other
parity tests. The shapes are drawn once from a fixed seed, so the ids are
stable."""
import numpy as np
import pytest
import torch

import mmsp_inputs as mi
from oracle import attention as A
from gpu_util import compare_attention, compare_grad, lib, needs_gpu, run_backward, run_forward, shard_rows

pytestmark = [pytest.mark.gpu, needs_gpu]


def _draw_cases(n_cases=10, seed=20261203):
    rng = np.random.default_rng(seed)
    cases = []
    for i in range(n_cases):
        P = int(rng.integers(1, 7))
        C = int(rng.choice([int(rng.integers(1, 64)), int(rng.integers(100, 200)), int(rng.integers(200, 340))]))
        G = int(rng.choice([1, 2, 3, 4, 7]))
        hkv = int(rng.choice([1, 2])) if G > 2 else int(rng.choice([1, 2, 4]))
        d = 64 if i % 5 == 4 else 128
        docs = int(rng.integers(0, 2)) == 1
        max_len = int(rng.integers(5, 3 * C + 2))
        cases.append((2 * P * C, P, G * hkv, hkv, d, docs, max_len, 1000 + i))
    return cases


CASES = _draw_cases()


def _id(c):
    N, P, hq, hkv, d, docs, max_len, _ = c
    return f"N{N}-P{P}-C{N // (2 * P)}-hq{hq}-hkv{hkv}-d{d}" + (f"-docs{max_len}" if docs else "")


@pytest.mark.parametrize("case", CASES, ids=[_id(c) for c in CASES])
def test_random_shape_matches_oracle(case):
    N, P, hq, hkv, d, docs, max_len, seed = case
    m = lib()
    seg = mi.random_segments(N, seed + 17)
    vis = mi.token_kinds(*seg) == mi.VISUAL
    q, k, v, do = mi.make_tensors(N, hq, hkv, d, seed, vis, device="cuda", with_dout=True)
    ds_dev, ds_host = None, None
    if docs:
        doc_len = mi.random_segments(N, seed, max_len=max_len)[0]
        ds_dev = torch.full((N,), -1, dtype=torch.int32, device="cuda")
        m.mmsp_doc_starts(doc_len, N, ds_dev)
        ds_host = A.document_starts(doc_len)
        np.testing.assert_array_equal(ds_dev.cpu().numpy(), ds_host)
    ql, kl, vl, dol = (shard_rows(x, N, P) for x in (q, k, v, do))
    o_acc, lse, o_out = run_forward(ql, kl, vl, P, doc_start=ds_dev)
    back = lambda x: shard_rows(x, N, P, inverse=True).float().cpu().numpy()
    cpu = [x.float().cpu().numpy() for x in (q, k, v, do)]
    if d != 128:  # the backward supports d = 128 only
        o_ref, lse_ref = A.causal_attention(*cpu[:3], doc_start=ds_host)
        compare_attention(back(o_acc), back(lse), o_ref, lse_ref, _id(case))
        return
    dq, dk, dv, _ = run_backward(ql, kl, vl, o_out, dol, lse, P, doc_start=ds_dev)
    ref = A.causal_attention_bwd(*cpu, doc_start=ds_host)
    compare_attention(back(o_acc), back(lse), ref["O"], ref["LSE"], _id(case))
    compare_grad(back(dq), ref["dQ"], "dQ " + _id(case))
    compare_grad(back(dk), ref["dK"], "dK " + _id(case))
    compare_grad(back(dv), ref["dV"], "dV " + _id(case))
