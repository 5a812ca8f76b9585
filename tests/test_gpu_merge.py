"""Standalone LSE merge kernel against the oracle merge."""
import numpy as np
import pytest
import torch

from oracle import merge as M
from gpu_util import lib, needs_gpu

pytestmark = [pytest.mark.gpu, needs_gpu]


def _parts(rows, H, d, seed):
    g = torch.Generator(device="cuda").manual_seed(seed)
    oa = torch.randn((rows, H, d), generator=g, device="cuda")
    ob = torch.randn((rows, H, d), generator=g, device="cuda")
    la = torch.randn((rows, H), generator=g, device="cuda") * 20
    lb = torch.randn((rows, H), generator=g, device="cuda") * 20
    # empties: a only, b only, both
    la[::7] = float("-inf")
    oa[::7] = 0
    lb[::5] = float("-inf")
    ob[::5] = 0
    return oa, la, ob, lb


@pytest.mark.parametrize("rows,H,d", [(1, 1, 128), (37, 3, 128), (1000, 28, 128), (999, 4, 64), (33, 5, 32),
                                      (64, 2, 4), (4096, 28, 128)])
def test_merge_matches_oracle(rows, H, d):
    m = lib()
    oa, la, ob, lb = _parts(rows, H, d, rows * 31 + d)
    o = torch.empty_like(oa)
    l = torch.empty_like(la)
    m.mmsp_lse_merge(oa, la, ob, lb, o, l, rows, H, d)
    m.mmsp_device_status()
    ro, rl = M.lse_merge(oa.double().cpu().numpy(), la.double().cpu().numpy(),
                         ob.double().cpu().numpy(), lb.double().cpu().numpy())
    lo = l.cpu().numpy()
    assert np.array_equal(np.isneginf(lo), np.isneginf(rl))
    fin = np.isfinite(rl)
    np.testing.assert_allclose(lo[fin], rl[fin], atol=2e-5, rtol=1e-6)
    np.testing.assert_allclose(o.cpu().numpy(), ro, atol=2e-5, rtol=1e-5)
    assert np.all(o.cpu().numpy()[np.isneginf(rl)] == 0)


def test_merge_in_place():
    m = lib()
    rows, H, d = 500, 7, 128
    oa, la, ob, lb = _parts(rows, H, d, 3)
    ro, rl = M.lse_merge(oa.double().cpu().numpy(), la.double().cpu().numpy(),
                         ob.double().cpu().numpy(), lb.double().cpu().numpy())
    m.mmsp_lse_merge(oa, la, ob, lb, oa, la, rows, H, d)
    m.mmsp_device_status()
    np.testing.assert_allclose(oa.cpu().numpy(), ro, atol=2e-5, rtol=1e-5)


def test_merge_zero_rows_is_noop():
    m = lib()
    x = torch.zeros(16, device="cuda")
    m.mmsp_lse_merge(x, x, x, x, x, x, 0, 1, 4)
    m.mmsp_device_status()
