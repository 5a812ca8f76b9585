"""RoPE fused into the shard gather (and its transposed scatter for the
gradients) on the GPU, through the C ABI, against the fp64 oracle, for both
pairings, every supported head size, document positions, ragged chunks, and
a million-token sequence (positions up to 2^20, where an fp32 angle would be
off by hundredths of a radian) on sampled rows.

Bar (derived from the arithmetic): the result is the fp32 rotation rounded
to bf16, so |gpu - exact| <= 2^-8 |exact| (half a bf16 ulp, relative) plus
the fp32 error of a cos - b sin, bounded by 2^-16 of the pair's norm (cos
and sin carry about 2^-21 absolute error); results near zero by
cancellation are bounded by the second term. Almost every element must also
equal the oracle rounded to bf16 exactly."""
import numpy as np
import pytest
import torch

import mmsp_inputs as mi
from oracle import attention as A
from oracle import rope as R
from gpu_util import lib, needs_gpu

pytestmark = [pytest.mark.gpu, needs_gpu]


def _pair_norm(ref64, interleaved):
    """|(a, b)| of the pair each element belongs to (rotation keeps it)."""
    r = np.asarray(ref64, np.float64)
    d = r.shape[-1]
    if interleaved:
        a, b = r[..., 0::2], r[..., 1::2]
        n = np.sqrt(a * a + b * b)
        return np.repeat(n, 2, axis=-1)
    a, b = r[..., : d // 2], r[..., d // 2:]
    n = np.sqrt(a * a + b * b)
    return np.concatenate([n, n], axis=-1)


def _check(got, ref64, interleaved, what):
    g = got.detach().float().cpu().numpy().astype(np.float64)
    r = np.asarray(ref64, np.float64)
    err = np.abs(g - r)
    bound = 2.0 ** -8 * np.abs(r) + 2.0 ** -16 * _pair_norm(r, interleaved)
    assert np.isfinite(g).all(), what + ": non-finite"
    assert (err <= bound).all(), f"{what}: worst excess {(err - bound).max():.3e}"
    exact = float((_bf16_ulps(got, r) == 0).float().mean())
    assert exact >= 0.99, f"{what}: only {exact:.5f} equal to the oracle rounded to bf16"


def _bf16_ulps(got, ref64):
    """Distance in bf16 units in the last place between the GPU's bf16 result
    and the fp64 oracle rounded to bf16."""
    ref = torch.as_tensor(np.asarray(ref64, np.float64)).to(torch.float32).to(torch.bfloat16)
    a = got.detach().cpu().view(torch.int16).to(torch.int32)
    b = ref.view(torch.int16).to(torch.int32)
    # map the sign-magnitude bit patterns onto a monotonic integer line
    a = torch.where(a < 0, -(a & 0x7FFF), a)
    b = torch.where(b < 0, -(b & 0x7FFF), b)
    return (a - b).abs()


def _x(N, H, d, seed):
    g = torch.Generator(device="cuda").manual_seed(seed)
    return torch.randn((N, H, d), generator=g, device="cuda").to(torch.bfloat16)


CASES = [
    # N, P, H, d, interleaved, documents
    (4096, 4, 28, 128, False, False),
    (4096, 4, 4, 128, True, False),
    (1200, 3, 4, 64, False, True),   # C = 200, positions restart per document
    (1200, 3, 4, 64, True, True),
    (144, 2, 7, 32, False, False),
    (144, 2, 3, 16, True, False),
    (96, 1, 2, 8, False, False),
    (512, 2, 1, 256, False, True),
]


@pytest.mark.parametrize("N,P,H,d,inter,docs", CASES)
def test_gather_and_gradient_scatter_match_oracle(N, P, H, d, inter, docs):
    m = lib()
    x = _x(N, H, d, seed=N + 7 * H + d)
    ds = ds_host = None
    if docs:
        doc_len = mi.random_segments(N, N + 1, max_len=300)[0]
        ds_host = A.document_starts(doc_len)
        ds = torch.as_tensor(ds_host.astype(np.int32)).cuda()
    y = torch.full_like(x, float("nan"))
    m.mmsp_shard_rope(x, y, N, P, H, d, 1e7, inter, doc_start=ds)
    torch.cuda.synchronize()
    ref = R.shard_rope(x.float().cpu().numpy(), N, P, 1e7, inter, ds_host)
    _check(y, ref, inter, "gather")
    # the transposed rotation, scattered back to global order
    g = _x(N, H, d, seed=N + 11)
    z = torch.full_like(g, float("nan"))
    m.mmsp_shard_rope(g, z, N, P, H, d, 1e7, inter, doc_start=ds, inverse=True)
    torch.cuda.synchronize()
    ref = R.unshard_rope_grad(g.float().cpu().numpy(), N, P, 1e7, inter, ds_host)
    _check(z, ref, inter, "gradient scatter")


def test_theta_10000_and_identity_at_position_zero():
    m = lib()
    N, P, H, d = 256, 2, 2, 64
    x = _x(N, H, d, seed=3)
    y = torch.empty_like(x)
    m.mmsp_shard_rope(x, y, N, P, H, d, 1e4, False)
    torch.cuda.synchronize()
    ref = R.shard_rope(x.float().cpu().numpy(), N, P, 1e4, False)
    _check(y, ref, False, "theta 1e4")


def test_million_token_positions_sampled():
    """N = 2^20 (P = 128): the angle pos * theta^(-2i/d) reaches 10^6 rad."""
    m = lib()
    N, P, H, d = 1 << 20, 128, 2, 128
    x = _x(N, H, d, seed=5)
    y = torch.empty_like(x)
    m.mmsp_shard_rope(x, y, N, P, H, d, 1e7, False)
    torch.cuda.synchronize()
    C = N // (2 * P)
    rows = mi.sample_rows(N, C, 512, seed=9)          # global positions
    g2l = torch.empty(N, dtype=torch.int32, device="cuda")
    m.mmsp_shard(None, None, N, P, global2local=g2l)
    loc = g2l[torch.as_tensor(rows, device="cuda")].long()
    ref = R.rope(x[torch.as_tensor(rows, device="cuda")].float().cpu().numpy(), rows, 1e7, False)
    _check(y[loc], ref, False, "2^20 tokens")


def test_invalid_arguments_launch_nothing():
    m = lib()
    x = torch.zeros((64, 2, 64), dtype=torch.bfloat16, device="cuda")
    y = torch.zeros_like(x)
    bad = [
        dict(d=48),                 # unsupported head size
        dict(theta=1.0),            # base must exceed 1
        dict(theta=float("inf")),
        dict(P=3),                  # N not divisible by 2P
    ]
    for b in bad:
        args = dict(N=64, P=2, H=2, d=64, theta=1e7)
        args.update(b)
        with pytest.raises(m.MmspError) as e:
            m.mmsp_shard_rope(x, y, args["N"], args["P"], args["H"], args["d"], args["theta"])
        assert e.value.status == 1
    with pytest.raises(m.MmspError):  # in place is not allowed (it is a permutation)
        m.mmsp_shard_rope(x, x, 64, 2, 2, 64)
    with pytest.raises(m.MmspError):  # misaligned
        m.mmsp_shard_rope(x.view(-1)[1:].data_ptr(), y, 32, 2, 1, 64)
    m.mmsp_shard_rope(x, y, 0, 2, 2, 64)  # N = 0: nothing to do
