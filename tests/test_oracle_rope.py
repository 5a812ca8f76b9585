"""Pins of the RoPE oracle (oracle/rope.py) to facts that do not come from
its own formula: hand-worked values, the complex-number form of the
rotation, the relative-position property that defines rotary embeddings,
the geometric frequency ladder, norm preservation, the adjoint of the
gather, and the two pairings' relation."""
import numpy as np
import pytest

from conftest import load_golden
from oracle import rope as R


def _vec(v):
    return np.asarray(v, np.float64).reshape(1, 1, -1)


def test_hand_worked_values():
    g = load_golden("rope_hand.txt")
    out = R.rope(_vec(g["c1_x"]), [1], theta=12345.0)
    np.testing.assert_allclose(out.ravel(), g["c1_out"], atol=1e-15)
    out = R.rope(_vec(g["c2_x"]), [1], theta=1e4, interleaved=False)
    np.testing.assert_allclose(out.ravel(), g["c2_out"], atol=1e-15)
    out = R.rope(_vec(g["c3_x"]), [1], theta=1e4, interleaved=True)
    np.testing.assert_allclose(out.ravel(), g["c3_out"], atol=1e-15)
    x = np.zeros((1, 1, 128))
    x[0, 0, 63] = 1.0  # first element of the last "half" pair (63, 127)
    out = R.rope(x, [2], theta=1e7)
    phi = g["c4_phi"][0]
    assert abs(out[0, 0, 127] - phi) < 1e-14
    assert abs(out[0, 0, 63] - (1 - phi * phi / 2)) < 1e-15


def test_position_zero_is_identity():
    x = np.random.default_rng(1).standard_normal((3, 2, 16))
    np.testing.assert_array_equal(R.rope(x, [0, 0, 0]), x)


@pytest.mark.parametrize("interleaved", [False, True])
def test_complex_multiplication_form(interleaved):
    """Pair (a, b) as a + ib, rotated by multiplying with e^(i phi)."""
    rng = np.random.default_rng(2)
    N, H, d, theta = 7, 3, 32, 1e7
    x = rng.standard_normal((N, H, d))
    pos = rng.integers(0, 1 << 20, N)
    out = R.rope(x, pos, theta, interleaved)
    first, second = R.pair_index(d, interleaved)
    for i in range(d // 2):
        z = x[:, :, first[i]] + 1j * x[:, :, second[i]]
        w = z * np.exp(1j * pos[:, None] * theta ** (-2.0 * i / d))
        np.testing.assert_allclose(out[:, :, first[i]], w.real, atol=1e-12)
        np.testing.assert_allclose(out[:, :, second[i]], w.imag, atol=1e-12)


@pytest.mark.parametrize("interleaved", [False, True])
def test_dot_product_depends_only_on_relative_position(interleaved):
    """<R(m) q, R(n) k> = <R(m - n) q, k>: the defining RoPE property."""
    rng = np.random.default_rng(3)
    q = rng.standard_normal((1, 1, 64))
    k = rng.standard_normal((1, 1, 64))
    for m, n in [(5, 2), (1000, 999), (70000, 12), (3, 3)]:
        lhs = (R.rope(q, [m], 1e7, interleaved) * R.rope(k, [n], 1e7, interleaved)).sum()
        rhs = (R.rope(q, [m - n], 1e7, interleaved) * k).sum()
        assert abs(lhs - rhs) < 1e-9 * (1 + abs(rhs))


def test_frequency_ladder():
    f = R.inv_freq(128, 1e7)
    assert f[0] == 1.0
    ratio = f[1:] / f[:-1]
    np.testing.assert_allclose(ratio, 1e7 ** (-2.0 / 128), rtol=1e-12)
    # one more step of the ladder would reach 1/theta
    assert abs(f[-1] * 1e7 ** (-2.0 / 128) - 1e-7) < 1e-20


def test_rotation_keeps_pair_norms_and_inverse_undoes_it():
    rng = np.random.default_rng(4)
    x = rng.standard_normal((5, 2, 32))
    pos = rng.integers(0, 1 << 21, 5)
    y = R.rope(x, pos, 1e7)
    first, second = R.pair_index(32, False)
    nx = x[:, :, first] ** 2 + x[:, :, second] ** 2
    ny = y[:, :, first] ** 2 + y[:, :, second] ** 2
    np.testing.assert_allclose(ny, nx, rtol=1e-12)
    np.testing.assert_allclose(R.rope(y, pos, 1e7, inverse=True), x, atol=1e-12)


def test_pairings_are_a_permutation_of_each_other():
    rng = np.random.default_rng(5)
    d = 16
    x = rng.standard_normal((4, 1, d))
    pos = [0, 1, 7, 1000]
    perm = np.empty(d, np.int64)  # interleaved slot -> half-split element
    perm[0::2] = np.arange(d // 2)
    perm[1::2] = np.arange(d // 2) + d // 2
    a = R.rope(x, pos, 1e4, interleaved=False)
    b = R.rope(x[:, :, perm], pos, 1e4, interleaved=True)
    np.testing.assert_allclose(b, a[:, :, perm], atol=1e-13)


def test_gather_and_gradient_scatter_are_adjoint():
    """<shard_rope(x), g> = <x, unshard_rope_grad(g)> (the backward of the
    fused gather), with and without document positions."""
    rng = np.random.default_rng(6)
    N, P, H, d = 48, 3, 2, 16
    x = rng.standard_normal((N, H, d))
    g = rng.standard_normal((N, H, d))
    from oracle import attention as A
    for ds in (None, A.document_starts([10, 1, 30, 7])):
        y = R.shard_rope(x, N, P, 1e7, False, ds)
        back = R.unshard_rope_grad(g, N, P, 1e7, False, ds)
        assert abs((y * g).sum() - (x * back).sum()) < 1e-10


def test_document_positions_restart():
    from oracle import attention as A
    ds = A.document_starts([3, 2])
    np.testing.assert_array_equal(R.positions(5, ds), [0, 1, 2, 0, 1])
    x = np.random.default_rng(7).standard_normal((5, 1, 8))
    y = R.rope(x, R.positions(5, ds))
    np.testing.assert_array_equal(y[3], x[3])  # a document's first token is not rotated
