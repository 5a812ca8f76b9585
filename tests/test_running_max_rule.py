"""The running-max rule of the forward softmax, replayed in fp32 on the CPU.

Per tile the kernel takes the tile's largest raw score mx, forms
mc = max(m, fl(mx * scale_log2)) and raises the stored max m to mc when
mc > m + margin (margin 8 with documents, 0 without). The document build
corrects the bf16 rounding of the row's largest probability in the
epilogue, recomputing it with the final m; that is right only if m never
changes after the tile that holds the row's largest score. These tests
check that invariant on random tile sequences (ties, masked tiles, long and
short rows), and that with margin 0 the largest probability's exponent
argument is the rounding residual of one product (so it rounds to 1.0)."""
import numpy as np
import pytest

f32 = np.float32
MARGINS = (8.0, 0.0)


def replay(tile_max, sl2, margin):
    """Stored max after each tile (m starts at -inf), fp32 throughout."""
    m = f32(-np.inf)
    after = []
    for mx in tile_max:
        mc = max(m, f32(f32(mx) * f32(sl2)))
        if mc > f32(m + f32(margin)):
            m = mc
        after.append(m)
    return after


def _rows(rng, n_rows=400):
    for _ in range(n_rows):
        n = int(rng.integers(1, 60))
        mx = (rng.standard_normal(n) * rng.choice([0.5, 3.0, 12.0])).astype(np.float32)
        if rng.random() < 0.3:  # ties with the eventual maximum
            mx[rng.integers(0, n)] = mx.max()
        if rng.random() < 0.3:  # fully masked tiles
            mx[rng.integers(0, n, size=max(1, n // 5))] = -np.inf
        if np.isneginf(mx).all():
            mx[0] = 0.5
        yield mx


@pytest.mark.parametrize("margin", MARGINS)
def test_stored_max_is_final_from_the_tile_holding_the_largest_score(margin):
    rng = np.random.default_rng(7 + int(margin))
    sl2 = f32(1.4426950408889634 / np.sqrt(128.0))
    for mx in _rows(rng):
        after = replay(mx, sl2, margin)
        first = int(np.argmax(mx))  # first tile holding the largest score
        assert all(a == after[-1] for a in after[first:]), (mx, after)


def test_without_margin_the_largest_probability_rounds_to_one():
    rng = np.random.default_rng(3)
    sl2 = f32(1.4426950408889634 / np.sqrt(128.0))
    for mx in _rows(rng):
        m = replay(mx, sl2, 0.0)[-1]
        top = f32(mx.max())
        # the kernel's exponent argument for that element: fma(top, sl2, -m),
        # formed exactly in fp64 and rounded once, as a fused multiply-add is
        x = f32(np.float64(top) * np.float64(sl2) - np.float64(m))
        assert abs(float(x)) <= 2.0 ** -23 * abs(float(m)) + 1e-30
        p = np.exp2(np.float64(x))
        # bf16 keeps 8 significant bits: within 2^-9 of 1, it rounds to 1.0
        assert abs(p - 1.0) < 2.0 ** -9
