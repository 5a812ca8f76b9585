"""Plant plausible mistakes in the oracle (on the CPU) and check that the pins
catch them: a pin that cannot fail pins nothing."""
import numpy as np
import pytest

from conftest import load_golden
from oracle import attention as A
from oracle import merge as M
import test_oracle_attention as TA


def test_interleaved_gqa_mapping_is_caught(monkeypatch):
    monkeypatch.setattr(A, "kv_head", lambda h, hq, hkv: h % hkv)
    with pytest.raises(AssertionError):
        TA.test_hand_worked_example()


def test_wrong_scale_is_caught(monkeypatch):
    real = A._rows_forward
    monkeypatch.setattr(A, "_rows_forward",
                        lambda qr, rows, K, V, scale, lo=None: real(qr, rows, K, V, scale * 2.0, lo))
    with pytest.raises(AssertionError):
        TA.test_matches_torch_sdpa_fp64(37, 4, 4, 16)


def test_dropped_merge_weight_is_caught():
    g = load_golden("merge_hand.txt")
    oa, ob = np.array(g["o_a"]), np.array(g["o_b"])
    # the page's sketch: plain sum of the normalised blocks
    wrong = oa + ob
    assert not np.allclose(wrong, g["o_out"])
    o, _ = M.lse_merge(oa, g["lse_a"][0], ob, g["lse_b"][0])
    assert np.allclose(o, g["o_out"])


def test_rope_wrong_frequency_exponent_is_caught(monkeypatch):
    import test_oracle_rope as TR
    from oracle import rope as R
    monkeypatch.setattr(R, "inv_freq", lambda d, theta: np.array([theta ** (-1.0 * i / d) for i in range(d // 2)]))
    with pytest.raises(AssertionError):
        TR.test_hand_worked_values()


def test_rope_wrong_rotation_sign_is_caught(monkeypatch):
    import test_oracle_rope as TR
    from oracle import rope as R
    real = R.rope
    monkeypatch.setattr(R, "rope", lambda x, pos, theta=1e7, interleaved=False, inverse=False:
                        real(x, pos, theta, interleaved, not inverse))
    with pytest.raises(AssertionError):
        TR.test_complex_multiplication_form(False)


def test_rope_swapped_pairing_is_caught(monkeypatch):
    import test_oracle_rope as TR
    from oracle import rope as R
    real = R.pair_index
    monkeypatch.setattr(R, "pair_index", lambda d, interleaved: real(d, not interleaved))
    with pytest.raises(AssertionError):
        TR.test_hand_worked_values()
