"""The parity checker itself (CPU only): the per-row and per-element bounds
reject one wrong row or one wrong element that the pooled relative-L2 bound
alone lets through.  Mistakes are planted in host copies only."""
import numpy as np
import pytest

import parity


def _pair(seed=0, rows=5120, d=128, noise=2e-3):
    # a reference output and a "GPU" copy at the bf16 rounding level
    rng = np.random.default_rng(seed)
    ref = rng.standard_normal((rows, d)) * rng.uniform(0.2, 2.0, (rows, 1))
    got = ref * (1.0 + noise * rng.standard_normal(ref.shape))
    return ref, got


def test_clean_copy_passes():
    ref, got = _pair()
    m = parity.check(got, ref, "bf16")
    assert m["rel_l2"] < 3e-3 and m["row_max"] < 5e-3 and m["elem_max"] < 2e-2


def test_one_wrong_row_passes_the_pooled_bound_but_fails_the_row_bound():
    ref, got = _pair(1)
    bad = got.copy()
    bad[1234] = -ref[1234]  # one row with error twice its own norm
    m = parity.metrics(bad, ref)
    assert m["rel_l2"] <= parity.BOUNDS["bf16"]["tol"]  # the old gate alone would accept it
    assert m["row_worst"] == 1234
    with pytest.raises(AssertionError, match="worst row"):
        parity.check(bad, ref, "bf16")


def test_one_wrong_element_fails_the_element_bound():
    ref, got = _pair(2)
    bad = got.copy()
    bad[77, 5] = ref[77, 5] + 0.5 * np.sqrt(np.mean(ref * ref)) + 0.5 * abs(ref[77, 5])
    m = parity.metrics(bad, ref)
    assert m["rel_l2"] <= parity.BOUNDS["bf16"]["tol"]
    with pytest.raises(AssertionError, match="worst element"):
        parity.check(bad, ref, "bf16", row_tol=1.0)


def test_shape_mismatch_and_leading_axes():
    ref, got = _pair(3, rows=64, d=64)
    m1 = parity.metrics(got.reshape(4, 16, 64), ref.reshape(4, 16, 64))
    m2 = parity.metrics(got, ref)
    assert m1 == m2
    with pytest.raises(ValueError):
        parity.metrics(got[:10], ref)


def test_zero_reference_rows_are_left_to_the_element_bound():
    ref, got = _pair(4, rows=256, d=64)
    ref[10] = 0.0
    got[10] = 1e-9
    m = parity.metrics(got, ref)
    assert m["row_max"] < 1e-2
