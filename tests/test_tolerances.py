"""The comparison helpers of the GPU tests (CPU only): what they accept and
what they must reject."""
import numpy as np
import pytest

from tests.gpu_utils import assert_close, assert_close_rows


def test_fixed_tolerance():
    ref = np.array([[1.0, -0.5, 0.0]])
    assert_close(ref + 0.0019, ref)
    with pytest.raises(AssertionError):
        assert_close(ref + np.array([[0.0, 0.0, 0.0021]]), ref)
    with pytest.raises(AssertionError):
        assert_close(np.array([[np.nan, 0, 0]]), ref)


def test_row_scaled_tolerance():
    rng = np.random.Generator(np.random.PCG64(3))
    for mag in (1e-2, 1.0, 1e2):
        ref = rng.standard_normal((4, 128)) * mag
        # bf16 rounding of every element passes at any magnitude
        u = ref.astype(np.float32).view(np.uint32).astype(np.uint64)
        bf16 = (((u + 0x7FFF + ((u >> 16) & 1)) >> 16) << 16).astype(np.uint32).view(np.float32)
        assert_close_rows(bf16.astype(np.float64), ref)
        # an error of 1% of the row's magnitude on a near-zero element fails at any magnitude
        bad = ref.copy()
        j = np.argmin(np.abs(ref[0]))
        bad[0, j] += 0.01 * np.max(np.abs(ref[0]))
        with pytest.raises(AssertionError):
            assert_close_rows(bad, ref)
    # a zero row must stay exactly zero
    with pytest.raises(AssertionError):
        assert_close_rows(np.array([[1e-9, 0.0]]), np.zeros((1, 2)))
