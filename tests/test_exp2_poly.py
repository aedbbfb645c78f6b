"""The polynomial exp2 the attention kernel runs on its FMA pipe, replayed
bit for bit in float32 on the CPU (no GPU): finite and non-negative for every
argument the softmax can produce (including -inf from masked columns) and
within its derived relative-error bound of exp2."""
import numpy as np

from paged_kv_cache_frame_b200.csrc import exp2_poly


def test_coefficients_are_the_remez_solution():
    c, err = exp2_poly.remez_rel()
    np.testing.assert_allclose(np.float32(c), np.float32(exp2_poly.COEFFS), rtol=0, atol=1e-7)
    assert err < 8e-5


def test_device_sequence_error_bound():
    assert exp2_poly.verify() < 8e-5


def test_masked_and_extreme_arguments():
    y = exp2_poly.emulate(np.array([-np.inf, -1e30, -126.0, -125.5, -0.5, 0.0, 0.5, 8.0, 8.49],
                                   dtype=np.float32))
    assert np.all(np.isfinite(y)) and np.all(y >= 0)
    assert y[0] < 1.2e-38 and y[1] < 1.2e-38
    np.testing.assert_allclose(y[3:], np.exp2([-125.5, -0.5, 0.0, 0.5, 8.0, 8.49]), rtol=8e-5)
