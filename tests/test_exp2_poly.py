"""The FMA-pipe 2^x of the prefill kernel against the mathematics (CPU only)."""
import numpy as np

from softmax_learned_covariance_b200 import exp2_poly


def test_kernel_coefficients_are_the_minimax_fit():
    c_fit, err = exp2_poly.remez_exp2(3)
    c_cu = exp2_poly.kernel_coefficients()
    assert np.max(np.abs(c_fit - c_cu)) < 1e-6
    assert err < 7.6e-5


def test_relative_error_bound_over_the_softmax_range():
    c = exp2_poly.kernel_coefficients()
    # the softmax evaluates x = z log2(e)/sqrt(d) - m_ref <= 8 (lazy rescale bound)
    x = np.concatenate([np.linspace(-124.0, 8.0, 2_000_001), np.arange(-124, 9, dtype=np.float64) + 0.5])
    y = exp2_poly.emulate_kernel_exp2(x, c).astype(np.float64)
    ref = np.exp2(x.astype(np.float32).astype(np.float64))
    rel = np.abs(y / ref - 1.0)
    assert rel.max() < 1.0e-4
    # whole numbers hit the polynomial at f = 0
    xi = np.arange(-124, 9, dtype=np.float64)
    yi = exp2_poly.emulate_kernel_exp2(xi, c).astype(np.float64)
    assert np.all(np.abs(yi / np.exp2(xi) - 1.0) < 1.0e-4)


def test_underflow_and_masked_scores_round_to_zero_in_fp16():
    c = exp2_poly.kernel_coefficients()
    x = np.array([-125.0, -126.5, -300.0, -1e30, -np.inf], dtype=np.float32)
    y = exp2_poly.emulate_kernel_exp2(x, c)
    assert np.all(np.isfinite(y)) and np.all(y >= 0)
    assert np.all(y.astype(np.float16) == 0)


def test_results_that_feed_fp16_match_the_exact_rounding_closely():
    # P is rounded to fp16 right after; the polynomial may move a rounding
    # decision by at most one fp16 ulp
    c = exp2_poly.kernel_coefficients()
    x = np.linspace(-24.0, 8.0, 200_001)
    y16 = exp2_poly.emulate_kernel_exp2(x, c).astype(np.float16).astype(np.float64)
    r16 = np.exp2(x).astype(np.float16).astype(np.float64)
    ulp = np.spacing(r16.astype(np.float16)).astype(np.float64)
    assert np.all(np.abs(y16 - r16) <= ulp)
