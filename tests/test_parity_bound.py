"""The output bound of the parity helpers (tests/parity.py), on the host: every
element of the GPU output within 2e-2 RMS(y) + 2^-8 |y| of the oracle's."""
import os
import sys

import numpy as np

sys.path.insert(0, os.path.dirname(os.path.abspath(__file__)))
import parity  # noqa: E402


def test_exact_match_scores_zero():
    y = np.random.default_rng(0).normal(size=(5, 7))
    assert parity.output_score(y, y) == 0.0


def test_bound_is_rms_term_plus_magnitude_term():
    yo = np.array([[0.0, 1.0, -1.0, 5.0]])
    rms = float(np.sqrt(np.mean(yo ** 2)))
    bound = parity.TOL_Y * rms + parity.TOL_Y_REL * np.abs(yo)
    inside = yo + 0.999 * bound * np.array([[1, -1, 1, -1]])
    outside = yo.copy()
    outside[0, 3] += 1.001 * bound[0, 3]
    assert parity.output_score(inside, yo) < parity.TOL_Y
    assert parity.output_score(outside, yo) >= parity.TOL_Y
    # the large element's allowance exceeds the RMS term alone
    assert bound[0, 3] > parity.TOL_Y * rms


def test_all_zero_oracle_needs_an_exact_zero():
    z = np.zeros((2, 3))
    assert parity.output_score(z, z) == 0.0
    assert parity.output_score(z + 1e-30, z) == float("inf")
