"""Host checks of the parity measures used by the GPU tests (kda_cases): each one
sees the kind of error it is meant to see."""
from __future__ import annotations

import numpy as np
import pytest

from kda_cases import FLOOR, check_outputs, output_errors


def _ref(T=40, H=3, d=16, seed=0):
    return np.random.default_rng(seed).standard_normal((T, H, d))


def test_exact_result_has_zero_error():
    y = _ref()
    e = output_errors(y.copy(), y, [0, 10, 40])
    assert e["normwise"] == e["rowwise"] == e["elementwise"] == 0.0


def test_row_measure_sees_a_small_row_that_normwise_misses():
    y = _ref()
    y[7, 1] *= 1e-2                      # a row whose outputs nearly cancel
    x = y.copy()
    x[7, 1] += 5e-3 * np.abs(y[7, 1]).max() * 10      # 5% of that row's own size
    e = output_errors(x, y)
    assert e["normwise"] < 2e-2 < e["rowwise"]
    assert e["worst_row"] == (7, 1)
    with pytest.raises(AssertionError):
        check_outputs("o", x, y, 2e-2)


def test_rows_below_the_floor_are_measured_against_it():
    y = _ref()
    y[3, 0] = 0.0
    x = y.copy()
    x[3, 0] = 0.5 * FLOOR * np.abs(y[:, 0]).max() * 2e-2
    e = output_errors(x, y)
    assert e["rowwise"] <= 2e-2 and np.isfinite(e["elementwise"])


def test_sequences_are_separate_blocks():
    y = _ref()
    y[:20] *= 1e-3                       # first sequence much smaller than the second
    x = y.copy()
    x[:20] *= 1.05                       # 5% error, relative to its own block only
    assert output_errors(x, y, [0, 20, 40])["normwise"] == pytest.approx(0.05, rel=1e-6)
    assert output_errors(x, y)["normwise"] < 1e-3
