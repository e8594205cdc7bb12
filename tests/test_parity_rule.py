"""The parity bars' rule for the two precision readings (host logic, no GPU).

Against the bf16 model the bars hold as stated; against float64 activations each measure may reach
the readings' own gap plus half a bar where that gap exceeds half a bar, and no further.
"""
import numpy as np
import pytest

from parity import MAX_ABS, check_readings


def _rows(seed):
    return np.random.default_rng(seed).standard_normal((6, 256))


def _bump(x, amount):
    y = x.copy()
    y[2, 7] += amount          # one element: moves the max-abs, barely the relative L1
    return y


def test_plain_bar_against_the_model_reading():
    f64 = _rows(1)
    check_readings(_bump(f64, 0.9 * MAX_ABS), {"bf16 model": f64}, "within")
    with pytest.raises(AssertionError):
        check_readings(_bump(f64, 1.2 * MAX_ABS), {"bf16 model": f64}, "beyond")


def test_float64_reading_bar_follows_the_readings_gap():
    f64 = _rows(2)
    model = _bump(f64, 1.5 * MAX_ABS)            # the readings themselves differ by more than the bar
    refs = {"bf16 model": model, "float64 activations": f64}
    check_readings(model, refs, "equal to the model")
    check_readings(_bump(model, 0.4 * MAX_ABS), refs, "a little further from float64")
    with pytest.raises(AssertionError):          # gap + 0.6 bar: beyond gap + bar / 2
        check_readings(_bump(model, 0.6 * MAX_ABS), refs, "too far from float64")


def test_small_gap_keeps_the_plain_bar():
    f64 = _rows(3)
    model = _bump(f64, 0.2 * MAX_ABS)
    refs = {"bf16 model": model, "float64 activations": f64}
    with pytest.raises(AssertionError):          # 0.2 + 0.9 bar from float64: beyond max(bar, 0.7 bar)
        check_readings(_bump(model, 0.9 * MAX_ABS), refs, "plain bar")
