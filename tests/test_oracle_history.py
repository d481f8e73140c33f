"""Pins of the oracle's amax history (supplied tensor scale of a requantizing
epilogue): shift semantics and the closed-form tensor scale."""
import numpy as np
import pytest

import oracle


def test_shift_and_scale_closed_form():
    h = np.zeros(4, np.float32)
    seq = [10.5, 3.0, 42.0, 1.0, 0.5, 0.25]
    for n, a in enumerate(seq):
        h, g = oracle.amax_history_push(h, a)
        window = seq[max(0, n - 3):n + 1][::-1]  # newest first, at most 4
        assert list(h[:len(window)]) == [np.float32(x) for x in window]
        # 10.5 * 2^k / 2688 = 2^(k - 8) exactly; 42 = 10.5 * 4 -> 2^-6
        assert g == float(np.float32(max(window)) / np.float32(2688.0))
    h, g = oracle.amax_history_push(np.zeros(1, np.float32), 10.5 * 2.0 ** 5)
    assert g == 2.0 ** -3


def test_length_one_is_the_previous_call():
    h = np.array([7.0], np.float32)
    h, g = oracle.amax_history_push(h, 2688.0)
    assert h[0] == 2688.0 and g == 1.0


def test_nonfinite_is_rejected_and_changes_nothing():
    h = np.array([1.0, 2.0], np.float32)
    with pytest.raises(ValueError):
        oracle.amax_history_push(h, float("inf"))
    with pytest.raises(ValueError):
        oracle.amax_history_push(h, float("nan"))
