"""Host-side mask comparison of the selection-accuracy diagnostic (no GPU)."""
import numpy as np
import pytest

from long_context_prefill_estimate_b200.diagnostics import csr_to_mask, mask_metrics


def test_csr_to_mask_hand_worked():
    # H = 1, Nb = 3: rows I=0 -> {0}, I=1 -> {1}, I=2 -> {0, 2}
    rp = np.array([0, 1, 2, 4], np.int32)
    ci = np.array([0, 1, 0, 2], np.int32)
    m = csr_to_mask(rp, ci, 1, 3)
    expect = np.array([[[1, 0, 0], [0, 1, 0], [1, 0, 1]]], bool)
    assert np.array_equal(m, expect)


def test_metrics_identical_disjoint_and_partial():
    ref = np.array([[[1, 0], [1, 1]]], bool)
    mass = np.array([[[1.0, 0.0], [0.25, 0.75]]])
    same = mask_metrics(ref, ref, mass)
    assert same["precision"][0] == same["recall"][0] == same["f1"][0] == 1.0
    assert same["captured_mass"][0] == pytest.approx(1.0)
    part = np.array([[[1, 0], [0, 1]]], bool)          # drops (1, 0)
    m = mask_metrics(part, ref, mass)
    assert m["precision"][0] == 1.0
    assert m["recall"][0] == pytest.approx(2 / 3)
    assert m["f1"][0] == pytest.approx(0.8)
    assert m["captured_mass"][0] == pytest.approx((1.0 + 0.75) / 2)
    other = np.array([[[0, 0], [1, 0]]], bool)
    m = mask_metrics(other, np.array([[[1, 0], [0, 1]]], bool), mass)
    assert m["precision"][0] == 0.0 and m["recall"][0] == 0.0 and m["f1"][0] == 0.0
