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


def _diag_row(a, tau):
    """[k*, cum_(k*-1), cum_(k*), tau*T, gap] of one row, from a plain sort."""
    order = sorted(range(len(a)), key=lambda j: (-a[j], j))
    s = np.asarray(a, np.float64)[order]
    cum = np.cumsum(s)
    k = int(np.argmax(cum >= tau * cum[-1])) + 1
    gap = s[k - 1] - s[k] if k < len(a) else np.inf
    return [k, cum[k - 2] if k > 1 else 0.0, cum[k - 1], tau * cum[-1], gap], sorted(order[:k])


def test_classify_masks_cases():
    from long_context_prefill_estimate_b200.diagnostics import classify_masks

    Nb, tau = 4, 0.75
    # one head per case; rows I = 0..2 agree, row I = 3 is the case (side b = the reference)
    cases = [
        # identical
        ([0.4, 0.3, 0.2, 0.1], [0.4, 0.3, 0.2, 0.1], None),
        # a score error of 3e-7 swaps two blocks next to the cut: a near tie
        ([0.4, 0.2, 0.2000001, 0.1999999], [0.4, 0.2000002, 0.1999998, 0.2], None),
        # side b's sum reaches tau*T exactly at the cut: a boundary row
        ([0.5, 0.25, 0.15, 0.1], [0.5, 0.25, 0.15, 0.1], [0, 1, 2]),
        # the same scores on both sides but a different set: unexplained
        ([0.7, 0.1, 0.1, 0.1], [0.7, 0.1, 0.1, 0.1], [0, 1, 2]),
    ]
    rows_a, rows_b, diag, A_a, A_b = [], [], [], [], []
    for b_scores, a_scores, a_override in cases:
        for I in range(Nb):
            sb = list(b_scores[:I + 1]) + [0.0] * (Nb - I - 1)
            sa = list(a_scores[:I + 1]) + [0.0] * (Nb - I - 1)
            d, sel_b = _diag_row(b_scores[:I + 1], tau)
            sel_a = _diag_row(a_scores[:I + 1], tau)[1]
            if I == Nb - 1 and a_override is not None:
                sel_a = a_override
            rows_a.append(sel_a)
            rows_b.append(sel_b)
            diag.append(d)
            A_a.append(sa)
            A_b.append(sb)
    counts, bad = classify_masks(rows_a, rows_b, np.array(diag), np.array(A_b), np.array(A_a))
    # the near-tie head also swaps its two near-equal blocks in row I = 2, whose sum there
    # sits within 1e-4 of tau*T, so that row counts as a boundary row
    assert counts["rows"] == 16 and counts["mismatch_rows"] == 4
    assert counts["near_tie_swaps"] == 1
    assert counts["mismatch_boundary"] == 2
    assert counts["sum_within_error"] == 0
    assert [r for r, _, _ in bad] == [15]
