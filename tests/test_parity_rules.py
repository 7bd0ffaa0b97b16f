"""The comparison rules the GPU parity tests apply (oracle/parity.py), checked on
hand-made cases: exact sets pass, a changed set fails unless the oracle's K-th
and (K+1)-th scores are near-tied, order changes pass only between near-tied
neighbours, padding is part of the set, and outputs fail above the tolerance
or when not finite."""
import numpy as np
import pytest

from oracle.parity import ATOL, NEAR_TIE_REL, ParityReport, compare_outputs, compare_selection

INF = np.inf


def one(idx, sbar, gap, mag=None):
    """A single (row, group) as the arrays compare_selection takes: idx, sbar
    [1, 1, K], gap [1, 1], smag [1, 1, K+1].  Unless given, the magnitudes are
    those of scores whose terms do not cancel: |score| (the (K+1)-th one's
    from the gap)."""
    if mag is None:
        sk = sbar[len(idx) - 1]
        mag = [abs(v) for v in sbar] + [abs(sk - gap) if np.isfinite(gap) else 0.0]
    return (np.array([[idx]], dtype=np.int32), np.array([[sbar]], dtype=np.float64),
            np.array([[gap]], dtype=np.float64), np.array([[mag]], dtype=np.float64))


def test_identical_selection_passes():
    ri, rs, rg, rm = one([4, 1, 7], [3.0, 2.0, 1.0], 0.5)
    rep = ParityReport()
    differs = compare_selection(ri, rs, rg, rm, ri.copy(), rep)
    assert rep.ok and not differs.any() and rep.near_ties == 0 and rep.set_mismatch == 0


def test_changed_set_fails_without_a_near_tie():
    ri, rs, rg, rm = one([4, 1, 7], [3.0, 2.0, 1.0], 0.5)
    rep = ParityReport()
    differs = compare_selection(ri, rs, rg, rm, np.array([[[4, 1, 9]]], dtype=np.int32), rep)
    assert not rep.ok and differs.all() and rep.set_mismatch == 1


def test_changed_set_is_accepted_at_a_near_tie():
    gap = 0.5 * NEAR_TIE_REL * 1.0                  # K-th score 1.0, (K+1)-th 1.0 - gap
    ri, rs, rg, rm = one([4, 1, 7], [3.0, 2.0, 1.0], gap)
    rep = ParityReport()
    differs = compare_selection(ri, rs, rg, rm, np.array([[[4, 1, 9]]], dtype=np.int32), rep)
    assert rep.ok and differs.all() and rep.near_ties == 1 and rep.set_mismatch == 1


def test_gap_just_above_the_near_tie_bound_fails():
    gap = 2.0 * NEAR_TIE_REL * 1.0
    ri, rs, rg, rm = one([4, 1, 7], [3.0, 2.0, 1.0], gap)
    rep = ParityReport()
    compare_selection(ri, rs, rg, rm, np.array([[[4, 1, 9]]], dtype=np.int32), rep)
    assert not rep.ok and rep.near_ties == 0


def test_order_swap_only_between_near_tied_neighbours():
    eps = 0.1 * NEAR_TIE_REL
    ri, rs, rg, rm = one([4, 1, 7], [3.0, 2.0, 2.0 - eps], 0.5)
    rep = ParityReport()
    compare_selection(ri, rs, rg, rm, np.array([[[4, 7, 1]]], dtype=np.int32), rep)
    assert rep.ok and rep.order_mismatch == 1
    ri, rs, rg, rm = one([4, 1, 7], [3.0, 2.0, 1.0], 0.5)
    rep = ParityReport()
    compare_selection(ri, rs, rg, rm, np.array([[[1, 4, 7]]], dtype=np.int32), rep)
    assert not rep.ok


def test_padding_is_part_of_the_set():
    # two visible chunks, K = 3: the third slot is padding on both sides
    ri, rs, rg, rm = one([5, 0, -1], [1.0, 0.5, 0.0], INF)
    rep = ParityReport()
    compare_selection(ri, rs, rg, rm, np.array([[[5, 0, -1]]], dtype=np.int32), rep)
    assert rep.ok and rep.near_ties == 0
    rep = ParityReport()
    compare_selection(ri, rs, rg, rm, np.array([[[5, 0, 3]]], dtype=np.int32), rep)
    assert not rep.ok


@pytest.mark.parametrize("dtype", ["bf16", "f32"])
def test_output_tolerance(dtype):
    ref = np.zeros((2, 3))
    rep = ParityReport()
    compare_outputs(ref, ref + 0.9 * ATOL[dtype], ATOL[dtype], rep)
    assert rep.ok and rep.max_abs_err == pytest.approx(0.9 * ATOL[dtype])
    rep = ParityReport()
    compare_outputs(ref, ref + 1.1 * ATOL[dtype], ATOL[dtype], rep)
    assert not rep.ok
    bad = ref.copy()
    bad[1, 2] = np.nan
    rep = ParityReport()
    compare_outputs(ref, bad, ATOL[dtype], rep)
    assert not rep.ok


def test_near_tie_is_relative_to_the_magnitude_of_the_score_terms():
    # K-th and (K+1)-th scores that cancel to nearly zero (1e-3 and 1e-3 - 1e-7)
    # out of terms of magnitude 5: the gap is 2e-8 of that magnitude, far below
    # what an fp32 evaluation resolves, so a swapped set is a near-tie; the same
    # gap between scores whose terms do not cancel is not.
    mag = [9.0, 7.0, 5.0, 5.0]
    ri, rs, rg, rm = one([4, 1, 7], [3.0, 2.0, 1e-3], 1e-7, mag)
    rep = ParityReport()
    differs = compare_selection(ri, rs, rg, rm, np.array([[[4, 1, 9]]], dtype=np.int32), rep)
    assert rep.ok and differs.all() and rep.near_ties == 1
    ri, rs, rg, rm = one([4, 1, 7], [3.0, 2.0, 1e-3], 1e-7)
    rep = ParityReport()
    compare_selection(ri, rs, rg, rm, np.array([[[4, 1, 9]]], dtype=np.int32), rep)
    assert not rep.ok and rep.near_ties == 0
