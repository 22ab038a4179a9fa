"""The selection comparator: which GPU selections it accepts against the oracle's scores."""
import numpy as np

from oracle.checks import TIE_ABS, TIE_REL, selection_ok

# 20 pages of 16 tokens; sink = page 0, recency = pages 18, 19; budget 4 of the 17 candidates
N_TOK, K, SINK, REC = 320, 4, 16, 32


def scores(*pairs, base=0.01):
    S = np.full(20, base)
    for j, v in pairs:
        S[j] = v
    return S


def check(sel, S):
    return selection_ok(sel, S, N_TOK, K, SINK, REC)


def test_exact_selection():
    S = scores((3, 0.5), (7, 0.4), (9, 0.3), (12, 0.2))
    ok, exact, ref = check([0, 3, 7, 9, 12, 18, 19], S)
    assert ok and exact and ref == [0, 3, 7, 9, 12, 18, 19]


def test_swap_inside_the_relative_band_is_accepted():
    S = scores((3, 0.5), (7, 0.4), (9, 0.3), (12, 0.2), (14, 0.2 * (1 - TIE_REL / 4)))
    ok, exact, _ = check([0, 3, 7, 9, 14, 18, 19], S)
    assert ok and not exact


def test_swap_outside_the_band_is_rejected():
    S = scores((3, 0.5), (7, 0.4), (9, 0.3), (12, 0.2), (14, 0.2 * (1 - 4 * TIE_REL)))
    ok, _, _ = check([0, 3, 7, 9, 14, 18, 19], S)
    assert not ok


def test_swap_of_a_sure_page_is_rejected():
    # 12 and 14 tie, but dropping page 9 (well above the k-th score) is a real error
    S = scores((3, 0.5), (7, 0.4), (9, 0.3), (12, 0.2), (14, 0.2))
    ok, _, _ = check([0, 3, 7, 12, 14, 18, 19], S)
    assert not ok


def test_scores_below_the_fixed_point_resolution_may_swap():
    # a peaked distribution: three clear pages, the rest far below the GPU's 2^-55 score unit
    S = scores((3, 0.9), (7, 0.05), (9, 0.04), base=0.0)
    S[10:18] = np.geomspace(1e-18, 1e-20, 8)
    ok_ref, exact, ref = check([0, 3, 7, 9, 10, 18, 19], S)
    assert ok_ref and exact and ref == [0, 3, 7, 9, 10, 18, 19]
    ok, _, _ = check([0, 3, 7, 11, 9, 18, 19], S)
    assert not ok  # not ascending: rejected whatever the scores
    ok, exact, _ = check([0, 3, 7, 9, 11, 18, 19], S)
    assert ok and not exact
    assert 1e-18 < TIE_ABS


def test_forced_pages_must_be_present():
    S = scores((3, 0.5), (7, 0.4), (9, 0.3), (12, 0.2), (14, 0.2))
    ok, _, _ = check([3, 7, 9, 12, 14, 18, 19], S)
    assert not ok


def test_wrong_length_is_rejected():
    S = scores((3, 0.5), (7, 0.4), (9, 0.3), (12, 0.2), (14, 0.2))
    ok, _, _ = check([0, 3, 7, 9, 12, 14, 18, 19], S)
    assert not ok
