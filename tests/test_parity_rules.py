"""The routing comparison rule itself (host logic, CPU)."""
import numpy as np

from parity import compare_route_row, compare_routes


def test_exact_match_and_order():
    a = np.array([0.1, 5.0, 3.0, -1.0, 4.0])
    assert compare_route_row(a, [1, 4, 2], 3) == (True, False)
    assert compare_route_row(a, [4, 1, 2], 3) == (False, False)  # order across clear gaps
    assert compare_route_row(a, [1, 4, 0], 3) == (False, False)  # wrong set


def test_tie_inside_topk_compares_as_set():
    a = np.array([2.0, 2.0 + 1e-9, 1.0, 0.0])
    assert compare_route_row(a, [1, 0, 2], 3) == (True, False)
    assert compare_route_row(a, [0, 1, 2], 3) == (True, False)


def test_tie_straddling_k_is_ambiguous_but_checked():
    a = np.array([3.0, 1.0, 1.0 + 1e-8, 0.0])
    assert compare_route_row(a, [0, 1], 2) == (True, True)
    assert compare_route_row(a, [0, 2], 2) == (True, True)
    assert compare_route_row(a, [0, 3], 2) == (False, True)   # 3 is not in the tie
    assert compare_route_row(a, [1, 0], 2) == (False, False)  # first cluster misplaced


def test_duplicates_and_range_rejected():
    a = np.array([3.0, 2.0, 1.0])
    assert compare_route_row(a, [0, 0], 2)[0] is False
    assert compare_route_row(a, [0, 3], 2)[0] is False


def test_full_topk_is_a_set():
    a = np.array([3.0, 2.0, 1.0])
    assert compare_route_row(a, [0, 1, 2], 3) == (True, False)


def test_compare_routes_counts():
    a = np.zeros((1, 1, 2, 3))
    a[0, 0, 0] = [3.0, 2.0, 1.0]
    a[0, 0, 1] = [1.0, 1.0, 0.0]
    idx = np.array([[[[0, 1], [1, 0]]]])
    rep = compare_routes(idx, a)
    assert rep.rows == 2 and not rep.mismatches and rep.ambiguous == 0
    idx2 = np.array([[[[1, 0], [0, 2]]]])
    rep = compare_routes(idx2, a)
    assert len(rep.mismatches) == 2
