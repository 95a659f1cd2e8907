"""Comparison rules between the CUDA path and the float64 oracle.

Routing: top-k is decided by floating point, and the GPU forms A^r in fp32
while the oracle uses float64, so rows whose k-th and (k+1)-th affinities
nearly tie may legitimately differ.  The rule, per row of the oracle's
affinities sorted descending a_(1) >= ... >= a_(R), with
thr(x, y) = rel * max(|x|, |y|, 1e-30), rel = 1e-4:

  * the sorted list is cut into clusters wherever a gap exceeds thr;
  * every cluster that lies wholly inside the first k positions must hold
    exactly the same regions, at the same positions as a set, on the GPU
    (so the set of the row and the order between clusters are bit-exact);
  * a cluster that straddles position k makes the row's set ambiguous: the
    GPU's pick there is only checked to be valid (distinct regions, each
    within thr of a_(k) or above it), and the row is counted as ambiguous.

Attention: O is compared with the oracle's token attention evaluated on the
GPU's own routing (so ambiguous rows are pinned too), max-abs error within
1e-4 for fp32 and 2e-2 for bf16.
"""
from __future__ import annotations

import dataclasses

import numpy as np

REL_GAP = 1e-4
TOL = {"f32": 1e-4, "bf16": 2e-2}

# (case, max-abs error, tolerance, ambiguous routing rows, routing rows) of
# every GPU parity comparison in this process, printed at the end of the
# pytest run (tests/conftest.py) so the margin to the tolerance is on record.
MARGINS: list[tuple[str, float, float, int, int]] = []


def record_margin(case: str, err: float, tol: float, ambiguous: int = 0, rows: int = 0) -> None:
    MARGINS.append((case, float(err), float(tol), int(ambiguous), int(rows)))


@dataclasses.dataclass
class RouteReport:
    rows: int = 0
    ambiguous: int = 0
    mismatches: list = dataclasses.field(default_factory=list)


def _thr(x: float, y: float) -> float:
    return REL_GAP * max(abs(x), abs(y), 1e-30)


def compare_route_row(a_row: np.ndarray, got: np.ndarray, k: int):
    """Returns (ok, ambiguous) for one row; see the module docstring."""
    R = a_row.shape[0]
    order = sorted(range(R), key=lambda s: (-a_row[s], s))
    vals = a_row[order]
    got = [int(x) for x in got]
    if len(set(got)) != k or any(g < 0 or g >= R for g in got):
        return False, False
    start = 0
    ambiguous = False
    for p in range(1, R + 1):
        if p == R or abs(vals[p - 1] - vals[p]) > _thr(vals[p - 1], vals[p]):
            lo, hi = start, p  # cluster [lo, hi)
            if lo >= k:
                break
            if hi <= k:
                if set(got[lo:hi]) != set(order[lo:hi]):
                    return False, False
            else:
                ambiguous = True
                members = set(order[lo:hi])
                if not set(got[lo:k]) <= members:
                    return False, True
            start = p
    return True, ambiguous


def compare_routes(idx_gpu: np.ndarray, a_oracle: np.ndarray) -> RouteReport:
    B, heads, R, k = idx_gpu.shape
    rep = RouteReport()
    for b in range(B):
        for h in range(heads):
            for r in range(R):
                ok, amb = compare_route_row(a_oracle[b, h, r], idx_gpu[b, h, r], k)
                rep.rows += 1
                rep.ambiguous += int(amb)
                if not ok:
                    rep.mismatches.append((b, h, r, list(idx_gpu[b, h, r])))
    return rep
