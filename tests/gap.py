"""Score-gap enforcement for parity inputs (test infrastructure).

The CUDA path sums squared entries in fp32, the oracle in fp64.  Their index
sets agree bit for bit whenever the scores on the two sides of the selection
boundary are separated by more than fp32 summation error.  The workloads ask
for sorted scores at least 1e-3 apart (relative).  Across all d scores that is
infeasible at d >= 256 with log-normal scales, and only the boundary matters
for the returned (ascending) index set, so:
  * the tiny fp32 workload spreads ALL sorted scores >= 1.0011x apart by
    per-column gains (constructive, see all_gaps_gain);
  * every other workload checks the relative gap at each boundary k that the
    test uses and, where it is below 1e-3, scales every column ranked below
    that boundary by (1 - 2^-7) before the final rounding, then re-checks
    (enforce_boundary_gaps).
Scores are measured with the oracle; the generator only applies the gains.
"""
from __future__ import annotations

import numpy as np

import oracle

MIN_GAP = 1e-3
NUDGE = 1.0 - 2.0 ** -7


def descending_order(s2: np.ndarray) -> np.ndarray:
    d = s2.size
    return np.lexsort((np.arange(d), -s2))


def boundary_gap(s2: np.ndarray, k: int) -> float:
    d = s2.size
    if k >= d:
        return float("inf")
    s = np.sqrt(s2[descending_order(s2)])
    if s[k - 1] == 0.0:
        return 0.0
    return float((s[k - 1] - s[k]) / s[k - 1])


def all_gaps_gain(s2: np.ndarray, ratio: float = 1.0011) -> np.ndarray:
    order = descending_order(s2)
    s = np.sqrt(s2[order])
    t = s.copy()
    for r in range(len(t) - 2, -1, -1):
        t[r] = max(t[r], ratio * t[r + 1])
    gain = np.ones_like(s2)
    gain[order] = t / s
    return gain


def min_adjacent_gap(s2: np.ndarray) -> float:
    s = np.sqrt(s2[descending_order(s2)])
    return float(np.min((s[:-1] - s[1:]) / s[:-1]))


def enforce_boundary_gaps(make, score_sets, ks, max_iter: int = 8):
    """make(gain) -> inputs; score_sets(inputs) -> list of fp64 score vectors
    (one per head, or one); gains have the shape [len(score_sets), d].
    Returns (inputs, gain)."""
    gain = None
    for _ in range(max_iter):
        inputs = make(None if gain is None else (gain[0] if gain.shape[0] == 1 else gain))
        sets = score_sets(inputs)
        if gain is None:
            gain = np.ones((len(sets), sets[0].size))
        bad = False
        for h, s2 in enumerate(sets):
            order = descending_order(s2)
            for k in ks:
                if boundary_gap(s2, k) < MIN_GAP:
                    gain[h, order[k:]] *= NUDGE
                    bad = True
        if not bad:
            return inputs, gain
    raise RuntimeError("could not open the score gap at the selection boundary")


def scores_2d(A) -> list:
    return [oracle.column_scores_sq(A)]


def scores_per_head(X) -> list:
    return [oracle.column_scores_sq(X[h]) for h in range(X.shape[0])]
