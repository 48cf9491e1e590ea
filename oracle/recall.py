"""Recall of bucketed top-k: the method's formulas (TEST INFRASTRUCTURE ONLY).

Source: "Approximate Top-k for Increased Parallelism" (arXiv 2412.04358),
pith.science review page:
  - Eq. (1) ("What carries the argument"): expected recall on inputs whose top
    values fall in buckets uniformly at random,
        E[R(k, b, k_b)] = (1/k) * (k_b + sum_{i=k_b}^{k-1} F(k_b - 1; i, 1/b)),
    with F read as the binomial CDF  F(x; m, p) = P[Binomial(m, p) <= x].
  - Eq. (2) (same section, and "What would settle it"): the worst case, when
    all top values sit in as few buckets as possible -- ceil(b*k/n) of them.
    The formula itself is not printed on the page; it is restated here from
    that description (a reading).
  - Referee report, major comment 1 / Appendix C note: Eq. (1) is read as a
    lower bound on the expected recall (an upper bound on the recall error).

Finite-n expectation (a reading that the pages imply but do not print): with
interleaved buckets every bucket has exactly s = n/b slots, so the bucket of the
rank-(i+1) element holds a hypergeometric, not binomial, number of the i larger
elements.  `expected_recall_exact` is that exact value; Eq. (1) is its
with-replacement approximation.
"""
from __future__ import annotations

import math
from fractions import Fraction

import numpy as np


def eq1_expected_recall(k: int, b: int, kb: int) -> float:
    """Eq. (1): (1/k) (k_b + sum_{i=k_b}^{k-1} P[Bin(i, 1/b) <= k_b - 1])."""
    if kb >= k:
        return 1.0
    p = 1.0 / b
    total = float(kb)
    for i in range(kb, k):
        cdf = 0.0
        for j in range(0, kb):
            cdf += math.comb(i, j) * p ** j * (1.0 - p) ** (i - j)
        total += cdf
    return total / k


def expected_recall_exact(n: int, k: int, b: int, kb: int) -> float:
    """Exact expected recall for iid continuous rows with b | n.

    The rank-(i+1) element is retrieved iff fewer than k_b of the i larger
    elements share its bucket; that count is Hypergeometric(N=n-1, K=s-1, i).
    An element of rank <= k that survives Stage 1 always survives Stage 2
    (fewer than k candidates can beat it), so recall = mean over ranks.
    """
    if n % b:
        raise ValueError("exact expectation is stated for b | n")
    s = n // b
    N, K = n - 1, s - 1
    total = Fraction(0)
    for i in range(k):
        denom = math.comb(N, i)
        num = 0
        for x in range(0, min(kb - 1, K, i) + 1):
            num += math.comb(K, x) * math.comb(N - K, i - x)
        total += Fraction(num, denom)
    return float(total / k)


def eq2_worst_recall(n: int, k: int, b: int, kb: int) -> float:
    """Eq. (2) as read from the page: all top-k values packed into the fewest
    buckets, ceil(k/s) of them with s = n/b slots each.  Each full bucket gives
    min(k_b, s) of them, the partly filled one min(k_b, k mod s)."""
    if n % b:
        raise ValueError("worst case is stated for b | n")
    s = n // b
    full, rest = divmod(k, s)
    return (min(kb, s) * full + min(kb, rest)) / k


def recall(selected_idx, exact_idx) -> np.ndarray:
    """Per-row recall |S_bucketed & S_exact| / |S_exact| (padding -1 ignored)."""
    sel = np.atleast_2d(np.asarray(selected_idx))
    ex = np.atleast_2d(np.asarray(exact_idx))
    out = np.empty(sel.shape[0])
    for r in range(sel.shape[0]):
        e = set(int(v) for v in ex[r] if v >= 0)
        s = set(int(v) for v in sel[r] if v >= 0)
        out[r] = len(e & s) / max(1, len(e))
    return out
