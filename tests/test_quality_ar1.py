"""Correlated rows (AR(1) Gaussian) and the bucket assignment study, on the CPU.

- the AR(1) input recipe against its definition (unit variance, lag-l
  correlation rho^l);
- contiguous assignment through a transposed copy (quality.contiguous_view)
  against contiguous buckets written out by definition on tiny rows;
- the page's assignment claim ("Approximate Top-k for Increased Parallelism",
  Appendix A.1 / Fig. 6) on the oracle: without correlation both assignments
  sit in the iid recall band; with it, interleaved recall does not fall below
  the iid expectation while contiguous recall collapses.
"""
import numpy as np
import pytest
import torch

from approximate_top_selection_b200 import inputs, quality
from oracle import recall as rc


@pytest.mark.parametrize("rho", [0.0, 0.5, 0.9, 0.99])
def test_ar1_recipe(rho):
    x = inputs.ar1_rows(4, 100000, rho, 3).numpy().astype(np.float64)
    assert abs(x.var() - 1.0) < (0.03 if rho < 0.95 else 0.08)
    for lag in (1, 2):
        c = np.mean([np.corrcoef(r[:-lag], r[lag:])[0, 1] for r in x])
        assert abs(c - rho ** lag) < 0.01
    # stationary from the first element on
    first = inputs.ar1_rows(4000, 2, rho, 5).numpy()[:, 0]
    assert abs(first.var() - 1.0) < 0.08


def _contiguous_by_definition(row, k, b, kb):
    n = row.size
    s = n // b
    cand = []
    for j in range(b):
        idx = np.arange(j * s, (j + 1) * s)
        order = sorted(idx, key=lambda i: (-row[i], i))
        cand.extend(order[:kb])
    cand = sorted(cand, key=lambda i: (-row[i], i))
    return cand[:k]


@pytest.mark.parametrize("n,k,b,kb", [(64, 8, 8, 1), (96, 10, 4, 3), (120, 30, 12, 2)])
def test_contiguous_view_is_contiguous_assignment(oracle_mod, n, k, b, kb):
    x = inputs.ar1_rows(6, n, 0.9, n + k)
    xc = quality.contiguous_view(x, b)
    _, ci = oracle_mod.bucketed(xc.numpy(), k, b, kb)
    got = quality.contiguous_index(torch.from_numpy(ci).long(), n, b).numpy()
    for r in range(x.shape[0]):
        want = _contiguous_by_definition(x[r].numpy(), k, b, kb)
        m = min(k, len(want))
        assert sorted(got[r, :m].tolist()) == sorted(want)


def _recalls(oracle_mod, rows, n, k, b, kb, rho, seed):
    x = inputs.ar1_rows(rows, n, rho, seed)
    _, ei = oracle_mod.exact(x.numpy(), k)
    _, ii = oracle_mod.bucketed(x.numpy(), k, b, kb)
    _, cp = oracle_mod.bucketed(quality.contiguous_view(x, b).numpy(), k, b, kb)
    ci = quality.contiguous_index(torch.from_numpy(cp).long(), n, b).numpy()
    return rc.recall(ii, ei), rc.recall(ci, ei)


def test_assignment_study_on_the_oracle(oracle_mod):
    rows, n, k, b, kb = 300, 8192, 128, 64, 2
    e = rc.expected_recall_exact(n, k, b, kb)
    ri, rcn = _recalls(oracle_mod, rows, n, k, b, kb, 0.0, 21)
    for r in (ri, rcn):
        assert abs(r.mean() - e) <= 4 * r.std() / np.sqrt(rows)
    for rho, seed in ((0.9, 22), (0.99, 23)):
        ri, rcn = _recalls(oracle_mod, rows, n, k, b, kb, rho, seed)
        assert ri.mean() >= e - 4 * ri.std() / np.sqrt(rows)
        assert rcn.mean() <= ri.mean() - 0.2
