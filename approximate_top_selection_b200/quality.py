"""Recall of the bucketed selection on correlated rows: interleaved against
contiguous bucket assignment.

"Approximate Top-k for Increased Parallelism" (pith.science review page,
"Core claim" and Appendix A.1 / Fig. 6): real scores are correlated along the
row, and the method relies on interleaved buckets (element i in bucket i mod b)
to spread the top values over the buckets; with contiguous buckets (element i
in bucket i div s, s = n / b) a run of large neighbours lands in one bucket and
recall drops.  The study draws stationary AR(1) Gaussian rows
(`inputs.ar1_rows`) and measures recall = |selected ∩ exact top-k| / k.

Contiguous assignment runs through the same CUDA kernel on a transposed copy of
the row: position t*b + j of the copy holds element j*s + t, so interleaved
bucket j of the copy is contiguous bucket j of the row, and a selected position
p maps back to (p mod b) * s + p div b.  (The copy's index order differs from
the row's, so ties may resolve differently; on continuous rows there are none
in practice.)  Recall itself is counted with PyTorch on the device: this is an
evaluation harness, not part of the selection path.

Run `python -m approximate_top_selection_b200.quality` on a GPU for the table.
"""
from __future__ import annotations

import argparse
import json

import torch

from . import _binding, inputs


def contiguous_view(x: torch.Tensor, b: int) -> torch.Tensor:
    """Copy of rows x [rows, n] (b | n) whose interleaved buckets are x's contiguous ones."""
    rows, n = x.shape
    if n % b:
        raise ValueError("contiguous buckets need b | n")
    return x.reshape(rows, b, n // b).transpose(1, 2).contiguous().reshape(rows, n)


def contiguous_index(p: torch.Tensor, n: int, b: int) -> torch.Tensor:
    """Row index of position p of contiguous_view (p >= 0)."""
    s = n // b
    return (p % b) * s + torch.div(p, b, rounding_mode="floor")


def _recall(sel: torch.Tensor, exact: torch.Tensor, k: int) -> torch.Tensor:
    hit = (sel[:, :, None] == exact[:, None, :]) & (sel[:, :, None] >= 0)
    count = hit.any(dim=2).sum(dim=1).to(torch.float64)
    # a tensor divisor keeps the division correctly rounded (count / k exactly)
    return count / torch.full_like(count, float(k))


def assignment_recall(x: torch.Tensor, k: int, b: int, kb: int):
    """Per-row recall (interleaved, contiguous) of the bucketed top-k of x [rows, n] on the GPU."""
    n = x.shape[1]
    _, exact = _binding.topk_exact(x, k)
    _, inter = _binding.topk_bucketed(x, k, b, kb)
    _, cpos = _binding.topk_bucketed(contiguous_view(x, b), k, b, kb)
    cont = torch.where(cpos >= 0, contiguous_index(cpos.long(), n, b), cpos.long()).to(torch.int32)
    return _recall(inter, exact, k), _recall(cont, exact, k)


def study(rows: int = 256, n: int = 131072, k: int = 512, b: int = 256, kb: int = 2,
          rhos=(0.0, 0.5, 0.9, 0.99, 0.999), seed: int = 0x6A0, device="cuda"):
    out = []
    for i, rho in enumerate(rhos):
        x = inputs.ar1_rows(rows, n, rho, seed + i, device=device)
        ri, rc = assignment_recall(x, k, b, kb)
        out.append({"rho": rho, "interleaved": float(ri.mean()), "contiguous": float(rc.mean()),
                    "interleaved_min": float(ri.min()), "contiguous_min": float(rc.min())})
    return out


def main():
    ap = argparse.ArgumentParser(description=__doc__.split("\n")[0])
    ap.add_argument("--rows", type=int, default=256)
    ap.add_argument("--n", type=int, default=131072)
    ap.add_argument("--k", type=int, default=512)
    ap.add_argument("--b", type=int, default=256)
    ap.add_argument("--kb", type=int, default=2)
    a = ap.parse_args()
    res = study(a.rows, a.n, a.k, a.b, a.kb)
    print(json.dumps({"rows": a.rows, "n": a.n, "k": a.k, "b": a.b, "kb": a.kb, "ar1": res}))


if __name__ == "__main__":
    main()
