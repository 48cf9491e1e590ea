"""Rows cut into column slices across ranks (vocabulary- or entity-parallel).

split_row_topk takes score rows; split_score_topk takes the key matrices of
the fused scorers, split by keys.

Each rank holds columns [offset, offset + n_local) of the same rows.  It runs
the bucketed selection on its slice, the (value, index) candidate lists of all
ranks are all-gathered -- the one exchange of the method when a row is split
-- and `topk_bucketed_merge` finishes with buckets taken by global index
modulo b ("Approximate Top-k for Increased Parallelism", pith.science review
page, "What carries the argument"; "The reading").  The result equals the
single-pass selection of the whole rows, bit for bit, for any cut points.

A slice's own selection may use local indices: its positions fall into the
same residue classes as their global indices shifted by one offset, so it
keeps the same elements; the merge adds the offsets.

The collectives are plain torch.distributed calls (NCCL between GPUs, into
device memory; with a host backend such as gloo the small candidate lists are
gathered on the host); every rank calls them in the same order.
"""
from __future__ import annotations

import torch
import torch.distributed as dist

from . import _binding


def column_slices(n_total: int, world: int) -> list[tuple[int, int]]:
    """Contiguous (offset, length) slices of [0, n_total), as even as possible."""
    if world < 1 or n_total < world:
        raise ValueError("need 1 <= world <= n_total")
    base, extra = divmod(n_total, world)
    out, off = [], 0
    for r in range(world):
        ln = base + (1 if r < extra else 0)
        out.append((off, ln))
        off += ln
    return out


def _on_device(group) -> bool:
    """NCCL gathers device tensors; host backends (gloo) gather host tensors."""
    return dist.get_backend(group) == "nccl"


def gather_offsets(offset: int, group=None, device=None) -> list[int]:
    """Every rank's column offset, in rank order."""
    world = dist.get_world_size(group)
    dev = device if _on_device(group) else "cpu"
    t = torch.tensor([int(offset)], dtype=torch.int64, device=dev)
    parts = [torch.empty_like(t) for _ in range(world)]
    dist.all_gather(parts, t, group=group)
    return [int(p.item()) for p in parts]


def gather_candidates(vals: torch.Tensor, idx: torch.Tensor, group=None):
    """All-gather per-rank candidate lists [rows, m] into [world, rows, m] on
    the lists' device.  NCCL gathers straight into device memory (one
    all_gather_into_tensor per array, ~8 bytes x m per row and rank); a host
    backend gathers copies on the host and the result is copied back."""
    world = dist.get_world_size(group)
    vals, idx = vals.contiguous(), idx.contiguous()
    if _on_device(group):
        out_v = torch.empty((world,) + tuple(vals.shape), dtype=vals.dtype, device=vals.device)
        out_i = torch.empty((world,) + tuple(idx.shape), dtype=idx.dtype, device=idx.device)
        dist.all_gather_into_tensor(out_v, vals, group=group)
        dist.all_gather_into_tensor(out_i, idx, group=group)
        return out_v, out_i
    hv, hi = vals.cpu(), idx.cpu()
    out_v = torch.empty((world,) + tuple(hv.shape), dtype=hv.dtype)
    out_i = torch.empty((world,) + tuple(hi.shape), dtype=hi.dtype)
    dist.all_gather(list(out_v.unbind(0)), hv, group=group)
    dist.all_gather(list(out_i.unbind(0)), hi, group=group)
    return out_v.to(vals.device), out_i.to(idx.device)


def _all_offsets(offset: int, offsets, group, device) -> list[int]:
    if offsets is None:
        return gather_offsets(offset, group, device=device)
    offsets = [int(o) for o in offsets]
    if len(offsets) != dist.get_world_size(group) or offsets[dist.get_rank(group)] != int(offset):
        raise ValueError("offsets must list every rank's column offset, this rank's included")
    return offsets


def split_row_topk(x_local: torch.Tensor, offset: int, n_total: int, k: int, b: int, kb: int,
                   group=None, offsets=None):
    """Bucketed top-k of rows whose columns are spread over the ranks.

    x_local: this rank's [rows, n_local] float32 slice on its GPU, starting at
    global column `offset`.  offsets: every rank's column offset in rank order,
    when the caller knows them (else they are all-gathered, which costs a
    host synchronisation per call).  Returns (values, global indices)
    [rows, k] on every rank.
    """
    v, i = _binding.topk_bucketed(x_local, k, b, kb)
    offs = _all_offsets(offset, offsets, group, x_local.device)
    V, I = gather_candidates(v, i, group)
    return _binding.topk_bucketed_merge(V, I, n_total, k, b, kb, part_offsets=offs)


def split_score_topk(q: torch.Tensor, K_local: torch.Tensor, offset: int, n_total: int, k: int, b: int,
                     kb: int, group=None, offsets=None):
    """Fused scoring and bucketed top-k with the keys split by rows across the
    ranks (entity- or sequence-parallel): this rank holds keys
    [offset, offset + n_local) of every row's key matrix.

    q: [rows, d] bf16, the same on every rank; K_local: [rows, n_local, d] or
    [n_local, d] bf16; offsets as in split_row_topk.  Returns (values, global
    indices) [rows, k] on every rank, equal to the selection over the ranks'
    own fp32 scores of their key slices.
    """
    v, i = _binding.score_topk(q, K_local, k, b, kb)
    offs = _all_offsets(offset, offsets, group, q.device)
    V, I = gather_candidates(v, i, group)
    return _binding.topk_bucketed_merge(V, I, n_total, k, b, kb, part_offsets=offs)
