"""Rows cut into column slices across ranks (host side, CPU).

The slicing and the all-gather layout of `approximate_top_selection_b200.sharded`
run here over two gloo ranks; each rank's selection and the final merge are
done by the oracle, so the test checks that slice offsets and gathered lists
line up such that the merge equals the single pass over the whole rows.
"""
import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

from approximate_top_selection_b200 import inputs, sharded


def test_column_slices_cover_the_row():
    for n, w in [(10, 1), (10, 3), (131072, 8), (1001, 7), (5, 5)]:
        s = sharded.column_slices(n, w)
        assert len(s) == w
        assert s[0][0] == 0 and sum(ln for _, ln in s) == n
        assert all(s[i][0] + s[i][1] == s[i + 1][0] for i in range(w - 1))
        assert max(ln for _, ln in s) - min(ln for _, ln in s) <= 1
    with pytest.raises(ValueError):
        sharded.column_slices(3, 4)


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    p = s.getsockname()[1]
    s.close()
    return p


CASES = [  # rows, n, k, b, kb, kind
    (4, 3001, 64, 128, 1, "normal"),
    (4, 2500, 40, 7, 3, "integer"),
    (3, 777, 100, 16, 2, "special"),
    (2, 4096, 512, 256, 4, "uniform"),
]


def _rows(kind, rows, n, seed):
    if kind == "normal":
        return inputs.normal_rows(rows, n, seed)
    if kind == "uniform":
        return inputs.uniform_rows(rows, n, seed)
    if kind == "integer":
        return inputs.integer_rows(rows, n, 9, seed)
    return inputs.special_rows(rows, n, seed)


def _worker(rank, world, port, out):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    import oracle

    oracle.build()
    oracle.set_threads(1)
    ok = []
    for ci, (rows, n, k, b, kb, kind) in enumerate(CASES):
        x = _rows(kind, rows, n, 1000 + ci).numpy()
        off, ln = sharded.column_slices(n, world)[rank]
        v, i = oracle.bucketed(np.ascontiguousarray(x[:, off:off + ln]), k, b, kb)  # local indices
        offsets = sharded.gather_offsets(off)
        V, I = sharded.gather_candidates(torch.from_numpy(v), torch.from_numpy(i))
        V, I = V.numpy(), I.numpy()
        ev, ei = oracle.bucketed(x, k, b, kb)
        good = True
        for r in range(rows):
            pv, pi = [], []
            for p in range(world):
                keep = I[p, r] >= 0
                pv.append(V[p, r][keep])
                pi.append(I[p, r][keep] + offsets[p])
            mv, mi = oracle.bucketed_pairs(np.concatenate(pv), np.concatenate(pi).astype(np.int32), k, b, kb)
            good &= np.array_equal(mi, ei[r]) and np.array_equal(mv.view(np.uint32), ev[r].view(np.uint32))
        ok.append(bool(good))
    out[rank] = ok
    dist.destroy_process_group()


@pytest.mark.parametrize("world", [2, 3])
def test_gloo_split_and_merge_equals_single_pass(world):
    ctx = mp.get_context("spawn")
    with ctx.Manager() as m:
        out = m.dict()
        port = _free_port()
        procs = [ctx.Process(target=_worker, args=(r, world, port, out)) for r in range(world)]
        for p in procs:
            p.start()
        for p in procs:
            p.join(180)
            assert p.exitcode == 0
        for r in range(world):
            assert out[r] == [True] * len(CASES)
