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


# ------------------------------------------------------------------ the product functions
# split_row_topk and split_score_topk themselves, over gloo ranks on the CPU:
# the GPU calls they make (topk_bucketed, score_topk, topk_bucketed_merge) are
# replaced by stand-ins that run the oracle, so that the offsets, the gather
# order and the arguments passed between the steps are what is checked.
def _oracle_stand_ins(oracle):
    def topk_bucketed(x, k, b, kb, **_):
        v, i = oracle.bucketed(np.ascontiguousarray(x.numpy()), k, b, kb)
        return torch.from_numpy(v), torch.from_numpy(i)

    def score_topk(q, K, k, b, kb, **_):
        bits = lambda t: t.contiguous().view(torch.int16).numpy().view(np.uint16)  # noqa: E731
        v, i, _ = oracle.score_topk(bits(q), bits(K), k, b, kb)
        return torch.from_numpy(v), torch.from_numpy(i)

    def topk_bucketed_merge(V, I, n_total, k, b, kb, part_offsets=None, **_):
        V, I = V.numpy(), I.numpy()
        parts, rows, _m = V.shape
        offs = part_offsets if part_offsets is not None else [0] * parts
        ov = np.empty((rows, k), np.float32)
        oi = np.empty((rows, k), np.int32)
        for r in range(rows):
            keep = [I[p, r] >= 0 for p in range(parts)]
            pv = np.concatenate([V[p, r][keep[p]] for p in range(parts)])
            pi = np.concatenate([I[p, r][keep[p]] + offs[p] for p in range(parts)]).astype(np.int32)
            ov[r], oi[r] = oracle.bucketed_pairs(pv, pi, k, b, kb)
        return torch.from_numpy(ov), torch.from_numpy(oi)

    return topk_bucketed, score_topk, topk_bucketed_merge


def _cuts(n, world, seed):
    """Cut points of [0, n) into `world` slices, not multiples of any b."""
    if world == 1:
        return [(0, n)]
    rng = np.random.default_rng(seed)
    inner = np.sort(rng.choice(np.arange(1, n), size=world - 1, replace=False))
    edges = [0] + [int(c) for c in inner] + [n]
    return [(edges[r], edges[r + 1] - edges[r]) for r in range(world)]


def _product_worker(rank, world, port, out):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    import oracle
    from approximate_top_selection_b200 import _binding

    oracle.build()
    oracle.set_threads(1)
    _binding.topk_bucketed, _binding.score_topk, _binding.topk_bucketed_merge = \
        _oracle_stand_ins(oracle)
    ok = []
    for ci, (rows, n, k, b, kb, kind) in enumerate(CASES):
        x = _rows(kind, rows, n, 2000 + ci)
        for cuts in (sharded.column_slices(n, world), _cuts(n, world, 50 + ci)):
            off, ln = cuts[rank]
            v, i = sharded.split_row_topk(x[:, off:off + ln].contiguous(), off, n, k, b, kb)
            ev, ei = oracle.bucketed(x.numpy(), k, b, kb)
            ok.append(bool(np.array_equal(i.numpy(), ei)
                           and np.array_equal(v.numpy().view(np.uint32), ev.view(np.uint32))))
    # keys split by rows of the key matrix: per-row keys and one shared matrix
    q, K = inputs.decode_inputs(1, 3, 1500, 128, 77)
    Q, Ks = inputs.link_inputs(4, 2048, 128, 78)
    bits = lambda t: t.contiguous().view(torch.int16).numpy().view(np.uint16)  # noqa: E731
    for (qq, KK, k, b, kb) in [(q, K, 100, 64, 2), (Q, Ks, 50, 128, 1)]:
        n = KK.shape[-2]
        off, ln = _cuts(n, world, 90 + n)[rank]
        K_local = KK[..., off:off + ln, :].contiguous()
        v, i = sharded.split_score_topk(qq, K_local, off, n, k, b, kb)
        ev, ei, _ = oracle.score_topk(bits(qq), bits(KK), k, b, kb)
        ok.append(bool(np.array_equal(i.numpy(), ei)
                       and np.array_equal(v.numpy().view(np.uint32), ev.view(np.uint32))))
    out[rank] = ok
    dist.destroy_process_group()


@pytest.mark.parametrize("world", [1, 2, 3])
def test_split_functions_equal_single_pass(world):
    """split_row_topk / split_score_topk, cut at even and at random points
    (offsets that are not multiples of b), equal the single pass."""
    ctx = mp.get_context("spawn")
    with ctx.Manager() as m:
        out = m.dict()
        port = _free_port()
        procs = [ctx.Process(target=_product_worker, args=(r, world, port, out))
                 for r in range(world)]
        for p in procs:
            p.start()
        for p in procs:
            p.join(180)
            assert p.exitcode == 0
        for r in range(world):
            assert out[r] == [True] * (2 * len(CASES) + 2)
