"""The multi-rank bench plumbing on the CPU (gloo, world size 2): time is
the maximum over ranks and throughput adds the ranks' bytes (weak scaling)."""
import os
import socket

import torch
import torch.distributed as dist
import torch.multiprocessing as mp


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    p = s.getsockname()[1]
    s.close()
    return p


def _worker(rank, world, port, out):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    import bench

    ms = [4.0, 6.5][rank]
    slowest = bench.max_over_ranks(ms, world, device="cpu")
    out[rank] = (slowest, bench.job_throughput(1e9, slowest, world))
    dist.destroy_process_group()


def test_two_gloo_ranks():
    ctx = mp.get_context("spawn")
    with ctx.Manager() as m:
        out = m.dict()
        port = _free_port()
        procs = [ctx.Process(target=_worker, args=(r, 2, port, out)) for r in range(2)]
        for p in procs:
            p.start()
        for p in procs:
            p.join(120)
            assert p.exitcode == 0
        for r in range(2):
            slowest, gbs = out[r]
            assert slowest == 6.5
            assert abs(gbs - 2 * 1e9 / 6.5e-3 / 1e9) < 1e-9


def _split_worker(rank, world, port, out):
    """The bench's row-split step over gloo ranks: each rank's Workload holds
    its column slice; the step (sharded.split_row_topk, with the GPU calls
    replaced by oracle stand-ins) must return the selection over the whole
    row of all ranks' slices."""
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    import numpy as np

    import bench
    import oracle
    from approximate_top_selection_b200 import _binding
    from test_sharded_rows import _oracle_stand_ins

    oracle.build()
    oracle.set_threads(1)
    _binding.topk_bucketed, _binding.score_topk, _binding.topk_bucketed_merge = \
        _oracle_stand_ins(oracle)
    bench.CONFIGS["vocab-split-small"] = dict(bench.CONFIGS["vocab-split"], rows=4, n=3000, k=20,
                                              b=16, kb=2)
    cpu = torch.device("cpu")
    w = bench.Workload("vocab-split-small", cpu, seed_offset=rank, rank=rank, world=world)
    v, i = w.step()
    whole = np.concatenate([bench.Workload("vocab-split-small", cpu, seed_offset=r, rank=r,
                                           world=world).x.numpy() for r in range(world)], axis=1)
    ev, ei = oracle.bucketed(whole, 20, 16, 2)
    out[rank] = bool(np.array_equal(i.numpy(), ei)
                     and np.array_equal(v.numpy().view(np.uint32), ev.view(np.uint32))
                     and (i.numpy() >= 3000).any())
    dist.destroy_process_group()


def test_split_workload_two_gloo_ranks():
    import sys

    sys.path.insert(0, os.path.dirname(os.path.abspath(__file__)))
    ctx = mp.get_context("spawn")
    with ctx.Manager() as m:
        out = m.dict()
        port = _free_port()
        procs = [ctx.Process(target=_split_worker, args=(r, 2, port, out)) for r in range(2)]
        for p in procs:
            p.start()
        for p in procs:
            p.join(120)
            assert p.exitcode == 0
        assert out[0] is True and out[1] is True
