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
