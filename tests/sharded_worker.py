"""Worker for tests/test_gpu_sharded.py: runs the row-split functions of
`approximate_top_selection_b200.sharded` on cuda:0 as one rank of a process
group and saves what they return.

    python tests/sharded_worker.py nccl1 <port> <out_dir>          (1 rank, NCCL)
    python tests/sharded_worker.py gloo2 <port> <out_dir> <rank>   (2 ranks, gloo)

Only the product path runs here (no oracle): the test compares the saved
results with the oracle in its own process.  The inputs are the seeded draws
of `inputs`, which the test draws again.
"""
import datetime
import os
import sys

import numpy as np
import torch
import torch.distributed as dist

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import approximate_top_selection_b200 as atk  # noqa: E402
from approximate_top_selection_b200 import inputs, sharded  # noqa: E402

DEV = torch.device("cuda", 0)

# (rows, n, k, b, kb, seed): float32 score rows cut into column slices
ROW_CASES = [(8, 300000, 100, 512, 2, 501), (5, 131072, 512, 256, 4, 502),
             (300, 4096, 64, 128, 1, 503)]
# (kind, rows, n, d, k, b, kb, seed): fused scoring with the keys cut by rows
SCORE_CASES = [("per-row", 4, 20000, 128, 200, 256, 2, 601),
               ("shared", 64, 16384, 256, 100, 1024, 1, 602)]


def row_input(rows, n, seed):
    return inputs.normal_rows(rows, n, seed)


def score_input(kind, rows, n, d, seed):
    if kind == "per-row":
        return inputs.decode_inputs(1, rows, n, d, seed)
    return inputs.link_inputs(rows, n, d, seed)


def cuts(n, world, mode, seed):
    """(offset, length) per rank: even slices, or cut at seeded random points."""
    if mode == "even" or world == 1:
        return sharded.column_slices(n, world)
    rng = np.random.default_rng(seed)
    inner = np.sort(rng.choice(np.arange(1, n), size=world - 1, replace=False))
    edges = [0] + [int(c) for c in inner] + [n]
    return [(edges[r], edges[r + 1] - edges[r]) for r in range(world)]


def run(world, rank, out_dir):
    res = {}
    for ci, (rows, n, k, b, kb, seed) in enumerate(ROW_CASES):
        x = row_input(rows, n, seed)
        for mode in ("even", "random"):
            off, ln = cuts(n, world, mode, seed)[rank]
            v, i = sharded.split_row_topk(x[:, off:off + ln].contiguous().to(DEV), off, n, k, b, kb)
            res["row%d_%s_v" % (ci, mode)] = v.cpu().numpy()
            res["row%d_%s_i" % (ci, mode)] = i.cpu().numpy()
        if world == 1:  # one rank holding only a slice of the row: the slice, global indices
            off, ln = n // 3, n // 2
            v, i = sharded.split_row_topk(x[:, off:off + ln].contiguous().to(DEV), off, n, k, b, kb)
            res["row%d_part_v" % ci] = v.cpu().numpy()
            res["row%d_part_i" % ci] = i.cpu().numpy()
    for ci, (kind, rows, n, d, k, b, kb, seed) in enumerate(SCORE_CASES):
        q, K = score_input(kind, rows, n, d, seed)
        for mode in ("even", "random"):
            off, ln = cuts(n, world, mode, seed)[rank]
            Kl = K[..., off:off + ln, :].contiguous().to(DEV)
            qd = q.to(DEV)
            v, i = sharded.split_score_topk(qd, Kl, off, n, k, b, kb)
            # this rank's own fp32 scores of its slice, for the bit-exact check
            _, _, s = atk.score_topk(qd, Kl, k, b, kb, return_scores=True)
            res["score%d_%s_v" % (ci, mode)] = v.cpu().numpy()
            res["score%d_%s_i" % (ci, mode)] = i.cpu().numpy()
            res["score%d_%s_s%d" % (ci, mode, rank)] = s.cpu().numpy()
    torch.cuda.synchronize()
    assert atk.topk_device_status() == 0
    np.savez(os.path.join(out_dir, "rank%d.npz" % rank), **res)


def main():
    mode, port, out_dir = sys.argv[1], int(sys.argv[2]), sys.argv[3]
    torch.cuda.set_device(0)
    atk.load_library()
    store = dist.TCPStore("127.0.0.1", port, is_master=(mode == "nccl1" or sys.argv[4] == "0"),
                          timeout=datetime.timedelta(seconds=120))
    if mode == "nccl1":
        dist.init_process_group("nccl", store=store, rank=0, world_size=1,
                                timeout=datetime.timedelta(seconds=120), device_id=DEV)
        run(1, 0, out_dir)
    else:
        rank = int(sys.argv[4])
        dist.init_process_group("gloo", store=store, rank=rank, world_size=2,
                                timeout=datetime.timedelta(seconds=120))
        run(2, rank, out_dir)
    dist.destroy_process_group()


if __name__ == "__main__":
    main()
