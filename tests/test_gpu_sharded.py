"""The row split across ranks, run as written: `sharded.split_row_topk` and
`sharded.split_score_topk` on cuda:0.

Two launches of tests/sharded_worker.py:
  - one rank with NCCL (the device all-gather, all_gather_into_tensor, of the
    product path), given the whole row and given only a slice of it;
  - two gloo ranks sharing the one GPU (each rank's kernels are independent;
    only the host gathers the candidate lists), cut at even and at random
    column offsets.
Each result is compared here with the oracle: for score rows bit for bit with
the single pass over the whole rows; for fused scoring bit for bit with the
oracle's selection over the ranks' own fp32 slice scores (which must also lie
within 2e-3 of the oracle's fp64 scores).  ("Approximate Top-k for Increased
Parallelism", pith.science review page, "What carries the argument": the
per-bucket top-k_b of a row is the top-k_b of the per-slice lists.)
"""
import os
import socket
import subprocess
import sys

import numpy as np
import pytest
import torch

pytestmark = pytest.mark.gpu

HERE = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, HERE)
import sharded_worker as W  # noqa: E402


def _port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    p = s.getsockname()[1]
    s.close()
    return p


def _launch(args_per_rank):
    env = dict(os.environ, NCCL_NVLS_ENABLE="0")
    procs = [subprocess.Popen([sys.executable, os.path.join(HERE, "sharded_worker.py"), *a],
                              env=env) for a in args_per_rank]
    rcs = []
    for p in procs:
        try:
            rcs.append(p.wait(timeout=600))
        except subprocess.TimeoutExpired:
            p.kill()
            rcs.append(-9)
    assert rcs == [0] * len(procs), rcs


def _bits(t):
    return t.contiguous().view(torch.int16).numpy().view(np.uint16)


def _same(v, want):
    return np.array_equal(np.asarray(v, np.float32).view(np.uint32), want.view(np.uint32))


def _check_rows(res, world, oracle_mod):
    for ci, (rows, n, k, b, kb, seed) in enumerate(W.ROW_CASES):
        x = W.row_input(rows, n, seed).numpy()
        ev, ei = oracle_mod.bucketed(x, k, b, kb)
        for mode in ("even", "random"):
            for r in range(world):
                assert np.array_equal(res[r]["row%d_%s_i" % (ci, mode)], ei), (ci, mode, r)
                assert _same(res[r]["row%d_%s_v" % (ci, mode)], ev), (ci, mode, r)
        if world == 1:
            off, ln = n // 3, n // 2
            idx = np.arange(off, off + ln, dtype=np.int32)
            for row in range(rows):
                pv, pi = oracle_mod.bucketed_pairs(np.ascontiguousarray(x[row, off:off + ln]), idx,
                                                   k, b, kb)
                assert np.array_equal(res[0]["row%d_part_i" % ci][row], pi), (ci, row)
                assert _same(res[0]["row%d_part_v" % ci][row], pv), (ci, row)


def _check_scores(res, world, oracle_mod):
    for ci, (kind, rows, n, d, k, b, kb, seed) in enumerate(W.SCORE_CASES):
        q, K = W.score_input(kind, rows, n, d, seed)
        ref = oracle_mod.scores(_bits(q), _bits(K))
        for mode in ("even", "random"):
            parts = [res[r]["score%d_%s_s%d" % (ci, mode, r)] for r in range(world)]
            s = np.concatenate(parts, axis=1)
            assert s.shape == (rows, n)
            qn = np.linalg.norm(q.float().numpy().astype(np.float64), axis=1)
            kn = np.linalg.norm(K.float().numpy().astype(np.float64), axis=-1)
            scale = qn[:, None] * (kn if kn.ndim == 2 else kn[None, :])
            tol = 2e-3 * np.maximum(np.abs(ref), 2.0 ** -10 * scale)
            assert np.all(np.abs(s.astype(np.float64) - ref) <= tol), (ci, mode)
            ev, ei = oracle_mod.bucketed(s, k, b, kb)
            for r in range(world):
                assert np.array_equal(res[r]["score%d_%s_i" % (ci, mode)], ei), (ci, mode, r)
                assert _same(res[r]["score%d_%s_v" % (ci, mode)], ev), (ci, mode, r)


def test_split_functions_one_nccl_rank(tmp_path, oracle_mod):
    if not torch.cuda.is_available():
        pytest.fail("this test needs a CUDA device")
    _launch([("nccl1", str(_port()), str(tmp_path))])
    res = [dict(np.load(tmp_path / "rank0.npz"))]
    _check_rows(res, 1, oracle_mod)
    _check_scores(res, 1, oracle_mod)


def test_split_functions_two_gloo_ranks_one_gpu(tmp_path, oracle_mod):
    if not torch.cuda.is_available():
        pytest.fail("this test needs a CUDA device")
    port = str(_port())
    _launch([("gloo2", port, str(tmp_path), "0"), ("gloo2", port, str(tmp_path), "1")])
    res = [dict(np.load(tmp_path / ("rank%d.npz" % r))) for r in range(2)]
    _check_rows(res, 2, oracle_mod)
    _check_scores(res, 2, oracle_mod)
