"""Benchmark: bucketed approximate top-k on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
                    [--config decode|tiny|vocab|link|long-b128-kb1 ...]

One step is one pass of the whole hot path over one batch of resident input.
The default workload is the sparse-attention decode selection: 16 x 32 rows,
each a bf16 query (d = 128) scored against its own 32768 x 128 bf16 key matrix
(4 GiB of keys in total, larger than L2), then bucketed top-k with k = 512,
b = 256, k_b = 2 -- one fused kernel launch per step.

The metric is "bucketed top-k GB/s of scores read": the bytes of score input the
step must read (the key matrices and queries for the fused step), plus the
output, divided by the step's device time.  rows/s and the recall against exact
top-k (with Eq. (1) of "Approximate Top-k for Increased Parallelism" beside it)
ride along.  Timing protocol after that paper's benchmark appendix: warm-up
launches, then device-side CUDA events around K steps.

Multi-GPU (`--gpus N`, one rank per GPU; started as one process it relaunches
itself under torch.distributed.run): every rank runs the same per-GPU workload
on its own inputs (rows are independent; no collective on the data path),
except `vocab-split`, whose rows are cut by columns across the ranks and merged
after one all-gather of the candidate pairs; the time is the maximum over
ranks and `value` counts the bytes of all ranks (weak scaling).

A one-GPU run also carries `sweep`: every score-row workload (vocabulary and
the long-context b x k_b grid, fp32 and bf16) and the fused link and re-rank
workloads, each timed on its own from CUDA-graph replays, with its roofline
fraction and clock record.
"""
from __future__ import annotations

import argparse
import json
import math
import os
import statistics
import subprocess
import sys
import threading
import time

import numpy as np
import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "bucketed top-k GB/s of scores read vs HBM peak; rows/s; recall@k vs Eq.(1)"

# name -> workload description.  kind: "score" (fused q.K + selection), "select",
# or "rerank" (exact scores of given candidate indices + top-k).
CONFIGS = {
    "tiny": dict(kind="select", rows=8, n=4096, k=64, b=128, kb=1, dist="normal"),
    "decode": dict(kind="score", batch=16, heads=32, n=32768, d=128, k=512, b=256, kb=2),
    "vocab": dict(kind="select", rows=256, n=131072, k=50, b=512, kb=1, dist="vocab"),
    "link": dict(kind="score", queries=1024, n=1 << 20, d=256, k=100, b=1024, kb=1),
    # reduced cases profiled with ncu --set full (inputs still larger than L2)
    "decode-quarter": dict(kind="score", batch=4, heads=32, n=32768, d=128, k=512, b=256, kb=2),
    "link-quarter": dict(kind="score", queries=1024, n=1 << 18, d=256, k=100, b=1024, kb=1),
    # exact re-ranking of reused supports against the decode key cache: per row
    # the union of 4 overlapping supports of 512 keys, top-512 of their scores
    "decode-rerank": dict(kind="rerank", batch=16, heads=32, n=32768, d=128, k=512, supports=4,
                          support=512),
    "decode-rerank-quarter": dict(kind="rerank", batch=4, heads=32, n=32768, d=128, k=512,
                                  supports=4, support=512),
}
for _b in (128, 256, 512):
    for _kb in (1, 2, 4):
        CONFIGS["long-b%d-kb%d" % (_b, _kb)] = dict(kind="select", rows=256, n=131072, k=512,
                                                    b=_b, kb=_kb, dist="uniform")
# vocabulary sampling with its tail: the selection, then one token per row drawn
# from the softmax (T = 1) of the selected logits
CONFIGS["vocab-sample"] = dict(CONFIGS["vocab"], sample=1.0)
# bfloat16 score rows (the page's Fig. 10 repeats its configurations in bf16)
for _name in ["vocab"] + ["long-b%d-kb%d" % (b, kb) for b in (128, 256, 512) for kb in (1, 2, 4)]:
    CONFIGS[_name + "-bf16"] = dict(CONFIGS[_name], dtype="bf16")
# vocabulary-parallel rows: every rank holds 131072 columns of each of the 256
# rows (a row of world x 131072 logits in all), selects on its slice,
# all-gathers the k (value, index) pairs per row and merges them by global
# index (sharded.split_row_topk).  Per-rank work is fixed: weak scaling.
CONFIGS["vocab-split"] = dict(CONFIGS["vocab"], kind="split")

L2_BYTES = 126 * 2 ** 20

# The cells of the score-row sweep that rides along with the default line.
SWEEP = (["vocab", "vocab-bf16", "vocab-sample"]
         + ["long-b%d-kb%d%s" % (b, kb, t) for t in ("", "-bf16") for b in (128, 256, 512)
            for kb in (1, 2, 4)]
         + ["link", "decode-rerank"])


def _peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            p = json.load(f)
        return float(p["hbm_gbs"]), float(p.get("bf16_tflops", 1590.0)), "measured"
    return 6650.0, 1590.0, "fallback"


class ClockSampler:
    """nvidia-smi sampling of SM clocks and throttle reasons during a region."""

    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.gpu = gpu_index
        self.proc = None
        self.lines = []

    def __enter__(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.gpu), "--query-gpu=" + self.FIELDS,
                 "--format=csv,noheader,nounits", "-lms", "50"],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            self.thread = threading.Thread(target=self._read, daemon=True)
            self.thread.start()
            time.sleep(0.15)
        except (OSError, FileNotFoundError):
            self.proc = None
        return self

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append(line.strip())

    def __exit__(self, *exc):
        if self.proc is not None:
            time.sleep(0.1)
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()
        return False

    def summary(self):
        if not self.lines:
            return None
        sm, mx, reasons = [], 0.0, set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for ln in self.lines:
            parts = [p.strip() for p in ln.split(",")]
            if len(parts) < 9:
                continue
            try:
                sm.append(float(parts[1]))
                mx = max(mx, float(parts[2]))
            except ValueError:
                continue
            for name, val in zip(names, parts[5:9]):
                if val.lower() == "active":
                    reasons.add(name)
        if not sm:
            return None
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": mx, "reasons": sorted(reasons),
                "samples": len(sm)}


# ---------------------------------------------------------------- workloads
class Workload:
    """Resident device inputs for one config, plus the step function."""

    def __init__(self, name: str, device, seed_offset: int = 0, rank: int = 0, world: int = 1):
        from approximate_top_selection_b200 import inputs

        self.name, self.cfg, self.device = name, CONFIGS[name], device
        self.rank, self.world = rank, world
        c = self.cfg
        seed = inputs.SEEDS[name.split("-")[0]] + seed_offset
        if c["kind"] == "rerank":
            self.rows = c["batch"] * c["heads"]
            self.q, self.K = inputs.decode_inputs(c["batch"], c["heads"], c["n"], c["d"], seed,
                                                  device=device)
            self.cand = inputs.support_union(self.rows, c["n"], c["supports"], c["support"],
                                             seed ^ 0xCA, device=device)
            distinct = sum(len(set(r.tolist())) for r in self.cand.cpu())
            # the distinct key rows each query gathers, the queries, the candidate lists
            self.in_bytes = distinct * c["d"] * 2 + self.q.numel() * 2 + self.cand.numel() * 4
        elif c["kind"] == "score":
            if "batch" in c:
                self.rows = c["batch"] * c["heads"]
                self.q, self.K = inputs.decode_inputs(c["batch"], c["heads"], c["n"], c["d"], seed,
                                                      device=device)
            else:
                self.rows = c["queries"]
                self.q, self.K = inputs.link_inputs(c["queries"], c["n"], c["d"], seed,
                                                    device=device)
            self.in_bytes = self.q.numel() * 2 + self.K.numel() * 2
        else:
            self.rows = c["rows"]
            if c["dist"] == "normal":
                self.x = inputs.normal_rows(c["rows"], c["n"], seed, device=device)
            elif c["dist"] == "vocab":
                self.x = inputs.vocab_logits(c["rows"], c["n"], seed, device=device)
            else:
                self.x = inputs.uniform_rows(c["rows"], c["n"], seed, device=device)
            if c.get("dtype") == "bf16":
                self.x = self.x.to(torch.bfloat16)
            self.in_bytes = self.x.numel() * self.x.element_size()
        # values (2 bytes for bf16 rows, else 4) + int32 indices
        self.out_bytes = self.rows * c["k"] * (6 if c.get("dtype") == "bf16" else 8)
        if c.get("sample"):
            g = torch.Generator(device=device).manual_seed(seed ^ 0x5EED)
            self.u = torch.rand(self.rows, generator=g, device=device, dtype=torch.float32)
            self.in_bytes += self.rows * 4
            self.out_bytes += self.rows * 4
        self.bytes = self.in_bytes + self.out_bytes

    def step(self, stream=None):
        import approximate_top_selection_b200 as atk

        c = self.cfg
        if c["kind"] == "score":
            return atk.score_topk(self.q, self.K, c["k"], c["b"], c["kb"], stream=stream)
        if c["kind"] == "rerank":
            return atk.score_rerank(self.q, self.K, self.cand, c["k"], stream=stream)
        if c.get("sample"):
            return atk.topk_sample(self.x, c["k"], c["b"], c["kb"], c["sample"], self.u, stream=stream)
        if c["kind"] == "split":
            return self.split_step(self.x)
        return atk.topk_bucketed(self.x, c["k"], c["b"], c["kb"], stream=stream)

    def split_step(self, x):
        """This rank's slice of the rows: local selection, all-gather of the
        candidate pairs, merge by global index."""
        from approximate_top_selection_b200 import sharded

        c = self.cfg
        return sharded.split_row_topk(x, self.rank * c["n"], self.world * c["n"], c["k"], c["b"],
                                      c["kb"], offsets=[r * c["n"] for r in range(self.world)])

    def oracle_step(self, rows: int):
        """A callable doing this workload's step with the oracle on its first `rows` rows."""
        import oracle

        c = self.cfg
        if c["kind"] in ("score", "rerank"):
            q = self.q[:rows].cpu().contiguous().view(torch.int16).numpy().view(np.uint16)
            K = (self.K[:rows] if self.K.dim() == 3 else self.K).cpu().contiguous().view(torch.int16)
            K = K.numpy().view(np.uint16)
            if c["kind"] == "rerank":
                cand = self.cand[:rows].cpu().numpy()
                return lambda: oracle.rerank(q, K, cand, c["k"])
            return lambda: oracle.score_topk(q, K, c["k"], c["b"], c["kb"])
        x = self.x[:rows].float().cpu().numpy()
        if c.get("sample"):
            u = self.u[:rows].cpu().numpy().astype(np.float64)

            def run():
                ov, oi = oracle.bucketed(x, c["k"], c["b"], c["kb"])
                oracle.sample_rows(ov, oi, c["sample"], u)
            return run
        return lambda: oracle.bucketed(x, c["k"], c["b"], c["kb"])

    def describe(self):
        c = dict(self.cfg)
        c["workload"] = self.name
        return c


def _uses_tensor_cores(cfg) -> bool:
    """Shared key matrix (link prediction): the tcgen05 GEMM path."""
    return cfg["kind"] == "score" and "queries" in cfg and cfg["n"] % cfg["b"] == 0


def _kernel_name(cfg) -> str:
    if cfg["kind"] == "score":
        if _uses_tensor_cores(cfg):  # CTA pairs from 256 queries on
            return "score_select_umma_pair" if cfg["queries"] >= 256 else "score_select_umma"
        return "score_select_gemv"
    if cfg["kind"] == "rerank":
        return "rerank_kernel"
    if cfg["kb"] > 2 and cfg["b"] >= 512 and cfg.get("dtype") != "bf16":
        return "bucket_select_wide"  # the 16-warp k_b > 2 kernel (bf16 rows: order-key queues)
    return "bucket_select_tma"


def _launches_per_step(cfg) -> int:
    # the tensor-core path adds a Stage-2 kernel, the row split a merge kernel;
    # the sampling draw runs inside the selection kernel
    return 2 if _uses_tensor_cores(cfg) or cfg["kind"] == "split" else 1


def _rotations(w: Workload) -> int:
    """Input copies cycled through so that every step reads its input from
    HBM: one copy when the input is at least twice the L2, else enough copies
    to span three L2s."""
    if w.in_bytes >= 2 * L2_BYTES:
        return 1
    return max(2, math.ceil(3 * L2_BYTES / w.in_bytes))


def _l2_note(w: Workload, nrot: int) -> str:
    if nrot == 1:
        return "inputs larger than twice the L2"
    return "%d rotating input copies (%.0f MiB) defeat L2" % (nrot, nrot * w.in_bytes / 2 ** 20)


def _config(w: Workload, nrot: int, graph: bool) -> dict:
    """The `config` object of a line: the workload, how L2 is defeated and
    how steps are launched (the same object for both arms)."""
    return dict(w.describe(), l2=_l2_note(w, nrot),
                launch="cuda-graph replay" if graph else "eager")


def _time_ms(fn, steps: int, warmup: int = 3) -> float:
    for _ in range(warmup):
        fn()
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record()
    for _ in range(steps):
        fn()
    e1.record()
    torch.cuda.synchronize()
    return e0.elapsed_time(e1) / steps


def exact_context(w: Workload, ms_bucketed: float, steps: int = 20):
    """Context for the page's claim (bucketed vs exact top-k): on the same
    resident input, this library's exact top-k and torch.topk (for the fused
    workloads: the PyTorch scores, materialised, then torch.topk)."""
    import approximate_top_selection_b200 as atk

    c = w.cfg
    out = {"bucketed_ms": ms_bucketed}
    if c["kind"] in ("select", "split"):
        x = w.x.float() if w.x.dtype != torch.float32 else w.x
        out["exact_topk_ms"] = _time_ms(lambda: atk.topk_exact(x, c["k"]), steps)
        out["torch_topk_ms"] = _time_ms(lambda: torch.topk(w.x, c["k"], dim=1), steps)
    elif c["kind"] == "rerank":
        ci = w.cand.long().clamp_min(0)

        def fn():  # gather the candidate keys, score them, top-k (repeats not removed)
            kc = torch.gather(w.K, 1, ci[:, :, None].expand(-1, -1, w.K.shape[2]))
            return torch.topk(torch.bmm(kc, w.q[:, :, None]).squeeze(-1).float(), c["k"], dim=1)
        out["torch_gather_scores_topk_ms"] = _time_ms(fn, max(3, steps // 4))
    else:
        if w.K.dim() == 3:
            fn = lambda: torch.topk(torch.bmm(w.K, w.q[:, :, None]).squeeze(-1).float(),  # noqa: E731
                                    c["k"], dim=1)
        else:
            fn = lambda: torch.topk((w.q @ w.K.T).float(), c["k"], dim=1)  # noqa: E731
        out["torch_scores_then_topk_ms"] = _time_ms(fn, max(3, steps // 4))
    for key in list(out):
        if key != "bucketed_ms":
            out["speedup_vs_" + key[:-3]] = out[key] / ms_bucketed
    return out


def recall_report(w: Workload):
    """Recall of the step's selection against exact top-k on the same scores."""
    import approximate_top_selection_b200 as atk
    from oracle import recall as rc

    c = w.cfg
    if c["kind"] == "rerank":
        return None  # exact on its candidates: nothing to compare with
    if c["kind"] == "score":
        rows = min(w.rows, 64)
        _, bi, s = atk.score_topk(w.q[:rows], w.K[:rows] if w.K.dim() == 3 else w.K, c["k"],
                                  c["b"], c["kb"], return_scores=True)
    else:
        rows = min(w.rows, 256)
        s = w.x[:rows]
        _, bi = atk.topk_bucketed(s, c["k"], c["b"], c["kb"])
    # bf16 widens to fp32 exactly, so the exact selection sees the same values
    _, ei = atk.topk_exact(s.float() if s.dtype != torch.float32 else s, c["k"])
    r = rc.recall(bi.cpu().numpy(), ei.cpu().numpy())
    n = c["n"]
    out = {"mean": float(r.mean()), "rows": rows, "eq1": rc.eq1_expected_recall(c["k"], c["b"], c["kb"])}
    if n % c["b"] == 0 and c["kind"] == "score" or c.get("dist") == "uniform":
        out["exact_expectation_iid"] = rc.expected_recall_exact(n, c["k"], c["b"], c["kb"])
    return out


def cpu_baseline(w: Workload, budget_s: float = 10.0):
    """The oracle, as it stands, on the host cores over a bounded row sample."""
    import oracle

    oracle.build()
    threads = oracle.max_threads()
    oracle.set_threads(threads)
    c = w.cfg

    def run(rows):
        step = w.oracle_step(rows)
        t0 = time.perf_counter()
        step()
        return time.perf_counter() - t0

    def sample(nthreads, budget):
        oracle.set_threads(nthreads)
        probe = min(w.rows, max(1, nthreads))
        t = run(probe)
        rows = int(min(w.rows, max(probe, probe * budget / max(t, 1e-6))))
        if rows > probe:
            t = run(rows)
        else:
            rows = probe
        return rows, t

    per_row = w.bytes / w.rows
    rows1, t1 = sample(1, budget_s / 4)
    rows, t = sample(threads, budget_s)
    return {"value": rows * per_row / t / 1e9, "unit": "GB/s", "cores": threads, "kind": "oracle",
            "sample": "%d of %d rows of the %s workload (%.1f s)" % (rows, w.rows, w.name, t),
            "rows_per_s": rows / t,
            "single_thread": {"value": rows1 * per_row / t1 / 1e9, "unit": "GB/s",
                              "rows_per_s": rows1 / t1,
                              "sample": "%d of %d rows (%.1f s)" % (rows1, w.rows, t1)}}


# ---------------------------------------------------------------- runs
def setup_dist(args):
    """One process per GPU: the NCCL process group from torchrun's variables.
    A row-split workload on one GPU still runs its collective, in a
    one-rank group."""
    import datetime

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    timeout = datetime.timedelta(seconds=120)
    if world > 1:
        torch.cuda.set_device(local)
        torch.distributed.init_process_group("nccl", timeout=timeout,
                                             device_id=torch.device("cuda", local))
    else:
        torch.cuda.set_device(0)
        if CONFIGS[args.config]["kind"] == "split":
            torch.distributed.init_process_group("nccl", store=torch.distributed.HashStore(),
                                                 rank=0, world_size=1, timeout=timeout,
                                                 device_id=torch.device("cuda", 0))
    return world, rank, local


def max_over_ranks(x: float, world: int, device="cuda") -> float:
    """Largest value over the ranks (the job's time is its slowest rank's)."""
    if world == 1:
        return x
    t = torch.tensor([x], dtype=torch.float64, device=device)
    torch.distributed.all_reduce(t, op=torch.distributed.ReduceOp.MAX)
    return float(t.item())


def job_throughput(bytes_per_rank: float, ms_per_step_max: float, world: int) -> float:
    """Whole-job GB/s: every rank processes its own workload (weak scaling),
    so the bytes add up over ranks and the time is the slowest rank's."""
    return bytes_per_rank * world / (ms_per_step_max * 1e-3) / 1e9


def barrier(world):
    if world > 1:
        torch.distributed.barrier()
    torch.cuda.synchronize()


def run_ours(args, world, rank, local):
    import approximate_top_selection_b200 as atk

    atk.load_library()
    dev = torch.device("cuda", local)
    w = Workload(args.config, dev, seed_offset=rank, rank=rank, world=world)
    nrot = _rotations(w)
    extra = [Workload(args.config, dev, seed_offset=rank + 101 * (j + 1), rank=rank, world=world)
             for j in range(nrot - 1)]
    works = [w] + extra
    stream = torch.cuda.current_stream()
    for i in range(args.warmup):
        works[i % nrot].step()
    run = [wk.step for wk in works]
    if args.graph:
        # One CUDA graph per input copy, each holding one step (the page's
        # Fig. 9 measures the same kernels with CUDA graphs): replays skip
        # the host side of every launch.
        gs = torch.cuda.Stream()
        gs.wait_stream(stream)
        with torch.cuda.stream(gs):
            for wk in works:  # workspace and kernel set-up for this stream
                wk.step()
        gs.synchronize()
        graphs = []
        for wk in works:
            g = torch.cuda.CUDAGraph()
            with torch.cuda.graph(g, stream=gs):
                wk.step()
            graphs.append(g)
        run = [g.replay for g in graphs]
        for i in range(args.warmup):
            run[i % nrot]()
    barrier(world)
    evs = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps + 1)]
    with ClockSampler(local) as clk:
        barrier(world)
        evs[0].record(stream)
        for i in range(args.steps):
            run[i % nrot]()
            evs[i + 1].record(stream)
        barrier(world)
    ms = evs[0].elapsed_time(evs[-1])
    ms = max_over_ranks(ms, world)
    ms_step = ms / args.steps
    dist = step_distribution(evs[i].elapsed_time(evs[i + 1]) for i in range(args.steps))
    dist = {key: max_over_ranks(v, world) for key, v in dist.items()}
    hbm, tflops_burst, peak_src = _peaks()
    achieved = w.bytes / (ms_step * 1e-3) / 1e9
    line = {
        "metric": METRIC,
        "value": job_throughput(w.bytes, ms_step, world),
        "unit": "GB/s",
        "n_gpus": world,
        "steps": args.steps,
        "warmup": args.warmup,
        "ms_per_step": ms_step,
        "step_ms": dist,
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": "bf16" if w.cfg.get("dtype") == "bf16" else "f32",
        "data": "synthetic (seeded; shapes of the pages' workloads)",
        "config": _config(w, nrot, args.graph),
        "rows_per_s": w.rows * world / (ms_step * 1e-3),
        "gpu_launches": args.steps * _launches_per_step(w.cfg),
        "roofline": _roofline(w, ms_step, achieved, hbm, peak_src, ms_step * args.steps * 1e-3),
        "clocks": clk.summary(),
    }
    if not args.no_recall:
        line["recall"] = recall_report(w)
    if args.context:
        line["context"] = exact_context(w, ms_step)
    if not args.no_e2e:
        line["e2e"] = e2e(w, args, world)
    if rank == 0 and world == 1 and not args.no_cpu:
        line["cpu_baseline"] = cpu_baseline(w)
    if world == 1 and not args.no_sweep:
        del run, works, extra, w
        if args.graph:
            del graphs, g
        torch.cuda.synchronize()
        torch.cuda.empty_cache()
        line["sweep"] = sweep(dev, local)
    return line


def _graph_of_steps(works, reps: int):
    """One CUDA graph holding `reps` passes over the input copies (one step
    per copy): a replay launches len(works) * reps steps with no host work."""
    side = torch.cuda.Stream()
    side.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(side):
        for wk in works:  # workspace and kernel set-up on the capturing stream
            wk.step()
    side.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=side):
        for _ in range(reps):
            for wk in works:
                wk.step()
    return g


def step_distribution(per_step_ms) -> dict:
    """Median and 90th percentile (nearest rank) of per-step times in ms."""
    xs = sorted(float(x) for x in per_step_ms)
    if not xs:
        return {"median": None, "p90": None}
    return {"median": statistics.median(xs), "p90": xs[max(0, math.ceil(0.9 * len(xs)) - 1)]}


def sweep_cell(name: str, dev, local: int, min_region_s: float = 0.25) -> dict:
    """One workload timed alone: CUDA-graph replays of back-to-back steps over
    rotating input copies, CUDA events around the replays, clocks sampled
    meanwhile."""
    w = Workload(name, dev)
    nrot = _rotations(w)
    works = [w] + [Workload(name, dev, seed_offset=101 * (j + 1)) for j in range(nrot - 1)]
    reps = max(1, 24 // nrot)
    g = _graph_of_steps(works, reps)
    per_replay = nrot * reps
    for _ in range(3):
        g.replay()
    est = _time_ms(g.replay, 3, warmup=0) / per_replay
    replays = max(3, math.ceil(min_region_s * 1e3 / (est * per_replay)))
    stream = torch.cuda.current_stream()
    evs = [torch.cuda.Event(enable_timing=True) for _ in range(replays + 1)]
    with ClockSampler(local) as clk:
        torch.cuda.synchronize()
        evs[0].record(stream)
        for i in range(replays):
            g.replay()
            evs[i + 1].record(stream)
        torch.cuda.synchronize()
    steps = replays * per_replay
    ms = evs[0].elapsed_time(evs[-1]) / steps
    # per step, from each replay's own events (one replay = per_replay steps)
    dist = step_distribution(evs[i].elapsed_time(evs[i + 1]) / per_replay for i in range(replays))
    hbm, _, peak_src = _peaks()
    gbs = w.bytes / (ms * 1e-3) / 1e9
    roof = _roofline(w, ms, gbs, hbm, peak_src, ms * steps * 1e-3)
    out = {"ms_per_step": ms, "GB/s": gbs, "rows_per_s": w.rows / (ms * 1e-3),
           "bound": roof["bound"], "achieved": roof["achieved"], "unit": roof["unit"],
           "frac": roof["frac"], "kernel": roof["kernel"], "steps": steps, "step_ms": dist,
           "l2": _l2_note(w, nrot), "clocks": clk.summary()}
    del g, works, w
    torch.cuda.synchronize()
    torch.cuda.empty_cache()
    return out


def sweep(dev, local: int) -> dict:
    """Every score-row cell (vocab, fp32 and bf16; the long-context b x k_b
    grid, fp32 and bf16) and the fused link and re-rank workloads, each timed
    on its own."""
    return {name: sweep_cell(name, dev, local) for name in SWEEP}


# Device sources of each timed kernel: a traffic figure stays valid while these
# files are unchanged since the capture.
_KERNEL_SOURCES = {
    "bucket_select_tma": ("common.cuh", "select_core.cuh", "bucket_select.cuh"),
    "bucket_select_wide": ("common.cuh", "select_core.cuh", "bucket_select.cuh"),
    "score_select_gemv": ("common.cuh", "select_core.cuh", "score_gemv.cuh"),
    "score_select_umma": ("common.cuh", "select_core.cuh", "score_umma.cuh"),
    "score_select_umma_pair": ("common.cuh", "select_core.cuh", "score_umma.cuh"),
    "rerank_kernel": ("common.cuh", "select_core.cuh", "rerank.cuh"),
}


def _source_hash(kernel: str) -> str:
    import hashlib

    h = hashlib.sha256()
    for f in _KERNEL_SOURCES.get(kernel, ()):
        with open(os.path.join(ROOT, "approximate_top_selection_b200", "csrc", f), "rb") as fh:
            h.update(fh.read())
    return h.hexdigest()[:16]


def _traffic(workload: str):
    """DRAM bytes per launch from the committed ncu summary, if the kernel's
    device sources have not changed since it was taken (else None)."""
    path = os.path.join(ROOT, "profiles", "traffic.md")
    if not os.path.exists(path):
        return None
    for line in open(path):
        cells = [c.strip() for c in line.strip().strip("|").split("|")]
        if len(cells) >= 4 and cells[0] == workload and cells[1] in _KERNEL_SOURCES \
                and cells[2] == _source_hash(cells[1]):
            try:
                return int(cells[3])
            except ValueError:
                return None
    return None


def _roofline(w: Workload, ms_step: float, achieved_gbs: float, hbm: float, peak_src: str,
              region_s: float):
    c = w.cfg
    if _uses_tensor_cores(c):
        flops = 2.0 * w.rows * c["n"] * c["d"]
        tf = flops / (ms_step * 1e-3) / 1e12
        peak, src = _tensor_peak(region_s)
        return {"bound": "tensor", "achieved": tf, "peak": peak, "unit": "TFLOP/s",
                "frac": tf / peak, "traffic": _traffic(w.name), "kernel": _kernel_name(c),
                "flops_per_step": flops, "peak_source": src}
    return {"bound": "hbm", "achieved": achieved_gbs, "peak": hbm, "unit": "GB/s",
            "frac": achieved_gbs / hbm, "traffic": _traffic(w.name), "kernel": _kernel_name(c),
            "peak_source": peak_src + " hbm_gbs"}


SUSTAINED_REGION_S = 2.0  # timed regions at least this long compare with the sustained peak


def _tensor_peak(region_s: float):
    """Dense bf16 peak: the burst figure for a timed region shorter than
    SUSTAINED_REGION_S, the sustained (power-capped) one for a longer one."""
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    long_region = region_s >= SUSTAINED_REGION_S
    if os.path.exists(path):
        with open(path) as f:
            p = json.load(f)
        if long_region and "bf16_tflops_sustained" in p:
            return float(p["bf16_tflops_sustained"]), "measured bf16_tflops_sustained"
        return float(p["bf16_tflops"]), "measured bf16_tflops"
    return (1400.0, "fallback (sustained)") if long_region else (1590.0, "fallback (burst)")


def e2e(w: Workload, args, world):
    """Same metric through the public API with host buffers: per step, pinned
    host -> device copy of the inputs, the call, device -> host of the result."""
    import approximate_top_selection_b200 as atk

    c = w.cfg
    steps = max(1, min(args.steps, args.e2e_steps))
    if c["kind"] in ("score", "rerank"):
        hq = torch.empty(w.q.shape, dtype=w.q.dtype, pin_memory=True)
        hK = torch.empty(w.K.shape, dtype=w.K.dtype, pin_memory=True)
        hq.copy_(w.q)
        hK.copy_(w.K)
        dq, dK = torch.empty_like(w.q), torch.empty_like(w.K)
        h2d = hq.numel() * 2 + hK.numel() * 2
        if c["kind"] == "rerank":
            hc = torch.empty(w.cand.shape, dtype=w.cand.dtype, pin_memory=True)
            hc.copy_(w.cand)
            dc = torch.empty_like(w.cand)
            h2d += hc.numel() * 4
    else:
        hx = torch.empty(w.x.shape, dtype=w.x.dtype, pin_memory=True)
        hx.copy_(w.x)
        dx = torch.empty_like(w.x)
        h2d = hx.numel() * hx.element_size()
        if c.get("sample"):
            hu = torch.empty(w.u.shape, dtype=w.u.dtype, pin_memory=True)
            hu.copy_(w.u)
            du = torch.empty_like(w.u)
            ht = torch.empty(w.rows, dtype=torch.int32, pin_memory=True)
            h2d += hu.numel() * 4
    hv = torch.empty(w.rows, c["k"], dtype=torch.bfloat16 if c.get("dtype") == "bf16" else torch.float32,
                     pin_memory=True)
    hi = torch.empty(w.rows, c["k"], dtype=torch.int32, pin_memory=True)
    stream = torch.cuda.current_stream()

    def one():
        if c["kind"] == "score":
            dq.copy_(hq, non_blocking=True)
            dK.copy_(hK, non_blocking=True)
            v, i = atk.score_topk(dq, dK, c["k"], c["b"], c["kb"])
        elif c["kind"] == "rerank":
            dq.copy_(hq, non_blocking=True)
            dK.copy_(hK, non_blocking=True)
            dc.copy_(hc, non_blocking=True)
            v, i = atk.score_rerank(dq, dK, dc, c["k"])
        elif c.get("sample"):
            dx.copy_(hx, non_blocking=True)
            du.copy_(hu, non_blocking=True)
            t, v, i = atk.topk_sample(dx, c["k"], c["b"], c["kb"], c["sample"], du)
            ht.copy_(t, non_blocking=True)
        elif c["kind"] == "split":
            dx.copy_(hx, non_blocking=True)
            v, i = w.split_step(dx)
        else:
            dx.copy_(hx, non_blocking=True)
            v, i = atk.topk_bucketed(dx, c["k"], c["b"], c["kb"])
        hv.copy_(v, non_blocking=True)
        hi.copy_(i, non_blocking=True)

    one()
    barrier(world)
    ev0, ev1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    ev0.record(stream)
    for _ in range(steps):
        one()
    ev1.record(stream)
    barrier(world)
    ms = max_over_ranks(ev0.elapsed_time(ev1), world) / steps
    return {"value": w.bytes * world / (ms * 1e-3) / 1e9, "unit": "GB/s",
            "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": w.out_bytes,
            "ms_per_step": ms, "steps": steps}


REFERENCE_BUDGET_S = 60.0  # host seconds for the reference arm's warm-up and timed steps


def run_reference(args, world, rank, local):
    """The oracle on the host cores, as it stands: every step is a bounded
    row sample of the same workload, sized so that the W warm-up and K timed
    steps take about REFERENCE_BUDGET_S together."""
    import oracle

    dev = torch.device("cuda", local) if torch.cuda.is_available() else torch.device("cpu")
    w = Workload(args.config, dev)
    oracle.build()
    threads = oracle.max_threads()
    oracle.set_threads(threads)
    probe = cpu_baseline(w, budget_s=1.0)
    per_step_s = min(1.0, max(0.02, REFERENCE_BUDGET_S / (args.steps + args.warmup)))
    rows = max(1, min(w.rows, int(probe["rows_per_s"] * per_step_s)))
    step = w.oracle_step(rows)
    for _ in range(args.warmup):
        step()
    t0 = time.perf_counter()
    for _ in range(args.steps):
        step()
    dt = (time.perf_counter() - t0) / args.steps
    per_row = w.bytes / w.rows
    value = rows * per_row / dt / 1e9
    sample = "%d of %d rows of the %s workload per step" % (rows, w.rows, w.name)
    return {"metric": METRIC, "value": value, "unit": "GB/s", "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": dt * 1e3, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f64 accumulate / f32 select",
            "data": "synthetic (seeded; shapes of the pages' workloads)", "impl": "reference",
            "config": _config(w, _rotations(w), args.graph),
            "rows_per_s": rows / dt,
            "cpu_baseline": {"value": value, "unit": "GB/s", "cores": threads, "kind": "oracle",
                             "sample": sample},
            "e2e": {"value": value, "unit": "GB/s", "h2d_bytes_per_step": 0,
                    "d2h_bytes_per_step": 0}}


def _json_stdout():
    """The one JSON line goes to the process's stdout; anything else a library
    writes there (NCCL prints its version at start-up, for instance) is sent
    to stderr instead, so that stdout holds exactly that line."""
    out = os.fdopen(os.dup(1), "w")
    sys.stdout.flush()
    os.dup2(2, 1)
    return out


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=200)
    ap.add_argument("--warmup", type=int, default=16)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--config", choices=sorted(CONFIGS), default="decode")
    ap.add_argument("--e2e-steps", type=int, default=5)
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-cpu", action="store_true")
    ap.add_argument("--no-recall", action="store_true")
    ap.add_argument("--graph", action="store_true",
                    help="time CUDA-graph replays of the step instead of eager launches")
    ap.add_argument("--context", action="store_true",
                    help="also time exact top-k (this library and torch.topk) on the same input")
    ap.add_argument("--no-sweep", action="store_true",
                    help="skip the per-workload sweep that rides along with a one-GPU line")
    args = ap.parse_args()
    if args.warmup < 3:
        ap.error("--warmup must be >= 3")
    if args.gpus < 1:
        ap.error("--gpus must be >= 1")
    if args.graph and CONFIGS[args.config]["kind"] == "split":
        ap.error("the row-split workload holds collectives: it is timed eagerly")
    if "WORLD_SIZE" not in os.environ and args.gpus > 1:
        relaunch_with_torchrun(args.gpus)  # does not return
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    if world != args.gpus:
        ap.error("--gpus %d but %d ranks were launched (WORLD_SIZE)" % (args.gpus, world))
    out = _json_stdout()
    if args.impl == "reference":
        if rank != 0:
            return
        line = run_reference(args, world, rank, int(os.environ.get("LOCAL_RANK", "0")))
        print(json.dumps(line), file=out, flush=True)
        return
    world, rank, local = setup_dist(args)
    line = run_ours(args, world, rank, local)
    if rank == 0:
        print(json.dumps(line), file=out, flush=True)
    if torch.distributed.is_initialized():
        torch.distributed.destroy_process_group()


def relaunch_with_torchrun(n: int) -> None:
    """`bench.py --gpus N` started as a single process: run it again as N
    ranks, one per GPU, under torch.distributed.run on this node."""
    import socket

    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    cmd = [sys.executable, "-m", "torch.distributed.run", "--nnodes=1", "--nproc-per-node", str(n),
           "--master-addr", "127.0.0.1", "--master-port", str(port), os.path.abspath(__file__),
           *sys.argv[1:]]
    sys.stdout.flush()
    os.execv(sys.executable, cmd)


if __name__ == "__main__":
    main()
