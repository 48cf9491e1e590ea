"""bench.py as the driver runs it (small workload): one JSON line per run
with the contract's keys, for the eager arm, the CUDA-graph arm and the
reference (oracle) arm."""
import json
import os
import subprocess
import sys

import pytest

sys.path.insert(0, os.path.dirname(os.path.dirname(os.path.abspath(__file__))))

pytestmark = pytest.mark.gpu

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
KEYS = {"metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step", "higher_is_better",
        "scaling", "vs_baseline", "dtype", "data", "config", "roofline", "gpu_launches", "clocks",
        "step_ms"}


def _run(*args):
    out = subprocess.run([sys.executable, "bench.py", *args], cwd=ROOT, capture_output=True,
                         text=True, timeout=600)
    assert out.returncode == 0, out.stderr[-2000:]
    lines = [ln for ln in out.stdout.splitlines() if ln.strip()]
    assert len(lines) == 1, out.stdout
    return json.loads(lines[0])


@pytest.mark.parametrize("extra", [[], ["--graph"]])
def test_bench_line(extra):
    d = _run("--config", "tiny", "--steps", "20", "--warmup", "3", "--no-cpu", "--no-sweep", *extra)
    assert KEYS <= set(d)
    assert d["value"] > 0 and d["n_gpus"] == 1 and d["steps"] == 20 and d["warmup"] == 3
    assert d["config"]["workload"] == "tiny"
    assert d["config"]["launch"] == ("cuda-graph replay" if extra else "eager")
    r = d["roofline"]
    assert r["bound"] == "hbm" and r["peak"] > 0 and r["frac"] > 0
    e = d["e2e"]
    assert e["h2d_bytes_per_step"] == 8 * 4096 * 4 and e["d2h_bytes_per_step"] == 8 * 64 * 8
    assert d["gpu_launches"] == 20
    st = d["step_ms"]
    assert 0 < st["median"] <= st["p90"]


def test_reference_line():
    d = _run("--impl", "reference", "--config", "tiny", "--steps", "2", "--warmup", "3")
    assert d["impl"] == "reference" and d["value"] > 0
    assert d["cpu_baseline"]["kind"] == "oracle" and d["cpu_baseline"]["cores"] >= 1
    assert d["e2e"]["h2d_bytes_per_step"] == 0
    assert d["steps"] == 2 and d["warmup"] == 3
    ours = _run("--config", "tiny", "--steps", "2", "--warmup", "3", "--no-cpu", "--no-sweep",
                "--no-e2e")
    assert d["config"] == ours["config"]
    assert (d["metric"], d["unit"], d["higher_is_better"]) == \
        (ours["metric"], ours["unit"], ours["higher_is_better"])


def test_default_line_carries_the_sweep():
    """The default workload's line, with the sweep of every score-row cell
    (fp32 and bf16) and the fused workloads, each with its own timing."""
    d = _run("--steps", "5", "--warmup", "3", "--no-cpu", "--no-e2e", "--no-recall")
    assert d["config"]["workload"] == "decode"
    sw = d["sweep"]
    import bench
    assert set(sw) == set(bench.SWEEP)
    for name, cell in sw.items():
        assert cell["ms_per_step"] > 0 and 0 < cell["frac"] < 1.5, name
        assert cell["bound"] in ("hbm", "tensor"), name
        assert 0 < cell["step_ms"]["median"] <= cell["step_ms"]["p90"], name


def test_split_workload_one_gpu():
    """The vocabulary-parallel workload in a one-rank group: selection on the
    slice, the NCCL all-gather, the merge kernel; two launches per step."""
    d = _run("--config", "vocab-split", "--steps", "10", "--warmup", "3", "--no-cpu",
             "--no-sweep")
    assert d["config"]["workload"] == "vocab-split" and d["gpu_launches"] == 20
    assert d["value"] > 0 and d["recall"]["mean"] > 0.9
