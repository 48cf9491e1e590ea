"""Host logic of the benchmark contract, on the CPU: which kernel a workload's
roofline names, the committed DRAM traffic lookup (valid only while the
kernel's device sources hash to the captured value), input rotation against
L2, and the launch count claimed per step."""
import math

import bench


def test_every_config_names_a_kernel_with_sources():
    for name, cfg in bench.CONFIGS.items():
        k = bench._kernel_name(cfg)
        assert k in bench._KERNEL_SOURCES, (name, k)
        assert len(bench._source_hash(k)) == 16


def test_kernel_choice_follows_the_library_dispatch():
    assert bench._kernel_name(bench.CONFIGS["decode"]) == "score_select_gemv"
    assert bench._kernel_name(bench.CONFIGS["link"]) == "score_select_umma_pair"
    assert bench._kernel_name(bench.CONFIGS["vocab"]) == "bucket_select_tma"
    assert bench._kernel_name(bench.CONFIGS["long-b512-kb4"]) == "bucket_select_wide"
    assert bench._kernel_name(bench.CONFIGS["long-b256-kb4"]) == "bucket_select_tma"
    assert bench._kernel_name(bench.CONFIGS["long-b512-kb4-bf16"]) == "bucket_select_tma"
    assert bench._kernel_name(bench.CONFIGS["decode-rerank"]) == "rerank_kernel"


def test_traffic_rows_match_the_current_sources():
    """Every traffic row of the committed summary refers to a known kernel;
    a row whose hash is current yields its byte count, others yield None."""
    rows = 0
    for line in open(bench.os.path.join(bench.ROOT, "profiles", "traffic.md")):
        cells = [c.strip() for c in line.strip().strip("|").split("|")]
        if len(cells) >= 4 and cells[1] in bench._KERNEL_SOURCES:
            rows += 1
            got = bench._traffic(cells[0])
            if cells[2] == bench._source_hash(cells[1]):
                assert got == int(cells[3])
            else:
                assert got is None
    assert rows >= 4
    assert bench._traffic("no-such-workload") is None


def test_launches_per_step():
    assert bench._launches_per_step(bench.CONFIGS["link"]) == 2
    assert bench._launches_per_step(bench.CONFIGS["decode"]) == 1
    assert bench._launches_per_step(bench.CONFIGS["vocab-sample"]) == 1  # draw fused
    assert bench._launches_per_step(bench.CONFIGS["vocab"]) == 1


class _W:
    def __init__(self, in_bytes):
        self.in_bytes = in_bytes


def test_rotations_defeat_l2():
    """Inputs under twice the L2 (the 128 MiB score rows among them) rotate
    over copies spanning at least three L2s; larger inputs stream as they are."""
    assert bench._rotations(_W(4 << 30)) == 1
    assert bench._rotations(_W(2 * bench.L2_BYTES)) == 1
    for b in (1 << 17, 64 << 20, 120 << 20, 128 << 20, 2 * bench.L2_BYTES - 1):
        n = bench._rotations(_W(b))
        assert n >= 2 and n * b >= 3 * bench.L2_BYTES


def test_tensor_peak_burst_or_sustained():
    """A timed region shorter than a couple of seconds compares with the burst
    GEMM peak, a longer one with the sustained (power-capped) figure."""
    short, src_s = bench._tensor_peak(0.05)
    long_, src_l = bench._tensor_peak(10.0)
    assert "sustained" not in src_s and short >= long_
    assert "sustained" in src_l


def test_sweep_cells_exist():
    for name in bench.SWEEP:
        assert name in bench.CONFIGS, name
    for b in (128, 256, 512):
        for kb in (1, 2, 4):
            assert "long-b%d-kb%d" % (b, kb) in bench.SWEEP
            assert "long-b%d-kb%d-bf16" % (b, kb) in bench.SWEEP
    assert {"vocab", "vocab-bf16"} <= set(bench.SWEEP)


def test_split_workload_launches():
    assert bench._launches_per_step(bench.CONFIGS["vocab-split"]) == 2
    assert bench._kernel_name(bench.CONFIGS["vocab-split"]) == "bucket_select_tma"


def test_job_throughput_is_weak_scaling():
    assert math.isclose(bench.job_throughput(1e9, 2.0, 4), 4 * 1e9 / 2e-3 / 1e9)


def test_step_distribution():
    """Median and nearest-rank 90th percentile of the per-step times."""
    d = bench.step_distribution([5.0, 1.0, 3.0, 2.0, 4.0])
    assert d == {"median": 3.0, "p90": 5.0}
    d = bench.step_distribution([float(x) for x in range(1, 21)])  # 1..20
    assert d["median"] == 10.5 and d["p90"] == 18.0
    assert bench.step_distribution([7.0]) == {"median": 7.0, "p90": 7.0}
    assert bench.step_distribution([]) == {"median": None, "p90": None}
