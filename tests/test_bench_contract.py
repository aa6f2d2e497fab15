"""bench.py keeps its contract: one JSON line with every key its consumers read.  The reference arm
(the fp64 oracle on host cores) runs here on CPU; the CUDA arm runs its small profiling case on
the GPU (the same code path as the full line, T = 5632)."""
import json
import os
import subprocess
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
REQUIRED = ("metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step", "higher_is_better",
            "scaling", "vs_baseline", "dtype", "data", "config", "e2e")


def _run(args, timeout):
    proc = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py")] + args, cwd=ROOT, capture_output=True,
                          text=True, timeout=timeout)
    assert proc.returncode == 0, proc.stderr[-2000:]
    lines = [ln for ln in proc.stdout.splitlines() if ln.startswith("{")]
    assert len(lines) == 1, proc.stdout[-2000:]
    return json.loads(lines[0])


@pytest.mark.slow
def test_reference_arm_line():
    line = _run(["--impl", "reference", "--steps", "1", "--warmup", "0"], timeout=600)
    for k in REQUIRED:
        assert k in line, k
    assert line["impl"] == "reference" and line["value"] > 0
    assert line["cpu_baseline"]["kind"] == "oracle" and line["e2e"]["h2d_bytes_per_step"] == 0


def test_gpus_2_launches_two_ranks_over_one_sharded_batch():
    """--gpus 2 without a torchrun environment re-launches bench.py as two ranks; the dry run (gloo,
    CPU, no kernels) shows that each rank holds a contiguous whole-group shard of ONE global batch,
    that the shards cover it, that R* is the global number of responses and that the collective
    settings are pinned."""
    env = {k: v for k, v in os.environ.items() if k not in ("WORLD_SIZE", "RANK", "LOCAL_RANK")}
    proc = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--gpus", "2", "--dry-run"], cwd=ROOT,
                          capture_output=True, text=True, timeout=600, env=env)
    assert proc.returncode == 0, proc.stderr[-2000:]
    lines = [ln for ln in proc.stdout.splitlines() if ln.startswith("{")]
    assert len(lines) == 1, proc.stdout[-2000:]
    line = json.loads(lines[0])
    assert line["n_gpus"] == 2 and line["dry_run"] is True
    (a0, a1), (b0, b1) = line["shards"]
    assert a0 == 0 and a1 == b0 and b1 == line["global_rows"] and 0 < a1 < b1
    assert line["rows_all_ranks"] == line["global_rows"]
    assert line["resp_normalizer"] == 16  # two sub-batches of 2 x 4 responses
    assert line["collectives"] == {"NCCL_ALGO": "Ring", "NCCL_PROTO": "Simple"}


def test_world_size_other_than_gpus_is_refused():
    env = dict(os.environ, WORLD_SIZE="1", RANK="0", LOCAL_RANK="0")
    proc = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--gpus", "2", "--dry-run"], cwd=ROOT,
                          capture_output=True, text=True, timeout=300, env=env)
    assert proc.returncode != 0 and "WORLD_SIZE=1" in proc.stderr


@pytest.mark.gpu
def test_cuda_arm_line_small_case():
    line = _run(["--small", "--steps", "2", "--warmup", "3", "--no-cpu-baseline"], timeout=900)
    for k in REQUIRED + ("roofline", "clocks", "gpu_launches"):
        assert k in line, k
    assert line["value"] > 0 and line["gpu_launches"] > 0
    roof = line["roofline"]
    for k in ("bound", "achieved", "peak", "unit", "frac", "traffic"):
        assert k in roof, k
    assert 0 < roof["frac"] < 2
    assert line["e2e"]["value"] > 0 and line["e2e"]["h2d_bytes_per_step"] > 0


@pytest.mark.slow
def test_dense_reference_arm_line():
    line = _run(["--impl", "reference", "--workload", "dense", "--steps", "1", "--warmup", "0"], timeout=600)
    for k in REQUIRED:
        assert k in line, k
    assert line["impl"] == "reference" and line["unit"] == "TFLOP/s" and line["value"] > 0


@pytest.mark.gpu
def test_dense_workload_line():
    line = _run(["--workload", "dense", "--steps", "3", "--warmup", "3", "--no-cpu-baseline"], timeout=900)
    for k in REQUIRED + ("roofline", "rmsnorm_roofline", "clocks", "gpu_launches"):
        assert k in line, k
    assert line["gpu_launches"] == 6 and line["value"] > 0
    assert 0 < line["roofline"]["frac"] < 2 and 0 < line["rmsnorm_roofline"]["frac"] < 2
    assert line["e2e"]["d2h_bytes_per_step"] == 76239 * 8960 * 2


@pytest.mark.slow
def test_decode_reference_arm_line():
    line = _run(["--impl", "reference", "--workload", "decode", "--steps", "1", "--warmup", "0"], timeout=600)
    for k in REQUIRED:
        assert k in line, k
    assert line["impl"] == "reference" and line["higher_is_better"] is False and line["value"] > 0


@pytest.mark.gpu
def test_decode_workload_line():
    line = _run(["--workload", "decode", "--steps", "20", "--warmup", "3"], timeout=900)
    for k in REQUIRED + ("roofline", "clocks", "gpu_launches", "cluster_kernel_ms", "rows_128_ms"):
        assert k in line, k
    # three launches per one-row call: zeroing of the status and the tagged maxima, the single
    # pass over W on every SM, then the combine
    assert line["gpu_launches"] == 3 * 20 and line["value"] < line["cluster_kernel_ms"]
    assert 0 < line["roofline"]["frac"] < 2 and line["e2e"]["h2d_bytes_per_step"] > 0


def test_d3_reference_arm_line():
    line = _run(["--impl", "reference", "--workload", "d3", "--steps", "1", "--warmup", "0"], timeout=600)
    for k in REQUIRED:
        assert k in line, k
    assert line["impl"] == "reference" and line["unit"] == "GB/s" and line["value"] > 0


@pytest.mark.gpu
def test_d3_workload_line():
    line = _run(["--workload", "d3", "--steps", "10", "--warmup", "3"], timeout=900)
    for k in REQUIRED + ("roofline", "clocks", "gpu_launches", "cpu_baseline"):
        assert k in line, k
    # two launches per call: the block partials, then their fixed-order sum
    assert line["gpu_launches"] == 2 * 10
    assert line["roofline"]["bound"] == "hbm" and 0 < line["roofline"]["frac"] < 2
    assert line["e2e"]["h2d_bytes_per_step"] == 9 * (1 << 24)
