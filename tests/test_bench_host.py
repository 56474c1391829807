"""Host-side logic of bench.py, without a GPU: the max over ranks on two gloo ranks, the
dense step's GEMM choice, and the reference arm's JSON line."""
import json
import os
import socket
import subprocess
import sys
from types import SimpleNamespace

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)
import bench  # noqa: E402
import workloads  # noqa: E402


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, out_dir):
    import torch.distributed as dist
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        bench.barrier(world)
        got = bench.max_over_ranks(1.5 + rank, world)   # each rank's own time
        bench.barrier(world)
        with open(os.path.join(out_dir, f"r{rank}"), "w") as f:
            f.write(repr(got))
    finally:
        dist.destroy_process_group()


def test_max_over_ranks_on_two_gloo_ranks(tmp_path):
    import torch.multiprocessing as mp
    port = _free_port()
    mp.spawn(_rank_main, args=(2, port, str(tmp_path)), nprocs=2, join=True)
    for r in range(2):
        assert float(open(tmp_path / f"r{r}").read()) == 2.5      # the slower rank's time


def test_gemm_path_follows_the_scales():
    dense, wgrad = workloads.dense(), workloads.wgrad()
    auto = SimpleNamespace(gemm="auto")
    assert bench.gemm_path(auto, dense) == "ue8m0"               # power-of-two on both sides
    assert bench.gemm_path(auto, wgrad) == "promoted"            # FP32 scales
    assert bench.gemm_path(SimpleNamespace(gemm="promoted"), dense) == "promoted"
    with pytest.raises(SystemExit):
        bench.gemm_path(SimpleNamespace(gemm="ue8m0"), wgrad)


def test_spread_of_per_step_times():
    got = bench._spread([0.30, 0.10, 0.20, 0.25])
    assert got == {"mean": 0.2125, "median": 0.225, "best": 0.1}


def test_library_ceiling_reports_instead_of_raising():
    """The cuBLASLt FP8 ceiling leg is context only: without a usable GPU it returns an
    'unavailable' entry and the bench line is still printed."""
    import torch
    if torch.cuda.is_available():
        pytest.skip("a GPU is present: the leg would measure instead")
    flushed = []
    got = bench.library_fp8_ceiling(lambda: flushed.append(1), n=256, reps=1)
    assert set(got) == {"unavailable"} and got["unavailable"]
    json.dumps(got)


def _run_bench(*args, env=None):
    e = dict(os.environ, **(env or {}))
    return subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), *args], cwd=ROOT,
                          env=e, capture_output=True, text=True, timeout=600)


def test_reference_arm_line_on_rank0_and_silence_elsewhere():
    r = _run_bench("--impl", "reference", "--steps", "2", "--warmup", "1", "--workload", "tiny")
    assert r.returncode == 0, r.stderr[-2000:]
    line = json.loads(r.stdout.strip().splitlines()[-1])
    for key in ("metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step",
                "higher_is_better", "scaling", "vs_baseline", "dtype", "data", "config",
                "cpu_baseline", "e2e"):
        assert key in line, key
    assert line["impl"] == "reference" and line["value"] > 0
    assert line["e2e"]["value"] == line["value"] and line["e2e"]["h2d_bytes_per_step"] == 0
    assert line["config"] == bench.bench_config(workloads.tiny(), 1)
    r1 = _run_bench("--impl", "reference", "--steps", "1", "--warmup", "1", "--workload", "tiny",
                    env={"RANK": "1", "WORLD_SIZE": "2"})
    assert r1.returncode == 0 and r1.stdout.strip() == ""
