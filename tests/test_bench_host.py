"""Host-side logic of bench.py, without a GPU: the max over ranks on two gloo ranks, the
dense step's GEMM choice, the reference arm's JSON line, and the timing loop's rule for
keeping the host ahead of the GPU (_enqueue_ahead, against a stand-in for torch.cuda)."""
import json
import os
import socket
import subprocess
import sys
from types import SimpleNamespace

import numpy as np
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


def test_bench_fp64_reference_agrees_with_the_oracle():
    """The bench's own float64 product (used by its spot check and accumulation study,
    which must not call the oracle) against the oracle's reference on oracle codes."""
    import oracle
    assert np.array_equal(bench._e4m3_values(), oracle.decode_table(), equal_nan=True)
    rng = np.random.default_rng(11)
    a = workloads.normal_bf16(rng, (5, 384), 1.0, 0.01)
    b = workloads.normal_bf16(rng, (256, 384), 0.02)
    qa, sa = oracle.quant_act_1x128(a, False)
    for rowwise in (False, True):
        qb, sb = oracle.quant_act_1x128(b, True) if rowwise else oracle.quant_weight_128x128(b, False)
        want, want_T = oracle.gemm_blockscaled_ref(qa, sa, qb, sb, b_rowwise=rowwise)
        got, got_T = bench._fp64_product(qa, sa, qb, sb, rowwise)
        assert np.allclose(got, want, rtol=1e-12, atol=0) and np.allclose(got_T, want_T, rtol=1e-12)


@pytest.mark.parametrize("out_fp32", [False, True])
def test_bench_band_is_the_parity_tests_band(out_fp32):
    import oracle
    rng = np.random.default_rng(12)
    C_ref = rng.standard_normal(4000) * np.exp2(rng.integers(-140, 20, 4000))
    C_ref[:10] = 0.0
    T = np.abs(C_ref) * np.exp2(rng.uniform(0, 12, 4000))
    C = C_ref * (1 + rng.standard_normal(4000) * np.exp2(rng.uniform(-30, -4, 4000)))
    C = C.astype(np.float32).astype(np.float64)
    want = oracle.check_fp32(C, C_ref, T) if out_fp32 else oracle.check_bf16(C, C_ref, T)[0]
    got = bench._within_band(C, C_ref, T, out_fp32)
    assert 0 < got.sum() < got.size
    assert np.array_equal(got, want)


def test_spot_check_on_host_tensors():
    import oracle
    import torch
    w = SimpleNamespace(M=256, b_rowwise=True, out_fp32=False)   # the step's mode wins
    rng = np.random.default_rng(13)
    qa, sa = oracle.quant_act_1x128(workloads.normal_bf16(rng, (256, 256), 1.0), False)
    qb, sb = oracle.quant_weight_128x128(workloads.normal_bf16(rng, (128, 256), 0.02), False)
    C_ref, _ = oracle.gemm_blockscaled_ref(qa, sa, qb, sb)
    t = torch.from_numpy
    C = t(C_ref.astype(np.float32)).to(torch.bfloat16)
    got = bench.spot_check(w, t(qa), t(sa), t(qb), t(sb), C)
    assert got["within_band"] and got["entries"] == 4 * 128
    C[128, 5] += 1.0                                   # a planted error in a checked row
    assert not bench.spot_check(w, t(qa), t(sa), t(qb), t(sb), C)["within_band"]
    # ROW-mode B scales (1x128 along K), as a caller with a Wgrad-style GEMM passes them
    qb_r, sb_r = oracle.quant_act_1x128(workloads.normal_bf16(rng, (128, 256), 1.0), False)
    C_r, _ = oracle.gemm_blockscaled_ref(qa, sa, qb_r, sb_r, b_rowwise=True)
    got = bench.spot_check(SimpleNamespace(M=256, out_fp32=True), t(qa), t(sa), t(qb_r), t(sb_r),
                           t(C_r.astype(np.float32)), b_rowwise=True)
    assert got["within_band"]


def test_accumulation_study_runs_on_host_stand_ins(monkeypatch):
    """The accumulation study's plumbing (row sampling, scale layouts, the float64 products
    of the same codes) on a small workload, with the library replaced by oracle-backed
    host stand-ins whose GEMMs are the exact product rounded to fp32: every reported
    error is then at fp32 rounding level."""
    import oracle
    import torch
    t = torch.from_numpy
    v = oracle.decode_table()

    def bits(x):
        return x.view(torch.int16).numpy().view(np.uint16)

    def gemm_blockscaled(qa, sa, qb, sb, out_dtype, b_rowwise):
        C, _ = bench._fp64_product(qa.numpy(), sa.numpy(), qb.numpy(), sb.numpy(), b_rowwise)
        return t(C.astype(np.float32))

    def gemm_nopromo(qa, sa, qb, sb):
        A = v[qa.numpy()] * sa.numpy().astype(np.float64)[:, None]
        B = v[qb.numpy()] * sb.numpy().astype(np.float64)[:, None]
        return t((A @ B.T).astype(np.float32))

    fake = SimpleNamespace(
        quant_act_1x128=lambda x, pow2: tuple(map(t, oracle.quant_act_1x128(bits(x), pow2))),
        quant_rowwise=lambda x: tuple(map(t, oracle.quant_rowwise(bits(x)))),
        gemm_blockscaled=gemm_blockscaled, gemm_nopromo=gemm_nopromo)
    monkeypatch.setattr(bench, "dev_bf16",
                        lambda b: t(np.ascontiguousarray(b).view(np.int16)).view(torch.bfloat16))
    monkeypatch.setattr(torch.cuda, "synchronize", lambda *a, **k: None)
    w = SimpleNamespace(M=96, N=256, a_std=1e-3, b_std=1.0)
    res = bench.accumulation_study(fake, rows_sampled=8, seeds=(0, 1), ks=(256, 512), w=w)
    assert res["rows_sampled"] == 8 and res["seeds"] == [0, 1]
    assert [r["K"] for r in res["results"]] == [256, 512]
    for r in res["results"]:
        for key in ("promoted_1x128", "promoted_1xK_codes", "no_promotion_1xK_codes"):
            mx, fro = r[key]["max_rel_T"], r[key]["rel_frobenius"]
            assert len(mx["per_seed"]) == 2 and mx["min"] <= mx["max"]
            assert 0 <= mx["max"] < 1e-7 and fro["max"] < 1e-6
    json.dumps(res)


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


class _FakeCuda:
    """Stand-in for torch.cuda in _enqueue_ahead: records the spin lengths and answers the
    spin's completion query from a script (True: the spin had ended before the host
    finished enqueueing)."""

    def __init__(self, caught_up):
        self.caught_up = list(caught_up)
        self.spins = []
        self.syncs = 0
        fake = self

        class Event:
            def record(self, stream):
                pass

            def query(self):
                return fake.caught_up.pop(0)

        self.Event = Event

    def current_stream(self):
        return object()

    def synchronize(self):
        self.syncs += 1

    def _sleep(self, cycles):
        self.spins.append(cycles)


def _run_enqueue_ahead(monkeypatch, caught_up, **kw):
    import torch
    fake = _FakeCuda(caught_up)
    for name in ("Event", "current_stream", "synchronize", "_sleep"):
        monkeypatch.setattr(torch.cuda, name, getattr(fake, name))
    calls = []
    out = bench._enqueue_ahead(lambda: calls.append(len(calls)) or len(calls), **kw)
    return fake, calls, out


def test_enqueue_ahead_keeps_the_first_run_when_the_spin_outlasted_the_host(monkeypatch):
    fake, calls, out = _run_enqueue_ahead(monkeypatch, [False], lead_ms=20.0)
    assert calls == [0] and out == 1
    assert fake.spins == [int(20.0 * 2.0e6)]
    assert fake.syncs == 2          # before the spin, and after the work before returning


def test_enqueue_ahead_doubles_the_spin_until_it_outlasts_the_host(monkeypatch):
    fake, calls, out = _run_enqueue_ahead(monkeypatch, [True, True, False], lead_ms=20.0)
    assert calls == [0, 1, 2] and out == 3      # the work of the last run is returned
    assert fake.spins == [int(ms * 2.0e6) for ms in (20.0, 40.0, 80.0)]


def test_enqueue_ahead_stops_at_its_longest_spin(monkeypatch):
    fake, calls, out = _run_enqueue_ahead(monkeypatch, [True] * 10, lead_ms=20.0, max_ms=80.0)
    assert len(calls) == 3 and fake.spins == [int(ms * 2.0e6) for ms in (20.0, 40.0, 80.0)]
