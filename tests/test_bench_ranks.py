"""Multi-rank host logic of bench.py on the CPU (gloo, world size 2): the job
time is the max over ranks, the value counts every rank's units, and the
reference arm prints from rank 0 only."""
import os
import subprocess
import sys

import pytest
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _worker(rank, world, port, q):
    import torch.distributed as dist
    sys.path.insert(0, ROOT)
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    import bench
    local_ms = 100.0 * (rank + 1)          # rank 1 is the slow one
    value, t_max = bench.job_rate(local_ms, 50, world, dist, "cpu")
    q.put((rank, value, t_max))
    dist.barrier()
    dist.destroy_process_group()


def test_job_rate_takes_max_over_ranks_gloo():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = 29500 + (os.getpid() % 1000)
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    res = sorted(q.get(timeout=120) for _ in procs)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    for rank, value, t_max in res:
        assert t_max == 200.0                       # the slowest rank's time
        assert value == pytest.approx(2 * 50 / 0.2)  # all ranks' units over the job time


def test_job_rate_single_rank():
    sys.path.insert(0, ROOT)
    import bench
    value, t_max = bench.job_rate(250.0, 100, 1)
    assert (value, t_max) == (400.0, 250.0)


def test_reference_arm_non_zero_rank_exits_silently():
    env = dict(os.environ, RANK="1", WORLD_SIZE="2", LOCAL_RANK="1")
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference",
                        "--steps", "3", "--warmup", "3", "--gpus", "2"],
                       capture_output=True, text=True, env=env, timeout=300)
    assert r.returncode == 0
    assert r.stdout.strip() == ""


def test_reference_arm_prints_the_contract_line():
    # rank 0 of a one-process run times the oracle and prints one JSON line
    # carrying the contract's keys, its own workload config and a cpu_baseline
    # and e2e that describe the same run
    import json
    env = {k: v for k, v in os.environ.items() if k not in ("RANK", "WORLD_SIZE", "LOCAL_RANK")}
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference",
                        "--workload", "corr_n2000_k8", "--steps", "3", "--warmup", "3"],
                       capture_output=True, text=True, env=env, timeout=600)
    assert r.returncode == 0, r.stderr[-2000:]
    lines = [l for l in r.stdout.splitlines() if l.startswith("{")]
    assert len(lines) == 1
    d = json.loads(lines[0])
    for key in ("metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step",
                "higher_is_better", "scaling", "vs_baseline", "dtype", "data", "config",
                "impl", "cpu_baseline", "e2e"):
        assert key in d, key
    assert d["impl"] == "reference" and d["n_gpus"] == 1
    assert d["steps"] == 3 and d["warmup"] == 3 and d["higher_is_better"] is True
    assert d["value"] > 0 and d["dtype"] == "f64"
    assert d["config"]["workload"] == "corr_n2000_k8" and d["config"]["n"] == 2000
    cb = d["cpu_baseline"]
    assert cb["kind"] == "oracle" and cb["value"] == d["value"] and cb["cores"] >= 1 and cb["sample"]
    assert d["e2e"] == {"value": d["value"], "unit": d["unit"],
                        "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}


def test_row_rooflines_and_config_on_the_cpu():
    # each row's fraction is its algorithmic bytes over its time, against the
    # given peak; the config names the workload and its sizes
    sys.path.insert(0, ROOT)
    import bench
    n, k, T, peak = 100000, 24, 1000, 6543.7
    sbytes = 4.0 * n * n
    rows = {"stats_ms": 8.0, "kmeans_steps": 10, "kmeans_ms_per_step": 16.0,
            "svrg_epoch_ms": 16.0, "tpdm_build_ms": 10.0}
    out, f16 = bench.row_rooflines(rows, n, k, T, peak)
    assert out["stats"]["GBs"] == pytest.approx(sbytes / 8e-3 / 1e9)
    assert out["stats"]["frac"] == pytest.approx(sbytes / 8e-3 / 1e9 / peak)
    assert out["kmeans_step"]["GBs"] == pytest.approx(2 * sbytes / 16e-3 / 1e9)
    assert out["svrg_epoch"]["GBs"] == pytest.approx(2 * sbytes / 16e-3 / 1e9)
    assert out["tpdm_build_writes"]["GBs"] == pytest.approx(sbytes / 10e-3 / 1e9)
    assert all(v["bound"] == "hbm" for v in out.values())
    assert f16 > 0
    cfg = bench.bench_config("corr_n100000_k24", 1)
    assert (cfg["workload"], cfg["n"], cfg["k"], cfg["T"]) == ("corr_n100000_k24", n, k, T)
    assert cfg["parallelism"] == "single"
    assert bench.bench_config("corr_n100000_k24", 8)["parallelism"].endswith("x8")


def test_bin_by_clock_groups_launches_by_the_nearest_sample():
    # launches of 10, 10, 12 and 14 ms from t = 100 s; samples at 100.000 s
    # (1965 MHz), 100.025 s (1600 MHz) and 100.035 s (1400 MHz): the launch
    # midpoints 100.005, 100.015, 100.026 and 100.039 take 1965, 1600, 1600
    # and 1400
    sys.path.insert(0, ROOT)
    import bench
    samples = [(100.0, 1965.0), (100.025, 1600.0), (100.035, 1400.0)]
    rows = bench.bin_by_clock([10.0, 10.0, 12.0, 14.0], 100.0, samples, 40.0, 6500.0)
    by = {tuple(r["sm_mhz_range"]): r for r in rows}
    assert by[(1800.0, None)]["launches"] == 1
    assert by[(1500.0, 1800.0)]["launches"] == 2 and by[(1500.0, 1800.0)]["ms"] == 11.0
    assert by[(0.0, 1500.0)]["launches"] == 1 and by[(0.0, 1500.0)]["ms"] == 14.0
    assert by[(0.0, 1500.0)]["GBs"] == pytest.approx(40.0 / 14.0 * 1e3)
    # no samples: one row over every launch
    assert bench.bin_by_clock([1.0, 3.0], 0.0, [], 1.0, 1.0)[0]["ms"] == 2.0
