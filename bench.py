#!/usr/bin/env python
"""SymNMF iterations/s and S-stream HBM GB/s at n = 100,000, k = 24, fp32.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
                    [--workload corr_n100000_k24] [--no-cpu-baseline]

A step is one iteration of the full-batch fit on a resident |corr| matrix:
one pass over S forming S H, the trace-identity loss, the gradient, the
AdaGrad accumulator and projected update, and the Gram of the new H.  The
timed region is one symnmf_fit call that runs K such passes (W warm-up passes
in a separate call first).  S (40 GB) exceeds L2 many times over, so no flush
is needed between iterations.

With N > 1 (torchrun, one process per GPU) every rank factorises its own
window (seed = rank): independent problems, weak scaling, no data-path
collective.  The max over ranks of the device time defines the job time.

--impl reference times the CPU oracle (the plain fp64 numpy restatement of
the method) on the host cores instead, on a bounded sample of the same
workload, scaled to the metric's unit.
"""
from __future__ import annotations

import argparse
import json
import math
import os
import statistics
import subprocess
import sys
import tempfile
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import numpy as np  # noqa: E402

import synth  # noqa: E402

METRIC = "SymNMF iterations/sec and S-stream HBM GB/s (% of peak) at n=1e5, k=24 fp32"
UNIT = "iterations/s"
SAMPLE_ROWS = 8192   # oracle sample: leading principal r x r block of the same window
# DRAM traffic of one launch of each S-stream kernel from ncu (dram__bytes_read.sum
# + dram__bytes_write.sum) at n = 20,000, k = 24, over its algorithmic bytes
# (4n^2 + 4nk = 1.602 GB); the full-size launch (40 GB S, too large to capture)
# is reported as the same ratio times its algorithmic bytes.  A kernel without
# an entry (changed since its capture) reports null.  Retake a capture whenever
# its kernel changes.
STREAM_TRAFFIC_RATIO = {
    "stream_tc_kernel": (1.618906e9 + 13.768704e6) / (4.0 * 20000 ** 2 + 4.0 * 20000 * 24),
}
STREAM_TRAFFIC_SOURCE = ("ncu dram__bytes_read.sum + dram__bytes_write.sum of one launch at "
                         "n = 20,000, k = 24, scaled to this launch by algorithmic bytes")


def parse():
    ap = argparse.ArgumentParser(description=__doc__, formatter_class=argparse.RawDescriptionHelpFormatter)
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=100)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", default="corr_n100000_k24")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-rows", action="store_true", help="skip the per-row timings")
    ap.add_argument("--sharded", action="store_true",
                    help="the row-sharded fit (the default with more than one GPU)")
    ap.add_argument("--replicas", action="store_true",
                    help="with more than one GPU: independent windows, one per GPU")
    ap.add_argument("--upper", action="store_true",
                    help="time the upper-triangle S-stream (upper_only = 1) in the main loop")
    ap.add_argument("--h16-min-n", type=int, default=None,
                    help="size from which full-batch fits run the fp16 S-stream "
                         "(sets SYMNMF_H16_MIN_N; the library's default is 20000, 0 = never)")
    args = ap.parse_args()
    if args.h16_min_n is not None:
        os.environ["SYMNMF_H16_MIN_N"] = str(args.h16_min_n)
    return args


# ----------------------------------------------------------------------------- plumbing
def dist_env():
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return world, rank, local


def peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            d = json.load(f)
        return float(d["hbm_gbs"]), "measured"
    except Exception:
        return 6650.0, "fallback"


class ClockSampler:
    """nvidia-smi clock/throttle samples every 200 ms while the timed region runs."""

    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.gpu = gpu_index
        self.proc = None
        self.out = None

    def start(self):
        try:
            self.out = tempfile.TemporaryFile(mode="w+")
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.gpu), f"--query-gpu={self.FIELDS}",
                 "--format=csv,noheader,nounits", "-lms", "200"],
                stdout=self.out, stderr=subprocess.DEVNULL)
        except Exception:
            self.proc = None

    def stop(self):
        if self.proc is None:
            return None
        time.sleep(0.25)
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        self.out.seek(0)
        rows = [r.split(",") for r in self.out.read().strip().splitlines() if r.strip()]
        sm, mx, reasons = [], 0.0, set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for r in rows:
            try:
                sm.append(float(r[1]))
                mx = max(mx, float(r[2]))
                for name, v in zip(names, r[5:9]):
                    if v.strip().lower() in ("active", "1"):
                        reasons.add(name)
            except (ValueError, IndexError):
                continue
        if not sm:
            return None
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": mx, "reasons": sorted(reasons),
                "samples": len(sm)}


def cpu_threads():
    try:
        from threadpoolctl import threadpool_info
        n = [i.get("num_threads", 0) for i in threadpool_info() if i.get("user_api") == "blas"]
        if n:
            return int(max(n))
    except Exception:
        pass
    return os.cpu_count() or 1


def oracle_sample(name: str, seed: int, steps: int, warmup: int):
    """Oracle fit on the leading r x r principal block of the same window.

    One oracle iteration costs O(r^2 k) (dominated by S H), so the per-
    iteration time at the full n is the sample time scaled by (n / r)^2.
    """
    import oracle
    spec = synth.WORKLOADS[name]
    n, k = spec["n"], spec["k"]
    r = min(SAMPLE_ROWS, n)
    R, _, _ = synth.workload(name, seed=seed)
    S = oracle.corr_abs(R[:, :r]).astype(np.float32)
    s_sum, sq, _ = oracle.stats(S)
    H0 = oracle.scale_matched_init(s_sum, r, k, 1000 + seed)
    if warmup > 0:
        oracle.fit_adagrad(S, k, H0, max_iters=warmup - 1, S_sqnorm=sq)
    t0 = time.perf_counter()
    oracle.fit_adagrad(S, k, H0, max_iters=max(steps - 1, 0), S_sqnorm=sq)
    dt = time.perf_counter() - t0
    per_iter_full = dt / max(steps, 1) * (n / r) ** 2
    return {
        "value": 1.0 / per_iter_full,
        "unit": UNIT,
        "cores": cpu_threads(),
        "kind": "oracle",
        "sample": (f"{steps} oracle fp64 full-batch iterations on the leading {r}x{r} principal "
                   f"block of the n={n} |corr| window (seed {seed}); per-iteration time scaled "
                   f"by (n/r)^2 = {(n / r) ** 2:.1f}"),
        "sample_seconds": dt,
        "sample_block": r,
        "sample_iters": steps,
        "scale_to_full": (n / r) ** 2,
    }


def job_rate(local_ms: float, units_per_rank: int, world: int, dist=None, device=None):
    """Whole-job throughput of a weak-scaled run: every rank processed
    `units_per_rank` units in `local_ms`; the job time is the max over ranks.
    Returns (units per second over all ranks, job time in ms)."""
    import torch
    t = torch.tensor([float(local_ms)], dtype=torch.float64, device=device)
    if world > 1 and dist is not None:
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
    t_max = float(t.item())
    return world * units_per_rank / (t_max / 1000.0), t_max


def _timed(torch, fn):
    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    torch.cuda.synchronize()
    a.record()
    out = fn()
    b.record()
    torch.cuda.synchronize()
    return a.elapsed_time(b), out


def stream_clock_bins(m, torch, dev, S, H0, n, k, peak):
    """The fit's S-stream launch time against the SM clock.  After a second of
    idle, a 60-iteration fit on S (the sustained regime, where the power cap
    lowers the SM clock) with every stream launch timed by CUDA events; then
    12 single-pass fits, each after 40 ms of idle (the pass follows the fit's
    statistics read of S).  nvidia-smi samples the clock every 50 ms; each
    back-to-back launch takes the sample nearest its midpoint, and launches
    are grouped by that clock.  The stream is the one the fit runs
    (`stream_kernel` in the row)."""
    import datetime
    gpu = int(os.environ.get("LOCAL_RANK", "0"))
    m.fit(S, k, seed=1000, max_iters=1, rel_tol=0.0)   # warm (workspace, attributes)
    out_f = tempfile.TemporaryFile(mode="w+")
    proc = subprocess.Popen(["nvidia-smi", "-i", str(gpu), "--query-gpu=timestamp,clocks.sm",
                             "--format=csv,noheader,nounits", "-lms", "50"],
                            stdout=out_f, stderr=subprocess.DEVNULL)
    try:
        torch.cuda.synchronize()
        time.sleep(1.0)
        _, st = m.fit(S, k, seed=1000, max_iters=59, rel_tol=0.0, stream_times=True)
        torch.cuda.synchronize()
        t_end = time.time()
        b2b = st["stream_ms_each"]
        t_start = t_end - st["loop_ms"] / 1e3   # the loop ends just before the call returns
        kind = m._lib.STREAM_KERNEL_NAMES.get(st.get("stream_kernel", 0), "stream_tc_kernel")
        spaced = []
        for _ in range(12):
            time.sleep(0.04)
            _, s1 = m.fit(S, k, seed=1000, max_iters=0, rel_tol=0.0, stream_times=True)
            torch.cuda.synchronize()
            spaced.append(s1["stream_ms_each"][0])
        time.sleep(0.1)
    finally:
        proc.terminate()
        try:
            proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            proc.kill()
    out_f.seek(0)
    samples = []
    for line in out_f.read().strip().splitlines():
        try:
            ts, mhz = line.split(",")[:2]
            t = datetime.datetime.strptime(ts.strip(), "%Y/%m/%d %H:%M:%S.%f").timestamp()
            samples.append((t, float(mhz)))
        except (ValueError, IndexError):
            continue
    gb = (4.0 * n * n + 4.0 * n * k) / 1e9
    return {"stream_kernel": kind, "spaced": _launch_row(spaced, [], gb, peak),
            "back_to_back": bin_by_clock(b2b, t_start, samples, gb, peak)}


def _launch_row(ms_list, mhz_list, gb, peak):
    ms = statistics.median(ms_list)
    return {"launches": len(ms_list), "ms": ms, "GBs": gb / ms * 1e3, "frac": gb / ms * 1e3 / peak,
            "sm_mhz": statistics.median(mhz_list) if mhz_list else None}


def bin_by_clock(ms_list, t_start, samples, gb, peak,
                 edges=((1800.0, None), (1500.0, 1800.0), (0.0, 1500.0))):
    """Back-to-back launch times (ms, in order from host time t_start) grouped
    by the clock sample (time, MHz) nearest each launch's midpoint."""
    if not samples:
        return [_launch_row(ms_list, [], gb, peak)]
    clk, t = [], t_start
    for ms in ms_list:
        mid = t + ms / 2e3
        clk.append(min(samples, key=lambda sm: abs(sm[0] - mid))[1])
        t += ms / 1e3
    out = []
    for lo, hi in edges:
        sel = [i for i in range(len(ms_list)) if clk[i] >= lo and (hi is None or clk[i] < hi)]
        if sel:
            r = _launch_row([ms_list[i] for i in sel], [clk[i] for i in sel], gb, peak)
            r["sm_mhz_range"] = [lo, hi]
            out.append(r)
    return out


def converge_row(m, torch, S, k, planted_dev, solver, **kw):
    """One fit to the relative-loss-change stop (rel < 1e-5), timed with CUDA
    events: passes or epochs, seconds, loss, ARI of its labels against the
    planted groups, and a sampled loss curve."""
    ms, (H, st) = _timed(torch, lambda: m.fit(S, k, seed=1000, solver=solver, rel_tol=1e-5,
                                              history=True, **kw))
    lab = m.labels(H)
    h = st["history"]
    pts = sorted({0, 1, 2, 5, 10, 20, 50, 100, 200, 500, 1000, 2000, 5000, 10000, len(h) - 1}
                 & set(range(len(h))))
    return lab, {
        "solver": solver, "seconds": ms / 1e3, "converged": bool(st["converged"]),
        "full_batch_passes": st["iters"], "epochs": st["epochs"], "evaluations": st["evaluations"],
        "block_final": st["block_final"], "loss": st["loss"], "rel_change": st["rel_change"],
        "s_sqnorm": st["s_sqnorm"], "explained": 1.0 - st["loss"] / st["s_sqnorm"],
        "ARI_vs_planted": m.ari(lab, planted_dev, max(k, int(planted_dev.max().item()) + 1))[0],
        "loss_curve": {str(i): float(h[i]) for i in pts}}


def measure_rows(m, torch, dev, S, H0, lab, n, k, T, rank, workload, planted=None):
    """One timing per remaining row of the path on the resident |corr| matrix
    (probe, labels, statistics, spherical k-means), on a TPDM of the
    heavy-tailed window of the same size (builder, one Block-SVRG epoch), and
    the rolling-window study at its own size (n = 5,000, 250 windows)."""
    out = {}
    # the S-stream against the SM clock (sustained back-to-back vs spaced launches)
    if n >= 50000:
        try:
            out["stream_clock_bins"] = stream_clock_bins(m, torch, dev, S, H0, n, k, peaks()[0])
        except Exception as exc:
            out["stream_clock_bins"] = {"error": f"{type(exc).__name__}: {exc}"}
    # statistics pre-pass: one read of S
    ws = m.workspace(m._lib.OP_STATS, n, device=dev)
    ms, _ = _timed(torch, lambda: m.stats(S, ws=ws))
    out["stats_ms"] = ms
    out["stats_GBs"] = 4.0 * n * n / (ms / 1e3) / 1e9
    # labels
    ms, _ = _timed(torch, lambda: m.labels(H0))
    out["labels_ms"] = ms
    # spectral probe of the k+2 leading eigenvalues (block Lanczos on the S-stream)
    p = m.fit_params(probe_block=16, probe_max_iter=12)
    wsp = m.workspace(m._lib.OP_SPECTRAL_PROBE, n, k + 2, params=p, device=dev)
    ms, ev = _timed(torch, lambda: m.spectral_probe(S, k + 2, block=16, max_iter=12, tol=1e-7, ws=wsp))
    info = m.probe_last_info()
    out["probe_ms"] = ms
    out["probe_s_passes"] = info["s_passes"]
    out["probe_block_steps"] = info["block_steps"]
    out["probe_GBs"] = info["s_passes"] * 4.0 * n * n / (ms / 1e3) / 1e9
    out["probe_top"] = [float(x) for x in ev[:3]]
    out["probe_gamma_k1"] = float(ev[k] / abs(ev[k + 1]))
    del wsp
    # TPDM of the heavy-tailed window (same n, T) into a second n x n buffer
    tname = workload.replace("corr", "tpdm")
    if tname in synth.WORKLOADS:
        Rt, _, _ = synth.workload(tname, seed=rank)
        Rt = torch.from_numpy(Rt).to(dev)
        S2 = m.alloc_S(n, dev)
        wst = m.workspace(m._lib.OP_BUILD_TPDM, n, 0, T, device=dev)
        m.build_tpdm(Rt, 0.05, 1, out=S2, ws=wst)   # warm-up (cudaFuncSetAttribute etc.)
        ms, _ = _timed(torch, lambda: m.build_tpdm(Rt, 0.05, 1, out=S2, ws=wst))
        out["tpdm_build_ms"] = ms
        out["tpdm_build_write_GBs"] = 4.0 * n * n / (ms / 1e3) / 1e9
        del wst, Rt
        # Block-SVRG epochs at the workload's block (snapshot + m block steps): a
        # 3-epoch fit minus a 1-epoch fit, so the fit's setup (statistics pass,
        # start, Gram of H0) is not counted as epoch time
        b = 8192 if n >= 100000 else 2048
        pf = m.fit_params(solver="block_svrg", block_rows=b, max_iters=3, rel_tol=0.0, grow=0)
        wsf = m.workspace(m._lib.OP_FIT, n, k, params=pf, device=dev)
        Hs = H0.clone()
        svrg = {}
        for E in (1, 3):
            Hs.copy_(H0)
            svrg[E] = _timed(torch, lambda: m.fit(S2, k, H0=Hs, out=Hs, solver="block_svrg",
                                                  block_rows=b, max_iters=E, rel_tol=0.0,
                                                  grow=False, ws=wsf))
        out["svrg_epoch_ms"] = (svrg[3][0] - svrg[1][0]) / 2.0
        out["svrg_fit_1epoch_ms"] = svrg[1][0]
        out["svrg_block_rows"] = b
        out["svrg_epochs"] = svrg[3][1][1]["epochs"]
        del wsf, Hs
        # the heavy-tailed workload to convergence: Block-SVRG at b = 8,192 with
        # growth until the snapshot loss changes by less than 1e-5 (cap 2,000 epochs)
        _, tplanted, _ = synth.workload(tname, seed=rank)
        tpl = torch.from_numpy(np.asarray(tplanted, dtype=np.int32)).to(dev)
        tlab, conv = converge_row(m, torch, S2, k, tpl, "block_svrg", block_rows=b, max_iters=2000)
        kl, _, _, _ = m.spherical_kmeans(S2, k, seed=rank, max_iters=30)
        conv["kmeans_vs_symnmf_ARI"] = m.ari(kl, tlab, k)[0]
        out["converge_tpdm_block_svrg"] = conv
        del S2, tpl
        torch.cuda.empty_cache()
    # spherical k-means on the resident |corr| matrix (two S passes per step),
    # and its agreement with the SymNMF labels (the pages quote about 0.83 on
    # their own data)
    wsk = m.workspace(m._lib.OP_SPHERICAL_KMEANS, n, k, device=dev)
    km_iters = 10
    ms, (klab, _, ksteps, kconv) = _timed(
        torch, lambda: m.spherical_kmeans(S, k, seed=rank, max_iters=km_iters, ws=wsk))
    out["kmeans_ms"] = ms
    out["kmeans_steps"] = ksteps
    out["kmeans_ms_per_step"] = ms / max(ksteps, 1)
    out["kmeans_S_GBs"] = (2 * ksteps - (1 if kconv else 0)) * 4.0 * n * n / (ms / 1e3) / 1e9
    out["kmeans_vs_symnmf_ARI"] = m.ari(klab, lab, k)[0]
    del wsk
    # the upper-triangle S-stream (upper_only = 1): the same fit reading only the
    # 128 x 128 tiles on or above the diagonal (S rounded to TF32 in the product)
    if k <= 24:
        pu = m.fit_params(max_iters=19, rel_tol=0.0, upper_only=1, timing=1)
        wsu = m.workspace(m._lib.OP_FIT, n, k, params=pu, device=dev)
        Hu = H0.clone()
        m.fit(S, k, H0=Hu, out=Hu, max_iters=2, rel_tol=0.0, upper_only=True, ws=wsu)   # warm-up
        Hu.copy_(H0)
        ms, (_, stu) = _timed(torch, lambda: m.fit(S, k, H0=Hu, out=Hu, max_iters=19, rel_tol=0.0,
                                                  upper_only=True, timing=True, ws=wsu))
        T = (n + 127) // 128
        tile_bytes = 4.0 * 128 * 128 * T * (T + 1) / 2      # the tiles read per pass
        kms = stu["stream_ms"] / max(stu["stream_launches"], 1)
        out["upper_triangle"] = {
            "iterations_per_s": 20 / (ms / 1e3), "ms_per_iteration": ms / 20,
            "tri_kernel_ms": kms, "tile_bytes_read": tile_bytes,
            "tri_kernel_GBs_over_bytes_read": (tile_bytes + 4.0 * n * k) / (kms / 1e3) / 1e9,
            "loss_after_19": stu["loss"]}
        del wsu, Hu
    # the |corr| workload to convergence: full-batch AdaGrad until the loss
    # changes by less than 1e-5 (cap 20,000 passes)
    if planted is not None:
        pl = torch.from_numpy(np.asarray(planted, dtype=np.int32)).to(dev)
        clab, conv = converge_row(m, torch, S, k, pl, "adagrad", max_iters=20000)
        conv["kmeans_vs_symnmf_ARI"] = m.ari(klab, clab, k)[0]
        out["converge_corr_adagrad"] = conv
        del pl
    # the rolling study: 250 windows of 250 days, |corr| and TPDM, 100-iteration
    # fits, ARI series, 3-sigma limit, cross-sector monitor
    st = synth.rolling_stream(seed=rank)
    Rr = torch.from_numpy(st.R).to(dev)
    groups = torch.from_numpy(st.groups_before.astype("int32")).to(dev)
    kw = dict(groups=groups, window=250, k=24, delta=50, calib_begin=50, calib_end=125,
              tail_frac=0.05, tail_sign=-1, stressed=list(st.stressed))
    m.rolling(Rr, n_windows=2, **kw)                  # warm-up
    ms, res = _timed(torch, lambda: m.rolling(Rr, **kw))
    W = res["n_windows"]
    out["rolling_windows"] = W
    out["rolling_s"] = ms / 1e3
    out["rolling_ms_per_window"] = ms / W
    for kind in ("corr", "tpdm"):
        r = res[kind]
        ad = r["ari_delta"]
        out[f"rolling_{kind}_build_ms_per_window"] = r["build_ms"] / W
        out[f"rolling_{kind}_fit_ms_per_window"] = r["fit_ms"] / W
        out[f"rolling_{kind}_calm_ari_delta"] = r["mean"]
        out[f"rolling_{kind}_limit"] = r["limit"]
        out[f"rolling_{kind}_flagged_windows"] = [int(w) for w in np.flatnonzero(r["flags"])][:12]
        out[f"rolling_{kind}_min_ari_delta"] = float(np.nanmin(ad))
        out[f"rolling_{kind}_cross_max"] = float(np.nanmax(r["cross"]))
        out[f"rolling_{kind}_cross_last"] = float(r["cross"][-1])
    out["rolling_kernel_launches"] = res["launches"]
    del Rr, groups
    torch.cuda.empty_cache()
    return out


def measure_n20000(m, torch, dev, rank):
    """The two n = 20,000 workloads at their stated sizes: the rank-24 |corr|
    window (T = 500) with 500 full-batch AdaGrad iterations and a 64-eigenvalue
    probe, and the heavy-tailed TPDM window (T = 1,000) with 50 Block-SVRG
    epochs at b = 2,048 (growth on)."""
    out = {}
    R, planted, spec = synth.workload("corr_n20000_k24", seed=rank)
    n, k = spec["n"], spec["k"]
    Rd = torch.from_numpy(R).to(dev)
    S = m.alloc_S(n, dev)
    m.build_corr(Rd, out=S)
    pl = torch.from_numpy(np.asarray(planted, dtype=np.int32)).to(dev)
    p = m.fit_params(max_iters=500, rel_tol=0.0)
    ws = m.workspace(m._lib.OP_FIT, n, k, params=p, device=dev)
    H = torch.empty((n, k), dtype=torch.float32, device=dev)
    m.fit(S, k, seed=1000 + rank, max_iters=5, rel_tol=0.0, out=H, ws=ws)   # warm-up
    ms, (H, st) = _timed(torch, lambda: m.fit(S, k, seed=1000 + rank, max_iters=500, rel_tol=0.0,
                                              out=H, ws=ws, timing=True))
    c2 = {"workload": "corr_n20000_k24", "iterations": 500, "ms": ms,
          "iterations_per_s": 501 / (ms / 1e3),
          "stream_ms_per_pass": st["stream_ms"] / max(st["stream_launches"], 1),
          "ARI_vs_planted": m.ari(m.labels(H), pl, k)[0], "loss": st["loss"]}
    c2["stream_GBs"] = (4.0 * n * n + 4.0 * n * k) / (c2["stream_ms_per_pass"] / 1e3) / 1e9
    pp = m.fit_params(probe_block=16, probe_max_iter=40)
    wsp = m.workspace(m._lib.OP_SPECTRAL_PROBE, n, 64, params=pp, device=dev)
    m.spectral_probe(S, 64, block=16, max_iter=40, tol=1e-7, ws=wsp)   # warm-up
    pms, ev = _timed(torch, lambda: m.spectral_probe(S, 64, block=16, max_iter=40, tol=1e-7, ws=wsp))
    info = m.probe_last_info()
    c2.update({"probe64_ms": pms, "probe64_s_passes": info["s_passes"],
               "probe64_GBs": info["s_passes"] * 4.0 * n * n / (pms / 1e3) / 1e9,
               "probe64_gamma_k25": float(ev[24] / abs(ev[25])), "probe64_top": [float(x) for x in ev[:2]]})
    out["corr_n20000_k24"] = c2
    del ws, wsp, Rd
    # heavy-tailed TPDM, Block-SVRG b = 2,048, 50 epochs
    R, planted, spec = synth.workload("tpdm_n20000_k24", seed=rank)
    Rd = torch.from_numpy(R).to(dev)
    m.build_tpdm(Rd, 0.05, 1, out=S)
    pl = torch.from_numpy(np.asarray(planted, dtype=np.int32)).to(dev)
    pf = m.fit_params(solver="block_svrg", block_rows=2048, max_iters=50, rel_tol=0.0)
    wsf = m.workspace(m._lib.OP_FIT, n, k, params=pf, device=dev)
    m.fit(S, k, seed=1000 + rank, solver="block_svrg", block_rows=2048, max_iters=2, rel_tol=0.0,
          out=H, ws=wsf)   # warm-up
    ms, (H, st) = _timed(torch, lambda: m.fit(S, k, seed=1000 + rank, solver="block_svrg",
                                              block_rows=2048, max_iters=50, rel_tol=0.0,
                                              out=H, ws=wsf))
    out["tpdm_n20000_k24"] = {"workload": "tpdm_n20000_k24", "epochs": st["epochs"],
                              "full_batch_passes": st["iters"], "block_final": st["block_final"],
                              "ms": ms, "epochs_per_s": 50 / (ms / 1e3),
                              "ARI_vs_planted": m.ari(m.labels(H), pl, k)[0], "loss": st["loss"]}
    del S, Rd, wsf
    torch.cuda.empty_cache()
    return out


def row_rooflines(rows, n, k, T, hbm_peak):
    """Algorithmic traffic (or flops) of each timed row over its time, as a fraction of
    the measured peaks: HBM copy bandwidth for streams, and for the |corr| Gram
    (fp16 operands, fp32 accumulation) the measured bf16 burst rate, which the
    fp16 kind runs at on this part (both 2.25 PFLOP/s nominal, dense)."""
    out = {}
    sbytes = 4.0 * n * n
    def hbm(name, bytes_, ms):
        if ms and ms > 0:
            gbs = bytes_ / (ms / 1e3) / 1e9
            out[name] = {"bound": "hbm", "GBs": gbs, "frac": gbs / hbm_peak}
    hbm("stats", sbytes, rows.get("stats_ms"))
    if "upper_triangle" in rows:
        u = rows["upper_triangle"]
        out["upper_triangle_stream"] = {"bound": "hbm", "GBs": u["tri_kernel_GBs_over_bytes_read"],
                                        "frac": u["tri_kernel_GBs_over_bytes_read"] / hbm_peak,
                                        "bytes": "tiles on or above the diagonal (about 2 n^2) + X"}
    if "probe_s_passes" in rows:
        hbm("probe", rows["probe_s_passes"] * sbytes, rows.get("probe_ms"))
    if "kmeans_steps" in rows:
        # two S passes per assignment step; the last step stops after its assignment
        hbm("kmeans_step", 2 * sbytes, rows.get("kmeans_ms_per_step"))
    if "svrg_epoch_ms" in rows:
        hbm("svrg_epoch", 2 * sbytes, rows.get("svrg_epoch_ms"))   # snapshot pass + all blocks
    if "tpdm_build_ms" in rows:
        hbm("tpdm_build_writes", sbytes, rows.get("tpdm_build_ms"))
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as f:
            f16 = float(json.load(f)["bf16_tflops"])
    except Exception:
        f16 = 1590.0
    return out, f16


def bench_config(workload, world):
    """The workload description both arms print."""
    spec = synth.WORKLOADS[workload]
    return {"workload": workload, "n": spec["n"], "k": spec["k"], "T": spec["T"], "solver": "adagrad",
            "lr": 0.1, "eps": 1e-10, "l2": "inputs larger than L2 (S is 4n^2 bytes)",
            "parallelism": f"independent windows x{world}" if world > 1 else "single"}


# ----------------------------------------------------------------------------- reference arm
def run_reference(args):
    world, rank, _ = dist_env()
    if rank != 0:
        return 0
    res = oracle_sample(args.workload, 0, args.steps, args.warmup)
    spec = synth.WORKLOADS[args.workload]
    line = {
        "metric": METRIC, "value": res["value"], "unit": UNIT, "n_gpus": args.gpus,
        "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": 1000.0 / res["value"], "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": bench_config(args.workload, args.gpus),
        "impl": "reference",
        "cpu_baseline": {k2: res[k2] for k2 in ("value", "unit", "cores", "kind", "sample")},
        "e2e": {"value": res["value"], "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
        # what was actually timed: ms_per_step above is this sample extrapolated to the full n
        "measured_sample": {"seconds": res["sample_seconds"], "iterations": res["sample_iters"],
                            "block_rows": res["sample_block"], "scale_to_full_n": res["scale_to_full"],
                            "ms_per_sample_iteration": 1000.0 * res["sample_seconds"] / max(res["sample_iters"], 1)},
    }
    print(json.dumps(line), flush=True)
    return 0


# ----------------------------------------------------------------------------- our arm
def run_ours(args):
    import torch
    import torch.distributed as dist

    world, rank, local = dist_env()
    if world > 1:
        dist.init_process_group("nccl", timeout=__import__("datetime").timedelta(seconds=600))
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    import symmetric_nmf_clustering_b200 as m

    spec = synth.WORKLOADS[args.workload]
    n, k, T = spec["n"], spec["k"], spec["T"]
    K, W = args.steps, args.warmup

    def barrier():
        if world > 1:
            dist.barrier()
        torch.cuda.synchronize()

    # --- inputs resident in HBM: the window, its |corr| matrix and the seeded start
    R_host, planted, _ = synth.workload(args.workload, seed=rank)
    R_pin = torch.from_numpy(R_host).pin_memory()
    R = R_pin.to(dev)
    S = m.alloc_S(n, dev)
    ws_corr = m.workspace(m._lib.OP_BUILD_CORR, n, 0, T, device=dev)
    e_b0, e_b1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e_b0.record()
    m.build_corr(R, out=S, ws=ws_corr)
    e_b1.record()
    torch.cuda.synchronize()
    build_ms = e_b0.elapsed_time(e_b1)
    del ws_corr

    H0, _ = m.fit(S, k, seed=1000 + rank, max_iters=0, rel_tol=0.0)
    up = bool(args.upper)
    p = m.fit_params(max_iters=K - 1, rel_tol=0.0, timing=1, upper_only=int(up))
    ws = m.workspace(m._lib.OP_FIT, n, k, params=p, device=dev)
    H = H0.clone()

    # --- warm-up
    for _ in range(1):
        H.copy_(H0)
        m.fit(S, k, H0=H, out=H, max_iters=max(W - 1, 0), rel_tol=0.0, ws=ws, upper_only=up)
    H.copy_(H0)
    barrier()

    # --- timed region: K fused iterations on resident inputs
    clocks = ClockSampler(local)
    clocks.start()
    time.sleep(0.3)
    barrier()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    torch.cuda.nvtx.range_push("timed")
    e0.record()
    H, st = m.fit(S, k, H0=H, out=H, max_iters=K - 1, rel_tol=0.0, timing=True, ws=ws,
                  upper_only=up)
    e1.record()
    torch.cuda.nvtx.range_pop()
    barrier()
    clk = clocks.stop()
    t_ms = e0.elapsed_time(e1)
    value, t_max = job_rate(t_ms, K, world, dist, dev)

    # dominant kernel: the S-stream, timed by events on its own stream inside the call
    launches = st["stream_launches"]
    stream_ms = st["stream_ms"] / max(launches, 1)
    alg_bytes = 4.0 * n * n + 4.0 * n * k          # S once + H once per launch
    if up:   # the tiles on or above the diagonal + X
        nt = (n + 127) // 128
        alg_bytes = 4.0 * 128 * 128 * nt * (nt + 1) / 2 + 4.0 * n * k
    achieved = alg_bytes / (stream_ms / 1000.0) / 1e9
    peak, peak_src = peaks()

    lab = m.labels(H)
    torch.cuda.synchronize()

    # --- library context: cuBLAS S @ H on the same matrix (the pages' kernel choice)
    mm_ms = None
    try:
        Sd = S if S.is_contiguous() else None
        if Sd is not None:
            Hc = H0.clone()
            torch.mm(Sd, Hc)
            torch.cuda.synchronize()
            a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            a.record()
            for _ in range(3):
                torch.mm(Sd, Hc)
            b.record()
            torch.cuda.synchronize()
            mm_ms = a.elapsed_time(b) / 3
    except Exception:
        mm_ms = None

    # --- end to end through the public API: pinned host window -> device, build
    #     S, K fit iterations, labels and loss back to the host
    e2e = None
    if not args.no_e2e:
        ws_corr = m.workspace(m._lib.OP_BUILD_CORR, n, 0, T, device=dev)
        lab_host = torch.empty(n, dtype=torch.int32).pin_memory()
        barrier()
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record()
        R.copy_(R_pin, non_blocking=True)
        m.build_corr(R, out=S, ws=ws_corr)
        He, st_e = m.fit(S, k, seed=1000 + rank, max_iters=K - 1, rel_tol=0.0, ws=ws)
        lab_host.copy_(m.labels(He), non_blocking=True)
        b.record()
        barrier()
        e2e_value, te_ms = job_rate(a.elapsed_time(b), K, world, dist, dev)
        e2e = {"value": e2e_value, "unit": UNIT,
               "h2d_bytes_per_step": int(R_pin.numel() * 4) / K,
               "d2h_bytes_per_step": int(n * 4 + 8) / K,
               "h2d_bytes_per_call": int(R_pin.numel() * 4),
               "d2h_bytes_per_call": int(n * 4 + 8),
               "note": "one call = window upload, |corr| build, K-iteration fit, labels + loss "
                       "download; per-step bytes = per-call bytes / K"}
        del ws_corr

    # --- the other rows of the path, each timed once on this GPU (CUDA events)
    # (a failure in a secondary row is reported in the line, not fatal to it)
    rows = None
    if not args.no_rows:
        try:
            rows = measure_rows(m, torch, dev, S, H0, lab, n, k, T, rank, args.workload, planted)
            if n == 100000:
                rows["n20000"] = measure_n20000(m, torch, dev, rank)
            rows["roofline"], f16_peak = row_rooflines(rows, n, k, T, peak)
            rows["roofline"]["corr_build"] = {
                "bound": "tensor", "f16_TFs": 3.0 * n * n * T / (build_ms / 1e3) / 1e12,
                "peak_TFs": f16_peak, "frac": 3.0 * n * n * T / (build_ms / 1e3) / 1e12 / f16_peak,
                "peak_source": "MEASURED_PEAKS.json bf16_tflops (burst); fp16 runs at the bf16 rate",
                "flops": "3 n^2 T (fp16 hi/lo split of 2^14 z, three products, upper triangle "
                         "of tiles)"}
        except Exception as exc:
            rows = {"error": f"{type(exc).__name__}: {exc}"}

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        try:
            res = oracle_sample(args.workload, 0, 20, 2)
            cpu = {k2: res[k2] for k2 in ("value", "unit", "cores", "kind", "sample")}
        except Exception as exc:
            cpu = {"error": f"{type(exc).__name__}: {exc}"}

    if world > 1:
        dist.barrier()
    if rank == 0:
        planted_dev = torch.from_numpy(np.asarray(planted, dtype=np.int32)).to(dev)
        ari_planted = m.ari(lab, planted_dev, max(k, int(planted.max()) + 1))[0]
        kname = m._lib.STREAM_KERNEL_NAMES.get(st.get("stream_kernel", 0), "stream_tc_kernel")
        ratio = STREAM_TRAFFIC_RATIO.get(kname)
        traffic = (ratio * alg_bytes
                   if ratio is not None and args.workload == "corr_n100000_k24" and k == 24 else None)
        line = {
            "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": K,
            "warmup": W, "ms_per_step": t_max / K, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f32", "data": "synthetic",
            "config": bench_config(args.workload, world),
            "roofline": {"bound": "hbm", "achieved": achieved, "peak": peak, "unit": "GB/s",
                         "frac": achieved / peak, "traffic": traffic,
                         "traffic_source": (STREAM_TRAFFIC_SOURCE if traffic is not None else
                                            "null: no ncu capture of this kernel since its last change"
                                            if ratio is None else
                                            "null: the capture's ratio applies to the n = 100,000, k = 24 launch only"),
                         "kernel": kname,
                         "peak_source": peak_src,
                         "alg_bytes_per_launch": alg_bytes, "launch_ms": stream_ms,
                         "frac_of_8000": achieved / 8000.0},
            "s_stream_gbs": achieved,
            "gpu_launches": st["kernel_launches"],
            "clocks": clk,
            "e2e": e2e,
            "cpu_baseline": cpu,
            "rows": rows,
            "context": {"pages_time_to_converge_s": {"corr": 13.0, "tpdm": 12.4,
                                                     "hardware": "4x GB200 (the pages' own data)"},
                        "corr_build_ms": build_ms,
                        "corr_build_f16_TFs": 3.0 * n * n * T / (build_ms / 1e3) / 1e12, "torch_mm_S_H_ms": mm_ms,
                        "ARI_vs_planted": ari_planted,
                        "final_loss": st["loss"], "loop_ms": st["loop_ms"]},
        }
        print(json.dumps(line), flush=True)
    if world > 1:
        dist.destroy_process_group()
    return 0


def run_sharded(args):
    """One n = 100,000 factorisation row-sharded over the N ranks ([CaS]
    "Factorization at scale", "Scale-out"): rank p streams its block of rows
    of S every iteration; (Gram, trace) are all-reduced and the new rows of H
    all-gathered over NCCL.  Strong scaling: the job's iterations per second."""
    import torch
    import torch.distributed as dist

    world, rank, local = dist_env()
    if world > 1:
        dist.init_process_group("nccl", timeout=__import__("datetime").timedelta(seconds=600))
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    import symmetric_nmf_clustering_b200 as m
    from symmetric_nmf_clustering_b200.sharded import fit_sharded, shard_rows

    spec = synth.WORKLOADS[args.workload]
    n, k, T = spec["n"], spec["k"], spec["T"]
    K, W = args.steps, args.warmup
    r0, r1 = shard_rows(n, world, rank)

    def barrier():
        if world > 1:
            dist.barrier()
        torch.cuda.synchronize()

    # every rank builds the window's |corr| matrix and keeps its block of rows
    R_host, planted, _ = synth.workload(args.workload, seed=0)
    R_pin = torch.from_numpy(R_host).pin_memory()
    R = R_pin.to(dev)
    S = m.alloc_S(n, dev)
    m.build_corr(R, out=S)
    S_rows = S[r0:r1]
    torch.cuda.synchronize()
    fit_sharded(S_rows, r0, n, k, seed=1000, max_iters=max(W - 1, 0), rel_tol=0.0)   # warm-up
    barrier()
    clocks = ClockSampler(local)
    clocks.start()
    time.sleep(0.3)
    barrier()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record()
    H, st = fit_sharded(S_rows, r0, n, k, seed=1000, max_iters=K - 1, rel_tol=0.0)
    e1.record()
    barrier()
    clk = clocks.stop()
    t = torch.tensor([e0.elapsed_time(e1)], dtype=torch.float64, device=dev)
    if world > 1:
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
    t_max = float(t.item())
    value = K / (t_max / 1000.0)

    # end to end: window upload, |corr| build, the sharded fit, labels and loss back
    lab_host = torch.empty(n, dtype=torch.int32).pin_memory()
    barrier()
    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    a.record()
    R.copy_(R_pin, non_blocking=True)
    m.build_corr(R, out=S)
    He, ste = fit_sharded(S_rows, r0, n, k, seed=1000, max_iters=K - 1, rel_tol=0.0)
    lab_host.copy_(m.labels(He), non_blocking=True)
    b.record()
    barrier()
    te = torch.tensor([a.elapsed_time(b)], dtype=torch.float64, device=dev)
    if world > 1:
        dist.all_reduce(te, op=dist.ReduceOp.MAX)
    e2e = {"value": K / (float(te.item()) / 1000.0), "unit": UNIT,
           "h2d_bytes_per_step": int(R_pin.numel() * 4) / K, "d2h_bytes_per_step": int(n * 4 + 8) / K,
           "note": "one call per rank = window upload, full |corr| build, K-iteration sharded fit, "
                   "labels + loss download; the job time is the max over ranks"}
    peak, peak_src = peaks()
    ms_step = t_max / K
    rank_bytes = 4.0 * (r1 - r0) * n + 4.0 * n * k
    if rank == 0:
        pl = torch.from_numpy(np.asarray(planted, dtype=np.int32)).to(dev)
        line = {
            "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": K, "warmup": W,
            "ms_per_step": ms_step, "higher_is_better": True, "scaling": "strong",
            "vs_baseline": None, "dtype": "f32", "data": "synthetic",
            "config": dict(bench_config(args.workload, world),
                           parallelism=f"row-sharded S x{world}, H replicated (NCCL)"),
            "roofline": {"bound": "hbm", "achieved": rank_bytes / (ms_step / 1000.0) / 1e9,
                         "peak": peak, "unit": "GB/s",
                         "frac": rank_bytes / (ms_step / 1000.0) / 1e9 / peak, "traffic": None,
                         "kernel": "stream_tc_kernel on rank 0's rows (whole-step time bounds the launch)",
                         "peak_source": peak_src, "alg_bytes_per_launch": rank_bytes},
            "gpu_launches": 4 * K + 3,
            "clocks": clk, "e2e": e2e, "cpu_baseline": None,
            "context": {"rows_rank0": [r0, r1], "final_loss": st["loss"],
                        "ARI_vs_planted": m.ari(m.labels(H), pl, k)[0]},
        }
        print(json.dumps(line), flush=True)
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()
    return 0


def main():
    args = parse()
    if args.impl == "reference":
        return run_reference(args)
    world, _, _ = dist_env()
    if args.sharded or (world > 1 and not args.replicas):
        return run_sharded(args)
    return run_ours(args)


if __name__ == "__main__":
    sys.exit(main())
