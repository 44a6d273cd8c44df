#!/usr/bin/env python
"""Benchmark of the Effort approximate GEMV on B200.

Headline workload: one approximate matvec out = W^T v with W 4096 x 14336 fp16
(Mistral-7B FFN w1/w3 shape, entries N(0, 0.02^2)), v fp32 Student-t(3) /
sqrt(3), effort 0.25, keep 1.0, batch 1.  A step is one call of the library's
gemv (one fused kernel: cutoff, dispatch and multiply) on inputs resident in
HBM.  Steps rotate over 10 prepared matrices and 8 vectors, so the bytes a
call reads are not in L2 from the previous use.  Steps are issued from CUDA
graphs (Python launch overhead would otherwise dominate a call of tens of
microseconds).  The timed region of exactly --steps steps is repeated
TIMED_REGIONS times; the line reports the median region (all of them are
listed).

Prints ONE JSON line (rank 0).  `--impl reference` times the CPU oracle
instead (the reference arm).  `--gpus N` under torchrun runs N independent
replicas (the path is single-GPU; no collective on the data path).
"""
import argparse
import hashlib
import json
import math
import os
import statistics
import subprocess
import sys
import tempfile
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "approx-GEMV µs & achieved HBM GB/s vs effort (4096×14336 fp16, batch 1)"
IN_DIM, OUT_DIM = 4096, 14336
EFFORT, KEEP = 0.25, 1.0
N_MATS, N_VECS, GRAPH_STEPS = 10, 8, 40
TIMED_REGIONS = 5
SWEEP = (1.0, 0.5, 0.4, 0.25, 0.15)
NOMINAL_HBM_GBS = 8000.0
FALLBACK_HBM_GBS = 6650.0


def args_parse():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=2000)
    ap.add_argument("--warmup", type=int, default=200)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-sweep", action="store_true")
    ap.add_argument("--ncu", action="store_true",
                    help="small profiling case: 4 prepared matrices, 8 warm calls then 4 calls, no timing")
    return ap.parse_args()


def hbm_peak():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(p) as f:
            return float(json.load(f)["hbm_gbs"]), "measured"
    except Exception:
        return FALLBACK_HBM_GBS, "fallback"


def workload_config():
    return {"workload": f"approx GEMV W {IN_DIM}x{OUT_DIM} fp16 N(0,0.02^2), v fp32 t3/sqrt(3), "
                        f"effort {EFFORT}, keep {KEEP}, batch 1",
            "in_dim": IN_DIM, "out_dim": OUT_DIM, "effort": EFFORT, "keep_fraction": KEEP,
            "l2": f"inputs larger than L2: {N_MATS} prepared matrices x {N_VECS} vectors rotated",
            "issue": f"CUDA graphs of {GRAPH_STEPS} steps",
            "timing": f"median of {TIMED_REGIONS} timed regions of --steps steps each"}


# ----------------------------------------------------------------- CPU oracle
def host_info():
    """The host the CPU numbers come from: usable cores, CPU model, memory."""
    nproc = len(os.sched_getaffinity(0)) if hasattr(os, "sched_getaffinity") else os.cpu_count()
    model = None
    try:
        out = subprocess.run(["lscpu"], capture_output=True, text=True, timeout=10).stdout
        for line in out.splitlines():
            if line.strip().startswith("Model name:"):
                model = line.split(":", 1)[1].strip()
                break
    except Exception:
        pass
    if not model:
        try:
            with open("/proc/cpuinfo") as f:
                for line in f:
                    if line.startswith("model name"):
                        model = line.split(":", 1)[1].strip()
                        break
        except Exception:
            pass
    mem_gb = None
    try:
        with open("/proc/meminfo") as f:
            for line in f:
                if line.startswith("MemAvailable:"):
                    mem_gb = int(line.split()[1]) / 1e6
    except Exception:
        pass
    return {"nproc": nproc, "cpu_model": model, "mem_available_gb": mem_gb}


def oracle_workload(rows=IN_DIM, seed=4, n_vecs=4):
    """The headline workload (or its first `rows` rows) prepared for the oracle
    (the offline step, not timed) and a few of its vectors."""
    from dynamic_approximate_gemv_b200 import inputs
    from oracle import effort_oracle as O
    Wn = inputs.weights(rows, OUT_DIM, seed)
    prep = O.Prepared(Wn.view(np.uint16), KEEP)
    vs = [inputs.vector(rows, 50 + k, "t3") for k in range(n_vecs)]
    return Wn, prep, vs


def time_oracle_calls(prep, vs, min_calls, budget_s=0.0):
    """Whole oracle matvecs (chart, cutoff, selection, float64 sum) back to back;
    returns seconds per call, calls and seconds."""
    from oracle import effort_oracle as O
    t0 = time.perf_counter()
    n = 0
    while n < min_calls or (time.perf_counter() - t0) < budget_s:
        O.effort_gemv(prep, vs[n % len(vs)], EFFORT)
        n += 1
    dt = time.perf_counter() - t0
    return (dt / n if n else 0.0), n, dt


def _oracle_worker(args):
    """One process of the all-core measurement: prepares its own copy of the
    workload, then times `calls` whole matvecs (wall-clock start and end)."""
    seed, calls = args
    sys.path.insert(0, ROOT)
    _, prep, vs = oracle_workload(seed=seed)
    from oracle import effort_oracle as O
    t0 = time.time()
    for k in range(calls):
        O.effort_gemv(prep, vs[k % len(vs)], EFFORT)
    return t0, time.time(), calls


def cpu_baseline(budget_s=12.0):
    """The oracle on the host cores: whole matvecs of the headline workload on
    one thread, the same on all cores (independent processes, one matvec each
    at a time), and a plain CPU dense GEMV (numpy float32 W^T v through its BLAS,
    and the oracle's float64 dense product) beside them."""
    import multiprocessing as mp
    info = host_info()
    Wn, prep, vs = oracle_workload()
    time_oracle_calls(prep, vs, 1)  # warm
    sec, n, dt = time_oracle_calls(prep, vs, 2, budget_s)
    # all cores: as many processes as memory allows (a prepared copy and one
    # call's temporaries take about 6 GB)
    procs = max(1, int(info["nproc"] or 1))
    if info["mem_available_gb"]:
        procs = min(procs, int(info["mem_available_gb"] // 8))
    procs = max(1, min(procs, 16))
    allc = None
    if procs > 1:
        ctx = mp.get_context("spawn")
        with ctx.Pool(procs) as pool:
            res = pool.map(_oracle_worker, [(4, 2)] * procs)
        t_start = min(r[0] for r in res)
        t_end = max(r[1] for r in res)
        calls = sum(r[2] for r in res)
        allc = {"processes": procs, "matvecs": calls, "seconds": t_end - t_start,
                "us_per_matvec": (t_end - t_start) / calls * 1e6}
    # plain dense GEMV on the CPU
    from oracle import effort_oracle as O
    W32 = Wn.astype(np.float32)
    v32 = vs[0].astype(np.float32)
    W32.T @ v32
    reps = 20
    t0 = time.perf_counter()
    for _ in range(reps):
        W32.T @ v32
    sgemv_us = (time.perf_counter() - t0) / reps * 1e6
    try:
        from threadpoolctl import threadpool_info
        blas_threads = max([d.get("num_threads", 1) for d in threadpool_info()] or [1])
    except Exception:
        blas_threads = None
    t0 = time.perf_counter()
    O.dense_gemv(Wn.view(np.uint16), vs[0])
    f64_us = (time.perf_counter() - t0) * 1e6
    return {"value": sec * 1e6, "unit": "us", "cores": 1, "kind": "oracle",
            "sample": f"{n} whole oracle matvecs of the {IN_DIM}x{OUT_DIM} workload ({dt:.1f} s), numpy, one "
                      f"thread (the oracle's own preparation of the matrix is the offline step, not timed)",
            "all_cores": allc, "host": info,
            "cpu_dense_gemv": {"numpy_f32_us": sgemv_us, "blas_threads": blas_threads,
                               "oracle_f64_us": f64_us}}


REFERENCE_BUDGET_S = 120.0  # the reference arm's oracle work, whatever --steps is


def run_reference(a):
    """The reference arm: the oracle, as it stands, on the host cores.  Each
    step is one whole oracle matvec of the workload when all --steps + warmup
    steps fit in REFERENCE_BUDGET_S; otherwise each step is the oracle on a
    row slice of the workload, the time per matvec is scaled to the full
    matrix, and the line says so (`extrapolated`).  ms_per_step is always the
    time a step really took."""
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return
    info = host_info()
    Wn, prep, vs = oracle_workload()
    sec_full, _, _ = time_oracle_calls(prep, vs, 1)
    warm = min(a.warmup, 1)
    if (a.steps + warm) * sec_full <= REFERENCE_BUDGET_S:
        time_oracle_calls(prep, vs, warm)
        sec, n, dt = time_oracle_calls(prep, vs, a.steps)
        value, step_ms, extra = sec * 1e6, sec * 1e3, None
        sample = f"{n} whole oracle matvecs of the {IN_DIM}x{OUT_DIM} workload ({dt:.1f} s), numpy, one thread"
    else:
        del prep
        rows = int(IN_DIM * REFERENCE_BUDGET_S / ((a.steps + warm) * sec_full))
        rows = max(16, min(IN_DIM, rows // 16 * 16))
        _, sprep, svs = oracle_workload(rows=rows)
        time_oracle_calls(sprep, svs, warm)
        sec, n, dt = time_oracle_calls(sprep, svs, a.steps)
        value, step_ms = sec * IN_DIM / rows * 1e6, sec * 1e3
        extra = {"rows_per_step": rows, "scale_to_full_matvec": IN_DIM / rows,
                 "whole_matvec_us_measured_once": sec_full * 1e6}
        sample = (f"{n} oracle matvecs on a {rows}x{OUT_DIM} row slice of the workload ({dt:.1f} s), time per "
                  f"matvec scaled by {IN_DIM / rows:g} to the full matrix; numpy, one thread")
    line = {"metric": METRIC, "value": value, "unit": "us", "n_gpus": a.gpus, "steps": a.steps, "warmup": a.warmup,
            "ms_per_step": step_ms, "higher_is_better": False, "scaling": "weak", "vs_baseline": None,
            "dtype": "f64", "data": "synthetic", "impl": "reference", "config": workload_config(),
            "cpu_baseline": {"value": value, "unit": "us", "cores": 1, "kind": "oracle", "sample": sample,
                             "host": info},
            "extrapolated": extra,
            "e2e": {"value": value, "unit": "us", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


# ----------------------------------------------------------------- bytes
def algorithmic_bytes(in_dim, out_dim, used, v_bytes=4):
    """Algorithmic bytes of one matvec: 3 bytes per used product (fp16 value
    and an 8-bit position), the 16 fp16 probes of every row, v and out."""
    return 3.0 * used + 2.0 * 16 * in_dim + v_bytes * in_dim + 4.0 * out_dim


def read_bytes(in_dim, out_dim, dense, sparse, v_bytes=4):
    """Bytes a call plans to read from the prepared matrix (whole dense
    panel rows at 2 bytes per entry, stored chunks at 3 bytes per slot), plus
    probes, v and out: what the kernel actually moves, which unlike the
    algorithmic figure cannot exceed a copy's bandwidth."""
    return float(dense) + float(sparse) + 2.0 * 16 * in_dim + v_bytes * in_dim + 4.0 * out_dim


def algorithmic_bytes_q8(in_dim, out_dim, used, v_bytes=4):
    """The same for a Q8 matrix: 2 bytes per used product (int8 value and an
    8-bit position), the probes, one binary16 scale per row, v and out."""
    return 2.0 * used + 2.0 * 16 * in_dim + 2.0 * in_dim + v_bytes * in_dim + 4.0 * out_dim


def read_bytes_q8(in_dim, out_dim, dense, sparse, v_bytes=4):
    """Planned reads of a Q8 call (int8 dense panel rows, 2-byte chunk slots,
    as the library reports them) plus probes, row scales, v and out."""
    return read_bytes(in_dim, out_dim, dense, sparse, v_bytes) + 2.0 * in_dim


# ----------------------------------------------------------------- other shapes
def measure_shape(E, dev, in_dim, out_dim, efforts, dist, n_mats=10, n_vecs=8, seed0=5000, keep=1.0, q8=False):
    """us per matvec and algorithmic GB/s on another workload shape: n_mats
    prepared matrices N(0, 0.02^2) fp16 and n_vecs vectors rotated through CUDA
    graphs of 40 steps (inputs larger than L2), as for the headline workload.
    q8: the same draws quantised per row to int8 with a binary16 scale
    (s_i = fp16(max |w_i| / 127), q = round(w / s_i) clipped to +-127)."""
    import torch
    from dynamic_approximate_gemv_b200 import inputs
    g = torch.Generator(device=dev)
    mats = []
    for m in range(n_mats):
        g.manual_seed(seed0 + m)
        W = torch.randn(in_dim, out_dim, device=dev, generator=g) * 0.02
        if q8:
            sc = (W.abs().amax(dim=1) / 127.0).to(torch.float16)
            sc[sc == 0] = 1.0
            q = torch.clamp(torch.round(W / sc.float()[:, None]), -127, 127).to(torch.int8)
            mats.append(E.PreparedMatrix.from_q8(q, sc, keep))
            del q, sc
        else:
            mats.append(E.PreparedMatrix(W.to(torch.float16), keep))
        del W
    vecs = [torch.from_numpy(inputs.vector(in_dim, seed0 + 100 + k, dist)).to(dev) for k in range(n_vecs)]
    outs = [torch.empty(out_dim, device=dev) for _ in range(n_mats)]
    cnt = torch.zeros(1, device=dev, dtype=torch.int64)
    res = {}
    steps = 40
    for e in efforts:
        used, dense, sparse = 0.0, 0.0, 0.0
        for k in range(steps):
            mats[k % n_mats].gemv(vecs[k % n_vecs], e, out=outs[k % n_mats], count=cnt)
            used += float(cnt.item())
            d, sp = mats[k % n_mats].last_call_bytes()
            dense += d
            sparse += sp
        used /= steps
        dense /= steps
        sparse /= steps
        s = torch.cuda.Stream(device=dev)
        s.wait_stream(torch.cuda.current_stream(dev))
        gr = torch.cuda.CUDAGraph()
        with torch.cuda.stream(s):
            for k in range(steps):
                mats[k % n_mats].gemv(vecs[k % n_vecs], e, out=outs[k % n_mats])
        torch.cuda.synchronize()
        with torch.cuda.graph(gr, stream=s):
            for k in range(steps):
                mats[k % n_mats].gemv(vecs[k % n_vecs], e, out=outs[k % n_mats])
        for _ in range(3):
            gr.replay()
        torch.cuda.synchronize()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        reps = 10
        e0.record()
        for _ in range(reps):
            gr.replay()
        e1.record()
        torch.cuda.synchronize()
        us = e0.elapsed_time(e1) * 1000.0 / (reps * steps)
        if q8:
            b = algorithmic_bytes_q8(in_dim, out_dim, used)
            rb = read_bytes_q8(in_dim, out_dim, dense, sparse)
            dense_b = 1.0 * in_dim * out_dim + 2.0 * in_dim + 4.0 * in_dim + 4.0 * out_dim
        else:
            b = algorithmic_bytes(in_dim, out_dim, used)
            rb = read_bytes(in_dim, out_dim, dense, sparse)
            dense_b = 2.0 * in_dim * out_dim + 4.0 * in_dim + 4.0 * out_dim
        res[str(e)] = {"us": us, "gbs_algorithmic": b / (us * 1e-6) / 1e9, "mean_used": used,
                       "read_bytes": {"dense": dense, "sparse": sparse, "total": rb},
                       "gbs_read": rb / (us * 1e-6) / 1e9,
                       "dense_roofline_us_measured_peak": dense_b / (hbm_peak()[0] * 1e9) * 1e6}
        del gr
    for m in mats:
        m.close()
    return res


# ----------------------------------------------------------------- decode chain
CHAIN_MATS = (("q", 0, 0), ("k", 0, 1), ("v", 0, 1), ("o", 0, 0), ("w1", 0, 2), ("w3", 0, 2), ("w2", 2, 0))


def rms_norm(y, eps=1e-5):
    """y / sqrt(mean(y^2) + eps), no gain (harness between matvecs)."""
    import torch
    return y * torch.rsqrt(torch.mean(y * y) + eps)


def effort_for(schedule, layer, name):
    """Effort of matrix `name` in layer `layer` under `schedule`.

    The pages treat effort as a setting that can change from layer to layer,
    matrix to matrix and token to token, not only one value for the whole
    model (the author's replies in Hacker News item 40067677).  A schedule is
    a number (one effort for every matvec), a mapping keyed by matrix name or
    by (layer, name), or a callable (layer, name) -> effort.
    """
    if callable(schedule):
        e = schedule(layer, name)
    elif isinstance(schedule, dict):
        e = schedule[(layer, name)] if (layer, name) in schedule else schedule[name]
    else:
        e = schedule
    e = float(e)
    if not 0.0 <= e <= 1.0:
        raise ValueError(f"effort {e} for layer {layer} matrix {name} is outside [0, 1]")
    return e


# An illustrative per-matrix schedule for the Mistral-7B shapes: the attention
# projections at 0.5 and the FFN at 0.19, which keeps the parameter-weighted
# mean effort near 0.25.  The pages give no schedule; this one only exercises
# the per-matrix setting.
CHAIN_EQUALIZER = {"q": 0.5, "k": 0.5, "v": 0.5, "o": 0.5, "w1": 0.19, "w3": 0.19, "w2": 0.19}


def chain_token(E, mats, x, effort):
    """One token through the stack: per layer x -> q, k, v; q -> o; o -> w1, w3;
    w1 * w3 -> w2; every matvec input RMS-normalised (no gain).  `effort` is a
    schedule (see effort_for)."""
    for l, L in enumerate(mats):
        e = {name: effort_for(effort, l, name) for name in L}
        xn = rms_norm(x)
        q = L["q"].gemv(xn, e["q"])
        L["k"].gemv(xn, e["k"])
        L["v"].gemv(xn, e["v"])
        o = L["o"].gemv(rms_norm(q), e["o"])
        h = rms_norm(o)
        a = L["w1"].gemv(h, e["w1"])
        b = L["w3"].gemv(h, e["w3"])
        x = rms_norm(L["w2"].gemv(rms_norm(a * b), e["w2"]))
    return x


def measure_chain(E, dev, layers=32, dims=(4096, 1024, 14336), effort=0.25, keep=0.8):
    """Decode stack of Mistral-7B shapes (random init): one token = 7 * layers
    dependent matvecs, timed as one CUDA graph replay per token."""
    import torch
    from dynamic_approximate_gemv_b200 import inputs
    g = torch.Generator(device=dev)
    mats, dense_bytes = [], 0.0
    for l in range(layers):
        L = {}
        for m, (name, a, b) in enumerate(CHAIN_MATS):
            g.manual_seed(1000 * l + m)
            W = (torch.randn(dims[a], dims[b], device=dev, generator=g) * 0.02).to(torch.float16)
            L[name] = E.PreparedMatrix(W, keep)
            dense_bytes += 2.0 * dims[a] * dims[b] + 4.0 * (dims[a] + dims[b])
            del W
        mats.append(L)
    x0 = torch.from_numpy(inputs.vector(dims[0], 9)).to(dev)
    s = torch.cuda.Stream(device=dev)
    s.wait_stream(torch.cuda.current_stream(dev))

    def token_us(schedule):
        with torch.cuda.stream(s):
            chain_token(E, mats, x0, schedule)
        torch.cuda.synchronize()
        gr = torch.cuda.CUDAGraph()
        with torch.cuda.graph(gr, stream=s):
            chain_token(E, mats, x0, schedule)
        for _ in range(3):
            gr.replay()
        torch.cuda.synchronize()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        reps = 10
        e0.record()
        for _ in range(reps):
            gr.replay()
        e1.record()
        torch.cuda.synchronize()
        del gr
        return e0.elapsed_time(e1) * 1000.0 / reps

    us = token_us(effort)
    us_eq = token_us(CHAIN_EQUALIZER)
    params = {name: dims[a] * dims[b] for name, a, b in CHAIN_MATS}
    eq_mean = sum(CHAIN_EQUALIZER[n] * params[n] for n in params) / sum(params.values())
    storage = sum(L[n].info()["device_bytes"] for L in mats for n in L) if hasattr(mats[0]["q"], "info") else None
    for L in mats:
        for n in L:
            L[n].close()
    return {"workload": f"{layers} layers of q {dims[0]}x{dims[0]}, k/v {dims[0]}x{dims[1]}, o {dims[0]}x{dims[0]}, "
                        f"w1/w3 {dims[0]}x{dims[2]}, w2 {dims[2]}x{dims[0]} fp16 N(0,0.02^2), keep {keep}, "
                        f"effort {effort}; {7 * layers} dependent matvecs per token, RMS-normalised inputs",
            "us_per_token": us, "matvecs_per_token": 7 * layers, "us_per_matvec": us / (7 * layers),
            "dense_roofline_us_per_token_measured_peak": dense_bytes / (hbm_peak()[0] * 1e9) * 1e6,
            "prepared_bytes": storage,
            "per_matrix_schedule": {"efforts": CHAIN_EQUALIZER, "parameter_weighted_mean_effort": eq_mean,
                                    "us_per_token": us_eq}}


# ----------------------------------------------------------------- ranks
def replica_seed(rank, m):
    """Seed of prepared matrix m on `rank`: each rank runs its own replica
    (the path does not shard; there is no data-path collective)."""
    return 1000 * (rank + 1) + m


def max_over_ranks(x, world, device):
    """The largest of the ranks' values (timing is the slowest rank's)."""
    if world == 1:
        return x
    import torch
    import torch.distributed as dist
    t = torch.tensor([x], device=device, dtype=torch.float64)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def whole_job_us_per_matvec(us_per_step_max, world):
    """Whole-job figure: every rank did one matvec per step, so the job did
    `world` matvecs in the slowest rank's step time."""
    return us_per_step_max / world


# ----------------------------------------------------------------- clocks
class ClockSampler:
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, index):
        self.index = index
        self.file = tempfile.NamedTemporaryFile("w+", suffix=".csv", delete=False)
        self.proc = None

    def start(self):
        try:
            self.proc = subprocess.Popen(["nvidia-smi", "-i", str(self.index), "--query-gpu=" + self.FIELDS,
                                          "--format=csv,noheader,nounits", "-lms", "100"],
                                         stdout=self.file, stderr=subprocess.DEVNULL)
        except Exception:
            self.proc = None

    def stop(self):
        if self.proc is None:
            return None
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except Exception:
            self.proc.kill()
        self.file.flush()
        rows = []
        with open(self.file.name) as f:
            for line in f:
                p = [x.strip() for x in line.split(",")]
                if len(p) < 9:
                    continue
                try:
                    rows.append((float(p[1]), float(p[2]), float(p[3]), p[5:9]))
                except ValueError:
                    continue
        os.unlink(self.file.name)
        if not rows:
            return None
        pmax = max(r[2] for r in rows)
        load = [r for r in rows if r[2] >= 0.5 * pmax] or rows
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[k] for r in load for k in range(4) if r[3][k].lower() == "active"})
        return {"sm_mhz": statistics.median(r[0] for r in load), "sm_max_mhz": max(r[1] for r in load),
                "reasons": reasons, "samples": len(load), "power_w_max": pmax}


# ----------------------------------------------------------------- GPU arm
def source_sha(*names):
    h = hashlib.sha256()
    for n in names:
        with open(os.path.join(ROOT, "dynamic_approximate_gemv_b200", "csrc", n), "rb") as f:
            h.update(f.read())
    return h.hexdigest()[:16]


def ncu_traffic(kernel):
    """DRAM bytes per launch from the committed ncu summary, if its source hash is current."""
    p = os.path.join(ROOT, "profiles", "traffic.json")
    try:
        with open(p) as f:
            rec = json.load(f)[kernel]
        if rec["source_sha"] != source_sha(*rec["sources"]):
            return None
        return float(rec["dram_bytes_per_launch"])
    except Exception:
        return None


def run_ncu_case():
    """Plain launches for an ncu capture: the headline shape, 4 matrices rotated
    (each call reads ~50 MB of a 330 MB prepared matrix; 4 x 50 MB > L2)."""
    import torch
    from dynamic_approximate_gemv_b200 import build, inputs
    build.build()
    import dynamic_approximate_gemv_b200 as E
    dev = torch.device("cuda", 0)
    g = torch.Generator(device=dev)
    mats = []
    for m in range(4):
        g.manual_seed(1000 + m)
        W = (torch.randn(IN_DIM, OUT_DIM, device=dev, generator=g) * 0.02).to(torch.float16)
        mats.append(E.PreparedMatrix(W, KEEP))
        del W
    vecs = [torch.from_numpy(inputs.vector(IN_DIM, 7 + k, "t3")).to(dev) for k in range(4)]
    out = torch.empty(OUT_DIM, device=dev)
    for k in range(12):
        mats[k % 4].gemv(vecs[k % 4], EFFORT, out=out)
    torch.cuda.synchronize()
    print("ncu case done", float(out.abs().sum()))


def main():
    a = args_parse()
    if a.impl == "reference":
        run_reference(a)
        return
    if a.ncu:
        run_ncu_case()
        return
    import torch
    import torch.distributed as dist

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        import datetime
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120))
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)

    from dynamic_approximate_gemv_b200 import build, inputs
    if rank == 0:
        build.build()
    if world > 1:
        dist.barrier()
    import dynamic_approximate_gemv_b200 as E

    def barrier():
        if world > 1:
            dist.barrier()

    def rank_max(x):
        return max_over_ranks(x, world, dev)

    g = torch.Generator(device=dev)
    mats, raws = [], []
    for m in range(N_MATS):
        g.manual_seed(replica_seed(rank, m))
        W = (torch.randn(IN_DIM, OUT_DIM, device=dev, generator=g) * 0.02).to(torch.float16)
        mats.append(E.PreparedMatrix(W, KEEP))
        raws.append(W)
    vecs = [torch.from_numpy(inputs.vector(IN_DIM, 7 + k, "t3")).to(dev) for k in range(N_VECS)]
    outs = [torch.empty(OUT_DIM, device=dev) for _ in range(N_MATS)]
    torch.cuda.synchronize()

    def step_pairs(n, offset=0):
        return [((offset + k) % N_MATS, (offset + k) % N_VECS) for k in range(n)]

    # per-step means over the rotation at one effort: used products, and the
    # bytes each call planned to read per path (dense rows, stored chunks)
    def rotation_stats(effort):
        cnt = torch.zeros(1, device=dev, dtype=torch.int64)
        used, dense, sparse = 0, 0, 0
        pairs = step_pairs(GRAPH_STEPS)
        for (mi, vi) in pairs:
            mats[mi].gemv(vecs[vi], effort, out=outs[mi], count=cnt)
            used += int(cnt.item())
            d, sp = mats[mi].last_call_bytes()
            dense += d
            sparse += sp
        n = len(pairs)
        return used / n, dense / n, sparse / n

    def capture(n_steps, effort, offset=0):
        gr = torch.cuda.CUDAGraph()
        s = torch.cuda.Stream(device=dev)
        s.wait_stream(torch.cuda.current_stream(dev))
        with torch.cuda.stream(s):
            for (mi, vi) in step_pairs(n_steps, offset):  # warm once outside capture
                mats[mi].gemv(vecs[vi], effort, out=outs[mi])
        torch.cuda.current_stream(dev).wait_stream(s)
        torch.cuda.synchronize()
        with torch.cuda.graph(gr, stream=s):
            for (mi, vi) in step_pairs(n_steps, offset):
                mats[mi].gemv(vecs[vi], effort, out=outs[mi])
        torch.cuda.synchronize()
        return gr

    def timed_steps(effort, steps, warmup, regions=1, sampler=None, min_seconds=0.0):
        """Times `regions` back-to-back regions of exactly `steps` steps (after
        `warmup` untimed ones); returns each region's milliseconds (max over
        ranks)."""
        full = capture(GRAPH_STEPS, effort)
        rem = steps % GRAPH_STEPS
        tail = capture(rem, effort, offset=0) if rem else None
        for _ in range(max(1, math.ceil(warmup / GRAPH_STEPS))):
            full.replay()
        torch.cuda.synchronize()
        out_ms = []
        for _ in range(regions):
            barrier()
            torch.cuda.synchronize()
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record()
            for _ in range(steps // GRAPH_STEPS):
                full.replay()
            if tail is not None:
                tail.replay()
            e1.record()
            torch.cuda.synchronize()
            barrier()
            out_ms.append(rank_max(e0.elapsed_time(e1)))
        # keep the same replay running until the clock sampler has a window of samples
        if sampler is not None and min_seconds > 0:
            t0 = time.perf_counter()
            while time.perf_counter() - t0 < min_seconds:
                for _ in range(50):
                    full.replay()
                torch.cuda.synchronize()
        return out_ms

    def phase_marks(effort, calls=12):
        """Medians (over calls, of the median over blocks) of the fused
        kernel's phase marks, in microseconds after the earliest block passed
        its wait on the preceding grid; one call at a time."""
        nb = mats[0].grid_blocks()
        marks = torch.zeros(nb, 16, dtype=torch.int64, device=dev)
        rows = []
        for k in range(calls):
            marks.zero_()
            mats[k % N_MATS].gemv_timed(vecs[k % N_VECS], effort, outs[0], marks)
            torch.cuda.synchronize()
            m = marks.cpu().numpy().astype(np.int64)
            rows.append(m - m[:, 1].min())
        R = np.stack(rows)
        names = {0: "start", 1: "wait", 2: "chart_histogram", 3: "barrier_B1", 4: "crossing_bin",
                 5: "crossing_entries", 6: "cutoff", 7: "dispatch", 8: "dense_streamed", 9: "sparse_streamed", 10: "accumulated",
                 11: "out_reduced", 13: "end"}
        res = {}
        for k, nm in names.items():
            col = R[:, :, k]
            if (col == 0).all() or (col < -10 ** 12).any():
                continue
            res[nm] = round(float(np.median(np.median(col.astype(np.float64), 1))) / 1e3, 2)
        return res

    peak, peak_kind = hbm_peak()
    sampler = ClockSampler(local)
    sampler.start()
    time.sleep(0.3)
    region_ms = timed_steps(EFFORT, a.steps, a.warmup, regions=TIMED_REGIONS, sampler=sampler, min_seconds=2.0)
    clocks = sampler.stop()
    ms = statistics.median(region_ms)
    us_per_step = ms * 1000.0 / a.steps
    value = whole_job_us_per_matvec(us_per_step, world)

    S_mean, D_mean, Sp_mean = rotation_stats(EFFORT)
    alg_bytes = algorithmic_bytes(IN_DIM, OUT_DIM, S_mean)
    rd_bytes = read_bytes(IN_DIM, OUT_DIM, D_mean, Sp_mean)
    launch_us = us_per_step  # one kernel per call
    achieved = alg_bytes / (launch_us * 1e-6) / 1e9
    traffic = ncu_traffic("k_effort")
    roofline = {"bound": "hbm", "achieved": achieved, "peak": peak, "unit": "GB/s", "frac": achieved / peak,
                "traffic": traffic, "kernel": "k_effort", "peak_kind": peak_kind,
                "frac_of_nominal_8000": achieved / NOMINAL_HBM_GBS,
                "algorithmic_bytes_per_launch": alg_bytes, "launch_us": launch_us,
                "read_bytes_per_launch": {"dense": D_mean, "sparse": Sp_mean, "total": rd_bytes},
                "read_gbs": rd_bytes / (launch_us * 1e-6) / 1e9}
    phases = phase_marks(EFFORT) if world == 1 else {}

    # dense baselines on the same rotation (raw fp16 matrices, 117 MB each)
    ws = E.Workspace(IN_DIM, OUT_DIM)
    vec16 = [v.to(torch.float16) for v in vecs]
    dense_outs = [torch.empty(OUT_DIM, device=dev) for _ in range(N_MATS)]
    mv_outs = [torch.empty(OUT_DIM, device=dev, dtype=torch.float16) for _ in range(N_MATS)]

    def time_graph(fn, n_rep=20):
        gr = torch.cuda.CUDAGraph()
        st = torch.cuda.Stream(device=dev)
        st.wait_stream(torch.cuda.current_stream(dev))
        with torch.cuda.stream(st):
            fn()
        torch.cuda.synchronize()
        with torch.cuda.graph(gr, stream=st):
            fn()
        for _ in range(3):
            gr.replay()
        torch.cuda.synchronize()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record()
        for _ in range(n_rep):
            gr.replay()
        e1.record()
        torch.cuda.synchronize()
        return e0.elapsed_time(e1) / n_rep

    def dense_all():
        for k in range(GRAPH_STEPS):
            E.dense_gemv(ws, raws[k % N_MATS], vecs[k % N_VECS], out=dense_outs[k % N_MATS])

    def mv_all():
        for k in range(GRAPH_STEPS):
            torch.mv(raws[k % N_MATS].t(), vec16[k % N_VECS], out=mv_outs[k % N_MATS])

    dense_us = time_graph(dense_all) * 1000.0 / GRAPH_STEPS
    mv_us = time_graph(mv_all) * 1000.0 / GRAPH_STEPS
    dense_bytes = 2.0 * IN_DIM * OUT_DIM + 4.0 * IN_DIM + 4.0 * OUT_DIM
    baselines = {"dense_roofline_us_measured_peak": dense_bytes / (peak * 1e9) * 1e6,
                 "dense_roofline_us_nominal_8000": dense_bytes / (NOMINAL_HBM_GBS * 1e9) * 1e6,
                 "k_dense_gemv_us": dense_us, "k_dense_gemv_gbs": dense_bytes / (dense_us * 1e-6) / 1e9,
                 "torch_mv_cublas_us": mv_us}

    sweep = {}
    if not a.no_sweep:
        for e in SWEEP:
            msw = statistics.median(timed_steps(e, 400, 80, regions=3))
            us = msw * 1000.0 / 400
            Se, De, Spe = rotation_stats(e)
            b = algorithmic_bytes(IN_DIM, OUT_DIM, Se)
            rb = read_bytes(IN_DIM, OUT_DIM, De, Spe)
            sweep[str(e)] = {"us": us, "gbs_algorithmic": b / (us * 1e-6) / 1e9, "mean_used": Se,
                             "read_bytes": {"dense": De, "sparse": Spe, "total": rb},
                             "gbs_read": rb / (us * 1e-6) / 1e9,
                             "vs_dense_roofline_measured": baselines["dense_roofline_us_measured_peak"] / us}

    # batched / MoE: 8 experts of the workload's shape (the first eight prepared
    # matrices), n vectors N(0,1) each routed to its top-2 experts by a seeded
    # N(0,1)/64 gate (ties to the lower expert), one cutoff per (vector, expert)
    # pair, all pairs in one batched call
    moe = {}
    if not a.no_sweep:
        n_exp = 8
        gate = inputs.gate(n_exp, IN_DIM, 300)
        ws_moe = E.Workspace(IN_DIM, OUT_DIM, max_pairs=32)
        for nv in (1, 4, 16):
            Vn = np.stack([inputs.vector(IN_DIM, 200 + 16 * nv + k) for k in range(nv)])
            order = np.argsort(-(gate.astype(np.float64) @ Vn.astype(np.float64).T), axis=0, kind="stable")
            hidx = [int(order[r, k]) for k in range(nv) for r in range(2)]
            vidx = [k for k in range(nv) for _ in range(2)]
            Vd = torch.from_numpy(Vn).to(dev)
            OUTd = torch.empty(2 * nv, OUT_DIM, device=dev)
            cnt_d = torch.zeros(2 * nv, device=dev, dtype=torch.int64)
            row = {}
            for e in (0.5, 0.25, 0.12):
                E.gemv_batched(ws_moe, mats[:n_exp], hidx, vidx, Vd, [e] * (2 * nv), OUT=OUTd, counts=cnt_d)
                torch.cuda.synchronize()
                used = float(cnt_d.sum().item())
                bd, bs = ws_moe.last_call_bytes()
                # the same pairs as separate calls: the sum of their reads
                pair_bytes = 0
                for k in range(2 * nv):
                    mats[hidx[k]].gemv(Vd[vidx[k]], e, out=OUTd[k])
                    pd_, ps_ = mats[hidx[k]].last_call_bytes()
                    pair_bytes += pd_ + ps_
                ms_call = time_graph(lambda: E.gemv_batched(ws_moe, mats[:n_exp], hidx, vidx, Vd, [e] * (2 * nv),
                                                            OUT=OUTd), n_rep=20)
                b = 3.0 * used + 2 * nv * (algorithmic_bytes(IN_DIM, OUT_DIM, 0.0))
                row[str(e)] = {"us_per_call": ms_call * 1000.0, "pairs": 2 * nv,
                               "gbs_algorithmic": b / (ms_call * 1e-3) / 1e9,
                               "read_bytes_call": bd + bs, "read_bytes_pairs_separately": pair_bytes,
                               "union_saving": 1.0 - (bd + bs) / pair_bytes if pair_bytes else None}
            moe[str(nv)] = row
        ws_moe.close()

    # the other shapes of the method's workloads
    shapes = {}
    if not a.no_sweep:
        shapes["attention 4096x4096, v N(0,1)"] = measure_shape(E, dev, 4096, 4096, SWEEP, "normal")
        shapes["FFN down 14336x4096, v t3/sqrt(3)"] = measure_shape(E, dev, 14336, 4096, (0.25, 0.15), "t3")
        shapes["FFN up 4096x14336, keep 0.75, v t3/sqrt(3)"] = measure_shape(E, dev, 4096, 14336, (0.25, 0.15),
                                                                             "t3", keep=0.75)
        # Q8 weights (row f3) on the headline shape; the int8 dense roofline is half the fp16 one
        try:
            shapes["Q8 FFN up 4096x14336, v t3/sqrt(3)"] = measure_shape(E, dev, 4096, 14336, (1.0, 0.5, 0.25, 0.15),
                                                                         "t3", q8=True)
        except Exception as ex:  # reported, not fatal: the headline line stands on its own
            shapes["Q8 FFN up 4096x14336, v t3/sqrt(3)"] = {"error": repr(ex)[:200]}

    # the decode chain (one token through 32 layers)
    chain = measure_chain(E, dev) if (not a.no_sweep and world == 1) else {}

    # end to end through the C ABI on host buffers (effort_gemv_host): every
    # step copies its v from pinned host memory into the device and copies out
    # back to pinned host memory; the library calls are
    # issued from a CUDA graph of GRAPH_STEPS calls, like the device-resident
    # steps, so the figure carries the transfers and not Python's call cost
    n_e2e = max(1, min(a.steps, 400) // GRAPH_STEPS) * GRAPH_STEPS
    hv = [torch.from_numpy(inputs.vector(IN_DIM, 7 + k, "t3")).pin_memory() for k in range(N_VECS)]
    hout = torch.empty(OUT_DIM, dtype=torch.float32).pin_memory()
    st = torch.cuda.Stream(device=dev)
    st.wait_stream(torch.cuda.current_stream(dev))
    with torch.cuda.stream(st):
        for k in range(GRAPH_STEPS):
            mats[k % N_MATS].gemv_host(hv[k % N_VECS], EFFORT, hout)
    torch.cuda.synchronize()
    g_e2e = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g_e2e, stream=st):
        for k in range(GRAPH_STEPS):
            mats[k % N_MATS].gemv_host(hv[k % N_VECS], EFFORT, hout)
    for _ in range(3):
        g_e2e.replay()
    torch.cuda.synchronize()
    barrier()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record()
    for _ in range(n_e2e // GRAPH_STEPS):
        g_e2e.replay()
    e1.record()
    torch.cuda.synchronize()
    barrier()
    e2e_us = rank_max(e0.elapsed_time(e1)) * 1000.0 / n_e2e / world
    del g_e2e

    cpu = None
    if rank == 0 and world == 1 and not a.no_cpu_baseline:
        cpu = cpu_baseline()

    if rank == 0:
        line = {"metric": METRIC, "value": value, "unit": "us", "n_gpus": world, "steps": a.steps,
                "warmup": a.warmup, "ms_per_step": us_per_step / 1000.0, "higher_is_better": False,
                "scaling": "weak", "vs_baseline": None, "dtype": "f32", "data": "synthetic",
                "config": workload_config(),
                "gbs": alg_bytes / (us_per_step * 1e-6) / 1e9,
                "timed_regions_us_per_step": [x * 1000.0 / a.steps for x in region_ms],
                "phases_us": phases,
                "roofline": roofline, "cpu_baseline": cpu,
                "e2e": {"value": e2e_us, "unit": "us", "h2d_bytes_per_step": 4 * IN_DIM,
                        "d2h_bytes_per_step": 4 * OUT_DIM,
                        "how": "effort_gemv_host (C ABI) on pinned host v and out, calls issued from CUDA graphs of "
                               f"{GRAPH_STEPS}; v copied in and out copied back every step"},
                "gpu_launches": a.steps, "clocks": clocks,
                "mean_used_products": S_mean, "baselines": baselines, "sweep": sweep,
                "shapes": shapes,
                "chain": chain,
                "moe": {"workload": "8 experts 4096x14336 fp16, n vectors N(0,1) routed top-2 by a seeded gate, "
                                    "one cutoff per pair, one batched call (two pairs on one expert share "
                                    "one grid and read the union of their prefixes once)",
                        "by_n_vectors": moe}}
        print(json.dumps(line), flush=True)
    for m in mats:
        m.close()
    ws.close()
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()


if __name__ == "__main__":
    main()
