"""Benchmark of the record-and-replay discrete adjoint on B200.

One step = the whole hot path on the 2^20-trajectory stellar-orbit ensemble (test particles in an
NFW halo + Miyamoto-Nagai disk, d = 6, 5 parameters per trajectory, fp64, Tsit5, rtol 1e-8,
atol 1e-10, t in [0, 20]): the record pass (adaptive solve + record of accepted steps + record
finalisation), the caller's loss cotangent dL/dy1 = 2 (x(20) - x*) (velocities 0), and the replay
gradient dL/dtheta [N, 5], dL/dy0 [N, 6].  `value` = trajectories whose gradient is delivered per
second.  Inputs are resident in HBM before the timed region; the record (~9 GB) is far larger than
the 126 MB L2, so no L2 flush is needed between steps.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
Under torchrun each rank solves its own 2^20 ensemble (weak scaling, no collective on the path).
"""
import argparse
import json
import os
import statistics
import subprocess
import sys
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "replay-gradient trajectories/s and forward-solve traj/s at 2^20; % FP64 peak"
UNIT = "traj/s"

# Algorithmic FP64 flops per accepted step of the replay adjoint on the stellar field (add, sub,
# mul, fma = 2, div, sqrt, log1p each counted as one operation), and per attempted step of the
# forward solve: counted from the definitions of the Tsit5 replay step, its reverse sweep and the
# field's f and vector-Jacobian product (tests/test_flop_counts.py re-derives these numbers).
FLOPS_ADJOINT_STEP = {"nfw_mn": 1254, "lorenz63": 432, "lotka_volterra": 344, "mlp": 48400,
                      "log_halo": 840}
FLOPS_FORWARD_ATTEMPT = {"nfw_mn": 611, "lorenz63": 254, "lotka_volterra": 181, "mlp": 16425,
                         "log_halo": 479}
# Forward sensitivities, per accepted step and all m columns: the tangent of the Tsit5 step,
# 48 d (stage tangents 35 d, result 13 d) + 6 c_t per column, c_t = the forward-mode rules' extra
# operations over f (the value part that the kernel recomputes alongside is not counted).
FLOPS_SENS_STEP = {"log_halo": 948}
# Verner 7, counted the same way from its table (nonzero a_ij per stage row 1, 2, 2, 3, 4, 5, 6,
# 7, 6; b has 7 nonzeros, b - b_hat 8): per attempt 117 d + 10 c_f + 5 (nine new stages and the
# fresh first stage of the next step); per accepted step of the replay adjoint 160 d + 8 c_f +
# 9 c_v (stages 2..9 recomputed, nine pullbacks).  c_f, c_v as for Tsit5.
FLOPS_VERN7_ATTEMPT = {"lorenz63": 436, "nfw_mn": 1047}
FLOPS_VERN7_ADJOINT = {"lorenz63": 724, "nfw_mn": 2015}
# Stiff fields: (d, c_f, c_v, c_J, c_Jv) -- f, its pullback, the Jacobian and the contraction of a
# Jacobian cotangent with dJ/d(y, theta), counted like c_f and c_v.
STIFF_COUNTS = {"robertson": (3, 8, 20, 9, 22), "hires": (8, 38, 77, 3, 32)}


# Jacobian sparsity patterns the fields declare to the kernels (bit c of row r: J[r][c] can be
# nonzero); the LU of the iteration matrix then works on that pattern and its fill-in only.
JAC_PATTERN = {"hires": (0x07, 0x03, 0x1C, 0x0E, 0x70, 0xF8, 0xE0, 0xE0)}


def lu_ops(d):
    """Dense LU without the pivot search: per column one reciprocal, k multipliers and 2 k^2 for
    the update of the k x k trailing block."""
    return sum(1 + k + 2 * k * k for k in range(d))


def pattern_ops(field, d):
    """(nnz(J), operations of one triangular solve pair, operations of the LU) on the field's
    Jacobian pattern with the fill-in of elimination without row exchanges; the dense figures
    (d^2, 2 d^2 - d, lu_ops(d)) for a field without a declared pattern.  Per column of the LU: one
    reciprocal, m multipliers and 2 m u updates (m rows below, u columns right in the pattern);
    a solve: 2 per strictly lower and strictly upper entry, and d multiplications by the pivots'
    reciprocals."""
    rows = JAC_PATTERN.get(field)
    if rows is None:
        return d * d, 2 * d * d - d, lu_ops(d)
    J = [[bool((rows[r] >> c) & 1) for c in range(d)] for r in range(d)]
    f = [[J[r][c] or r == c for c in range(d)] for r in range(d)]
    for col in range(d):
        for i in range(col + 1, d):
            if f[i][col]:
                for j in range(col + 1, d):
                    if f[col][j]:
                        f[i][j] = True
    lu = 0
    for col in range(d):
        m = sum(f[r][col] for r in range(col + 1, d))
        u = sum(f[col][q] for q in range(col + 1, d))
        lu += 1 + m + 2 * m * u
    nl = sum(f[r][c] for r in range(d) for c in range(r))
    nu = sum(f[r][c] for r in range(d) for c in range(r + 1, d))
    return sum(map(sum, J)), 2 * (nl + nu) + d, lu


def stiff_flops(method, field):
    """Operations per attempted step and per accepted step of the replay adjoint, counted from the
    step's definition (one solve = 2 d^2 - d):
      ROS34PW2 attempt  c_J + 4 c_f + 17 d^2 + 53 d + LU(d) + 6
      ROS34PW2 adjoint  c_J + c_Jv + 4 c_f + 4 c_v + 51 d^2 + 92 d + LU(d) + 1
      Rosenbrock23 attempt  c_J + 2 c_f + 7 d^2 + 20 d + LU(d) + 7
      Rosenbrock23 adjoint  c_J + c_Jv + 2 c_f + 2 c_v + 12 d^2 + 12 d + LU(d) + 3
    Rosenbrock23's d^2 terms are the iteration matrix (d^2 + d), three solves in the attempt and
    four (two of them transposed) in the adjoint, and the adjoint's two outer products into the
    Jacobian cotangent (3 d^2): on a field with a declared Jacobian pattern they become nnz(J) + d,
    the pattern's solves and 3 nnz(J), and LU(d) the pattern's elimination (pattern_ops) -- the
    work of the kernels, which touch nothing else.  (ROS34PW2 is counted dense: its J G products
    run over every entry, and no patterned field takes it.)"""
    d, cf, cv, cj, cjv = STIFF_COUNTS[field]
    if method == "ros34pw2":
        lu = lu_ops(d)
        return (cj + 4 * cf + 17 * d * d + 53 * d + lu + 6,
                cj + cjv + 4 * cf + 4 * cv + 51 * d * d + 92 * d + lu + 1)
    nnz, solve, lu = pattern_ops(field, d)
    w = nnz + d
    return (cj + 2 * cf + w + 3 * solve + 22 * d + lu + 7,
            cj + cjv + 2 * cf + 2 * cv + w + 4 * solve + 3 * nnz + 15 * d + lu + 3)
# The MLP field (4-32-32-4, tanh) counted by hand: f = 1,280 multiply-adds + 68 bias adds + 64
# tanh = 2,692 ops; its pullback = the two transposed products (2 x 1,280 flops), the weight
# outer products (2 x 1,280), 2 x 64 for tanh' and 68 bias cotangents = 5,316 ops; per accepted
# step 88 d + 6 c_f + 6 c_v = 48,400 (FP32), per attempt 67 d + 6 c_f + 5 = 16,425.
# FP64 peak: 148 SMs x 64 FP64 FMA lanes/SM/clk x 2 flop x clock (1965 MHz max) = 37.2 TFLOP/s,
# the datasheet FP64 figure of B200; the same formula at the measured SM clock is reported too.
SMS, FP64_LANES, FP32_LANES = 148, 64, 128
# DRAM bytes (read + write) per accepted step, from one ncu capture of each kernel on the
# 2^18-trajectory case of this workload; both kernels move a fixed number of bytes per accepted
# step, so a launch's traffic is this times its accepted steps.  Record kernel: 64 B of record
# per step written plus inputs; adjoint: the 64 B entry read per step plus chunk table and inputs.
# Every figure comes from a capture after the last change to its kernel (a figure that a kernel
# change leaves stale is withheld as None until captured again); the Verner 7 Lorenz record
# keeps part of its record in L2 at the captured size, so it has none.
TRAFFIC_PER_STEP = {
    "nfw_mn": {"record": 67.3, "adjoint": 85.1},
    "robertson": {"record": 38.9, "adjoint": 42.2},
    "robertson_rb23": {"record": 39.8, "adjoint": 43.6},
    "hires": {"record": 80.5, "adjoint": 81.6},            # captured at 16,384 trajectories
    "lorenz63_vern7": {"adjoint": 45.2},                   # its record pass stays partly in L2
}
# FP64 pipe occupancy (sm__pipe_fp64_cycles_active, % of peak) of the same captures: how busy the
# pipe is, transcendental sequences included, next to the algorithmic fraction
PIPE_BUSY_NCU = {
    "nfw_mn": {"record": 0.564, "adjoint": 0.741},
    "robertson": {"record": 0.408, "adjoint": 0.474},
    "robertson_rb23": {"record": 0.299, "adjoint": 0.459},
    "hires": {"record": 0.204, "adjoint": 0.253},          # 16,384 trajectories: one wave
    "lorenz63_vern7": {"record": 0.439, "adjoint": 0.552},
    "log_halo": {"sens": 0.790},
}
# forward sensitivities: DRAM bytes per trajectory (inputs and outputs; nothing per step), from
# an ncu capture of the 2^18-orbit case
TRAFFIC_SENS_PER_TRAJ = {"log_halo": 94.3}
# library kernels per step: record = k_solve + the pass summary (3 kernels: step and chunk
# offsets side by side, longest record, worst status) + k_chunk_table + the longest-first order
# (k_bin_count, the one-block scan of the length bins, k_bin_scatter) (8); replay gradient =
# k_theta_check + k_replay_forward (exits at once: the theta is the recorded one) + k_adjoint (3).
LAUNCHES_PER_STEP = 11


def fp64_peak_tflops(mhz):
    return pipe_peak_tflops(mhz, FP64_LANES)


def pipe_peak_tflops(mhz, lanes):
    return SMS * lanes * 2 * mhz * 1e6 / 1e12


class ClockSampler:
    """nvidia-smi clocks / throttle reasons sampled every 200 ms around the timed region.  The
    sampler is started (and its first sample awaited) before the region begins, and samples taken
    within 250 ms of the region's ends count, so that short regions still carry a reading."""
    Q = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
         "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
         "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index):
        self.gpu = gpu_index
        self.proc = None
        self.samples = []
        self.t0 = self.t1 = None

    def _reader(self):
        for line in self.proc.stdout:
            if line.strip():
                self.samples.append((time.perf_counter(), line))

    def __enter__(self):
        import threading
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.gpu), "--query-gpu=" + self.Q,
                 "--format=csv,noheader,nounits", "-lms", "200"],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except OSError:
            self.proc = None
        if self.proc is not None:
            self.thread = threading.Thread(target=self._reader, daemon=True)
            self.thread.start()
            deadline = time.perf_counter() + 3.0
            while not self.samples and time.perf_counter() < deadline:
                time.sleep(0.01)
        self.t0 = time.perf_counter()
        return self

    def __exit__(self, *a):
        self.t1 = time.perf_counter()
        if self.proc is not None:
            time.sleep(0.25)
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()
            self.thread.join(timeout=5)

    def summary(self):
        sm, smax, reasons = [], None, set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        lines = [l for (ts, l) in self.samples
                 if self.t0 is not None and self.t0 - 0.25 <= ts <= self.t1 + 0.25]
        for l in lines:
            f = [x.strip() for x in l.split(",")]
            if len(f) < 9:
                continue
            try:
                sm.append(float(f[1]))
                smax = float(f[2])
            except ValueError:
                continue
            for n, v in zip(names, f[5:9]):
                if v.lower() == "active":
                    reasons.add(n)
        if not sm:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["unavailable"], "samples": 0}
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": smax, "reasons": sorted(reasons),
                "samples": len(sm)}


DESCR = {"nfw_mn": "stellar orbits: NFW halo + Miyamoto-Nagai disk",
         "nfw_mn_f32": "stellar orbits: NFW halo + Miyamoto-Nagai disk",
         "lorenz63": "Lorenz-63", "lotka_volterra": "Lotka-Volterra",
         "robertson": "Robertson kinetics (stiff)", "mlp": "neural RHS 4-32-32-4 tanh, shared weights",
         "log_halo": "stellar orbits in a flattened logarithmic halo, theta = (v_c, q) shared",
         "lorenz63_vern7": "Lorenz-63, Verner 7(6) pair",
         "robertson_rb23": "Robertson kinetics (stiff), Rosenbrock23",
         "hires": "HIRES kinetics (stiff, 8 components), Rosenbrock23, shared rate constants",
         "nfw_mn_vern7": "stellar orbits: NFW halo + Miyamoto-Nagai disk, Verner 7(6) pair"}


def workload_config(ws, N=1 << 20, name="nfw_mn", w=None, step=None):
    if w is None:
        spec = "d=6, m=5 per trajectory, fp64, Tsit5 rtol=1e-8 atol=1e-10, t=[0,20]"
    else:
        spec = "d=%d, m=%d %s, %s, %s rtol=%g atol=%g, t=[%g,%g]" % (
            w.d, w.m, "shared" if w.theta_shared else "per trajectory",
            "fp64" if w.dtype == np.float64 else "fp32", w.method, w.rtol, w.atol, w.t0, w.t1)
    step = step or "record + loss cotangent + replay gradient"
    return {"workload": "%s %s, N=%d per GPU, %s; step = %s" % (name, DESCR[name], N, spec, step),
            "global_batch": ws * N,
            "parallelism": "independent trajectories, %d rank(s)" % ws,
            "l2": "inputs larger than L2 (the record is several GB)" if name.startswith("nfw")
                  else ("flushed between steps" if name == "log_halo"
                        else "record size reported in record_gb")}


def dist_env():
    ws = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return ws, rank, local


def run_reference(args):
    """The CPU oracle as it stands, on the host cores, on a bounded sample of the same workload."""
    ws, rank, _ = dist_env()
    if rank != 0:
        return
    from differentiable_adaptive_ode_b200 import workloads as W
    from oracle import oracle as orc
    nthreads = orc.host_threads()
    w_full = W.by_name(args.workload)
    sens = WORKLOADS[args.workload].get("step") == "sens"

    def one_step(w):
        if sens:
            orc.solve_sens(w.field, w.theta, w.y0, w.t0, w.t1, w.rtol, w.atol, dtype=w.dtype,
                           theta_shared=w.theta_shared, nthreads=nthreads)
        else:
            r = orc.solve(w.field, w.method, w.theta, w.y0, w.t0, w.t1, w.rtol, w.atol,
                          keep_record=True, nthreads=nthreads, dtype=w.dtype,
                          theta_shared=w.theta_shared)
            tgt = w.target if w.target is not None else np.zeros_like(r["y1"])
            lam = W.loss_cotangent(w, r["y1"], tgt)
            orc.replay_grad(w.field, w.method, w.theta, w.y0, r["H"], r["S"], lam,
                            nthreads=nthreads, dtype=w.dtype, theta_shared=w.theta_shared)

    n_sample = args.ref_sample
    if n_sample <= 0:
        # a sample of about 3 s of host work per step (so that the whole run stays within
        # minutes), from a 256-trajectory calibration, between 64 and 4096 trajectories
        t0 = time.perf_counter()
        one_step(W.by_name(args.workload, N=256))
        per = (time.perf_counter() - t0) / 256
        n_sample = int(min(4096, max(64, 3.0 / max(per, 1e-9))))
    w = W.by_name(args.workload, N=n_sample)
    times = []
    for i in range(args.warmup + args.steps):
        t0 = time.perf_counter()
        one_step(w)
        dt = time.perf_counter() - t0
        if i >= args.warmup:
            times.append(dt)
    t = statistics.median(times)
    v = n_sample / t
    line = {"metric": METRIC, "value": v, "unit": UNIT, "impl": "reference", "n_gpus": args.gpus,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": t * 1e3,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
            "dtype": "f64" if w.dtype == np.float64 else "f32", "data": "synthetic",
            "config": dict(workload_config(1, w_full.N, args.workload, w_full,
                                           SENS_STEP if sens else None),
                           sample="%d trajectories per step" % n_sample),
            "cpu_baseline": {"value": v, "unit": UNIT, "cores": nthreads, "kind": "oracle",
                             "sample": "%d trajectories of the %s ensemble per step: %s"
                                       % (n_sample, args.workload,
                                          "solve with forward sensitivities" if sens else
                                          "record solve + replay gradient")},
            "e2e": {"value": v, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


def cpu_baseline_sample(seconds_target=15.0, single_core_n=1 << 14):
    """Oracle throughput (record + replay gradient) on a bounded sample, all host threads; and on
    one thread over the first 2^14 trajectories of the same ensemble, scaled linearly."""
    from differentiable_adaptive_ode_b200 import workloads as W
    from oracle import oracle as orc
    nthreads = orc.host_threads()

    def run(w, threads):
        t0 = time.perf_counter()
        r = orc.solve(w.field, w.method, w.theta, w.y0, w.t0, w.t1, w.rtol, w.atol,
                      keep_record=True, nthreads=threads)
        lam = W.loss_cotangent(w, r["y1"], w.target)
        orc.replay_grad(w.field, w.method, w.theta, w.y0, r["H"], r["S"], lam, nthreads=threads)
        return time.perf_counter() - t0

    n = 256
    while True:
        dt = run(W.nfw_mn(N=n), nthreads)
        if dt > seconds_target / 4 or n >= 1 << 16:
            break
        n *= 2
    out = {"value": n / dt, "unit": UNIT, "cores": nthreads, "kind": "oracle",
           "sample": "%d trajectories of the 2^20 stellar ensemble (record solve + replay "
                     "gradient), %.1f s" % (n, dt)}
    if single_core_n:
        w1 = W.subset(W.nfw_mn(), np.arange(single_core_n))
        dt1 = run(w1, 1)
        out["single_core"] = {"value": single_core_n / dt1, "unit": UNIT, "cores": 1,
                              "sample": "the first %d trajectories of the 2^20 stellar ensemble "
                                        "on one thread, %.1f s" % (single_core_n, dt1),
                              "full_ensemble_s_scaled": dt1 * (1 << 20) / single_core_n}
    return out


# Per-workload constants: the field/method, the FP pipe that bounds the hot kernels and the
# algorithmic operations per unit (counted from the definitions; see the constants above).
WORKLOADS = {
    "nfw_mn": dict(dtype="f64", fwd=FLOPS_FORWARD_ATTEMPT["nfw_mn"], adj=FLOPS_ADJOINT_STEP["nfw_mn"]),
    "nfw_mn_f32": dict(dtype="f32", fwd=FLOPS_FORWARD_ATTEMPT["nfw_mn"],
                       adj=FLOPS_ADJOINT_STEP["nfw_mn"]),
    "lorenz63": dict(dtype="f64", fwd=FLOPS_FORWARD_ATTEMPT["lorenz63"],
                     adj=FLOPS_ADJOINT_STEP["lorenz63"]),
    "lotka_volterra": dict(dtype="f64", fwd=FLOPS_FORWARD_ATTEMPT["lotka_volterra"],
                           adj=FLOPS_ADJOINT_STEP["lotka_volterra"]),
    "robertson": dict(dtype="f64", fwd=stiff_flops("ros34pw2", "robertson")[0],
                      adj=stiff_flops("ros34pw2", "robertson")[1]),
    "robertson_rb23": dict(dtype="f64", fwd=stiff_flops("rosenbrock23", "robertson")[0],
                           adj=stiff_flops("rosenbrock23", "robertson")[1]),
    "hires": dict(dtype="f64", fwd=stiff_flops("rosenbrock23", "hires")[0],
                  adj=stiff_flops("rosenbrock23", "hires")[1]),
    "mlp": dict(dtype="f32", fwd=FLOPS_FORWARD_ATTEMPT["mlp"], adj=FLOPS_ADJOINT_STEP["mlp"]),
    "lorenz63_vern7": dict(dtype="f64", fwd=FLOPS_VERN7_ATTEMPT["lorenz63"],
                           adj=FLOPS_VERN7_ADJOINT["lorenz63"]),
    "nfw_mn_vern7": dict(dtype="f64", fwd=FLOPS_VERN7_ATTEMPT["nfw_mn"],
                         adj=FLOPS_VERN7_ADJOINT["nfw_mn"]),
    "log_halo": dict(dtype="f64", fwd=FLOPS_FORWARD_ATTEMPT["log_halo"],
                     adj=FLOPS_ADJOINT_STEP["log_halo"], sens=FLOPS_SENS_STEP["log_halo"],
                     step="sens"),
}
SENS_STEP = ("forward solve with the sensitivities S = dy/dtheta (6 x 2 per orbit) in the same "
             "kernel, step size controlled on the orbit")
L2_FLUSH_BYTES = 256 << 20


def run_sens(args, w, wl, G, torch, dev, stream, ws, rank):
    """Forward sensitivities ("Differentiable astrophysics at scale" §3): one step = one
    gs_solve_forward_sens over the ensemble, L2 flushed between steps (inside the timed region)."""
    N, d, m = w.N, w.d, w.m
    dt = torch.float64
    sys_ = G.system(w.field, w.method, "f64", w.theta_shared)
    th = torch.as_tensor(w.theta, dtype=dt, device=dev)
    y0 = torch.as_tensor(w.y0, dtype=dt, device=dev)
    y1 = torch.empty((N, d), dtype=dt, device=dev)
    S1 = torch.empty((N, d, m), dtype=dt, device=dev)
    S = torch.empty(N, dtype=torch.int32, device=dev)
    rj = torch.empty(N, dtype=torch.int32, device=dev)
    st = torch.empty(N, dtype=torch.int32, device=dev)
    flush = torch.empty(L2_FLUSH_BYTES // 4, dtype=torch.int32, device=dev)
    # the caller's start order: orbits by decreasing attempts of the previous solve (scheduling
    # only), formed on the device after every step
    order = torch.arange(N, dtype=torch.int32, device=dev)
    opts = G.options(start_order=order)

    def step():
        G.gs_solve_forward_sens(sys_, N, th, y0, w.t0, w.t1, w.rtol, w.atol, y1, S1, None, S, rj,
                                st, opts=opts)
        order.copy_(torch.argsort(S + rj, descending=True))

    for _ in range(args.warmup):
        flush.zero_()
        step()
    torch.cuda.synchronize()

    def barrier():
        if ws > 1:
            torch.distributed.barrier()
        torch.cuda.synchronize()

    kev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
           for _ in range(args.steps)]
    barrier()
    with ClockSampler(dev.index) as clk:
        start = torch.cuda.Event(enable_timing=True)
        stop = torch.cuda.Event(enable_timing=True)
        start.record(stream)
        for i in range(args.steps):
            flush.zero_()
            kev[i][0].record(stream)
            step()
            kev[i][1].record(stream)
        stop.record(stream)
        barrier()
    total_ms = start.elapsed_time(stop)
    if ws > 1:
        t = torch.tensor([total_ms], device=dev)
        torch.distributed.all_reduce(t, op=torch.distributed.ReduceOp.MAX)
        total_ms = float(t.item())
    ms_step = total_ms / args.steps
    value = ws * N * args.steps / (total_ms / 1e3)
    kernel_ms = statistics.median(a.elapsed_time(b) for a, b in kev)
    assert int((st != 0).sum().item()) == 0, "some trajectory failed"
    accepted = int(S.sum().item())
    attempts = accepted + int(rj.sum().item())

    # ---- breakdown (not part of `value`): the orbit alone, and the reverse-mode route (record +
    # replay gradient of one scalar loss on the final positions) on the same ensemble
    def timeit(fn, reps=max(3, args.steps // 2)):
        fn()
        torch.cuda.synchronize()
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record(stream)
        for _ in range(reps):
            fn()
        b.record(stream)
        torch.cuda.synchronize()
        return a.elapsed_time(b) / reps

    fwd_ms = timeit(lambda: G.gs_solve_forward(sys_, N, th, y0, w.t0, w.t1, w.rtol, w.atol, y1))
    rec = G.Record()
    target = torch.as_tensor(w.target, dtype=dt, device=dev)
    mask = torch.as_tensor(w.loss_mask, dtype=dt, device=dev)
    lam = torch.empty((N, d), dtype=dt, device=dev)
    gt = torch.empty((m,), dtype=dt, device=dev)
    gy = torch.empty((N, d), dtype=dt, device=dev)

    def reverse():
        G.gs_solve_record(sys_, N, th, y0, w.t0, w.t1, w.rtol, w.atol, y1, rec=rec)
        torch.mul(torch.sub(y1, target), mask, out=lam).mul_(2.0)
        G.gs_replay_grad(rec, th, lam, gt, gy)

    rev_ms = timeit(reverse)
    rec.close()
    breakdown = {"sens_step": ms_step, "sens_kernel": kernel_ms, "forward_only": fwd_ms,
                 "record_plus_replay_grad": rev_ms}

    # ---- end to end through the public API with host buffers (pinned), copies inside the region
    # two stream pipelines with their own buffers, steps alternating between them, so that one
    # step's host<->device copies overlap the other's kernel (every step still copies its inputs
    # in and its orbits and sensitivities out)
    h_th = torch.as_tensor(w.theta, dtype=dt).pin_memory()
    h_y0 = torch.as_tensor(w.y0, dtype=dt).pin_memory()
    pipes = []
    for _ in range(2):
        pipes.append(dict(s=torch.cuda.Stream(), th=torch.empty_like(th), y0=torch.empty_like(y0),
                          y1=torch.empty_like(y1), S1=torch.empty_like(S1),
                          S=torch.empty_like(S), rj=torch.empty_like(rj), st=torch.empty_like(st),
                          order=order.clone(),
                          h_y1=torch.empty((N, d), dtype=dt).pin_memory(),
                          h_S1=torch.empty((N, d, m), dtype=dt).pin_memory()))

    def e2e_step(q):
        with torch.cuda.stream(q["s"]):
            q["th"].copy_(h_th, non_blocking=True)
            q["y0"].copy_(h_y0, non_blocking=True)
            G.gs_solve_forward_sens(sys_, N, q["th"], q["y0"], w.t0, w.t1, w.rtol, w.atol,
                                    q["y1"], q["S1"], None, q["S"], q["rj"], q["st"],
                                    opts=G.options(start_order=q["order"]))
            q["order"].copy_(torch.argsort(q["S"] + q["rj"], descending=True))
            q["h_y1"].copy_(q["y1"], non_blocking=True)
            q["h_S1"].copy_(q["S1"], non_blocking=True)

    for q in pipes:
        e2e_step(q)
    e2e_steps = max(4, args.steps // 2)
    barrier()
    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    a.record(stream)
    for q in pipes:
        q["s"].wait_event(a)
    for i in range(e2e_steps):
        e2e_step(pipes[i % 2])
    for q in pipes:
        ev = torch.cuda.Event()
        ev.record(q["s"])
        stream.wait_event(ev)
    b.record(stream)
    barrier()
    e2e_ms = a.elapsed_time(b) / e2e_steps
    h_y1, h_S1 = pipes[0]["h_y1"], pipes[0]["h_S1"]
    if ws > 1:
        t = torch.tensor([e2e_ms], device=dev)
        torch.distributed.all_reduce(t, op=torch.distributed.ReduceOp.MAX)
        e2e_ms = float(t.item())

    clocks = clk.summary()
    peak = pipe_peak_tflops(1965.0, FP64_LANES)
    at_clock = pipe_peak_tflops(clocks["sm_mhz"], FP64_LANES) if clocks.get("sm_mhz") else None
    flops = wl["fwd"] * attempts + wl["sens"] * accepted
    achieved = flops / (kernel_ms / 1e3) / 1e12
    roofline = {"kernel": "k_solve<log_halo, double, Tsit5, sens>", "bound": "alu",
                "achieved": achieved, "peak": peak, "unit": "TFLOP/s", "frac": achieved / peak,
                "pipe_busy_ncu": PIPE_BUSY_NCU.get(args.workload, {}).get("sens"),
                "traffic": (TRAFFIC_SENS_PER_TRAJ[args.workload] * N
                            if TRAFFIC_SENS_PER_TRAJ.get(args.workload) else None),
                "traffic_source": "ncu dram bytes per trajectory on the 2^18 case x trajectories",
                "peak_source": "derived: 148 SM x 64 FP64 FMA lanes/clk x 2 x 1965 MHz (FP64 pipe)",
                "flops_per_unit": {"attempted step": wl["fwd"], "accepted step (sensitivities)":
                                   wl["sens"]},
                "kernel_ms": kernel_ms,
                "frac_at_measured_clock": achieved / at_clock if at_clock else None}
    line = {
        "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": ws, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": ms_step, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": dict(workload_config(ws, N, args.workload, w, SENS_STEP),
                       l2="flushed between steps (%d MiB write inside the timed region)"
                          % (L2_FLUSH_BYTES >> 20),
                       accepted_steps=accepted, attempts=attempts),
        "roofline": roofline,
        "breakdown_ms": breakdown,
        "forward_traj_per_s": ws * N / (fwd_ms / 1e3),
        "e2e": {"value": ws * N / (e2e_ms / 1e3), "unit": UNIT,
                "h2d_bytes_per_step": (h_th.numel() + h_y0.numel()) * 8,
                "d2h_bytes_per_step": (h_y1.numel() + h_S1.numel()) * 8},
        "gpu_launches": args.steps,
        "clocks": clocks,
    }
    if rank == 0 and ws == 1 and not args.no_cpu_baseline:
        line["cpu_baseline"] = cpu_baseline_sens(w)
    else:
        line["cpu_baseline"] = None
    return line


def cpu_baseline_sens(w_full, seconds_target=15.0):
    """Oracle throughput (solve with forward sensitivities) on a bounded sample, all host threads."""
    from differentiable_adaptive_ode_b200 import workloads as W
    from oracle import oracle as orc
    nthreads = orc.host_threads()
    n = 256
    while True:
        w = W.subset(w_full, np.arange(n))
        t0 = time.perf_counter()
        orc.solve_sens(w.field, w.theta, w.y0, w.t0, w.t1, w.rtol, w.atol,
                       theta_shared=w.theta_shared, nthreads=nthreads)
        dt = time.perf_counter() - t0
        if dt > seconds_target / 4 or n >= 1 << 16:
            return {"value": n / dt, "unit": UNIT, "cores": nthreads, "kind": "oracle",
                    "sample": "%d orbits of the 2^20 logarithmic-halo ensemble (solve with "
                              "forward sensitivities), %.1f s" % (n, dt)}
        n *= 2


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=10)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--workload", default="nfw_mn", choices=sorted(WORKLOADS))
    ap.add_argument("--N", type=int, default=0, help="trajectories per GPU (0: the workload's)")
    ap.add_argument("--ref-sample", type=int, default=0,
                    help="trajectories per reference step (0: about 3 s of host work)")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    args = ap.parse_args()
    if args.impl == "reference":
        return run_reference(args)
    args.warmup = max(3, args.warmup)

    import torch
    from differentiable_adaptive_ode_b200 import gradsolve as G
    from differentiable_adaptive_ode_b200 import workloads as W

    ws, rank, local = dist_env()
    if ws > 1:
        import datetime
        import torch.distributed as dist
        torch.cuda.set_device(local)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=torch.device("cuda", local))
    else:
        torch.cuda.set_device(0)
    dev = torch.device("cuda", torch.cuda.current_device())
    stream = torch.cuda.current_stream()

    wl = WORKLOADS[args.workload]
    w = W.by_name(args.workload, N=args.N or None)
    w = W.by_name(args.workload, N=w.N, seed=w.seed + 1000 * rank)   # each rank: its own ensemble
    if wl.get("step") == "sens":
        line = run_sens(args, w, wl, G, torch, dev, stream, ws, rank)
        if ws > 1:
            torch.distributed.destroy_process_group()
        if rank == 0:
            print(json.dumps(line), flush=True)
        return
    N, d, m = w.N, w.d, w.m
    f64 = w.dtype == np.float64
    dt = torch.float64 if f64 else torch.float32
    rsz = 8 if f64 else 4
    sys_ = G.system(w.field, w.method, "f64" if f64 else "f32", w.theta_shared)
    th = torch.as_tensor(w.theta, dtype=dt, device=dev)
    y0 = torch.as_tensor(w.y0, dtype=dt, device=dev)
    y1 = torch.empty((N, d), dtype=dt, device=dev)
    # the caller's loss targets: drawn, or solved on the GPU at nominal / teacher parameters
    if w.target is not None:
        target = torch.as_tensor(w.target, dtype=dt, device=dev)
    elif w.target_kind == "nominal_y0":
        y0n = torch.as_tensor(np.tile(w.notes["nominal_y0"], (N, 1)), dtype=dt, device=dev)
        target = torch.empty((N, d), dtype=dt, device=dev)
        G.gs_solve_forward(sys_, N, th, y0n, w.t0, w.t1, w.rtol, w.atol, target)
    elif w.target_kind == "nominal_solve":
        thn = torch.as_tensor(np.tile(w.nominal_theta, (N, 1)), dtype=dt, device=dev)
        target = torch.empty((N, d), dtype=dt, device=dev)
        G.gs_solve_forward(sys_, N, thn, y0, w.t0, w.t1, w.rtol, w.atol, target)
    else:
        thn = torch.as_tensor(w.nominal_theta, dtype=dt, device=dev)
        target = torch.empty((N, d), dtype=dt, device=dev)
        G.gs_solve_forward(sys_, N, thn, y0, w.t0, w.t1, w.rtol, w.atol, target)
    mask = torch.as_tensor(w.loss_mask if w.loss_mask is not None else np.ones(d), dtype=dt,
                           device=dev)
    scale = 2.0 * w.loss_scale
    lam = torch.empty((N, d), dtype=dt, device=dev)
    gt = torch.empty((m,) if w.theta_shared else (N, m), dtype=dt, device=dev)
    gy = torch.empty((N, d), dtype=dt, device=dev)
    rec = G.Record()

    def loss_cotangent():
        torch.mul(torch.sub(y1, target), mask, out=lam).mul_(scale)

    # a parameter vector shared by the whole ensemble is shared across ranks too: its cotangent is
    # summed over the ranks' ensembles (the one exchange of the path; m values)
    reduce_shared = ws > 1 and w.theta_shared
    if reduce_shared:
        from differentiable_adaptive_ode_b200.ensemble import allreduce_theta_bar

    def step():
        G.gs_solve_record(sys_, N, th, y0, w.t0, w.t1, w.rtol, w.atol, y1, rec=rec)
        loss_cotangent()
        G.gs_replay_grad(rec, th, lam, gt, gy)
        if reduce_shared:
            allreduce_theta_bar(gt)

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()

    def barrier():
        if ws > 1:
            torch.distributed.barrier()
        torch.cuda.synchronize()

    # ---- timed: whole steps
    adj_ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
              for _ in range(args.steps)]
    solve_ms = []
    barrier()
    with ClockSampler(dev.index) as clk:
        start = torch.cuda.Event(enable_timing=True)
        stop = torch.cuda.Event(enable_timing=True)
        start.record(stream)
        for i in range(args.steps):
            G.gs_solve_record(sys_, N, th, y0, w.t0, w.t1, w.rtol, w.atol, y1, rec=rec)
            solve_ms.append(rec.info().solve_ms)     # the record kernel alone (library events)
            loss_cotangent()
            adj_ev[i][0].record(stream)
            G.gs_replay_grad(rec, th, lam, gt, gy)
            adj_ev[i][1].record(stream)
            if reduce_shared:
                allreduce_theta_bar(gt)
        stop.record(stream)
        barrier()
    total_ms = start.elapsed_time(stop)
    if ws > 1:
        t = torch.tensor([total_ms], device=dev)
        torch.distributed.all_reduce(t, op=torch.distributed.ReduceOp.MAX)
        total_ms = float(t.item())
    ms_step = total_ms / args.steps
    value = ws * N * args.steps / (total_ms / 1e3)
    adj_ms = statistics.median(a.elapsed_time(b) for a, b in adj_ev)
    info = rec.info()
    total_steps = int(info.total_steps)

    # ---- breakdown (not part of `value`): forward-only solve, record alone, replay alone
    def timeit(fn, reps=max(3, args.steps // 2)):
        fn()
        torch.cuda.synchronize()
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record(stream)
        for _ in range(reps):
            fn()
        b.record(stream)
        torch.cuda.synchronize()
        return a.elapsed_time(b) / reps

    S = torch.empty(N, dtype=torch.int32, device=dev)
    rj = torch.empty(N, dtype=torch.int32, device=dev)
    stt = torch.empty(N, dtype=torch.int32, device=dev)
    # the forward-only solve of the same ensemble starts its trajectories in the record's
    # longest-first order (scheduling only), as a caller repeating solves would
    fwd_order = rec.order().clone()
    fwd_opts = G.options(start_order=fwd_order)
    fwd_ms = timeit(lambda: G.gs_solve_forward(sys_, N, th, y0, w.t0, w.t1, w.rtol, w.atol, y1, S,
                                               rj, stt, opts=fwd_opts))
    attempts = int(S.sum().item() + rj.sum().item())
    rec_ms = timeit(lambda: G.gs_solve_record(sys_, N, th, y0, w.t0, w.t1, w.rtol, w.atol, y1,
                                              rec=rec))
    loss_cotangent()
    grad_ms = timeit(lambda: G.gs_replay_grad(rec, th, lam, gt, gy))
    breakdown = {"forward_only": fwd_ms, "record": rec_ms, "replay_grad": grad_ms, "step": ms_step}

    # a record made from nothing ([GS] §4.7 reports the one-time record separately): a new record
    # object per repetition -- its allocations, a pool sized by default for 64 steps per
    # trajectory (trajectories that find it full are parked and resumed once it has grown), no
    # longest-first order yet -- then the first gradient.  Wall-clock through completion, the best
    # of five (host-side costs -- allocation, the driver -- vary from one repetition to the next).
    def fresh(with_grad):
        best = None
        for _ in range(5):
            torch.cuda.synchronize()
            t0 = time.perf_counter()
            r = G.Record()
            G.gs_solve_record(sys_, N, th, y0, w.t0, w.t1, w.rtol, w.atol, y1, rec=r)
            if with_grad:
                loss_cotangent()
                G.gs_replay_grad(r, th, lam, gt, gy)
            torch.cuda.synchronize()
            dt_ = (time.perf_counter() - t0) * 1e3
            breakdown["fresh_record_solve_kernels"] = r.info().solve_ms
            r.close()
            best = dt_ if best is None else min(best, dt_)
        return best

    def reused_wall():
        best = None
        for _ in range(5):
            torch.cuda.synchronize()
            t0 = time.perf_counter()
            G.gs_solve_record(sys_, N, th, y0, w.t0, w.t1, w.rtol, w.atol, y1, rec=rec)
            torch.cuda.synchronize()
            dt_ = (time.perf_counter() - t0) * 1e3
            best = dt_ if best is None else min(best, dt_)
        return best

    breakdown["fresh_record_wall"] = fresh(False)
    breakdown["fresh_record_plus_first_gradient_wall"] = fresh(True)
    breakdown["reused_record_wall"] = reused_wall()
    # the same forward-only solve started in index order: what a first solve, which knows no
    # longest-first order yet, pays for scheduling alone
    ident = torch.arange(N, dtype=torch.int32, device=dev)
    breakdown["forward_only_index_order"] = timeit(
        lambda: G.gs_solve_forward(sys_, N, th, y0, w.t0, w.t1, w.rtol, w.atol, y1, S, rj, stt,
                                   opts=G.options(start_order=ident)))
    # outputs at 8 requested times ([GS] §3.4) and the gradient of a loss on them
    tau = [w.t0 + (w.t1 - w.t0) * (j + 1) / 8.0 for j in range(8)]
    yout = torch.empty((N, len(tau), d), dtype=dt, device=dev)
    lam_out = (mask.expand(N, len(tau), d) * 0.125).contiguous()
    breakdown["outputs_8_times"] = timeit(lambda: G.gs_replay_outputs(rec, th, y0, tau, yout))
    breakdown["replay_grad_outputs_8_times"] = timeit(
        lambda: G.gs_replay_grad_outputs(rec, th, tau, lam_out, None, gt, gy))

    # ---- end to end through the public API with host buffers (pinned), copies inside the region.
    # Two stream pipelines with their own buffers and records, steps alternating between them, so
    # that one step's host<->device copies overlap the other's kernels (every step still copies
    # its inputs in and its gradients out).
    h_th = torch.as_tensor(w.theta, dtype=dt).pin_memory()
    h_y0 = torch.as_tensor(w.y0, dtype=dt).pin_memory()
    pipes = []
    for _ in range(2):
        pipes.append(dict(s=torch.cuda.Stream(), th=torch.empty_like(th), y0=torch.empty_like(y0),
                          y1=torch.empty_like(y1), lam=torch.empty_like(lam),
                          gt=torch.empty_like(gt), gy=torch.empty_like(gy), rec=G.Record(),
                          h_gt=torch.empty(tuple(gt.shape), dtype=dt).pin_memory(),
                          h_gy=torch.empty((N, d), dtype=dt).pin_memory()))

    def e2e_step(q):
        with torch.cuda.stream(q["s"]):
            q["th"].copy_(h_th, non_blocking=True)
            q["y0"].copy_(h_y0, non_blocking=True)
            G.gs_solve_record(sys_, N, q["th"], q["y0"], w.t0, w.t1, w.rtol, w.atol, q["y1"],
                              rec=q["rec"])
            torch.mul(torch.sub(q["y1"], target), mask, out=q["lam"]).mul_(scale)
            G.gs_replay_grad(q["rec"], q["th"], q["lam"], q["gt"], q["gy"])
            if reduce_shared:
                allreduce_theta_bar(q["gt"])
            q["h_gt"].copy_(q["gt"], non_blocking=True)
            q["h_gy"].copy_(q["gy"], non_blocking=True)

    for q in pipes:   # untimed: each pipeline's record is sized once
        e2e_step(q)
    e2e_steps = max(4, args.steps // 2)
    barrier()
    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    a.record(stream)
    for q in pipes:
        q["s"].wait_event(a)
    for i in range(e2e_steps):
        e2e_step(pipes[i % 2])
    for q in pipes:
        ev = torch.cuda.Event()
        ev.record(q["s"])
        stream.wait_event(ev)
    b.record(stream)
    barrier()
    e2e_ms = a.elapsed_time(b) / e2e_steps
    h_gt, h_gy = pipes[0]["h_gt"], pipes[0]["h_gy"]
    for q in pipes:
        q["rec"].close()
    if ws > 1:
        t = torch.tensor([e2e_ms], device=dev)
        torch.distributed.all_reduce(t, op=torch.distributed.ReduceOp.MAX)
        e2e_ms = float(t.item())
    h2d = (h_th.numel() + h_y0.numel()) * rsz
    d2h = (h_gt.numel() + h_gy.numel()) * rsz

    clocks = clk.summary()
    lanes = FP64_LANES if f64 else FP32_LANES
    peak_max = pipe_peak_tflops(1965.0, lanes)
    at_clock = pipe_peak_tflops(clocks["sm_mhz"], lanes) if clocks.get("sm_mhz") else None
    pipe = "FP64" if f64 else "FP32"

    def roof(name, per_unit, units, ms, unit_name, traffic, busy=None):
        achieved = per_unit * units / (ms / 1e3) / 1e12 if per_unit else None
        return {"kernel": name, "bound": "alu", "achieved": achieved, "peak": peak_max,
                "pipe_busy_ncu": busy,
                "unit": "TFLOP/s", "frac": achieved / peak_max if achieved else None,
                "traffic": traffic,
                "traffic_source": "ncu dram bytes per accepted step of one capture x steps",
                "peak_source": "derived: 148 SM x %d %s FMA lanes/clk x 2 x 1965 MHz (%s pipe)"
                               % (lanes, pipe, pipe),
                "flops_per_unit": per_unit, "unit_counted": unit_name, "kernel_ms": ms,
                "frac_at_measured_clock": achieved / at_clock if (achieved and at_clock) else None}

    method = {"tsit5": "Tsit5", "vern7": "Vern7", "ros34pw2": "ROS34PW2",
              "rosenbrock23": "Rosenbrock23"}[w.method]
    rec_kernel_ms = statistics.median(solve_ms)
    traffic = TRAFFIC_PER_STEP.get(args.workload, {})
    roof_rec = roof("k_solve<%s, %s, %s, record>" % (w.field, "double" if f64 else "float", method),
                    wl["fwd"], attempts, rec_kernel_ms, "attempted step",
                    (traffic.get("record") or 0) * total_steps or None,
                    PIPE_BUSY_NCU.get(args.workload, {}).get("record"))
    roof_adj = roof("k_adjoint<%s, %s, %s>" % (w.field, "double" if f64 else "float", method),
                    wl["adj"], total_steps, adj_ms, "accepted step",
                    (traffic.get("adjoint") or 0) * total_steps or None,
                    PIPE_BUSY_NCU.get(args.workload, {}).get("adjoint"))
    dominant, other = (roof_rec, roof_adj) if rec_kernel_ms >= adj_ms else (roof_adj, roof_rec)
    line = {
        "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": ws, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": ms_step, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f64" if f64 else "f32",
        "data": "synthetic",
        "config": dict(workload_config(ws, N, args.workload, w), accepted_steps=total_steps,
                       attempts_forward=attempts, record_gb=round(info.pool_bytes / 1e9, 2)),
        "roofline": dominant,
        "roofline_other": other,
        "breakdown_ms": breakdown,
        "forward_traj_per_s": ws * N / (fwd_ms / 1e3),
        "replay_grad_traj_per_s": ws * N / (grad_ms / 1e3),
        "record_traj_per_s": ws * N / (rec_ms / 1e3),
        "forward_pipe_frac": (wl["fwd"] * attempts / (fwd_ms / 1e3) / 1e12 / peak_max
                              if wl["fwd"] else None),
        "e2e": {"value": ws * N / (e2e_ms / 1e3), "unit": UNIT, "h2d_bytes_per_step": h2d,
                "d2h_bytes_per_step": d2h},
        "gpu_launches": args.steps * LAUNCHES_PER_STEP,
        "clocks": clocks,
    }
    if rank == 0 and ws == 1 and not args.no_cpu_baseline and args.workload == "nfw_mn":
        line["cpu_baseline"] = cpu_baseline_sample()
    else:
        line["cpu_baseline"] = None
    rec.close()
    if ws > 1:
        torch.distributed.destroy_process_group()
    if rank == 0:
        print(json.dumps(line), flush=True)


if __name__ == "__main__":
    main()
