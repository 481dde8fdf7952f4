#!/usr/bin/env python
"""Throughput of the gated grouped causal FIR forward (Hyena-MR: B=1, L=8192, D=4096, d_g=64,
l_h=128, l_b=64, bf16) on B200, one process per GPU.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload mr] [--impl reference]

A step is one pass of the whole forward (one kernel launch) over one batch of synthetic
inputs already resident in HBM.  Three input sets rotate from step to step (3 x 256 MiB, more
than the 126 MB L2), so no step reads the previous step's inputs from L2.  The timed region is
bracketed by a barrier and a device synchronisation, timed with CUDA events on the launching
stream, and reduced as the max over ranks.  Under torchrun each rank runs an independent
replica on its own batch (weak scaling, no collective on the data path).

Rank 0 prints one JSON line.  Besides the throughput it reports the roofline of the kernel
(algorithmic bytes / mean launch time vs the measured HBM copy bandwidth, with the median and
minimum of a separate pass that times each launch on its own), SM clocks sampled
through NVML during the timed region, an end-to-end figure through
``hyena_conv_fwd_from_host`` (pinned host buffers, copies inside the timed region) and the
fp64 oracle timed on the host cores as a CPU baseline.  Beside the forward it reports the
backward (``backward``), the forward on the other configurations of the workload table
(``configs``: SE, MR batched, MR with 2^20 tokens, each with its roofline) and two
longer-filter cases (``long_filters``: the Hyena-LI-shaped
workload through the FFT entry point, and l_h = 513 on the tensor-core path) and, as context,
the pages' naive baseline (``comparator``: PyTorch's depthwise F.conv1d with the gating
products, on the same inputs).
``--impl reference`` times only the oracle, one l_b-row chunk of the workload per step.
"""
import argparse
import ctypes
import hashlib
import json
import os
import statistics
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "Hyena-MR fwd tokens/s (D=4096, L=8192, ℓ_h=128); HBM GB/s vs peak"
UNIT = "tokens/s"
FALLBACK_HBM_GBS = 6650.0
KERNEL_SOURCES = ["fir_tc.cuh", "ptx.cuh"]  # device code of the timed kernel


def parse():
    p = argparse.ArgumentParser(description=__doc__.split("\n\n")[0])
    p.add_argument("--gpus", type=int, default=1)
    p.add_argument("--steps", type=int, default=2000)
    p.add_argument("--warmup", type=int, default=20)
    p.add_argument("--workload", default="mr")
    p.add_argument("--algo", default="auto", choices=["auto", "tensor", "window", "direct", "fft"],
                   help="forward algorithm of the timed launches (auto = the library's choice)")
    p.add_argument("--impl", default="ours", choices=["ours", "reference"])
    p.add_argument("--e2e-steps", type=int, default=10)
    p.add_argument("--cpu-seconds", type=float, default=10.0,
                   help="target CPU time of the oracle baseline sample")
    p.add_argument("--no-cpu-baseline", action="store_true")
    p.add_argument("--no-e2e", action="store_true")
    p.add_argument("--bwd-steps", type=int, default=200,
                   help="timed steps of the backward (hyena_conv_bwd); 0 skips it")
    p.add_argument("--comparator-steps", type=int, default=5,
                   help="timed steps of the torch F.conv1d comparator; 0 skips")
    p.add_argument("--long-steps", type=int, default=20,
                   help="timed steps of the long-filter measurements (FFT, l_h = 513); 0 skips")
    p.add_argument("--stat-launches", type=int, default=300,
                   help="launches timed one by one for the median and minimum (>= 100)")
    p.add_argument("--config-steps", type=int, default=20,
                   help="timed steps of the other configurations (SE, MR batched, MR 1M); 0 skips")
    return p.parse_args()


def kernel_source_hash():
    h = hashlib.sha256()
    for name in KERNEL_SOURCES:
        with open(os.path.join(ROOT, "gated_causal_fir_b200", "csrc", name), "rb") as f:
            h.update(f.read())
    return h.hexdigest()[:16]


def measured_peak_hbm():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            return float(json.load(f)["hbm_gbs"]), "measured"
    except (OSError, KeyError, ValueError):
        return FALLBACK_HBM_GBS, "fallback"


def committed_traffic(kernel, workload):
    """DRAM bytes per launch from the committed ncu summary, if it was taken on the current
    kernel source (else None)."""
    path = os.path.join(ROOT, "profiles", "%s_%s_traffic.json" % (kernel, workload))
    try:
        with open(path) as f:
            rec = json.load(f)
    except (OSError, ValueError):
        return None
    if rec.get("kernel_source_hash") != kernel_source_hash():
        return None
    return rec.get("traffic_bytes_per_launch")


class ClockSampler:
    """Polls SM clock, power and clock-event reasons through NVML in a thread."""

    REASONS = {0x1: "gpu_idle", 0x2: "applications_clocks_setting", 0x4: "sw_power_cap",
               0x8: "hw_slowdown", 0x10: "sync_boost", 0x20: "sw_thermal_slowdown",
               0x40: "hw_thermal_slowdown", 0x80: "hw_power_brake_slowdown",
               0x100: "display_clock_setting"}

    def __init__(self, index, period_s=0.005):
        self.samples, self.period, self.ok = [], period_s, False
        self._stop = threading.Event()
        try:
            import pynvml
            pynvml.nvmlInit()
            self.nv = pynvml
            self.h = pynvml.nvmlDeviceGetHandleByIndex(index)
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self.h, pynvml.NVML_CLOCK_SM)
            self.ok = True
        except Exception as e:  # no NVML: report it instead of clocks
            self.err = repr(e)

    def _run(self):
        nv = self.nv
        while not self._stop.is_set():
            try:
                sm = nv.nvmlDeviceGetClockInfo(self.h, nv.NVML_CLOCK_SM)
                rs = nv.nvmlDeviceGetCurrentClocksEventReasons(self.h)
                self.samples.append((time.perf_counter(), sm, rs))
            except Exception:
                pass
            time.sleep(self.period)

    def start(self):
        if self.ok:
            self.t = threading.Thread(target=self._run, daemon=True)
            self.t.start()
        return self

    def stop(self):
        if self.ok:
            self._stop.set()
            self.t.join()

    def summary(self, t0, t1):
        if not self.ok:
            return {"error": "NVML unavailable: " + self.err}
        win = [s for s in self.samples if t0 <= s[0] <= t1] or self.samples
        reasons = set()
        for _, _, rs in win:
            for bit, name in self.REASONS.items():
                if rs & bit and name != "gpu_idle":
                    reasons.add(name)
        return {"sm_mhz": statistics.median(s[1] for s in win) if win else None,
                "sm_max_mhz": self.max_mhz, "reasons": sorted(reasons), "samples": len(win),
                "source": "NVML, %.0f ms period, during the timed region" % (1e3 * self.period)}


def cpu_baseline(wl, q, k, v, h, target_s):
    """Time the fp64 oracle, as it stands, on this host's cores over whole copies of the
    workload (repeated until ~target_s of work); returns (record, oracle output of one pass)."""
    import oracle
    qh, kh, vh, hh = (x.cpu() for x in (q, k, v, h))
    reps, t_total, y_ref = 0, 0.0, None
    while reps < 20 and (reps == 0 or t_total < target_s):
        t = time.perf_counter()
        y_ref = oracle.gated_fir(qh, kh, vh, hh, wl.d_g)
        t_total += time.perf_counter() - t
        reps += 1
    rec = {"value": wl.tokens * reps / t_total, "unit": UNIT, "cores": oracle.max_threads(),
           "kind": "oracle",
           "sample": "whole %s workload x%d (%.1f s of fp64 direct sums, OpenMP)"
                     % (wl.name, reps, t_total)}
    # the same oracle on one thread, over the last rows of the first sequence (full sums)
    n_rows = min(256, wl.L)
    rows = [(0, t) for t in range(wl.L - n_rows, wl.L)]
    t = time.perf_counter()
    oracle.gated_fir_rows(qh, kh, vh, hh, wl.d_g, rows, nthreads=1)
    dt = time.perf_counter() - t
    rec["single_thread"] = {"value": n_rows / dt, "unit": UNIT, "cores": 1,
                            "sample": "rows %d..%d of sequence 0, all %d channels"
                                      % (wl.L - n_rows, wl.L - 1, wl.D)}
    return rec, y_ref


def time_conv1d_comparator(args, wl, sets, stream, y_ours):
    """Context, not the product: the pages' naive baseline, PyTorch's depthwise F.conv1d
    (cuDNN; weight = each channel's filter reversed, left padding l_h - 1) with the two gating
    products around it, in the I/O dtype on the same inputs, timed with CUDA events over
    rotating input sets.  Its transposes to and from the [B, D, L] layout conv1d wants are part
    of the step."""
    import torch
    import torch.nn.functional as F
    h = sets[0][3]
    w = h.repeat_interleave(wl.d_g, dim=0).flip(-1).unsqueeze(1).to(sets[0][0].dtype)

    def step(q, k, v):
        x = (k * v).transpose(1, 2)
        z = F.conv1d(F.pad(x, (wl.l_h - 1, 0)), w, groups=wl.D)
        return q * z.transpose(1, 2)

    with torch.cuda.stream(stream):
        y = step(*sets[0][:3])
        for i in range(2):
            step(*sets[i % len(sets)][:3])
        torch.cuda.synchronize()
        diff = float((y.float() - y_ours.float()).abs().max())
        scale = float(y_ours.float().abs().max())
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        K = args.comparator_steps
        e0.record(stream)
        for i in range(K):
            step(*sets[i % len(sets)][:3])
        e1.record(stream)
        torch.cuda.synchronize()
    ms = e0.elapsed_time(e1) / K
    return {"kind": "torch F.conv1d depthwise (cuDNN) + gating, %s" % wl.dtype,
            "ms_per_step": ms, "value": wl.tokens / (ms / 1e3), "unit": UNIT, "steps": K,
            "max_abs_diff_vs_kernel": diff, "max_abs_kernel_output": scale}


def run_reference(args, wl, rank, world):
    """The oracle arm: one l_b-row chunk of the workload per step, on the host cores."""
    import oracle
    import torch
    from gated_causal_fir_b200.workloads import make_inputs
    if rank != 0:
        return
    q, k, v, h = make_inputs(wl, device="cpu")
    n_chunks = (wl.L + wl.l_b - 1) // wl.l_b

    def step(i):
        b = i % wl.B
        t0 = ((i // wl.B) % n_chunks) * wl.l_b
        t1 = min(wl.L, t0 + wl.l_b)
        s = max(0, t0 - (wl.l_h - 1))
        oracle.gated_fir(q[b, s:t1], k[b, s:t1], v[b, s:t1], h, wl.d_g)
        return t1 - t0

    for i in range(args.warmup):
        step(i)
    t = time.perf_counter()
    rows = sum(step(args.warmup + i) for i in range(args.steps))
    dt = time.perf_counter() - t
    value = rows / dt
    cores = oracle.max_threads()
    sample = "one %d-row chunk (all %d channels, with %d history rows) per step" % (
        wl.l_b, wl.D, wl.l_h - 1)
    print(json.dumps({
        "impl": "reference", "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": 1e3 * dt / args.steps,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic", "config": workload_config(wl, world),
        "cpu_baseline": {"value": value, "unit": UNIT, "cores": cores, "kind": "oracle",
                         "sample": sample},
        "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }), flush=True)
    del torch


def launch_stats(launch, n, stream):
    """Per-launch durations of n back-to-back launches (one CUDA event between consecutive
    launches on the launching stream): mean, median and minimum in microseconds."""
    import torch
    ev = [torch.cuda.Event(enable_timing=True) for _ in range(n + 1)]
    torch.cuda.synchronize()
    ev[0].record(stream)
    for i in range(n):
        launch(i)
        ev[i + 1].record(stream)
    torch.cuda.synchronize()
    us = [1e3 * ev[i].elapsed_time(ev[i + 1]) for i in range(n)]
    return {"launches": n, "mean_us": statistics.fmean(us), "median_us": statistics.median(us),
            "min_us": min(us)}


def time_configs(args, stream, dev, D, g, _native, peak, peak_kind):
    """The forward on the other configurations of the workload table (SE, MR batched, MR with
    2^20 tokens), timed like the headline: CUDA events over K back-to-back launches on the
    launching stream (max over ranks), plus per-launch median and minimum.  Inputs: three
    rotating sets where they fit in a few GiB, one set beyond (then every step's inputs exceed
    the 126 MB L2 on their own).  Algorithmic bytes per launch: q, k, v read and y written, plus
    the filters."""
    import torch
    from gated_causal_fir_b200.workloads import WORKLOADS, make_inputs
    sh = ctypes.c_void_p(stream.cuda_stream)
    out = {}
    for name in ("se", "mr_batched", "mr_1m"):
        wl = WORKLOADS[name]
        nsets = 3 if wl.algorithmic_bytes() * 3 < (8 << 30) else 1
        sets = [make_inputs(wl, device=dev, seed=wl.seed + 101 * s, l_slice=1 << 16)
                for s in range(nsets)]
        ys = [torch.empty_like(x[0]) for x in sets]
        # the inputs are made on torch's current stream and read on `stream` (non-blocking):
        # they must be complete, and their temporaries retired, before the first launch
        torch.cuda.synchronize()
        code = g.HYENA_DTYPE_F32 if wl.dtype == "f32" else g.HYENA_DTYPE_BF16
        algo = g.hyena_select_algo(wl.B, wl.L, wl.D, wl.d_g, wl.l_h, wl.l_b, code)
        cfn = _native.lib().hyena_conv_fwd_f32 if wl.dtype == "f32" else _native.lib().hyena_conv_fwd
        cargs = [(x[0].data_ptr(), x[1].data_ptr(), x[2].data_ptr(), x[3].data_ptr(),
                  y.data_ptr(), wl.B, wl.L, wl.D, wl.d_g, wl.l_h, wl.l_b, sh)
                 for x, y in zip(sets, ys)]

        def launch(i):
            rc = cfn(*cargs[i % nsets])
            if rc != 0:
                raise _native.HyenaError(name, rc)

        for i in range(max(3, args.warmup)):
            launch(i)
        torch.cuda.synchronize()
        K = args.config_steps
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        D.barrier()
        torch.cuda.synchronize()
        e0.record(stream)
        for i in range(K):
            launch(i)
        e1.record(stream)
        torch.cuda.synchronize()
        ms = D.max_over_ranks(e0.elapsed_time(e1), device=dev) / K
        stats = launch_stats(launch, max(100, K) if wl.tokens <= (1 << 16) else K, stream)
        nbytes = wl.algorithmic_bytes()
        achieved = nbytes / (ms / 1e3) / 1e9
        kernel = {g.HYENA_ALGO_TENSOR: "fir_tc_kernel", g.HYENA_ALGO_WINDOW: "fir_window_kernel",
                  g.HYENA_ALGO_DIRECT: "fir_tiled_kernel", g.HYENA_ALGO_FFT: "fir_fftblk_kernel"}[algo]
        out[name] = {"workload": wl.describe(), "ms_per_step": ms, "steps": K,
                     "value": D.env_world()[2] * wl.tokens / (ms / 1e3), "unit": UNIT,
                     "gpu_launches": K, "kernel": kernel, "launch_stats": stats,
                     "l2": "%d rotating input sets" % nsets,
                     "roofline": {"bound": "hbm", "achieved": achieved, "peak": peak,
                                  "unit": "GB/s", "frac": achieved / peak,
                                  "algorithmic_bytes_per_launch": nbytes,
                                  "peak_source": peak_kind}}
        del sets, ys, cargs
        torch.cuda.empty_cache()
    return out


def time_long_filters(args, stream, dev, D, g, _native, peak, peak_kind):
    """Filters longer than the MR workload's, on one GPU, timed like the forward (CUDA events on
    the launching stream over back-to-back calls, two rotating input sets):

    * ``li_fft``: the Hyena-LI-shaped workload (B=1, L=8192, D=4096, d_g=64, l_h=8192) through
      hyena_conv_fwd_fft (four-step FFT, caller workspace);
    * ``mr_lh513``, ``mr_lh514``: the MR shape with l_h = 513 (four history tiles on the
      tensor-core path) and 514 (five, with one band set and two k/v stages) (AUTO);
    * ``mr_lh641``, ``mr_lh642``: the longest filter of the tensor-core path, and one tap
      longer, past the tensor band: AUTO runs the single-pass block FFT (no workspace).

    Algorithmic bytes per call: q, k, v read and y written (4 B L D bf16 elements); the FFT's
    spectra in the workspace are overhead, not counted."""
    import torch
    from gated_causal_fir_b200.workloads import WORKLOADS, custom, make_inputs
    sh = ctypes.c_void_p(stream.cuda_stream)
    out = {}
    for name, wl, fft in (("li_fft", WORKLOADS["li"], True),
                          ("mr_lh513", custom("mr_lh513", 1, 8192, 4096, 64, 513, 64, "bf16",
                                              "mr", seed=6), False),
                          ("mr_lh514", custom("mr_lh514", 1, 8192, 4096, 64, 514, 64, "bf16",
                                              "mr", seed=7), False),
                          ("mr_lh641", custom("mr_lh641", 1, 8192, 4096, 64, 641, 64, "bf16",
                                              "mr", seed=8), False),
                          ("mr_lh642", custom("mr_lh642", 1, 8192, 4096, 64, 642, 64, "bf16",
                                              "mr", seed=9), False)):
        sets = [make_inputs(wl, device=dev, seed=wl.seed + 101 * s) for s in range(2)]
        ys = [torch.empty_like(x[0]) for x in sets]
        torch.cuda.synchronize()  # inputs complete before `stream` reads them
        if fft:
            need = g.hyena_conv_fwd_fft_workspace_bytes(wl.B, wl.L, wl.D, wl.d_g, wl.l_h)
            ws = torch.empty(need, dtype=torch.uint8, device=dev)
            torch.cuda.synchronize()
            cfn = _native.lib().hyena_conv_fwd_fft
            cargs = [(x[0].data_ptr(), x[1].data_ptr(), x[2].data_ptr(), x[3].data_ptr(),
                      y.data_ptr(), wl.B, wl.L, wl.D, wl.d_g, wl.l_h, wl.l_b, 0, ws.data_ptr(),
                      need, sh) for x, y in zip(sets, ys)]
            kernels = ["fft_pass1_kernel (filters)", "fft_pass2_kernel (filters)",
                       "fft_pass1_kernel", "fft_pass2_kernel", "fft_pass3_kernel"]
        else:
            cfn = _native.lib().hyena_conv_fwd
            cargs = [(x[0].data_ptr(), x[1].data_ptr(), x[2].data_ptr(), x[3].data_ptr(),
                      y.data_ptr(), wl.B, wl.L, wl.D, wl.d_g, wl.l_h, wl.l_b, sh)
                     for x, y in zip(sets, ys)]
            algo = g.hyena_select_algo(wl.B, wl.L, wl.D, wl.d_g, wl.l_h, wl.l_b)
            kernels = [{g.HYENA_ALGO_TENSOR: "fir_tc_kernel", g.HYENA_ALGO_FFT: "fir_fftblk_kernel",
                        g.HYENA_ALGO_DIRECT: "fir_tiled_kernel"}[algo]]
        for i in range(max(3, args.warmup)):
            if cfn(*cargs[i % 2]) != 0:
                raise _native.HyenaError(name, cfn(*cargs[i % 2]))
        torch.cuda.synchronize()
        K = args.long_steps
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        D.barrier()
        torch.cuda.synchronize()
        e0.record(stream)
        for i in range(K):
            cfn(*cargs[i % 2])
        e1.record(stream)
        torch.cuda.synchronize()
        ms = D.max_over_ranks(e0.elapsed_time(e1), device=dev) / K
        nbytes = 4 * wl.B * wl.L * wl.D * 2
        achieved = nbytes / (ms / 1e3) / 1e9
        out[name] = {"workload": wl.describe(), "ms_per_step": ms, "steps": K,
                     "value": D.env_world()[2] * wl.tokens / (ms / 1e3), "unit": UNIT,
                     "gpu_launches": len(kernels) * K, "kernels": kernels,
                     "roofline": {"bound": "hbm", "achieved": achieved, "peak": peak,
                                  "unit": "GB/s", "frac": achieved / peak,
                                  "algorithmic_bytes_per_step": nbytes,
                                  "peak_source": peak_kind}}
        del sets, ys
    return out


def time_backward(args, wl, sets, stream, dev, D, g, _native, peak, peak_kind):
    """The backward (hyena_conv_bwd: dq, dk, dv, dh) over the same rotating input sets, timed
    like the forward: CUDA events on the launching stream, max over ranks.

    Algorithmic bytes per step: read q, k, v, dy, write dq, dk, dv (7 tensors of B L D
    elements), plus h read and dh written (G l_h fp32 each); the workspace of partials is
    overhead, not counted."""
    import torch
    from gated_causal_fir_b200.workloads import make_grad
    code = g.HYENA_DTYPE_F32 if wl.dtype == "f32" else g.HYENA_DTYPE_BF16
    sh = ctypes.c_void_p(stream.cuda_stream)
    ws_bytes = g.hyena_conv_bwd_workspace_bytes(wl.B, wl.L, wl.D, wl.d_g, wl.l_h)
    ws = torch.empty(max(ws_bytes, 256), dtype=torch.uint8, device=dev)
    bufs = []
    for n, (q, k, v, h, _) in enumerate(sets):
        dy = make_grad(wl, device=dev, seed=wl.seed + 977 * n)
        dq, dk, dv, dh = (torch.empty_like(q), torch.empty_like(q), torch.empty_like(q),
                          torch.empty_like(h))
        torch.cuda.synchronize()  # dy complete before `stream` reads it
        g.hyena_conv_bwd(q, k, v, h, dy, wl.d_g, wl.l_b, workspace=ws,
                         grads=(dq, dk, dv, dh), stream=stream)  # binding checks, once
        bufs.append((q, k, v, h, dy, dq, dk, dv, dh))
    cfn = _native.lib().hyena_conv_bwd
    algo = g.hyena_select_bwd_algo(wl.B, wl.L, wl.D, wl.d_g, wl.l_h, wl.l_b, code)
    kernels = {
        g.HYENA_ALGO_TENSOR: ["fir_tc_kernel (dq)", "fir_tc_bwd_kernel",
                              "fir_bwd_tc_reduce_kernel"],
        g.HYENA_ALGO_WINDOW: ["forward kernel (dq)", "fir_bwd_window_kernel",
                              "fir_bwd_dh_reduce_kernel"],
    }.get(algo, ["forward kernel (dq)", "fir_tiled_kernel (dk, dv)", "fir_bwd_dh_partial_kernel",
                 "fir_bwd_dh_reduce_kernel"])
    cargs = [tuple(t.data_ptr() for t in b) + (wl.B, wl.L, wl.D, wl.d_g, wl.l_h, wl.l_b, code,
                                                ws.data_ptr(), ws.numel(), sh) for b in bufs]

    def launch(i):
        rc = cfn(*cargs[i % 3])
        if rc != 0:
            raise _native.HyenaError("hyena_conv_bwd", rc)

    for i in range(max(3, args.warmup)):
        launch(i)
    torch.cuda.synchronize()
    K = args.bwd_steps
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    D.barrier()
    torch.cuda.synchronize()
    e0.record(stream)
    for i in range(K):
        launch(i)
    e1.record(stream)
    torch.cuda.synchronize()
    ms = D.max_over_ranks(e0.elapsed_time(e1), device=dev) / K
    world = D.env_world()[2]
    elem = 4 if wl.dtype == "f32" else 2
    nbytes = 7 * wl.B * wl.L * wl.D * elem + 2 * wl.G * wl.l_h * 4
    achieved = nbytes / (ms / 1e3) / 1e9
    return {"metric": "%s bwd tokens/s (dq, dk, dv, dh)" % wl.describe(),
            "value": world * wl.tokens / (ms / 1e3), "unit": UNIT, "ms_per_step": ms,
            "steps": K, "gpu_launches": len(kernels) * K, "kernels": kernels,
            "algo": g.ALGO_NAMES[algo],
            "roofline": {"bound": "hbm", "achieved": achieved, "peak": peak, "unit": "GB/s",
                         "frac": achieved / peak, "algorithmic_bytes_per_step": nbytes,
                         "peak_source": peak_kind,
                         "note": "whole backward (all its kernels) per step"}}


def workload_config(wl, world):
    """The workload a line measures (the same keys on both arms of the bench)."""
    return {"workload": wl.describe(), "B": wl.B, "L": wl.L, "D": wl.D, "d_g": wl.d_g,
            "l_h": wl.l_h, "l_b": wl.l_b, "io_dtype": wl.dtype, "filters": wl.filt,
            "l2": "3 rotating input sets (%.0f MiB) > 126 MB L2"
                  % (3 * wl.algorithmic_bytes() / 2 ** 20),
            "parallelism": "replicas x%d" % world}


def main():
    args = parse()
    from gated_causal_fir_b200 import dist as D
    from gated_causal_fir_b200.workloads import WORKLOADS, make_inputs

    wl = WORKLOADS[args.workload]
    if args.impl == "reference":
        rank, _, world = D.env_world()
        run_reference(args, wl, rank, world)
        return

    import torch
    rank, local_rank, world = D.init("nccl")
    torch.cuda.set_device(local_rank)
    dev = torch.device("cuda", local_rank)

    import gated_causal_fir_b200 as g
    from gated_causal_fir_b200 import _native
    _native.lib()  # fail loudly here if the library is missing

    # Inputs: three independent sets per rank, resident before the timed region.
    sets = []
    for s in range(3):
        q, k, v, h = make_inputs(wl, device=dev, seed=D.rank_seed(wl.seed + 101 * s, rank),
                                 l_slice=1 << 16)
        sets.append((q, k, v, h, torch.empty_like(q)))
    # The inputs are made on torch's current stream and read on `stream` (a non-blocking
    # stream): they must be complete, and their temporaries retired, before the first launch.
    torch.cuda.synchronize()
    dcode = g.HYENA_DTYPE_F32 if wl.dtype == "f32" else g.HYENA_DTYPE_BF16
    algo = g.hyena_select_algo(wl.B, wl.L, wl.D, wl.d_g, wl.l_h, wl.l_b, dcode)
    forced = {"auto": None, "tensor": g.HYENA_ALGO_TENSOR, "window": g.HYENA_ALGO_WINDOW,
              "direct": g.HYENA_ALGO_DIRECT, "fft": g.HYENA_ALGO_FFT}[args.algo]
    fwd = g.hyena_conv_fwd_f32 if wl.dtype == "f32" else g.hyena_conv_fwd
    stream = torch.cuda.Stream(device=dev)

    # The timed loop calls the C ABI entry point directly with the argument tuples prepared
    # here: the per-call Python of the torch binding (shape checks, ctypes marshalling) costs
    # about as much host time as one kernel, and a host-bound loop would time the host.
    for x in sets:  # same checks the binding makes, once per input set
        fwd(*x[:4], wl.d_g, wl.l_b, y=x[4], stream=stream)
    cfn = _native.lib().hyena_conv_fwd_f32 if wl.dtype == "f32" else _native.lib().hyena_conv_fwd
    sh = ctypes.c_void_p(stream.cuda_stream)
    cargs = [(q.data_ptr(), k.data_ptr(), v.data_ptr(), h.data_ptr(), y.data_ptr(), wl.B, wl.L,
              wl.D, wl.d_g, wl.l_h, wl.l_b, sh) for q, k, v, h, y in sets]
    if forced is not None:  # the same launches through hyena_conv_fwd_ex with the algorithm
        for x in sets:
            g.hyena_conv_fwd_ex(*x[:4], wl.d_g, wl.l_b, algo=forced, y=x[4], stream=stream)
        cfn = _native.lib().hyena_conv_fwd_ex
        cargs = [c[:11] + (dcode, forced, sh) for c in cargs]
        algo = forced

    def launch(i):
        rc = cfn(*cargs[i % 3])
        if rc != 0:
            raise _native.HyenaError("hyena_conv_fwd", rc)

    torch.cuda.synchronize()
    for i in range(args.warmup):
        launch(i)
    torch.cuda.synchronize()
    assert g.hyena_device_status(clear=True) == 0, "device status raised during warm-up"

    K = args.steps
    start, stop = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    clocks = ClockSampler(local_rank).start()
    D.barrier()
    torch.cuda.synchronize()
    t_wall0 = time.perf_counter()
    start.record(stream)
    for i in range(K):
        launch(i)
    stop.record(stream)
    torch.cuda.synchronize()
    t_wall1 = time.perf_counter()
    D.barrier()
    clocks.stop()
    elapsed_ms = start.elapsed_time(stop)
    status = g.hyena_device_status(clear=True)
    max_ms = D.max_over_ranks(elapsed_ms, device=dev)
    # The timed region launches this kernel and nothing else, back to back on one stream: its
    # mean launch duration is the region's event time over K.
    mean_launch_ms = max_ms / K

    # Per-launch median and minimum (outside the timed region, the same launches one by one).
    stats = launch_stats(launch, max(100, args.stat_launches, K), stream)
    assert g.hyena_device_status(clear=True) == 0, "device status raised during the launches"

    # End to end through the host-buffer entry point, pinned buffers, copies timed.
    e2e = None
    if not args.no_e2e and args.e2e_steps > 0:
        qh, kh, vh, hh = (x.cpu().pin_memory() for x in sets[0][:4])
        yh = torch.empty_like(qh).pin_memory()
        g.hyena_conv_fwd_from_host(qh, kh, vh, hh, wl.d_g, wl.l_b, out=yh, device=dev,
                                   stream=stream, chunk=2048)
        torch.cuda.synchronize()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        D.barrier()
        torch.cuda.synchronize()
        e0.record(stream)
        for _ in range(args.e2e_steps):
            g.hyena_conv_fwd_from_host(qh, kh, vh, hh, wl.d_g, wl.l_b, out=yh, device=dev,
                                       stream=stream, chunk=2048)
        e1.record(stream)
        torch.cuda.synchronize()
        e2e_ms = D.max_over_ranks(e0.elapsed_time(e1), device=dev)
        # bytes the call copies: h once, every row of q, k, v once (a chunk's history rows
        # are copied on the device from the previous chunk), every row of y once
        e2e = {"value": world * wl.tokens * args.e2e_steps / (e2e_ms / 1e3), "unit": UNIT,
               "h2d_bytes_per_step": sum(x.numel() * x.element_size() for x in (qh, kh, vh, hh)),
               "d2h_bytes_per_step": yh.numel() * yh.element_size(),
               "steps": args.e2e_steps,
               "api": "hyena_conv_fwd_from_host (C ABI; 2048-row chunks, three streams)"}

    bwd = None
    if args.bwd_steps > 0:
        peak, peak_kind = measured_peak_hbm()
        bwd = time_backward(args, wl, sets, stream, dev, D, g, _native, peak, peak_kind)

    comparator = None
    if args.comparator_steps > 0 and rank == 0 and world == 1 and wl.B * wl.L * wl.D <= 1 << 26:
        q, k, v, h, y = sets[0]
        fwd(q, k, v, h, wl.d_g, wl.l_b, y=y, stream=stream)
        comparator = time_conv1d_comparator(args, wl, sets, stream, y)

    configs = None
    if args.config_steps > 0 and wl.name == "mr":
        peak, peak_kind = measured_peak_hbm()
        configs = time_configs(args, stream, dev, D, g, _native, peak, peak_kind)

    long_filters = None
    if args.long_steps > 0 and wl.name == "mr":
        peak, peak_kind = measured_peak_hbm()
        long_filters = time_long_filters(args, stream, dev, D, g, _native, peak, peak_kind)

    cpu, parity = None, None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        cpu, y_ref = cpu_baseline(wl, *sets[0][:4], target_s=args.cpu_seconds)
        q, k, v, h, y = sets[0]
        fwd(q, k, v, h, wl.d_g, wl.l_b, y=y, stream=stream)
        torch.cuda.synchronize()
        import numpy as np
        err = np.abs(y.double().cpu().numpy() - y_ref)
        parity = {"max_err_over_bound": float((err / (1e-2 + 1e-2 * np.abs(y_ref))).max()),
                  "bound": "|y - y_oracle| <= 1e-2 + 1e-2 |y_oracle|", "checked": "all outputs"}

    D.barrier()
    if rank == 0:
        peak, peak_kind = measured_peak_hbm()
        bytes_per_launch = wl.algorithmic_bytes()
        achieved = bytes_per_launch / (mean_launch_ms / 1e3) / 1e9
        kernel = {g.HYENA_ALGO_TENSOR: "fir_tc_kernel", g.HYENA_ALGO_WINDOW: "fir_window_kernel",
                  g.HYENA_ALGO_DIRECT: "fir_tiled_kernel", g.HYENA_ALGO_FFT: "fir_fftblk_kernel"}[algo]
        traffic = committed_traffic(kernel, wl.name)
        # the step in SM clock cycles (time x median sampled SM clock): comparable across boxes
        # whose clocks differ
        clock_summary = clocks.summary(t_wall0, t_wall1)
        try:
            clock_summary["sm_cycles_per_step"] = (max_ms / K) * 1e3 * clock_summary["sm_mhz"]
        except (KeyError, TypeError):
            pass
        line = {
            "metric": METRIC if wl.name == "mr" else
            "gated causal FIR fwd tokens/s (%s); HBM GB/s vs peak" % wl.describe(),
            "value": world * wl.tokens * K / (max_ms / 1e3), "unit": UNIT,
            "n_gpus": world, "steps": K, "warmup": args.warmup, "ms_per_step": max_ms / K,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
            "dtype": wl.dtype, "data": "synthetic", "config": workload_config(wl, world),
            "mma": "f16 x f16 -> f32 (tensor path)" if algo == g.HYENA_ALGO_TENSOR
            else "fp32 FFMA",
            "roofline": {"bound": "hbm", "achieved": achieved, "peak": peak, "unit": "GB/s",
                         "frac": achieved / peak, "traffic": traffic,
                         "peak_source": "%s (MEASURED_PEAKS hbm_gbs)" % peak_kind
                         if peak_kind == "measured" else "fallback 6.65 TB/s",
                         "algorithmic_bytes_per_launch": bytes_per_launch,
                         "mean_launch_us": 1e3 * mean_launch_ms, "kernel": kernel,
                         "median_launch_us": stats["median_us"], "min_launch_us": stats["min_us"],
                         "launch_stats": stats},
            "cpu_baseline": cpu, "e2e": e2e, "gpu_launches": K,
            "clocks": clock_summary,
            "backward": bwd, "configs": configs, "long_filters": long_filters,
            "comparator": comparator,
            "kernel_algo": g.ALGO_NAMES[algo], "device_status": status, "parity": parity,
            "wall_s_timed_region": t_wall1 - t_wall0,
        }
        print(json.dumps(line), flush=True)
    D.finalize()


if __name__ == "__main__":
    main()
