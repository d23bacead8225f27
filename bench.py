#!/usr/bin/env python3
"""Benchmark of the quantized-GEMM hot path on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

One step is one pass of the whole hot path over one batch of decode tokens
(M = 16 rows of a 4096-wide activation, LLaMA-7B linear shapes):
    quantize_rowwise_int8  X fp16 [16,4096]           -> Xq int8, x_scale
    gemm_w8a8              Xq @ Wq[4096x4096] + bias   -> fp16 [16,4096]
    gemm_w8a16             X  @ Wq[4096x11008]         -> fp16 [16,11008]
    gemm_w4a16             X  @ W4[4096x11008] (g=64)  -> fp16 [16,11008]
(the offline weight quantization is done once, before timing).  The metric is
the step's algorithmic HBM traffic divided by its time (GB/s): decode is
memory-bound, so this is the fraction of the B200 HBM roofline the path
reaches.  The prefill W8A8 GEMM (M=8192, N=11008, K=4096, bf16 out) is timed
as well and reported in TOPS under "kernels"; the other shapes of the
workload table (M = 1/8/256/2048, N = 4096, the quantizer at M = 2048/8192)
are timed alone under "shapes".

Inputs are seeded synthetic draws.  Four rotating weight sets (about 350 MB,
more than twice the 126 MB L2) are cycled so that no step finds its weights in
L2.  Steps are captured in CUDA graphs (launch-bound µs kernels) holding only
the kernel launches; every graph is replayed once before timing.  Within a
step, W4A16 -> W8A16 run on a second stream beside quantize -> W8A8 (they
share only X), joined before the next step (--one-stream: all four in order
on one stream).  CUDA events
on the launch stream bracket the timed steps: five timed regions of exactly
--steps steps each, the median reported (all five in the JSON line).
Each kernel is then timed alone (a graph of 64 back-to-back launches over
enough weight copies that they never fit in L2, bracketed by events) for the
per-kernel roofline figures.
N > 1 runs one independent replica per GPU (weak scaling, no data-path
collective); the time is the maximum over ranks.

--impl reference times the CPU oracle (plain C, fp64/int64) on the host cores
for the same workload and metric, on a bounded row sample of each step.
"""
from __future__ import annotations

import argparse
import datetime
import hashlib
import json
import math
import os
import subprocess
import sys
import tempfile
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "W8A8 INT8 TOPS and W8A16/W4A16 decode HBM GB/s, % of B200 roofline"
M_DEC, K_DIM, N_SQ, N_FF = 16, 4096, 4096, 11008
GROUP = 64
WORKLOAD = "decode linear pass M=16: quantize X[16,4096] + W8A8 4096x4096 + W8A16 4096x11008 + W4A16 4096x11008 (g64)"
PREFILL = (8192, 11008, 4096)
WEIGHT_SETS = 4
REPEATS = 5  # timed windows per measurement; the median is reported
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}


def step_bytes(M=M_DEC, K=K_DIM, n_sq=N_SQ, n_ff=N_FF, g=GROUP):
    """Algorithmic HBM bytes of one step, per kernel (each operand read once, each output written once)."""
    return {
        "quantize_rowwise_int8": 2 * M * K + M * K + 4 * M,
        "gemm_w8a8": n_sq * K + M * K + 4 * M + 4 * n_sq + 4 * n_sq + 2 * M * n_sq,
        "gemm_w8a16": n_ff * K + 2 * M * K + 4 * n_ff + 2 * M * n_ff,
        "gemm_w4a16": n_ff * K // 2 + 2 * 2 * (K // g) * n_ff + 2 * M * K + 2 * M * n_ff,
    }


def max_over_ranks(ms: float, world: int, device) -> float:
    """A rank's elapsed milliseconds -> the maximum over all ranks (every rank
    calls this at the same point; one all_reduce MAX on the process group)."""
    if world <= 1:
        return ms
    import torch
    t = torch.tensor([ms], device=device, dtype=torch.float64)
    torch.distributed.all_reduce(t, op=torch.distributed.ReduceOp.MAX)
    return float(t.item())


def job_throughput(world: int, bytes_per_step: float, steps: int, elapsed_ms: float) -> float:
    """Whole-job GB/s: each of `world` replicas moves bytes_per_step per step;
    the job's time is the slowest rank's."""
    return world * bytes_per_step * steps / (elapsed_ms * 1e-3) / 1e9


def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            d = json.load(f)
        return {"hbm_gbs": float(d["hbm_gbs"]), "bf16_tflops": float(d["bf16_tflops"]),
                "bf16_tflops_sustained": float(d.get("bf16_tflops_sustained", d["bf16_tflops"])),
                "source": "measured"}
    return dict(FALLBACK_PEAKS, source="fallback")


def kernel_traffic(kernel: str):
    """ncu DRAM bytes per launch for `kernel` if the capture matches the current source, else None."""
    path = os.path.join(ROOT, "profiles", "ncu_traffic.json")
    if not os.path.exists(path):
        return None
    with open(path) as f:
        d = json.load(f)
    e = d.get(kernel)
    if not e:
        return None
    return e["dram_bytes_per_launch"] if sources_digest(e["sources"]) == e["sources_sha256_16"] else None


def sources_digest(paths):
    """sha256 (16 hex) over the given source files, in order; None if one is missing."""
    h = hashlib.sha256()
    for rel in paths:
        p = os.path.join(ROOT, rel)
        if not os.path.exists(p):
            return None
        h.update(open(p, "rb").read())
    return h.hexdigest()[:16]


# ---------------------------------------------------------------------------
# host<->device copies of the end-to-end loop
# ---------------------------------------------------------------------------
class CudaRuntime:
    """The CUDA runtime library torch loaded, called through ctypes for the e2e
    loop's host<->device copies and its cross-stream ordering: a raw
    cudaMemcpyAsync / cudaEventRecord / cudaStreamWaitEvent costs well under a
    microsecond of host time, where torch's copy_() and stream contexts cost
    several each.  Handles are plain integers (torch's `cuda_stream`, events
    created here)."""
    H2D, D2H = 1, 2  # cudaMemcpyKind
    DISABLE_TIMING = 2  # cudaEventDisableTiming

    def __init__(self):
        import ctypes
        self._ct = ctypes
        lib = ctypes.CDLL(self._loaded_path())
        vp, i = ctypes.c_void_p, ctypes.c_int
        sig = {"cudaMemcpyAsync": [vp, vp, ctypes.c_size_t, i, vp], "cudaEventRecord": [vp, vp],
               "cudaStreamWaitEvent": [vp, vp, ctypes.c_uint],
               "cudaEventCreateWithFlags": [ctypes.POINTER(vp), ctypes.c_uint], "cudaEventDestroy": [vp],
               "cudaGetErrorString": [i]}
        for name, args in sig.items():
            getattr(lib, name).argtypes = args
            getattr(lib, name).restype = ctypes.c_char_p if name == "cudaGetErrorString" else i
        self.lib = lib
        self.memcpy = lib.cudaMemcpyAsync
        self.record = lib.cudaEventRecord
        self.wait = lib.cudaStreamWaitEvent

    @staticmethod
    def _loaded_path() -> str:
        """The libcudart already mapped into this process (torch's), else the soname."""
        try:
            with open("/proc/self/maps") as f:
                for line in f:
                    path = line.split()[-1]
                    if "/libcudart.so" in path:
                        return path
        except OSError:
            pass
        return "libcudart.so.12"

    def check(self, rc: int, what: str) -> None:
        if rc:
            raise RuntimeError(f"{what}: {self.lib.cudaGetErrorString(rc).decode()} ({rc})")

    def event(self) -> int:
        e = self._ct.c_void_p()
        self.check(self.lib.cudaEventCreateWithFlags(self._ct.byref(e), self.DISABLE_TIMING), "cudaEventCreate")
        return e.value

    def destroy(self, events) -> None:
        for e in events:
            self.check(self.lib.cudaEventDestroy(e), "cudaEventDestroy")


# ---------------------------------------------------------------------------
# clocks during the timed region
# ---------------------------------------------------------------------------
class ClockSampler:
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu: str):
        self.gpu = gpu  # nvidia-smi -i accepts an index or a UUID
        self.proc = None
        self.tmp = None

    def start(self):
        try:
            self.tmp = tempfile.NamedTemporaryFile("w+", suffix=".csv", delete=False)
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                 "-i", str(self.gpu), "-lms", "50"], stdout=self.tmp, stderr=subprocess.DEVNULL)
        except (OSError, FileNotFoundError):
            self.proc = None

    def stop(self):
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        self.tmp.flush()
        rows = []
        with open(self.tmp.name) as f:
            for line in f:
                p = [x.strip() for x in line.split(",")]
                if len(p) >= 9 and p[1].replace(".", "").isdigit():
                    rows.append(p)
        os.unlink(self.tmp.name)
        if not rows:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["no samples"], "samples": 0}
        sm = [float(r[1]) for r in rows]
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[i] for r in rows for i in range(4) if r[5 + i].lower() == "active"})
        return {"sm_mhz": float(np.median(sm)), "sm_max_mhz": float(rows[0][2]), "reasons": reasons,
                "samples": len(rows), "power_w_max": max(float(r[3]) for r in rows if r[3] not in ("", "[N/A]"))}


# ---------------------------------------------------------------------------
# our arm
# ---------------------------------------------------------------------------
def run_ours(args, rank, world, local_rank):
    import torch
    import int4_quantized_gemm_b200 as qg
    import workloads as W

    torch.cuda.set_device(local_rank)
    dev = torch.device("cuda", local_rank)
    M, K = M_DEC, K_DIM
    seed0 = 1000 * (rank + 1)

    # ---- weights (offline step a2, done by the library's own quantizers, untimed) ----
    sets = []
    for r in range(WEIGHT_SETS):
        s = seed0 + 10 * r
        w_sq = W.torch_weights(N_SQ, K, s + 1, dev)
        wq, ws = qg.quantize_rowwise_int8(w_sq)
        b = W.torch_bias(N_SQ, s + 1, dev)
        w_ff = W.torch_weights(N_FF, K, s + 3, dev)
        wq8, ws8 = qg.quantize_rowwise_int8(w_ff)
        w4 = W.torch_weights(N_FF, K, s + 4, dev, per_column_factor=False)
        qw, sc, ze = qg.quantize_block_asym4(w4)
        del w_sq, w_ff, w4
        x = W.torch_activations(M, K, s + 5, dev, outliers=True)
        sets.append(dict(x=x, wq=wq.contiguous(), ws=ws, b=b, wq8=wq8.contiguous(), ws8=ws8,
                         qw=qw, sc=sc, ze=ze,
                         xq=torch.empty((M, K), dtype=torch.int8, device=dev),
                         xs=torch.empty(M, dtype=torch.float32, device=dev),
                         y1=torch.empty((M, N_SQ), dtype=torch.float16, device=dev),
                         y2=torch.empty((M, N_FF), dtype=torch.float16, device=dev),
                         y3=torch.empty((M, N_FF), dtype=torch.float16, device=dev)))
    torch.cuda.synchronize()

    # The weights are quantized once, above, and synchronized: no kernel that
    # runs from here on writes them, which is the contract of the static-weights
    # flag (the decode kernels then stream weights across kernel boundaries).
    sw = not args.no_static_weights

    # One step: quantize -> W8A8 on the step's stream and, unless --one-stream,
    # W4A16 -> W8A16 on a second stream forked from it and joined back before
    # the step ends (the two chains share only X, so their ramps and tails
    # overlap; measured on B200 30.4 against 32.1 us per step on one stream).
    side = torch.cuda.Stream(device=dev)
    two = not args.one_stream

    def step(d):
        cur = torch.cuda.current_stream()
        if two:
            side.wait_stream(cur)
            with torch.cuda.stream(side):
                qg.gemm_w4a16(d["x"], d["qw"], d["sc"], d["ze"], out=d["y3"], static_weights=sw)
                qg.gemm_w8a16(d["x"], d["wq8"], d["ws8"], out=d["y2"], static_weights=sw)
        qg.quantize_rowwise_int8(d["x"], out=d["xq"], scale_out=d["xs"])
        qg.gemm_w8a8(d["xq"], d["wq"], d["xs"], d["ws"], d["b"], out_dtype=torch.float16, out=d["y1"],
                     static_weights=sw)
        if two:
            cur.wait_stream(side)
        else:
            qg.gemm_w8a16(d["x"], d["wq8"], d["ws8"], out=d["y2"], static_weights=sw)
            qg.gemm_w4a16(d["x"], d["qw"], d["sc"], d["ze"], out=d["y3"], static_weights=sw)

    # eager warm-up (module load, tensor-map paths)
    for d in sets:
        step(d)
    torch.cuda.synchronize()
    qg.check_device_errors()

    # ---- CUDA graphs of the steps: a chunk of C steps, the remainder, the warm-up ----
    K_steps, W_steps = args.steps, args.warmup
    C = min(64, K_steps)
    stream = torch.cuda.Stream(device=dev)
    stream.wait_stream(torch.cuda.current_stream())

    def capture(nsteps):
        g = torch.cuda.CUDAGraph()
        with torch.cuda.stream(stream):
            with torch.cuda.graph(g, stream=stream):
                for i in range(nsteps):
                    step(sets[i % WEIGHT_SETS])
        return g

    g_chunk = capture(C)
    rem = K_steps % C
    g_rem = capture(rem) if rem else None
    g_warm = capture(W_steps)
    torch.cuda.synchronize()

    visible = [v for v in os.environ.get("CUDA_VISIBLE_DEVICES", "").split(",") if v.strip()]
    sampler = ClockSampler(visible[local_rank] if local_rank < len(visible) else str(local_rank))
    # warm-up: the warm-up steps, then one replay of each graph the timed region
    # replays (a graph's first launch also uploads it to the device)
    with torch.cuda.stream(stream):
        g_warm.replay()
        g_chunk.replay()
        if g_rem is not None:
            g_rem.replay()
    stream.synchronize()
    # REPEATS timed regions of exactly K steps each, every one bracketed by a
    # barrier and a device synchronization; the reported time is the median
    # over the repeats of the slowest rank's elapsed time
    rep_ms = []
    sampler.start()
    time.sleep(0.05)
    for _ in range(REPEATS):
        if world > 1:
            torch.distributed.barrier()
        torch.cuda.synchronize()
        t0 = torch.cuda.Event(enable_timing=True)
        t1 = torch.cuda.Event(enable_timing=True)
        with torch.cuda.stream(stream):
            t0.record(stream)
            for _ in range(K_steps // C):
                g_chunk.replay()
            if g_rem is not None:
                g_rem.replay()
            t1.record(stream)
        stream.synchronize()
        if world > 1:
            torch.distributed.barrier()
        torch.cuda.synchronize()
        rep_ms.append(max_over_ranks(t0.elapsed_time(t1), world, dev))
    clocks = sampler.stop()
    elapsed_ms = float(np.median(rep_ms))
    qg.check_device_errors()

    # per-kernel durations: each kernel alone, C launches back to back over
    # rotating operand copies in one graph, bracketed by CUDA events on the
    # launch stream.  The W8A8 weights of the four step sets (67 MB) would fit
    # in L2, so extra copies are made until each kernel's working set exceeds it.
    names = ["quantize_rowwise_int8", "gemm_w8a8", "gemm_w8a16", "gemm_w4a16"]
    extra_w8a8 = []
    for r in range(max(0, int(np.ceil(300e6 / (N_SQ * K))) - WEIGHT_SETS)):
        wq_e, ws_e = qg.quantize_rowwise_int8(W.torch_weights(N_SQ, K, seed0 + 700 + r, dev))
        extra_w8a8.append((wq_e.contiguous(), ws_e))
    w8a8_sets = [(d["wq"], d["ws"]) for d in sets] + extra_w8a8
    extra_w4 = []  # the W4A16 weights of the four sets (103 MB) fit in L2 as well
    for r in range(max(0, int(np.ceil(300e6 / (N_FF * K // 2))) - WEIGHT_SETS)):
        extra_w4.append(qg.quantize_block_asym4(W.torch_weights(N_FF, K, seed0 + 800 + r, dev,
                                                                per_column_factor=False)))
    w4_sets = [(d["qw"], d["sc"], d["ze"]) for d in sets] + extra_w4
    torch.cuda.synchronize()  # the extra weight copies are complete before any flagged call
    calls = {
        "quantize_rowwise_int8": lambda d: qg.quantize_rowwise_int8(d["x"], out=d["xq"], scale_out=d["xs"]),
        "gemm_w8a8": lambda d, i=0: qg.gemm_w8a8(d["xq"], w8a8_sets[i % len(w8a8_sets)][0], d["xs"],
                                                  w8a8_sets[i % len(w8a8_sets)][1], d["b"],
                                                  out_dtype=torch.float16, out=d["y1"], static_weights=sw),
        "gemm_w8a16": lambda d: qg.gemm_w8a16(d["x"], d["wq8"], d["ws8"], out=d["y2"], static_weights=sw),
        "gemm_w4a16": lambda d, i=0: qg.gemm_w4a16(d["x"], *w4_sets[i % len(w4_sets)], out=d["y3"],
                                                    static_weights=sw),
    }
    dur_us = {}
    for n in names:
        gk = torch.cuda.CUDAGraph()
        with torch.cuda.stream(stream):
            with torch.cuda.graph(gk, stream=stream):
                for i in range(C):
                    if n in ("gemm_w8a8", "gemm_w4a16"):
                        calls[n](sets[i % WEIGHT_SETS], i)
                    else:
                        calls[n](sets[i % WEIGHT_SETS])
        reps = max(1, min(10, (K_steps + C - 1) // C))
        with torch.cuda.stream(stream):
            gk.replay()  # upload + warm-up
        times = []
        for _ in range(REPEATS):
            ka = torch.cuda.Event(enable_timing=True)
            kb = torch.cuda.Event(enable_timing=True)
            with torch.cuda.stream(stream):
                ka.record(stream)
                for _ in range(reps):
                    gk.replay()
                kb.record(stream)
            stream.synchronize()
            times.append(ka.elapsed_time(kb) * 1e3 / (reps * C))
        dur_us[n] = float(np.median(times))
        del gk
    del extra_w8a8, w8a8_sets, extra_w4, w4_sets
    qg.check_device_errors()

    sb = step_bytes()
    bytes_per_step = sum(sb.values())
    value = job_throughput(world, bytes_per_step, K_steps, elapsed_ms)
    peaks = load_peaks()
    kernels = {}
    for n in names:
        gbs = sb[n] / (dur_us[n] * 1e-6) / 1e9
        kernels[n] = {"us": round(dur_us[n], 3), "bytes": sb[n], "GB/s": round(gbs, 1),
                      "frac_hbm": round(gbs / peaks["hbm_gbs"], 4)}
    dominant = max(["gemm_w8a8", "gemm_w8a16", "gemm_w4a16"], key=lambda n: dur_us[n])
    dom_gbs = sb[dominant] / (dur_us[dominant] * 1e-6) / 1e9
    roofline = {"bound": "hbm", "kernel": dominant, "achieved": round(dom_gbs, 1),
                "peak": peaks["hbm_gbs"], "unit": "GB/s", "frac": round(dom_gbs / peaks["hbm_gbs"], 4),
                "traffic": kernel_traffic(dominant), "peak_source": peaks["source"] + " (burst copy)"}

    # ---- the widened rows (decode M=16, K=4096), each alone: C launches over
    # rotating weight copies (together larger than L2) in one graph ----
    if not args.skip_next_rows:
        kernels.update(time_next_rows(qg, W, torch, dev, stream, peaks, seed0))
    qg.check_device_errors()
    # ---- the other shapes of the workload table, each kernel alone ----
    sweep = None
    if not args.skip_sweep:
        sampler = ClockSampler(visible[local_rank] if local_rank < len(visible) else str(local_rank))
        sampler.start()
        time.sleep(0.05)
        sweep = time_config_sweep(qg, W, torch, dev, stream, peaks, seed0, sw)
        sweep["clocks"] = sampler.stop()
    qg.check_device_errors()

    # ---- end to end through the public API with host buffers ----
    K_e2e = min(K_steps, 2000)
    hx = [d["x"].cpu().pin_memory() for d in sets]
    # the three outputs of a step are column slices of one [M, 4096 + 2 x 11008]
    # buffer (written through the output leading dimension), read back in one copy
    n_all = N_SQ + 2 * N_FF
    ycat = [torch.empty((M, n_all), dtype=torch.float16, device=dev) for _ in sets]
    hy = [torch.empty((M, n_all), dtype=torch.float16).pin_memory() for _ in sets]
    yv = [(y[:, :N_SQ], y[:, N_SQ:N_SQ + N_FF], y[:, N_SQ + N_FF:]) for y in ycat]
    xdev = [torch.empty((M, K), dtype=torch.float16, device=dev) for _ in sets]

    # transfers on their own streams, so a step's download and the next step's
    # upload overlap the kernels; events order each buffer's reuse.  Copies and
    # events go straight to the CUDA runtime (CudaRuntime): through torch they
    # cost more host time per step than the kernel launches.
    rt = CudaRuntime()
    comp = torch.cuda.current_stream(dev)
    h2d, d2h, side2 = (torch.cuda.Stream(device=dev) for _ in range(3))
    s_comp, s_h2d, s_d2h, s_side = comp.cuda_stream, h2d.cuda_stream, d2h.cuda_stream, side2.cuda_stream
    ev_in = [rt.event() for _ in sets]    # input uploaded
    ev_out = [rt.event() for _ in sets]   # kernels done (input free, outputs ready)
    ev_done = [rt.event() for _ in sets]  # outputs downloaded (output buffer free)
    ev_fork = [rt.event() for _ in sets]  # the second kernel chain may start
    ev_join = [rt.event() for _ in sets]  # the second kernel chain is done
    x_bytes, y_bytes = 2 * M * K, 2 * M * n_all
    hx_p, xd_p = [t.data_ptr() for t in hx], [t.data_ptr() for t in xdev]
    hy_p, yc_p = [t.data_ptr() for t in hy], [t.data_ptr() for t in ycat]
    H2D, D2H = CudaRuntime.H2D, CudaRuntime.D2H

    # The serving pattern: device buffers allocated once, each step's kernels
    # bound to them once as launch plans (qg_plan_*), in the step's two-stream
    # schedule; outputs written in place.
    plans = [(qg.plan_quantize_rowwise_int8(xdev[r], out=d["xq"], scale_out=d["xs"]),
              qg.plan_gemm_w8a8(d["xq"], d["wq"], d["xs"], d["ws"], d["b"], out_dtype=torch.float16,
                                out=yv[r][0], static_weights=sw),
              qg.plan_gemm_w4a16(xdev[r], d["qw"], d["sc"], d["ze"], out=yv[r][2], static_weights=sw),
              qg.plan_gemm_w8a16(xdev[r], d["wq8"], d["ws8"], out=yv[r][1], static_weights=sw))
             for r, d in enumerate(sets)]

    def kernels_planned(r, d):
        rc = (rt.record(ev_fork[r], s_comp), rt.wait(s_side, ev_fork[r], 0))
        if any(rc):
            rt.check(next(c for c in rc if c), "e2e fork")
        pq, pa, pc, pb = plans[r]
        pc.launch(s_side)
        pb.launch(s_side)
        pq.launch(s_comp)
        pa.launch(s_comp)
        rc = (rt.record(ev_join[r], s_side), rt.wait(s_comp, ev_join[r], 0))
        if any(rc):
            rt.check(next(c for c in rc if c), "e2e join")

    def kernels_direct(r, d):  # the per-call binding, one stream
        qg.quantize_rowwise_int8(xdev[r], out=d["xq"], scale_out=d["xs"])
        qg.gemm_w8a8(d["xq"], d["wq"], d["xs"], d["ws"], d["b"], out_dtype=torch.float16, out=yv[r][0],
                     static_weights=sw)
        qg.gemm_w8a16(xdev[r], d["wq8"], d["ws8"], out=yv[r][1], static_weights=sw)
        qg.gemm_w4a16(xdev[r], d["qw"], d["sc"], d["ze"], out=yv[r][2], static_weights=sw)

    def e2e_step(i, kernels):
        d, r = sets[i % WEIGHT_SETS], i % WEIGHT_SETS
        rc = (rt.wait(s_h2d, ev_out[r], 0), rt.memcpy(xd_p[r], hx_p[r], x_bytes, H2D, s_h2d),
              rt.record(ev_in[r], s_h2d), rt.wait(s_comp, ev_in[r], 0), rt.wait(s_comp, ev_done[r], 0))
        if any(rc):
            rt.check(next(c for c in rc if c), "e2e upload")
        kernels(r, d)
        rc = (rt.record(ev_out[r], s_comp), rt.wait(s_d2h, ev_out[r], 0),
              rt.memcpy(hy_p[r], yc_p[r], y_bytes, D2H, s_d2h), rt.record(ev_done[r], s_d2h))
        if any(rc):
            rt.check(next(c for c in rc if c), "e2e download")

    def time_e2e(kernels):
        for e in ev_out + ev_done:
            rt.check(rt.record(e, s_comp), "cudaEventRecord")
        for i in range(max(3, W_steps)):
            e2e_step(i, kernels)
        torch.cuda.synchronize()
        if world > 1:
            torch.distributed.barrier()
        a = torch.cuda.Event(enable_timing=True)
        b = torch.cuda.Event(enable_timing=True)
        a.record(comp)
        for i in range(K_e2e):
            e2e_step(i, kernels)
        for e in ev_done:  # the timed region ends when every download has landed
            rt.check(rt.wait(s_comp, e, 0), "cudaStreamWaitEvent")
        b.record(comp)
        torch.cuda.synchronize()
        return max_over_ranks(a.elapsed_time(b), world, dev)

    e2e_ms = time_e2e(kernels_planned)
    direct_ms = time_e2e(kernels_direct)
    qg.check_device_errors()
    for pl in plans:
        for p in pl:
            p.close()
    rt.destroy(ev_in + ev_out + ev_done + ev_fork + ev_join)
    e2e = {"value": round(job_throughput(world, bytes_per_step, K_e2e, e2e_ms), 1), "unit": "GB/s",
           "h2d_bytes_per_step": x_bytes, "d2h_bytes_per_step": y_bytes, "steps": K_e2e,
           "api": "int4_quantized_gemm_b200 launch plans (qg_plan_*) -> libqg C ABI, the step's two-stream "
                  "schedule, no graph; pinned-host copies and stream ordering through the CUDA runtime",
           "direct_calls": {"value": round(job_throughput(world, bytes_per_step, K_e2e, direct_ms), 1),
                            "unit": "GB/s", "api": "the per-call binding (quantize_rowwise_int8, gemm_*), one "
                                                   "stream, same copies"}}

    # ---- prefill W8A8 (compute-bound), two rotating operand sets > L2; timed
    # last, after the memory-bound kernels, whose timings its power draw would depress ----
    Mp, Np, Kp = PREFILL
    pre = []
    for r in range(2):
        s = seed0 + 500 + r
        xq, xs = qg.quantize_rowwise_int8(W.torch_activations(Mp, Kp, s, dev, outliers=True))
        wq, ws = qg.quantize_rowwise_int8(W.torch_weights(Np, Kp, s, dev))
        pre.append(dict(xq=xq.contiguous(), xs=xs, wq=wq.contiguous(), ws=ws, b=W.torch_bias(Np, s, dev),
                        y=torch.empty((Mp, Np), dtype=torch.bfloat16, device=dev)))
    torch.cuda.synchronize()
    P = 8
    pev = [torch.cuda.Event(enable_timing=True, external=True) for _ in range(P + 1)]
    gp = torch.cuda.CUDAGraph()
    for i in range(2):
        d = pre[i]
        qg.gemm_w8a8(d["xq"], d["wq"], d["xs"], d["ws"], d["b"], out_dtype=torch.bfloat16, out=d["y"])
    torch.cuda.synchronize()
    with torch.cuda.stream(stream):
        with torch.cuda.graph(gp, stream=stream):
            for i in range(P):
                d = pre[i % 2]
                pev[i].record()
                qg.gemm_w8a8(d["xq"], d["wq"], d["xs"], d["ws"], d["b"], out_dtype=torch.bfloat16, out=d["y"])
            pev[P].record()
    for _ in range(3):
        gp.replay()
    gp.replay()
    torch.cuda.synchronize()
    pre_us = float(np.mean([pev[i].elapsed_time(pev[i + 1]) for i in range(P)])) * 1e3
    pre_tops = 2.0 * Mp * Np * Kp / (pre_us * 1e-6) / 1e12
    i8_peak = 2.0 * peaks["bf16_tflops"]  # dense int8 = 2x dense bf16 (nominal 4.5 vs 2.25 PF/s)
    kernels["gemm_w8a8_prefill_8192x11008x4096_bf16"] = {
        "us": round(pre_us, 2), "TOPS": round(pre_tops, 1), "peak_TOPS": i8_peak,
        "frac": round(pre_tops / i8_peak, 4), "frac_of_nominal_4500": round(pre_tops / 4500.0, 4),
        "peak_source": peaks["source"] + " bf16 x 2"}
    qg.check_device_errors()
    del pre

    result = {
        "metric": METRIC, "value": round(value, 1), "unit": "GB/s", "n_gpus": world, "steps": K_steps,
        "warmup": W_steps, "ms_per_step": round(elapsed_ms / K_steps, 6), "repeats": REPEATS,
        "ms_per_step_repeats": [round(t / K_steps, 6) for t in rep_ms], "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "i8xi8->i32, f16xf16->f32 (int8/int4 weights)",
        "data": "synthetic (seeded; LLaMA-7B linear shapes; no dataset or trained weights)",
        "config": {"workload": WORKLOAD, "M": M, "K": K, "N": [N_SQ, N_FF, N_FF], "group": GROUP,
                   "static_weights": sw, "schedule": "quantize->W8A8 | W4A16->W8A16 (two streams, joined per step)"
                   if two else "one stream: quantize, W8A8, W8A16, W4A16",
                   "weight_sets_rotated": WEIGHT_SETS, "l2": "inputs larger than L2 (4 rotating weight sets, ~350 MB)",
                   "parallelism": f"replicas x{world}", "bytes_per_step": bytes_per_step},
        "roofline": roofline, "kernels": kernels, "e2e": e2e,
        "gpu_launches": 4 * K_steps, "gpu_launches_note": "per timed region of K steps (each repeat)",
        "clocks": clocks,
    }
    if sweep is not None:
        result["shapes"] = sweep
    return result


def copies_beyond_l2(nbytes: int) -> int:
    """How many copies of an operand of `nbytes` to cycle through so that the
    set is well beyond the 126 MB L2 (at least 4)."""
    return max(4, int(np.ceil(300e6 / nbytes)))


def graph_time(torch, stream, make, nbytes):
    """Per-launch device time (us) of make(i)() for i cycling over
    copies_beyond_l2(nbytes) operand copies: the launches are captured in one
    CUDA graph (two passes over the copies); after one warm-up replay, REPEATS
    windows of two replays are bracketed by CUDA events on `stream` and the
    median window gives the time."""
    R = copies_beyond_l2(nbytes)
    calls = [make(i) for i in range(R)]
    torch.cuda.synchronize()  # operands written before the first call (static-weights contract)
    for c in calls:
        c()
    torch.cuda.synchronize()
    C = 2 * R
    g = torch.cuda.CUDAGraph()
    with torch.cuda.stream(stream):
        with torch.cuda.graph(g, stream=stream):
            for i in range(C):
                calls[i % R]()
    with torch.cuda.stream(stream):
        g.replay()  # upload + warm-up
    times = []
    for _ in range(REPEATS):
        a = torch.cuda.Event(enable_timing=True)
        b = torch.cuda.Event(enable_timing=True)
        with torch.cuda.stream(stream):
            a.record(stream)
            for _ in range(2):
                g.replay()
            b.record(stream)
        stream.synchronize()
        times.append(a.elapsed_time(b) * 1e3 / (2 * C))
    del g, calls
    return float(np.median(times))


def time_next_rows(qg, W, torch, dev, stream, peaks, seed0):
    """Per-launch device time of the fused quantize + W8A8, zero-point W8A8,
    W4A8, symmetric W4A16 and GELU-epilogue W4A16 kernels at the decode shape
    (M=16, K=4096): for each, a graph of launches cycling through enough
    weight copies that they never fit in L2, timed with CUDA events."""
    M, K = M_DEC, K_DIM

    def timed(make, nbytes):
        return graph_time(torch, stream, make, nbytes)

    out = {}

    def record(name, us, nbytes):
        gbs = nbytes / (us * 1e-6) / 1e9
        out[name] = {"us": round(us, 3), "bytes": int(nbytes), "GB/s": round(gbs, 1),
                     "frac_hbm": round(gbs / peaks["hbm_gbs"], 4)}

    x = W.torch_activations(M, K, seed0 + 900, dev, outliers=True)
    xrelu = torch.relu(x)
    # fused quantize + W8A8 (N = 4096)
    N = N_SQ
    R = max(4, int(np.ceil(300e6 / (N * K))))
    ws8 = [qg.quantize_rowwise_int8(W.torch_weights(N, K, seed0 + 910 + i, dev)) for i in range(R)]
    b = W.torch_bias(N, seed0 + 911, dev)
    y = torch.empty((M, N), dtype=torch.float16, device=dev)
    nb = N * K + 2 * M * K + 2 * M * N + 8 * N
    record("quantize_gemm_w8a8_16x4096x4096_fused",
           timed(lambda i: (lambda: qg.quantize_gemm_w8a8(x, ws8[i % R][0], ws8[i % R][1], b, out=y)), N * K), nb)
    del ws8
    # zero-point W8A8 (both operands asymmetric, N = 4096)
    xq, xs, xz, xsum = qg.quantize_rowwise_asym_int8(xrelu)
    wz = [qg.quantize_rowwise_asym_int8(W.torch_weights(N, K, seed0 + 920 + i, dev)) for i in range(R)]
    nb = N * K + M * K + 2 * M * N + 16 * N + 12 * M
    record("gemm_w8a8_zp_16x4096x4096",
           timed(lambda i: (lambda: qg.gemm_w8a8_zp(xq, xs, xz, xsum, wz[i % R][0], wz[i % R][1], wz[i % R][2],
                                                    wz[i % R][3], b, out=y)), N * K), nb)
    del wz
    # int4 weights at N = 11008
    N = N_FF
    xq16, xs16 = qg.quantize_rowwise_int8(x)
    y = torch.empty((M, N), dtype=torch.float16, device=dev)
    b = W.torch_bias(N, seed0 + 931, dev)
    R = max(4, int(np.ceil(300e6 / (N * K // 2))))
    w4c = [qg.quantize_channel_sym4(W.torch_weights(N, K, seed0 + 930 + i, dev)) for i in range(R)]
    nb = N * K // 2 + M * K + 2 * M * N + 8 * N + 4 * M
    record("gemm_w4a8_16x11008x4096",
           timed(lambda i: (lambda: qg.gemm_w4a8(xq16, w4c[i % R][0], xs16, w4c[i % R][1], b, out=y)), N * K // 2), nb)
    del w4c
    w4s = [qg.quantize_block_sym4(W.torch_weights(N, K, seed0 + 940 + i, dev, per_column_factor=False))
           for i in range(R)]
    nb = N * K // 2 + 2 * (K // GROUP) * N + 2 * M * K + 2 * M * N
    record("gemm_w4a16_sym_16x11008x4096",
           timed(lambda i: (lambda: qg.gemm_w4a16_sym(x, w4s[i % R][0], w4s[i % R][1], out=y)), N * K // 2), nb)
    del w4s
    w4a = [qg.quantize_block_asym4(W.torch_weights(N, K, seed0 + 950 + i, dev, per_column_factor=False))
           for i in range(R)]
    nb = N * K // 2 + 4 * (K // GROUP) * N + 2 * M * K + 2 * M * N + 4 * N
    record("gemm_w4a16_gelu_16x11008x4096",
           timed(lambda i: (lambda: qg.gemm_w4a16_act(x, w4a[i % R][0], w4a[i % R][1], w4a[i % R][2], bias=b,
                                                      activation="gelu", out=y)), N * K // 2), nb)
    del w4a
    torch.cuda.synchronize()
    return out


def time_config_sweep(qg, W, torch, dev, stream, peaks, seed0, sw=False):
    """The remaining shapes of the workload table, each kernel alone (graph of
    launches over operand copies beyond L2, CUDA events): W8A8 decode at
    M = 1 and 8 (N = K = 4096, fp16 out, bias); W8A8 prefill at M = 2048 with
    N = 4096 and 11008 and at M = 8192 with N = 4096 (bf16 out, bias); W8A16
    at M = 1, 16, 256 with N = 4096 and at M = 1, 256 with N = 11008; W4A16 at
    M = 1 with N = 11008; the per-row quantizer alone at M = 2048 and 8192.
    Memory-bound shapes report GB/s against the measured HBM copy bandwidth;
    the prefill and M = 256 shapes also report TFLOP/s (TOPS) against the
    measured dense bf16 peak (x2 for int8).  sw: the three base GEMMs are called
    with the static-weights flag (their weights are written and synchronized
    before the first call)."""
    K = K_DIM
    hbm, f16_peak = peaks["hbm_gbs"], peaks["bf16_tflops"]
    out = {}

    def rec(name, us, nbytes, ops=None, tc_peak=None):
        gbs = nbytes / (us * 1e-6) / 1e9
        d = {"us": round(us, 3), "bytes": int(nbytes), "GB/s": round(gbs, 1), "frac_hbm": round(gbs / hbm, 4)}
        if ops is not None:
            t = ops / (us * 1e-6) / 1e12
            d.update({"TFLOP/s": round(t, 1), "peak_TFLOP/s": tc_peak, "frac_tensor": round(t / tc_peak, 4)})
        out[name] = d

    # per-row quantizer alone at prefill batch sizes (rotating inputs beyond L2)
    for M in (2048, 8192):
        nb = 3 * M * K + 4 * M
        R = copies_beyond_l2(nb)
        xs_ = [W.torch_activations(M, K, seed0 + 1100 + i, dev, outliers=True) for i in range(R)]
        xq = torch.empty((M, K), dtype=torch.int8, device=dev)
        sc = torch.empty(M, dtype=torch.float32, device=dev)
        rec(f"quantize_rowwise_int8_{M}x{K}",
            graph_time(torch, stream, lambda i: (lambda: qg.quantize_rowwise_int8(xs_[i], out=xq, scale_out=sc)), nb),
            nb)
        del xs_, xq, sc
    # W8A8: decode batches here, the prefill shapes last (their power draw
    # would otherwise carry over into the memory-bound timings)
    def w8a8_shape(M, N, dt):
        R = copies_beyond_l2(N * K)
        ws8 = [qg.quantize_rowwise_int8(W.torch_weights(N, K, seed0 + 1200 + i, dev)) for i in range(R)]
        xq, xsc = qg.quantize_rowwise_int8(W.torch_activations(M, K, seed0 + 1210, dev, outliers=True))
        b = W.torch_bias(N, seed0 + 1211, dev)
        y = torch.empty((M, N), dtype=dt, device=dev)
        nb = N * K + M * K + y.element_size() * M * N + 8 * N + 4 * M
        us = graph_time(torch, stream, lambda i: (lambda: qg.gemm_w8a8(xq, ws8[i][0], xsc, ws8[i][1], b,
                                                                       out_dtype=dt, out=y, static_weights=sw)),
                        N * K)
        big = M > 64
        rec(f"gemm_w8a8_{M}x{N}x{K}_{'bf16' if dt == torch.bfloat16 else 'f16'}", us, nb,
            2.0 * M * N * K if big else None, 2.0 * f16_peak if big else None)
        del ws8, xq, xsc, y

    w8a8_shape(1, N_SQ, torch.float16)
    w8a8_shape(8, N_SQ, torch.float16)
    # W8A16
    for M, N in ((1, N_SQ), (16, N_SQ), (256, N_SQ), (1, N_FF), (256, N_FF)):
        R = copies_beyond_l2(N * K)
        ws8 = [qg.quantize_rowwise_int8(W.torch_weights(N, K, seed0 + 1300 + i, dev)) for i in range(R)]
        x = W.torch_activations(M, K, seed0 + 1310, dev)
        y = torch.empty((M, N), dtype=torch.float16, device=dev)
        nb = N * K + 2 * M * K + 2 * M * N + 4 * N
        us = graph_time(torch, stream,
                        lambda i: (lambda: qg.gemm_w8a16(x, ws8[i][0], ws8[i][1], out=y, static_weights=sw)), N * K)
        rec(f"gemm_w8a16_{M}x{N}x{K}", us, nb, 2.0 * M * N * K if M > 64 else None, f16_peak if M > 64 else None)
        del ws8, x, y
    # W4A16 (group 64) at M = 1
    M, N = 1, N_FF
    R = copies_beyond_l2(N * K // 2)
    w4 = [qg.quantize_block_asym4(W.torch_weights(N, K, seed0 + 1400 + i, dev, per_column_factor=False))
          for i in range(R)]
    x = W.torch_activations(M, K, seed0 + 1410, dev)
    y = torch.empty((M, N), dtype=torch.float16, device=dev)
    nb = N * K // 2 + 4 * (K // GROUP) * N + 2 * M * K + 2 * M * N
    rec(f"gemm_w4a16_{M}x{N}x{K}",
        graph_time(torch, stream, lambda i: (lambda: qg.gemm_w4a16(x, w4[i][0], w4[i][1], w4[i][2], out=y,
                                                                   static_weights=sw)), N * K // 2),
        nb)
    del w4, x, y
    for M, N in ((2048, N_SQ), (2048, N_FF), (8192, N_SQ)):
        w8a8_shape(M, N, torch.bfloat16)
    torch.cuda.synchronize()
    return out


# ---------------------------------------------------------------------------
# one small case per invocation, for ncu captures (--profile-case)
# ---------------------------------------------------------------------------
PROFILE_CASES = {
    # name: (op, M, N, K, weight-only token tile width or 0, static weights)
    "quantize_8192x4096": ("quant", 8192, 0, 4096, 0, False),
    "quantize_16x4096": ("quant", 16, 0, 4096, 0, False),
    "w4a8_16x11008x4096": ("w4a8", 16, 11008, 4096, 0, False),
    "w8a8_16x4096x4096": ("w8a8", 16, 4096, 4096, 0, True),
    "w8a8_2048x4096x4096": ("w8a8", 2048, 4096, 4096, 0, False),
    "w8a8_8192x11008x4096": ("w8a8", 8192, 11008, 4096, 0, False),
    "w8a16_16x11008x4096": ("w8a16", 16, 11008, 4096, 0, True),
    "w8a16_256x4096x4096": ("w8a16", 256, 4096, 4096, 0, False),
    "w8a16_256x11008x4096": ("w8a16", 256, 11008, 4096, 0, False),
    "w4a16_16x11008x4096": ("w4a16", 16, 11008, 4096, 0, True),
}


def run_profile_case(name, launches=3):
    """Draw the case's operands on the device (torch), then launch its kernel
    `launches` times; an ncu capture takes the last one (-k <kernel> -s 2 -c 1).
    Operands are random codes and scales (the timing does not depend on the
    values)."""
    import torch
    import int4_quantized_gemm_b200 as qg
    op, M, N, K, bn, sw = PROFILE_CASES[name]
    if bn:
        qg.set_tuning("QG_WONLY_BN", bn)
    dev = "cuda"
    g = torch.Generator(device=dev)
    g.manual_seed(0)
    x = torch.randn(M, K, device=dev, generator=g).half()
    if op == "quant":
        xq = torch.empty(M, K, dtype=torch.int8, device=dev)
        sc = torch.empty(M, device=dev)
        call = lambda: qg.quantize_rowwise_int8(x, out=xq, scale_out=sc)
    elif op == "w8a8":
        xq = torch.randint(-127, 128, (M, K), dtype=torch.int8, device=dev, generator=g)
        wq = torch.randint(-127, 128, (N, K), dtype=torch.int8, device=dev, generator=g)
        xs = torch.rand(M, device=dev, generator=g) * 0.01
        ws = torch.rand(N, device=dev, generator=g) * 0.01
        b = torch.randn(N, device=dev, generator=g)
        y = torch.empty(M, N, dtype=torch.bfloat16 if M > 64 else torch.float16, device=dev)
        call = lambda: qg.gemm_w8a8(xq, wq, xs, ws, b, out_dtype=y.dtype, out=y, static_weights=sw)
    elif op == "w4a8":
        xq = torch.randint(-127, 128, (M, K), dtype=torch.int8, device=dev, generator=g)
        qw = torch.randint(-2 ** 31, 2 ** 31 - 1, (N, K // 8), dtype=torch.int32, device=dev, generator=g)
        xs = torch.rand(M, device=dev, generator=g) * 0.01
        ws = torch.rand(N, device=dev, generator=g) * 0.01
        y = torch.empty(M, N, dtype=torch.float16, device=dev)
        call = lambda: qg.gemm_w4a8(xq, qw, xs, ws, None, out_dtype=torch.float16, out=y)
    elif op == "w8a16":
        wq = torch.randint(-127, 128, (N, K), dtype=torch.int8, device=dev, generator=g)
        ws = torch.rand(N, device=dev, generator=g) * 0.01
        y = torch.empty(M, N, dtype=torch.float16, device=dev)
        call = lambda: qg.gemm_w8a16(x, wq, ws, out=y, static_weights=sw)
    else:
        qw = torch.randint(-2 ** 31, 2 ** 31 - 1, (N, K // 8), dtype=torch.int32, device=dev, generator=g)
        sc = (torch.rand(K // 64, N, device=dev, generator=g) * 0.01 + 0.001).half()
        ze = torch.randint(0, 16, (K // 64, N), device=dev, generator=g).half()
        y = torch.empty(M, N, dtype=torch.float16, device=dev)
        call = lambda: qg.gemm_w4a16(x, qw, sc, ze, out=y, static_weights=sw)
    torch.cuda.synchronize()
    for _ in range(launches):
        call()
    torch.cuda.synchronize()
    qg.check_device_errors()
    print(json.dumps({"profile_case": name, "launches": launches, "ok": True}))


# ---------------------------------------------------------------------------
# CPU oracle on the host cores (cpu_baseline leg and the reference arm)
# ---------------------------------------------------------------------------
class OracleStep:
    """The oracle's decode step on a sample: `rows` of the 16 rows and the first
    1/`col_div` of the output columns of each GEMM (full K).  Its time scales
    with rows x columns (multiply-adds), which is how it is extrapolated."""

    def __init__(self, seed=1, col_div=1):
        import oracle
        import workloads as W
        self.o = oracle
        self.threads = oracle.max_threads()
        self.col_div = col_div
        M, K = M_DEC, K_DIM
        self.x = W.activations(M, K, seed, outliers=True)
        n1, n2 = max(1, N_SQ // col_div), max(1, N_FF // col_div)
        wq, ws = oracle.quantize_rowwise_int8(W.weights(N_SQ, K, seed))
        self.wq, self.ws, self.b = wq[:n1], ws[:n1], W.bias(N_SQ, seed)[:n1]
        wq8, ws8 = oracle.quantize_rowwise_int8(W.weights(N_FF, K, seed + 2))
        self.wq8, self.ws8 = wq8[:n2], ws8[:n2]
        qw, sc, ze, _ = oracle.quantize_block_asym4(W.weights(N_FF, K, seed + 3, per_column_factor=False), GROUP)
        self.qw = qw[:n2]
        self.sc = np.ascontiguousarray(sc[:, :n2])
        self.ze = np.ascontiguousarray(ze[:, :n2])

    def run(self, rows):
        o = self.o
        x = self.x[:rows]
        xq, xs = o.quantize_rowwise_int8(x)
        o.w8a8_f64(xq, self.wq, xs, self.ws, self.b)
        o.w8a16_f64(x, self.wq8, self.ws8, None)
        o.w4a16_f64(x, self.qw, self.sc, self.ze, GROUP, None)

    def time_rows(self, rows):
        t = time.perf_counter()
        self.run(rows)
        return time.perf_counter() - t

    def full_step_seconds(self, seconds, rows):
        return seconds * (M_DEC / rows) * self.col_div


def _sample_text(rows, col_div):
    cols = "all" if col_div == 1 else f"1/{col_div} of the"
    return f"{rows} of {M_DEC} rows x {cols} output columns of each GEMM (full K), extrapolated by multiply-adds"


def cpu_baseline(budget_s=15.0):
    st = OracleStep()
    t1 = st.time_rows(1)
    rows = int(max(1, min(M_DEC, math.floor(budget_s / max(t1, 1e-6)))))
    t = st.time_rows(rows)
    step_s = st.full_step_seconds(t, rows)
    value = sum(step_bytes().values()) / step_s / 1e9
    return {"value": round(value, 4), "unit": "GB/s", "cores": st.threads, "kind": "oracle",
            "sample": _sample_text(rows, 1) + f"; {t:.1f} s measured, {step_s:.1f} s per full step"}


def run_reference(args, total_budget_s=120.0):
    probe = OracleStep(col_div=16)
    t1 = probe.full_step_seconds(probe.time_rows(1), 1)  # seconds per full step (extrapolated)
    per_step = total_budget_s / max(1, args.steps + args.warmup)
    # the sample: as many rows as fit, and a column fraction when one row is too much
    frac_needed = per_step / t1 * M_DEC  # rows that fit at full width
    if frac_needed >= 1:
        st, rows = OracleStep(), int(min(M_DEC, math.floor(frac_needed)))
    else:
        col_div = min(256, 2 ** math.ceil(math.log2(1.0 / frac_needed)))
        st, rows = (probe if col_div == 16 else OracleStep(col_div=col_div)), 1
    for _ in range(args.warmup):
        st.run(rows)
    t = time.perf_counter()
    for _ in range(args.steps):
        st.run(rows)
    el = time.perf_counter() - t
    step_s = st.full_step_seconds(el / args.steps, rows)
    value = sum(step_bytes().values()) / step_s / 1e9
    sample = _sample_text(rows, st.col_div)
    return {
        "impl": "reference", "metric": METRIC, "value": round(value, 4), "unit": "GB/s", "n_gpus": 1,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(step_s * 1e3, 3),
        "extrapolated": f"value and ms_per_step are extrapolated from the timed sample ({sample}); "
                        f"the sample steps took {el / args.steps * 1e3:.1f} ms each",
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": "int64 / fp64 (CPU oracle)", "data": "synthetic (seeded)",
        "config": {"workload": WORKLOAD, "M": M_DEC, "K": K_DIM, "N": [N_SQ, N_FF, N_FF], "group": GROUP},
        "cpu_baseline": {"value": round(value, 4), "unit": "GB/s", "cores": st.threads, "kind": "oracle",
                         "sample": sample},
        "e2e": {"value": round(value, 4), "unit": "GB/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }


def main():
    ap = argparse.ArgumentParser(description=__doc__, formatter_class=argparse.RawDescriptionHelpFormatter)
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20000)
    ap.add_argument("--warmup", type=int, default=200)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--no-cpu-baseline", action="store_true", help="skip the oracle timing leg")
    ap.add_argument("--skip-next-rows", action="store_true",
                    help="skip the per-launch timing of the widened rows (fused quantize, zero-point, W4A8, ...)")
    ap.add_argument("--no-static-weights", action="store_true",
                    help="call the GEMMs without QG_FLAG_STATIC_WEIGHTS (weights are then loaded only after "
                         "the preceding kernel has finished)")
    ap.add_argument("--one-stream", action="store_true",
                    help="run the four kernels of a step on one stream (default: W4A16 -> W8A16 on a second stream "
                         "beside quantize -> W8A8, joined at the end of each step)")
    ap.add_argument("--skip-sweep", action="store_true",
                    help="skip the per-launch timing of the other workload shapes (M = 1/8/256/2048, N = 4096, ...)")
    ap.add_argument("--profile-case", choices=sorted(PROFILE_CASES),
                    help="launch one small case three times and exit (for ncu captures)")
    args = ap.parse_args()
    if args.profile_case:
        run_profile_case(args.profile_case)
        return
    if args.warmup < 3:
        ap.error("--warmup must be at least 3")
    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))

    if args.impl == "reference":
        if rank != 0:
            return
        print(json.dumps(run_reference(args)), flush=True)
        return

    if world > 1:
        import torch
        torch.cuda.set_device(local_rank)
        torch.distributed.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                             device_id=torch.device("cuda", local_rank))
    try:
        res = run_ours(args, rank, world, local_rank)
        if rank == 0:
            if world == 1 and not args.no_cpu_baseline:
                res["cpu_baseline"] = cpu_baseline()
            print(json.dumps(res), flush=True)
    finally:
        if world > 1:
            import torch
            torch.distributed.barrier()
            torch.distributed.destroy_process_group()


if __name__ == "__main__":
    main()
