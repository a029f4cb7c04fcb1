"""Benchmark of the fused linear-layer GEMM + epilogue on B200.

A step is one pass of the whole path over one batch of synthetic input:
forward (X.W + bias, ReLU, relu_aux mask) then backward DRELU_BGRAD
(dY2.W2 masked by relu_aux, dZ and the fp32 bias gradient). The default
workload is the FFN training-step shape (bf16, T=4096, K=4096, N=11008,
D2=4096); --workload selects the other shapes (pr1, square, large,
skinny-1/8/64/256).

python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME]
                [--impl ours|reference] [--ablation]

Prints ONE JSON line (rank 0). Timing: every step is bracketed by CUDA
events on the stream the kernels are launched on; an L2 flush (a 256 MiB
write, then a 256 MiB read of another buffer) runs between steps, outside
the events. The region of K steps is
bracketed by a barrier and device synchronisation; the max over ranks is
reported. Multi-GPU runs are independent replicas (the path has no
exchange step): value = units of all ranks / slowest rank's time.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import math
import os
import statistics
import subprocess
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

import torch  # noqa: E402

from gemm_epilogues_tcgen05_b200 import synth  # noqa: E402

FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}
L2_FLUSH_BYTES = 256 << 20
QUEUE_CHUNK = 32                 # steps queued behind one GPU sleep
QUEUE_SLEEP_CYCLES = 3_000_000   # ~1.5 ms at 2 GHz: longer than the host needs to queue a chunk


# ------------------------------------------------------------------ setup
def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            d = json.load(f)
        return d, "measured"
    except Exception:
        return dict(FALLBACK_PEAKS), "fallback"


def kernel_source_hash() -> str:
    h = hashlib.sha256()
    csrc = os.path.join(ROOT, "gemm_epilogues_tcgen05_b200", "csrc")
    for fn in sorted(os.listdir(csrc)):
        with open(os.path.join(csrc, fn), "rb") as f:
            h.update(fn.encode())
            h.update(f.read())
    return h.hexdigest()[:16]


def step_spec(w: synth.Workload, args=None):
    """Which epilogs a step of this workload runs. --fwd-epilog GELU_BIAS
    times that forward alone (the library has no GELU backward)."""
    if args is not None and getattr(args, "ffn_step", False):
        return "FFN_STEP", True
    if args is not None and getattr(args, "wgrad", False):
        return "WGRAD", False
    if args is not None and getattr(args, "fwd_epilog", None):
        return args.fwd_epilog, False
    if w.name in ("ffn", "pr1"):
        return "RELU_AUX_BIAS", True
    if w.name == "square":
        return "RELU_BIAS", False
    if w.name in ("large", "large-proxy"):
        return "RELU_AUX_BIAS", False
    if w.name.startswith("skinny"):
        return "RELU_BIAS", True
    raise ValueError(w.name)


def algorithmic(w: synth.Workload, fwd_epi: str, bwd: bool):
    """FLOPs and bytes per step (inputs read once, outputs written once)."""
    e = 2  # bytes per 16-bit element
    aux_bytes = w.T * math.ceil(w.N / 32) * 4
    f_fwd = 2.0 * w.T * w.N * w.K
    b_fwd = e * (w.T * w.K + w.K * w.N + w.N + w.T * w.N) + (aux_bytes if fwd_epi == "RELU_AUX_BIAS" else 0)
    if fwd_epi == "GELU_AUX_BIAS":  # the pre-activation written as the auxiliary output
        b_fwd += e * w.T * w.N
    if fwd_epi == "WGRAD":  # dW = X^T dZ: reads X and dZ, writes dW
        b_fwd = e * (w.T * w.K + w.T * w.N + w.K * w.N)
    if fwd_epi == "FFN_STEP":  # two-layer block, D = K, F = N: 2 forward and 4 backward products
        T, D, F = w.T, w.K, w.N
        g = 2.0 * T * D * F
        fwd_b = e * (T * D + F * D + F + T * F) + aux_bytes + e * (T * F + D * F + D + T * D)
        bwd_b = (e * (T * D + D * F + T * F) + aux_bytes + 4 * F +        # dZ1, db1
                 e * (T * D + T * F + D * F) + e * T * D + 4 * D +       # dW2, db2 (second read of dY)
                 e * (T * F + T * D + F * D) + e * (T * F + F * D + T * D))  # dW1, dX
        return {"fwd": {"flops": 2 * g, "bytes": float(fwd_b)}, "bwd": {"flops": 4 * g, "bytes": float(bwd_b)}}
    out = {"fwd": {"flops": f_fwd, "bytes": float(b_fwd)}}
    if bwd:
        f_bwd = 2.0 * w.T * w.N * w.D2
        b_bwd = e * (w.T * w.D2 + w.D2 * w.N + w.T * w.N) + aux_bytes + 4 * w.N
        out["bwd"] = {"flops": f_bwd, "bytes": float(b_bwd)}
    return out


# ----------------------------------------------------------------- clocks
REASON_BITS = {"hw_slowdown": 0x8, "hw_thermal_slowdown": 0x40, "sw_thermal_slowdown": 0x20, "sw_power_cap": 0x4}


def summarise_clock_samples(samples, t0, t1, t_warm0=None):
    """samples: (time, sm_mhz, max_mhz, power_w, reasons bitmask). Median SM
    clock and the active reasons inside [t0, t1] (the timed region), and over
    [t_warm0, t1] (warm-up and timed region) when given; falls back to every
    sample if none falls inside."""
    def stats(lo, hi):
        inside = [x for x in samples if lo <= x[0] <= hi]
        return inside

    inside = stats(t0, t1)
    wide = stats(t_warm0, t1) if t_warm0 is not None else inside
    use = inside or wide or list(samples)
    if not use:
        return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["no samples"]}
    reasons = sorted({n for x in use for n, b in REASON_BITS.items() if x[4] & b})
    out = {"sm_mhz": statistics.median(x[1] for x in use), "sm_max_mhz": max(x[2] for x in use),
           "samples": len(inside), "reasons": reasons, "power_w_max": max(x[3] for x in use)}
    if t_warm0 is not None and wide:
        out["warmup_and_timed"] = {
            "samples": len(wide), "sm_mhz": statistics.median(x[1] for x in wide),
            "sm_mhz_min": min(x[1] for x in wide),
            "reasons": sorted({n for x in wide for n, b in REASON_BITS.items() if x[4] & b})}
    return out


class ClockSampler:
    """Polls the GPU's SM clock, power and clock-event reasons through NVML
    every 5 ms in a thread (reads only; no setting is changed), from before
    the warm-up to the end of the timed region. Falls back to nvidia-smi at
    its shortest period when NVML cannot be loaded."""
    FIELDS = ("index,uuid,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")
    PERIOD_S = 0.005

    def __init__(self, uuid: str | None):
        self.uuid = uuid
        self.samples = []
        self.stop_flag = threading.Event()
        self.t = None
        self.proc = None
        self.source = None

    def start(self):
        try:
            import pynvml

            pynvml.nvmlInit()
            h = None
            if self.uuid:
                try:
                    u = self.uuid if self.uuid.startswith("GPU-") else "GPU-" + self.uuid
                    h = pynvml.nvmlDeviceGetHandleByUUID(u)
                except Exception:
                    h = None
            if h is None:
                h = pynvml.nvmlDeviceGetHandleByIndex(0)
            self.source = "nvml, 5 ms"
            self.t = threading.Thread(target=self._poll_nvml, args=(pynvml, h), daemon=True)
            self.t.start()
            return
        except Exception:
            pass
        try:
            self.proc = subprocess.Popen(["nvidia-smi", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                                          "-lms", "20"], stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            self.source = "nvidia-smi, 20 ms"
            self.t = threading.Thread(target=self._read_smi, daemon=True)
            self.t.start()
        except Exception:
            self.proc = None

    def _poll_nvml(self, nv, h):
        clk = getattr(nv, "nvmlDeviceGetCurrentClocksEventReasons", None) or nv.nvmlDeviceGetCurrentClocksThrottleReasons
        mx = nv.nvmlDeviceGetMaxClockInfo(h, nv.NVML_CLOCK_SM)
        while not self.stop_flag.is_set():
            try:
                self.samples.append((time.time(), float(nv.nvmlDeviceGetClockInfo(h, nv.NVML_CLOCK_SM)), float(mx),
                                     nv.nvmlDeviceGetPowerUsage(h) / 1000.0, int(clk(h))))
            except Exception:
                pass
            time.sleep(self.PERIOD_S)

    def _read_smi(self):
        for line in self.proc.stdout:
            parts = [p.strip() for p in line.split(",")]
            if len(parts) < 10 or (self.uuid and self.uuid not in parts[1]):
                continue
            try:
                bits = sum(b for n, b in REASON_BITS.items()
                           if parts[6 + list(REASON_BITS).index(n)].lower().startswith("active"))
                self.samples.append((time.time(), float(parts[2]), float(parts[3]), float(parts[4]), bits))
            except ValueError:
                continue

    def stop(self, t0, t1, t_warm0=None):
        self.stop_flag.set()
        if self.proc:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except Exception:
                self.proc.kill()
        if self.t:
            self.t.join(timeout=2)
        if self.source is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["no clock source"]}
        out = summarise_clock_samples(self.samples, t0, t1, t_warm0)
        out["source"] = self.source
        return out


def roofline(w, fwd_epi, res, peaks, peak_src):
    """The JSON line's roofline object for the dominant call (the slower of
    the two): HBM-bound for the few-row workloads, tensor-bound otherwise,
    against the measured peak that fits the run's regime."""
    alg = res["alg"]
    # dominant kernel: the one of the two calls that takes longer
    part = "fwd" if res["fwd_ms"] >= res["bwd_ms"] else "bwd"
    part_ms = res[f"{part}_ms"]
    skinny = w.name.startswith("skinny")
    if skinny:
        achieved = alg[part]["bytes"] / (part_ms / 1e3) / 1e9
        peak = float(peaks.get("hbm_gbs", FALLBACK_PEAKS["hbm_gbs"]))
        roof = {"bound": "hbm", "achieved": achieved, "peak": peak, "unit": "GB/s", "frac": achieved / peak}
    else:
        achieved = alg[part]["flops"] / (part_ms / 1e3) / 1e12
        # fp16 dense peak = bf16 dense peak. The burst figure is for a kernel
        # that runs before the 1 kW power cap settles the clocks; a launch of
        # a millisecond or more, or a timed region during which the sampled
        # clocks report the power cap active (back-to-back steps), is a
        # sustained load and is measured against the sustained figure.
        burst = float(peaks.get("bf16_tflops", FALLBACK_PEAKS["bf16_tflops"]))
        sustained = float(peaks.get("bf16_tflops_sustained", FALLBACK_PEAKS["bf16_tflops_sustained"]))
        long_launch = part_ms >= 1.0
        capped = "sw_power_cap" in ((res.get("clocks") or {}).get("reasons") or [])
        peak = sustained if (long_launch or capped) else burst
        kind = ("sustained (launch >= 1 ms)" if long_launch else
                "sustained (power cap active in the timed region)" if capped else "burst (launch < 1 ms)")
        roof = {"bound": "tensor", "achieved": achieved, "peak": peak, "unit": "TFLOP/s", "frac": achieved / peak,
                "frac_of_burst": achieved / burst, "peak_kind": kind}
    kname = {0: "tile_kernel", 1: "skinny_kernel", 2: "tile2_kernel (CTA pair)"}[res["kernel"]]
    roof["kernel"] = f"{part}: {kname} " + (fwd_epi if part == "fwd" else "DRELU_BGRAD" +
                                              (" + dbias finish" if res["kernel"] != 1 else ""))
    if fwd_epi == "FFN_STEP":
        roof["kernel"] = (f"{part}: " + ("layer 1 RELU_AUX_BIAS + layer 2 BIAS" if part == "fwd" else
                                         "DRELU_BGRAD, WGRAD (+db2), WGRAD, NONE") + f" ({kname} kernels)")
    roof["peak_source"] = "measured (MEASURED_PEAKS.json)" if peak_src == "measured" else "fallback"
    roof["traffic"] = measured_traffic(w, part, fwd_epi)
    # roofline time of the whole step: slower of FLOPs at the tensor peak and bytes at HBM
    t_roof = sum(max(v["flops"] / (float(peaks.get("bf16_tflops", 1590.0)) * 1e12),
                     v["bytes"] / (float(peaks.get("hbm_gbs", 6650.0)) * 1e9)) for v in alg.values())
    roof["step_roofline_frac"] = t_roof * 1e3 / res["step_ms"]
    return roof


# ------------------------------------------------------- across the ranks
def max_over_ranks(values, device, world: int) -> list[float]:
    """Each entry's maximum over all ranks (the slowest rank's time): an
    all-reduce with MAX on the default process group when world > 1."""
    t = torch.tensor([float(v) for v in values], device=device, dtype=torch.float64)
    if world > 1:
        torch.distributed.all_reduce(t, op=torch.distributed.ReduceOp.MAX)
    return [float(x) for x in t.tolist()]


def whole_job_tflops(flops_per_rank_step: float, world: int, slowest_step_ms: float) -> float:
    """Every rank runs its own replica of the step (weak scaling): the units of
    all ranks divided by the slowest rank's step time."""
    return flops_per_rank_step * world / (slowest_step_ms / 1e3) / 1e12


# ----------------------------------------------------------------- our arm
def run_ours(args, w: synth.Workload, rank: int, world: int, dev: torch.device):
    from gemm_epilogues_tcgen05_b200 import Plan, binding

    fwd_epi, has_bwd = step_spec(w, args)
    dt = w.torch_dtype
    inp = synth.make_inputs(w, device=dev)
    X, W, b = inp["X"], inp["W"], inp["bias"]
    Y = torch.empty((w.T, w.N), dtype=dt, device=dev)
    aux_words = math.ceil(w.N / 32)
    aux = torch.zeros((w.T, aux_words), dtype=torch.int32, device=dev)
    # plan cost: the first plan in a process also pays the library's one-time
    # initialisation (module load, driver entry points), reported apart
    t_plan = time.perf_counter()
    Plan(w.T, w.N, w.K, dt, "RELU_AUX_BIAS").free()
    plan_first_ms = (time.perf_counter() - t_plan) * 1e3
    t_plan = time.perf_counter()
    fplan = Plan(w.T, w.N, w.K, dt, "RELU_AUX_BIAS" if args.ffn_step else fwd_epi)
    plan_ms = (time.perf_counter() - t_plan) * 1e3
    bplan = None
    if has_bwd and not args.ffn_step:
        dY2, W2 = inp["dY2"], inp["W2"]
        dZ = torch.empty((w.T, w.N), dtype=dt, device=dev)
        dbias = torch.empty((w.N,), dtype=torch.float32, device=dev)
        t_plan = time.perf_counter()
        bplan = Plan(w.T, w.N, w.D2, dt, "DRELU_BGRAD")
        plan_ms = (plan_ms + (time.perf_counter() - t_plan) * 1e3) / 2
        if fwd_epi != "RELU_AUX_BIAS":  # the backward's mask comes from an untimed RELU_AUX_BIAS forward
            with Plan(w.T, w.N, w.K, dt, "RELU_AUX_BIAS") as mplan:
                mplan.gemm_epi_execute(X, W, b, Y, aux)
    if args.ablation:
        T1 = torch.empty((w.T, w.N), dtype=dt, device=dev)
        T2 = torch.empty((w.T, w.N), dtype=dt, device=dev)
        G = torch.empty((w.T, w.N), dtype=dt, device=dev)
    # L2 flush between steps: a 256 MiB write, then a read of another 256 MiB
    # buffer, so that L2 holds none of the step's inputs and no dirty line of
    # the flush itself is written back to HBM inside the timed events (with
    # the write alone, the T = 256, N = 11008, K = 4096 call measured 41.7 instead of
    # 34.8 us: the write-back of the flush's ~126 MB of dirty lines)
    flush_w = torch.empty(L2_FLUSH_BYTES, dtype=torch.uint8, device=dev)
    flush_r = torch.zeros(L2_FLUSH_BYTES // 8, dtype=torch.int64, device=dev)
    flush_sum = torch.empty((), dtype=torch.int64, device=dev)

    def flush_l2():
        flush_w.zero_()
        torch.sum(flush_r, dim=0, out=flush_sum)

    stream = torch.cuda.current_stream(dev)
    fwd_aux = (aux if fwd_epi == "RELU_AUX_BIAS" else
               torch.empty((w.T, w.N), dtype=dt, device=dev) if fwd_epi == "GELU_AUX_BIAS" else None)

    # prebuilt C calls: the timed loop does no per-call argument checking
    step_plans = None
    if args.ffn_step:  # a whole two-layer block step, weights in the [out, in] layout; D = K, F = N
        fplan.free()
        T, D, F = w.T, w.K, w.N
        si = synth.ffn_step_inputs(T, D, F, w.dtype, seed=w.seed, device=dev)
        t0 = time.perf_counter()
        sp = [Plan(T, F, D, dt, "RELU_AUX_BIAS", w_nk=True), Plan(T, D, F, dt, "BIAS", w_nk=True),
              Plan(T, F, D, dt, "DRELU_BGRAD"), Plan(T, F, D, dt, "WGRAD"), Plan(T, D, F, dt, "WGRAD"),
              Plan(T, D, F, dt, "NONE")]
        plan_ms = (time.perf_counter() - t0) * 1e3 / len(sp)
        H = torch.empty((T, F), dtype=dt, device=dev)
        aux1 = torch.empty((T, math.ceil(F / 32)), dtype=torch.int32, device=dev)
        Ys = torch.empty((T, D), dtype=dt, device=dev)
        dZ1 = torch.empty((T, F), dtype=dt, device=dev)
        db1 = torch.empty((F,), dtype=torch.float32, device=dev)
        dW2 = torch.empty((D, F), dtype=dt, device=dev)
        db2 = torch.empty((D,), dtype=torch.float32, device=dev)
        dW1 = torch.empty((F, D), dtype=dt, device=dev)
        dX = torch.empty((T, D), dtype=dt, device=dev)
        fcall = [sp[0].execute_call(si["X"], si["W1"], si["b1"], H, aux1, stream),
                 sp[1].execute_call(H, si["W2"], si["b2"], Ys, None, stream)]
        bcall = [sp[2].drelu_bgrad_call(si["dY"], si["W2"], aux1, dZ1, db1, stream),
                 sp[3].wgrad_call(si["dY"], H, dW2, db2, stream),
                 sp[4].wgrad_call(dZ1, si["X"], dW1, None, stream),
                 sp[5].execute_call(dZ1, si["W1"], None, dX, None, stream)]
        fplan, bplan = sp[0], sp[2]
        step_plans = sp
    elif args.wgrad:  # the weight gradient alone: dW (K x N) = X^T dZ, dZ a stand-in for the backward's
        fplan.free()
        dZw = synth.masked_grad(w.T, w.N, w.D2 or w.K, dt, seed=w.seed + 21, device=dev)
        fplan = Plan(w.T, w.N, w.K, dt, "WGRAD")
        dW = torch.empty((w.K, w.N), dtype=dt, device=dev)
        fcall = fplan.wgrad_call(X, dZw, dW, None, stream)
        bcall = None
    elif args.ablation:
        fcall = fplan.unfused_call(X, W, b, T1, T2 if fwd_epi != "BIAS" else Y, Y, fwd_aux, stream)
        bcall = bplan.drelu_bgrad_unfused_call(dY2, W2, aux, G, dZ, dbias, stream) if bplan is not None else None
    else:
        fcall = fplan.execute_call(X, W, b, Y, fwd_aux, stream)
        bcall = bplan.drelu_bgrad_call(dY2, W2, aux, dZ, dbias, stream) if bplan is not None else None

    def call(c):
        for fn, a in (c if isinstance(c, list) else [c]):
            rc = fn(*a)
            if rc != 0:
                raise RuntimeError(f"library call failed ({rc}): {binding.gemm_epi_last_error()}")

    def step(ev):
        ev[0].record(stream)
        call(fcall)
        ev[1].record(stream)
        if bcall is not None:
            call(bcall)
        ev[2].record(stream)

    def new_events():
        return [torch.cuda.Event(enable_timing=True) for _ in range(3)]

    def run_steps(evlist):
        # Steps are queued in chunks behind a short GPU sleep, so that the host
        # is ahead of the device and the events time the kernels, not the
        # host's launch latency (the e2e figure includes that).
        for c0 in range(0, len(evlist), QUEUE_CHUNK):
            torch.cuda._sleep(QUEUE_SLEEP_CYCLES)
            for ev in evlist[c0:c0 + QUEUE_CHUNK]:
                flush_l2()
                step(ev)

    uuid = None
    try:
        uuid = str(torch.cuda.get_device_properties(dev).uuid)
    except Exception:
        pass
    sampler = ClockSampler(uuid) if rank == 0 else None
    if sampler:
        sampler.start()
        time.sleep(0.05)
    torch.cuda.synchronize(dev)
    warm0 = time.time()
    run_steps([new_events() for _ in range(args.warmup)])
    torch.cuda.synchronize(dev)
    for p in (step_plans if args.ffn_step else (fplan, bplan)):
        if p is not None and p.status() != 0:
            raise RuntimeError("watchdog fired during warm-up")

    evs = [new_events() for _ in range(args.steps)]
    if world > 1:
        torch.distributed.barrier()
    torch.cuda.synchronize(dev)
    wall0 = time.time()
    run_steps(evs)
    torch.cuda.synchronize(dev)
    wall1 = time.time()
    if world > 1:
        torch.distributed.barrier()
    clocks = sampler.stop(wall0, wall1, warm0) if sampler else None
    for p in (step_plans if args.ffn_step else (fplan, bplan)):
        if p is not None and p.status() != 0:
            raise RuntimeError("watchdog fired during the timed region")

    fwd_ms = [e[0].elapsed_time(e[1]) for e in evs]
    bwd_ms = [e[1].elapsed_time(e[2]) for e in evs] if bplan is not None else [0.0] * args.steps
    spread = {"fwd_ms_median": statistics.median(fwd_ms), "fwd_ms_max": max(fwd_ms),
              "bwd_ms_median": statistics.median(bwd_ms), "bwd_ms_max": max(bwd_ms)}
    step_ms = sum(fwd_ms) / args.steps + sum(bwd_ms) / args.steps
    step_ms, fwd_avg, bwd_avg = max_over_ranks([step_ms, sum(fwd_ms) / args.steps, sum(bwd_ms) / args.steps], dev,
                                               world)

    alg = algorithmic(w, fwd_epi, bplan is not None)
    flops_step = sum(v["flops"] for v in alg.values())
    # our kernels per step, as the plans report them (the L2 flush between
    # steps is torch's and sits outside the timed events)
    launches_per_step = fplan.info()["launches"] + (bplan.info()["launches"] if bplan is not None else 0)
    if args.ffn_step:  # 2 forward GEMMs; DRELU_BGRAD, 2 WGRAD (+2 reduction launches for db2), NONE
        launches_per_step = 8
    if args.ablation:  # GEMM + bias + ReLU kernels; GEMM + mask + two column-sum kernels
        launches_per_step = (2 if fwd_epi == "BIAS" else 3) + (4 if bplan is not None else 0)

    # e2e: host buffers (pinned), H2D of the step's inputs, both calls, D2H of every output
    e2e = (run_e2e(args, w, fwd_epi, fplan, bplan, inp, dev, stream)
           if not (args.ablation or args.wgrad or args.ffn_step) else None)

    kernel = fplan.info()["kernel"]
    if args.ffn_step:
        for p in step_plans:
            p.free()
    else:
        fplan.free()
        if bplan is not None:
            bplan.free()
    return {"step_ms": step_ms, "fwd_ms": fwd_avg, "bwd_ms": bwd_avg, "alg": alg, "flops_step": flops_step,
            "kernel": kernel,
            "launches": launches_per_step * args.steps, "clocks": clocks, "e2e": e2e, "plan_ms": plan_ms,
            "plan_first_ms": plan_first_ms, "spread": spread,
            "wall_s": wall1 - wall0}


def run_e2e(args, w, fwd_epi, fplan, bplan, inp_dev, dev, stream):
    """End to end through the public calls with host buffers: every step copies
    all of its inputs from pinned host memory, runs the forward (and backward)
    call, and copies every output back. Steps are pipelined the way a training
    or serving loop runs them: inputs go up on one copy stream, results come
    down on another, the calls run on the compute stream, and two buffer sets
    alternate, so step i's results travel while step i+1's inputs do (the link
    is full duplex). Events order every reuse of a buffer set."""
    steps = max(1, min(args.steps, 20))
    host = {k: v.cpu().pin_memory() for k, v in inp_dev.items()}
    dt = w.torch_dtype
    aux_words = math.ceil(w.N / 32)
    h2d_s, d2h_s = torch.cuda.Stream(dev), torch.cuda.Stream(dev)

    spec = fplan.aux_spec()  # the forward's auxiliary output: mask words, or GELU's pre-activation
    has_aux = spec is not None

    def buffers():
        b = {"in": {k: torch.empty_like(v, device=dev) for k, v in host.items()},
             "Y": torch.empty((w.T, w.N), dtype=dt, device=dev),
             "aux": (torch.empty(spec[0], dtype=spec[1], device=dev) if has_aux and fwd_epi != "RELU_AUX_BIAS"
                     else torch.empty((w.T, aux_words), dtype=torch.int32, device=dev))}
        if bplan is not None:
            b["dZ"] = torch.empty((w.T, w.N), dtype=dt, device=dev)
            b["dbias"] = torch.empty((w.N,), dtype=torch.float32, device=dev)
        return b

    sets = [buffers(), buffers()]
    keys = ["Y"] + (["aux"] if has_aux else []) + (["dZ", "dbias"] if bplan is not None else [])
    hout = [{k: torch.empty_like(s[k], device="cpu").pin_memory() for k in keys} for s in sets]
    if bplan is not None and fwd_epi != "RELU_AUX_BIAS":  # the backward's mask, from an untimed forward
        with type(fplan)(w.T, w.N, w.K, dt, "RELU_AUX_BIAS") as mplan:
            for s_ in sets:
                mplan.gemm_epi_execute(inp_dev["X"], inp_dev["W"], inp_dev["bias"], s_["Y"], s_["aux"])
    h2d = sum(v.numel() * v.element_size() for v in host.values())
    d2h = sum(h.numel() * h.element_size() for h in hout[0].values())
    ev = lambda: torch.cuda.Event()  # noqa: E731
    computed = [None, None]  # event: the set's inputs consumed and outputs written
    drained = [None, None]   # event: the set's outputs copied to the host

    def one(i):
        b, ho = sets[i % 2], hout[i % 2]
        with torch.cuda.stream(h2d_s):
            if computed[i % 2] is not None:
                h2d_s.wait_event(computed[i % 2])  # inputs of step i-2 no longer read
            for k, v in host.items():
                b["in"][k].copy_(v, non_blocking=True)
            up = ev()
            up.record(h2d_s)
        stream.wait_event(up)
        if drained[i % 2] is not None:
            stream.wait_event(drained[i % 2])  # outputs of step i-2 already on the host
        fplan.gemm_epi_execute(b["in"]["X"], b["in"]["W"], b["in"]["bias"], b["Y"], b["aux"] if has_aux else None,
                               stream)
        if bplan is not None:
            bplan.drelu_bgrad_execute(b["in"]["dY2"], b["in"]["W2"], b["aux"], b["dZ"], b["dbias"], stream)
        done = ev()
        done.record(stream)
        computed[i % 2] = done
        with torch.cuda.stream(d2h_s):
            d2h_s.wait_event(done)
            for k in keys:
                ho[k].copy_(b[k], non_blocking=True)
            down = ev()
            down.record(d2h_s)
        drained[i % 2] = down

    for i in range(2):
        one(i)
    torch.cuda.synchronize(dev)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    h2d_s.wait_event(e0)
    d2h_s.wait_event(e0)
    for i in range(steps):
        one(i)
    stream.wait_stream(h2d_s)
    stream.wait_stream(d2h_s)
    e1.record(stream)
    torch.cuda.synchronize(dev)
    ms = e0.elapsed_time(e1) / steps
    return {"ms_per_step": ms, "steps": steps, "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
            "pipelined": "inputs up, results down and the calls on three streams, two buffer sets"}


# ------------------------------------------------------------ CPU oracle
def oracle_step_rows(w: synth.Workload, inp_cpu: dict, rows, fwd_epi: str, has_bwd: bool, threads: int):
    """The oracle on a sample of rows (every column): forward, then backward."""
    import numpy as np

    import oracle

    bits = synth.bits_u16
    dto = oracle.BF16 if w.dtype == "bf16" else oracle.F16
    t0 = time.perf_counter()
    f = oracle.linear_fwd(bits(inp_cpu["X"]), bits(inp_cpu["W"]), bits(inp_cpu["bias"]), dto, "RELU_AUX_BIAS",
                          rows=rows, threads=threads)
    macs = len(rows) * w.N * w.K
    if has_bwd:
        aux = np.zeros((w.T, math.ceil(w.N / 32)), dtype=np.uint32)
        aux[rows] = oracle.relu_aux_words(f["bits"])
        oracle.drelu_bgrad(bits(inp_cpu["dY2"]), bits(inp_cpu["W2"]), aux, dto, w.N, rows=rows, threads=threads)
        macs += len(rows) * w.N * w.D2
    return time.perf_counter() - t0, 2.0 * macs


def cpu_baseline(w: synth.Workload, fwd_epi: str, has_bwd: bool, target_s: float = 15.0):
    import oracle

    oracle.build()
    threads = oracle.default_threads()
    inp = synth.make_inputs(w, device="cpu")
    # grow the row sample until one run takes about target_s (each run also
    # pays a fixed cost for decoding W, so scale from the last measurement)
    rows = list(range(min(w.T, 8)))
    dt, fl = oracle_step_rows(w, inp, rows, fwd_epi, has_bwd, threads)
    for _ in range(3):
        if dt >= 0.6 * target_s or len(rows) >= w.T:
            break
        want = int(min(w.T, max(len(rows) + 1, len(rows) * target_s / max(dt, 1e-6))))
        rows = synth.sample_indices(w.T, want, seed=w.seed)
        dt, fl = oracle_step_rows(w, inp, rows, fwd_epi, has_bwd, threads)
    full_flops = 2.0 * w.T * w.N * w.K + (2.0 * w.T * w.N * w.D2 if has_bwd else 0.0)
    return {"value": fl / dt / 1e12, "unit": "TFLOP/s", "cores": threads, "kind": "oracle",
            "sample": f"{len(rows)} of {w.T} rows (every column), forward{' + backward' if has_bwd else ''}, "
                      f"fp64, {dt:.1f} s",
            # the whole step at the sample's rate (an extrapolation, not a measurement)
            "extrapolated_full_step_s": full_flops / (fl / dt)}


def run_reference(args, w: synth.Workload):
    """--impl reference: the oracle as it stands, on a bounded row sample per step."""
    import oracle

    fwd_epi, has_bwd = step_spec(w, args)
    oracle.build()
    threads = oracle.default_threads()
    inp = synth.make_inputs(w, device="cpu")
    budget = 150.0 / max(1, args.steps + args.warmup)  # seconds per step for a run of a few minutes
    n = min(w.T, 4)
    dt, _ = oracle_step_rows(w, inp, list(range(n)), fwd_epi, has_bwd, threads)
    rows_per_step = int(max(1, min(w.T, n * budget / max(dt, 1e-6))))
    times, flops = [], 0.0
    for i in range(args.warmup + args.steps):
        rows = synth.sample_indices(w.T, rows_per_step, seed=w.seed + 1000 + i)
        dt, fl = oracle_step_rows(w, inp, rows, fwd_epi, has_bwd, threads)
        if i >= args.warmup:
            times.append(dt)
            flops = fl
    ms = 1e3 * sum(times) / len(times)
    value = flops / (ms / 1e3) / 1e12
    sample = f"{rows_per_step} of {w.T} rows per step (every column), fp64"
    return {"metric": metric_name(w), "value": value, "unit": "TFLOP/s", "n_gpus": 0, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": ms, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "f64", "data": "synthetic", "impl": "reference",
            "config": config_of(w, fwd_epi, has_bwd, args),
            "cpu_baseline": {"value": value, "unit": "TFLOP/s", "cores": threads, "kind": "oracle", "sample": sample},
            "e2e": {"value": value, "unit": "TFLOP/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}


def metric_name(w: synth.Workload) -> str:
    return "fused GEMM+epilogue TFLOP/s (fwd RELU_AUX_BIAS, bwd DRELU_BGRAD), % of roofline"


def config_of(w, fwd_epi, has_bwd, args):
    desc = f"{w.name}: fwd {fwd_epi} T={w.T} K={w.K} N={w.N}"
    if fwd_epi == "FFN_STEP":
        desc = (f"{w.name}: two-layer block step, T={w.T} D={w.K} F={w.N} {w.dtype}, weights [out, in]: "
                f"H = relu(X W1^T + b1), Y = H W2^T + b2; dZ1, db1 = DRELU_BGRAD(dY, W2); dW2, db2; dW1; dX")
    if fwd_epi == "WGRAD":
        desc = (f"{w.name}: WGRAD dW (K x N) = X^T dZ over T={w.T}, K={w.K} N={w.N}; dZ a seeded stand-in "
                f"(N(0, D2/N), half zeros)")
    if has_bwd and fwd_epi != "FFN_STEP":
        desc += f" + bwd DRELU_BGRAD D2={w.D2}"
    desc += f", {w.dtype}"
    if args.ablation:
        desc += ", UNFUSED ablation (GEMM, then separate bias / ReLU+mask / mask / column-sum kernels)"
    return {"workload": desc, "T": w.T, "K": w.K, "N": w.N, "D2": w.D2, "dtype": w.dtype,
            "l2": ("flushed between steps outside the timed events: a 256 MiB write, then a read of another "
                   "256 MiB buffer (no dirty line of the flush is written back inside the events)"),
            "inputs": ("seeded synthetic: X~N(0,1), W1~N(0,1/D), W2~N(0,1/F), biases~N(0,0.1), dY~N(0,1)"
                       if fwd_epi == "FFN_STEP" else
                       "seeded synthetic: X~N(0,1), W~N(0,1/K), bias~N(0,0.1), dY2~N(0,1), W2~N(0,1/N)")}


# -------------------------------------------------------------------- main
def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=2000)
    ap.add_argument("--warmup", type=int, default=20)
    ap.add_argument("--workload", default="ffn", choices=sorted(synth.WORKLOADS))
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--ablation", action="store_true", help="time the unfused path instead")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--ffn-step", action="store_true",
                    help="time a whole two-layer block step (2 forward, 4 backward products) on the workload's shape")
    ap.add_argument("--wgrad", action="store_true",
                    help="time the weight gradient dW = X^T dZ alone on the workload's shape")
    ap.add_argument("--fwd-epilog", choices=["BIAS", "RELU_BIAS", "RELU_AUX_BIAS", "GELU_BIAS", "GELU_AUX_BIAS"],
                    default=None,
                    help="time this forward epilog alone on the workload's shape instead of its own step")
    args = ap.parse_args()
    if args.warmup < 3:
        ap.error("--warmup must be at least 3")
    w = synth.WORKLOADS[args.workload]
    fwd_epi, has_bwd = step_spec(w, args)

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))

    if args.impl == "reference":
        if rank == 0:
            print(json.dumps(run_reference(args, w)), flush=True)
        return

    if not torch.cuda.is_available():
        print(json.dumps({"metric": metric_name(w), "error": "no CUDA device"}))
        sys.exit(1)
    dev = torch.device("cuda", local)
    torch.cuda.set_device(dev)
    if world > 1:
        import datetime

        torch.distributed.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                             device_id=dev)
    res = run_ours(args, w, rank, world, dev)
    peaks, peak_src = load_peaks()
    if world > 1:
        torch.distributed.barrier()
        torch.distributed.destroy_process_group()
    if rank != 0:
        return

    value = whole_job_tflops(res["flops_step"], world, res["step_ms"])
    roof = roofline(w, fwd_epi, res, peaks, peak_src)

    line = {"metric": metric_name(w), "value": value, "unit": "TFLOP/s", "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": res["step_ms"], "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": w.dtype, "data": "synthetic",
            "config": config_of(w, fwd_epi, has_bwd, args),
            "parallelism": f"replicas x{world} (no exchange step)",
            "fwd_ms": res["fwd_ms"], "bwd_ms": res["bwd_ms"], "per_step_spread_rank0": res["spread"], "roofline": roof,
            "gpu_launches": res["launches"], "clocks": res["clocks"]}
    if res.get("plan_ms") is not None:
        line["plan_ms"] = res["plan_ms"]  # host time to create one plan (created once, reused every step)
        line["plan_first_ms"] = res["plan_first_ms"]  # the process's first plan, with one-time initialisation
    if res["e2e"]:
        e = res["e2e"]
        line["e2e"] = {"value": res["flops_step"] / (e["ms_per_step"] / 1e3) / 1e12, "unit": "TFLOP/s",
                       "h2d_bytes_per_step": e["h2d_bytes_per_step"], "d2h_bytes_per_step": e["d2h_bytes_per_step"],
                       "ms_per_step": e["ms_per_step"], "steps": e["steps"], "copies": e.get("pipelined")}
    if not args.no_cpu_baseline and world == 1:
        line["cpu_baseline"] = cpu_baseline(w, fwd_epi, has_bwd)
    print(json.dumps(line), flush=True)


def measured_traffic(w, part, fwd_epi):
    """DRAM bytes per launch of the timed call (keys "<workload>:fwd:<epilog>",
    "<workload>:bwd", "<workload>:wgrad") from the committed ncu summaries, if
    they were taken on the current kernel sources; else None."""
    path = os.path.join(ROOT, "profiles", "traffic.json")
    try:
        with open(path) as f:
            d = json.load(f)
    except Exception:
        return None
    current = kernel_source_hash()
    want = (f"{w.name}:wgrad" if fwd_epi == "WGRAD" else f"{w.name}:bwd" if part == "bwd"
            else f"{w.name}:fwd:{fwd_epi}")
    entry = d.get(want)
    if isinstance(entry, dict) and entry.get("source_hash") == current:
        return entry.get("dram_bytes_per_launch")
    return None


if __name__ == "__main__":
    main()
