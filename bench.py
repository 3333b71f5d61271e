"""Benchmark of the selective-scan hot path on B200 (one JSON line on stdout).

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

A step is one selective scan (discretise, recurrence, output, final state)
over the long-context workload, the largest single-GPU configuration: batch
1, length 1,048,576, 2048 channels, 16 states, bf16 inputs/outputs with fp32
state and arithmetic (12.95 GB of algorithmic traffic per step).  Inputs stay
resident in HBM and are far larger than L2, so no L2 flush is needed between
steps.  Timing is by CUDA events on the launching stream; for N > 1 (one
process per GPU under torchrun) every rank runs its own independent
workload, there is no collective on the data path, and the time is the max
over ranks.

Also reported on the same line:
  roofline   the scan call's algorithmic HBM bytes against the measured copy
             bandwidth (the metric's roof), with the FP32 FMA pipe under "alu"
  configs    every configuration of the workload list: tiny fp32, mid, large,
             long (the headline) and the decode chain, each with its time,
             token-channels/s and HBM fraction
  length_sweep  ns per token-channel of the long workload's generator for
             L = 2^14 .. 2^20 (linear scaling in length)
  e2e        the same metric through the public API from pinned host buffers,
             host<->device copies of each step's inputs and outputs included
  decode     the single-token state update on 256 x 5120 x 16 states, 1000
             steps with fresh inputs, captured in a CUDA graph
  variants, ssd  the scan's options and Mamba-2's scalar-A scan on the mid shape
  cpu_baseline  the fp64 CPU oracle on a strided channel subset of the workload
  clocks     SM clock and clock-event reasons sampled during the timed region
"""
from __future__ import annotations

import argparse
import hashlib
import json
import math
import os
import statistics
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

METRIC = "selective-scan token·channels/s and achieved HBM GB/s (% of B200 peak)"
UNIT = "token·channels/s"
FALLBACK_HBM_GBS = 6650.0
FALLBACK_BF16_TFLOPS = 1590.0
FMA_LANES_PER_SM = 128          # FP32 FMA results per clock per SM (sm_100)
FLOP_PER_STATE_STEP = 8         # 4 FMA per state and token: decay, input term, state update, output
FLOP_PER_TOKEN_CHANNEL = 4      # skip term and output scaling


def parse_args():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", default="long_bf16")
    ap.add_argument("--length", type=int, default=0,
                    help="override the workload's sequence length (smaller cases of the same generator, for profiling)")
    ap.add_argument("--decode-steps", type=int, default=1000)
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-decode", action="store_true")
    ap.add_argument("--no-variants", action="store_true",
                    help="skip the timings of the scan's options (general A, other discretisations, state counts)")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-configs", action="store_true", help="skip the per-configuration timings")
    ap.add_argument("--no-mimo", action="store_true", help="skip the multi-input multi-output leg")
    ap.add_argument("--no-sweep", action="store_true", help="skip the length sweep of the line")
    ap.add_argument("--no-ssd", action="store_true", help="skip Mamba-2's scalar-A scan (state space duality) leg")
    ap.add_argument("--only-backward", action="store_true",
                    help="run only the backward on the workload's shape (steps = timed calls) and print its object")
    ap.add_argument("--only-complex", action="store_true",
                    help="time only the complex-valued state scan on --workload (a small case for ncu)")
    ap.add_argument("--only-mimo", action="store_true",
                    help="time only the multi-input multi-output scan and step (a small case for ncu)")
    ap.add_argument("--only-ssd", action="store_true",
                    help="run only the scalar-A scan leg (steps/warmup as given) and print its object")
    ap.add_argument("--length-sweep", action="store_true",
                    help="instead of the benchmark line: ns per token-channel of the long-context workload's "
                         "generator (1 x L x 2048, bf16) for L = 2^14 .. 2^20 (linear scaling in length)")
    return ap.parse_args()


def measured_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            return json.load(f)
    except (OSError, ValueError):
        return {}


# device code of each profiled kernel (its launch shape -- tile, stages, warps --
# is in the kernel's template arguments, which the ncu summaries record)
KERNEL_SOURCES = {
    "scan_chunks_kernel": ("common.cuh", "scan.cuh"),
    "state_update_kernel": ("common.cuh", "scan.cuh", "decode.cuh"),
    "ssd_chunk_kernel": ("common.cuh", "ssd.cuh"),
    "scan_backward_kernel": ("common.cuh", "scan.cuh", "backward.cuh"),
}


def source_hash(kernel: str = "scan_chunks_kernel") -> str:
    """Hash of a kernel's device source: profile figures apply only to this exact code."""
    h = hashlib.sha256()
    csrc = os.path.join(ROOT, "selective_state_space_29_b200", "csrc")
    for name in KERNEL_SOURCES[kernel]:
        with open(os.path.join(csrc, name), "rb") as f:
            h.update(name.encode() + b"\0" + f.read())
    return h.hexdigest()[:16]


def profiled_traffic(kernel: str, workload: str):
    """dram bytes per launch from the committed ncu summary, if it was taken on
    the current source of that kernel; else None."""
    path = os.path.join(ROOT, "profiles", "traffic.json")
    try:
        with open(path) as f:
            rec = json.load(f)
    except (OSError, ValueError):
        return None
    for r in rec.get("entries", []):
        if r.get("kernel") == kernel and r.get("workload") == workload and r.get("source_hash") == source_hash(kernel):
            return r.get("dram_bytes_per_launch")
    return None


# --- clocks ---------------------------------------------------------------------

_REASONS = {0x1: "gpu_idle", 0x2: "applications_clocks_setting", 0x4: "sw_power_cap", 0x8: "hw_slowdown",
            0x10: "sync_boost", 0x20: "sw_thermal_slowdown", 0x40: "hw_thermal_slowdown",
            0x80: "hw_power_brake_slowdown", 0x100: "display_clock_setting"}


class ClockSampler:
    """Reads SM clock and clock-event reasons through NVML while running."""

    def __init__(self, torch_device_index: int, period_s: float = 0.005):
        self.samples = []
        self.max_mhz = None
        self.period = period_s
        self._stop = threading.Event()
        self._thread = None
        self.handle = None
        try:
            import pynvml
            import torch
            pynvml.nvmlInit()
            props = torch.cuda.get_device_properties(torch_device_index)
            uuid = str(getattr(props, "uuid", ""))
            try:
                self.handle = pynvml.nvmlDeviceGetHandleByUUID(("GPU-" + uuid) if uuid and not uuid.startswith("GPU-") else uuid)
            except Exception:
                vis = os.environ.get("CUDA_VISIBLE_DEVICES", "")
                idx = int(vis.split(",")[torch_device_index]) if vis and vis.split(",")[0].isdigit() else torch_device_index
                self.handle = pynvml.nvmlDeviceGetHandleByIndex(idx)
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self.handle, pynvml.NVML_CLOCK_SM)
            self._nvml = pynvml
        except Exception:
            self.handle = None

    def _read(self):
        p = self._nvml
        mhz = p.nvmlDeviceGetClockInfo(self.handle, p.NVML_CLOCK_SM)
        try:
            reasons = p.nvmlDeviceGetCurrentClocksEventReasons(self.handle)
        except Exception:
            reasons = p.nvmlDeviceGetCurrentClocksThrottleReasons(self.handle)
        return mhz, int(reasons)

    def _run(self):
        while not self._stop.is_set():
            try:
                self.samples.append(self._read())
            except Exception:
                pass
            time.sleep(self.period)

    def start(self):
        if self.handle is not None:
            self._thread = threading.Thread(target=self._run, daemon=True)
            self._thread.start()

    def stop(self):
        if self._thread is not None:
            self._stop.set()
            self._thread.join()
            try:
                self.samples.append(self._read())
            except Exception:
                pass

    def summary(self):
        if not self.samples:
            return {"sm_mhz": None, "sm_max_mhz": self.max_mhz, "reasons": [], "samples": 0}
        mhz = [s[0] for s in self.samples]
        bits = 0
        for _, r in self.samples:
            bits |= r
        names = [n for b, n in _REASONS.items() if bits & b and b != 0x1]
        return {"sm_mhz": statistics.median(mhz), "sm_max_mhz": self.max_mhz, "reasons": names,
                "samples": len(self.samples)}


# --- distributed plumbing -------------------------------------------------------------

def dist_setup(n_gpus: int):
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world != n_gpus:
        raise SystemExit(f"--gpus {n_gpus} but WORLD_SIZE={world}; launch N>1 with torchrun")
    return rank, world, local


def init_pg(world: int, local: int):
    import datetime

    import torch
    import torch.distributed as dist
    if world > 1:
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=torch.device("cuda", local))
    return dist


def barrier(dist, world):
    if world > 1:
        dist.barrier()


def max_over_ranks(dist, world, value: float, device="cuda") -> float:
    """Slowest rank's time: every rank calls this at the same point."""
    if world == 1:
        return value
    import torch
    t = torch.tensor([value], device=device, dtype=torch.float64)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def weak_scaling_value(world: int, units_per_rank: int, ms_per_step_max: float) -> float:
    """Whole-job throughput: units all ranks processed / the slowest rank's time."""
    return world * units_per_rank / (ms_per_step_max * 1e-3)


def rank_seed(base: int, rank: int) -> int:
    """Each rank draws its own independent workload."""
    return base + 1000 * rank


# --- algorithmic work -------------------------------------------------------------------

def scan_bytes(w) -> int:
    es = 2 if w.dtype == "bf16" else 4
    tc = w.batch * w.length * w.channels
    return (3 * tc * es                                 # u, delta read; y written
            + 2 * w.batch * w.length * w.nstate * es    # B, C read
            + w.channels * w.nstate * 4 + w.channels * 4  # A, D
            + w.batch * w.channels * w.nstate * 4)      # final state written


def scan_flops(w) -> int:
    tc = w.batch * w.length * w.channels
    return tc * (FLOP_PER_STATE_STEP * w.nstate + FLOP_PER_TOKEN_CHANNEL)


def decode_bytes_per_step(w) -> int:
    es = 2 if w.dtype == "bf16" else 4
    rows = w.batch * w.channels
    return (2 * rows * w.nstate * 4          # state read and written
            + 3 * rows * es                   # x, delta read; y written
            + 2 * w.batch * w.nstate * es     # B, C
            + w.channels * w.nstate * 4 + w.channels * 4)  # A, D


# --- CPU oracle baseline -------------------------------------------------------------------

def oracle_single_thread_tiny(budget_s: float = 1.0) -> dict:
    """tc/s of the fp64 oracle on one host thread over the tiny fp32 workload."""
    import oracle
    from selective_state_space_29_b200 import workloads as wl
    orc = oracle.get()
    w = wl.SCAN_WORKLOADS["tiny_f32"]
    inp = {k: v.to("cpu", copy=True).double().numpy() for k, v in wl.scan_inputs(w, "cpu").items()}
    reps, t0 = 0, time.perf_counter()
    while True:
        orc.scan(inp["u"], inp["delta"], inp["A"], inp["B"], inp["C"], inp["D"], nthreads=1)
        reps += 1
        dt = time.perf_counter() - t0
        if dt >= budget_s:
            break
    tc = w.batch * w.length * w.channels
    return {"value": reps * tc / dt, "unit": UNIT, "cores": 1, "reps": reps}


# --- our implementation ---------------------------------------------------------------

def time_calls(fn, stream, dist, world, reps: int, warmup: int = 3) -> float:
    """Mean device time of one call (ms), CUDA events on the launching stream
    around each call, max over ranks."""
    import torch
    for _ in range(warmup):
        fn()
    torch.cuda.synchronize()
    barrier(dist, world)
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(reps)]
    for a, b in ev:
        a.record(stream)
        fn()
        b.record(stream)
    torch.cuda.synchronize()
    return max_over_ranks(dist, world, statistics.mean(a.elapsed_time(b) for a, b in ev))


def scan_caller(lib, m, inp, y, hf, w, length, stream):
    """One mamba_selective_scan call over the first `length` tokens of the
    workload's tensors (contiguous prefixes for batch 1)."""
    dtc = m.dtype_code(w.torch_dtype)
    ptrs = [inp[k].data_ptr() for k in ("u", "delta", "A", "B", "C", "D")] + [y.data_ptr(), hf.data_ptr()]
    sh = stream.cuda_stream

    def call():
        st = lib.mamba_selective_scan(*ptrs, w.batch, length, w.channels, w.nstate, dtc, sh)
        if st != 0:
            raise m.MambaError(st, "mamba_selective_scan")
    return call


def hbm_entry(nbytes: int, ms: float, hbm_peak: float) -> dict:
    ach = nbytes / (ms * 1e-3) / 1e9
    return {"achieved_gbs": round(ach, 1), "frac": round(ach / hbm_peak, 4), "algorithmic_bytes": nbytes}


def run_configs(args, headline, dev, stream, dist, world, rank, hbm_peak, decode_res):
    """Time, token-channels/s and HBM fraction of every configuration of the
    workload list; the headline's own figures are reused, not re-measured."""
    import torch

    from selective_state_space_29_b200 import mamba_ssm as m
    from selective_state_space_29_b200 import workloads as wl
    lib = m.library()
    res = {}
    reps = {"tiny_f32": 200, "mid_bf16": 50, "large_bf16": 20}
    for name in ("tiny_f32", "mid_bf16", "large_bf16", "long_bf16"):
        w = wl.SCAN_WORKLOADS[name]
        if name == headline["name"]:
            ms = headline["ms"]
        else:
            inp = wl.scan_inputs(w, dev, seed=rank_seed(w.seed, rank))
            y = torch.empty_like(inp["u"])
            hf = torch.empty((w.batch, w.channels, w.nstate), device=dev, dtype=torch.float32)
            ms = time_calls(scan_caller(lib, m, inp, y, hf, w, w.length, stream), stream, dist, world,
                            reps.get(name, 5))
            del inp, y, hf
        tc = w.batch * w.length * w.channels
        e = {"ms_per_call": round(ms, 5), "token_channels_per_s": world * tc / (ms * 1e-3),
             "shape": f"batch {w.batch}, len {w.length}, channels {w.channels}, state {w.nstate}, {w.dtype} I/O"}
        e.update({"hbm_" + k: v for k, v in hbm_entry(scan_bytes(w), ms, hbm_peak).items()})
        if name == "tiny_f32":
            e["note"] = "16,384 token-channels: launch latency, not bandwidth, sets the time"
        res[name] = e
    if decode_res is not None:
        r = decode_res["roofline"]
        res["decode_bf16"] = {"ms_per_step": decode_res["ms_per_step"],
                              "updates_per_s": decode_res["updates_per_s"],
                              "hbm_achieved_gbs": r["achieved"], "hbm_frac": r["frac"],
                              "hbm_algorithmic_bytes": r["algorithmic_bytes_per_launch"]}
    return res


def run_length_sweep_on(inp, y, hf, w, dev, stream, dist, world, steps: int = 20) -> dict:
    """ns per token-channel of the long workload's generator over its first L
    tokens, L = 2^14 .. len, on the already resident input."""
    from selective_state_space_29_b200 import mamba_ssm as m
    lib = m.library()
    dtc = m.dtype_code(w.torch_dtype)
    rows = []
    L = 1 << 14
    while L <= w.length:
        reps = max(5, min(steps, int(2e9 // (w.channels * L))))
        ms = time_calls(scan_caller(lib, m, inp, y, hf, w, L, stream), stream, dist, world, reps)
        plan = m.mamba_scan_plan(w.batch, L, w.channels, w.nstate, 0, dtc)
        rows.append({"len": L, "ms": round(ms, 5), "ns_per_tc": round(ms * 1e6 / (w.channels * L), 6),
                     "reps": reps, "supers": int(plan.supers)})
        L *= 2
    v = [r["ns_per_tc"] for r in rows]
    ref = v[-1]
    return {"rows": rows, "workload": f"{w.name} generator, batch 1, {w.channels} channels, prefixes of one input",
            "max_over_min_ns_per_tc": round(max(v) / min(v), 4),
            "max_dev_from_longest": round(max(abs(x / ref - 1.0) for x in v), 4),
            "linear_within_10pct": bool(all(abs(x / ref - 1.0) <= 0.10 for x in v))}


def oracle_strided_rate(inp, w, stride: int, budget_s: float):
    """tc/s of the fp64 oracle over every `stride`-th channel of batch row 0
    (whole rows: per-channel independence makes each exact), growing the
    number of channels until it takes budget_s seconds or covers the stride."""
    import torch

    import oracle
    orc = oracle.get()
    all_ch = list(range(0, w.channels, stride))
    n = min(len(all_ch), 16)
    while True:
        ch = torch.tensor(all_ch[:n], device=inp["u"].device)
        arrs = [inp["u"][:1].index_select(2, ch), inp["delta"][:1].index_select(2, ch),
                inp["A"].index_select(0, ch), inp["B"][:1], inp["C"][:1], inp["D"].index_select(0, ch)]
        arrs = [a.to(torch.float64).cpu().numpy() for a in arrs]
        t0 = time.perf_counter()
        orc.scan(*arrs)
        dt = time.perf_counter() - t0
        del arrs
        if dt >= budget_s or n >= len(all_ch):
            break
        n = min(len(all_ch), max(2 * n, int(n * budget_s / max(dt, 1e-3))))
    tc = n * w.length
    return {"value": tc / dt, "rows": n, "seconds": dt, "tc": tc}, orc.max_threads()


def run_ours(args):
    import torch

    from selective_state_space_29_b200 import mamba_ssm as m
    from selective_state_space_29_b200 import workloads as wl

    rank, world, local = dist_setup(args.gpus)
    torch.cuda.set_device(local)
    dist = init_pg(world, local)
    dev = torch.device("cuda", local)
    peaks = measured_peaks()
    hbm_peak = float(peaks.get("hbm_gbs", FALLBACK_HBM_GBS))
    hbm_src = "measured" if "hbm_gbs" in peaks else "fallback"

    w = wl.SCAN_WORKLOADS[args.workload]
    if args.length > 0:
        w = w.with_(length=args.length, name=f"{w.name}_len{args.length}")
    inp = wl.scan_inputs(w, dev, seed=rank_seed(w.seed, rank))
    y = torch.empty_like(inp["u"])
    hf = torch.empty((w.batch, w.channels, w.nstate), device=dev, dtype=torch.float32)
    dtc = m.dtype_code(w.torch_dtype)
    plan = m.mamba_scan_plan(w.batch, w.length, w.channels, w.nstate, 0, dtc)
    lib = m.library()
    stream = torch.cuda.current_stream(dev)
    step = scan_caller(lib, m, inp, y, hf, w, w.length, stream)

    for _ in range(max(args.warmup, 3)):
        step()
    torch.cuda.synchronize()
    barrier(dist, world)
    K = args.steps
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(K)]
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    sampler = ClockSampler(local)
    torch.cuda.synchronize()
    barrier(dist, world)
    sampler.start()
    e0.record(stream)
    for i in range(K):
        ev[i][0].record(stream)
        step()
        ev[i][1].record(stream)
    e1.record(stream)
    torch.cuda.synchronize()
    sampler.stop()
    barrier(dist, world)
    total_ms = e0.elapsed_time(e1)
    call_ms = statistics.mean(a.elapsed_time(b) for a, b in ev)
    total_ms_max = max_over_ranks(dist, world, total_ms)
    ms_step = total_ms_max / K
    tc = w.batch * w.length * w.channels
    value = weak_scaling_value(world, tc, ms_step)
    if m.mamba_get_device_error(clear=False) != 0:
        raise RuntimeError("device error word set during the benchmark")
    clocks = sampler.summary()

    # roofline of the scan call (per launch, from the per-call event timing):
    # the metric's roof is HBM; the FP32 pipe figure is kept beside it
    sms = torch.cuda.get_device_properties(dev).multi_processor_count
    max_mhz = clocks.get("sm_max_mhz") or float(peaks.get("sm_max_mhz", 1965.0))
    alu_peak = sms * FMA_LANES_PER_SM * 2 * max_mhz * 1e6 / 1e12        # TFLOP/s
    flops = scan_flops(w)
    nbytes = scan_bytes(w)
    alu_ach = flops / (call_ms * 1e-3) / 1e12
    hbm_ach = nbytes / (call_ms * 1e-3) / 1e9
    roofline = {"bound": "hbm", "achieved": round(hbm_ach, 1), "peak": hbm_peak, "unit": "GB/s",
                "frac": round(hbm_ach / hbm_peak, 4),
                "traffic": profiled_traffic("scan_chunks_kernel", args.workload),
                "peak_source": ("measured (MEASURED_PEAKS.json hbm_gbs)" if hbm_src == "measured" else
                                f"fallback: the profiling recipe's {FALLBACK_HBM_GBS:.0f} GB/s (no MEASURED_PEAKS.json)"),
                "kernel": "scan_chunks_kernel (timed per call: the call's pre-pass included)",
                "call_ms": round(call_ms, 5), "algorithmic_bytes_per_launch": nbytes,
                "bytes_per_tc": round(nbytes / tc, 4),
                "alu": {"achieved": round(alu_ach, 3), "peak": round(alu_peak, 3), "unit": "TFLOP/s",
                        "frac": round(alu_ach / alu_peak, 4), "flop_per_launch": flops,
                        "peak_source": f"derived: {sms} SMs x {FMA_LANES_PER_SM} FP32 FMA/clk x 2 x "
                                       f"{max_mhz:.0f} MHz"}}

    out = {"metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": K, "warmup": args.warmup,
           "ms_per_step": ms_step, "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
           "dtype": "f32", "data": "synthetic",
           "config": {"workload": f"{w.name}: batch {w.batch}, len {w.length}, channels {w.channels}, "
                                  f"state {w.nstate}, {w.dtype} I/O, fp32 state",
                      "batch": w.batch, "len": w.length, "channels": w.channels, "nstate": w.nstate,
                      "io_dtype": w.dtype, "state_dtype": "f32", "global_batch": w.batch * world,
                      "l2": f"inputs larger than L2 ({nbytes / 1e6:.0f} MB per step), no flush",
                      "parallelism": f"independent workload per GPU x{world}", "plan": plan.as_dict()},
           "roofline": roofline, "gpu_launches": int(K * plan.kernels), "clocks": clocks}

    # the long workload's length sweep, on the resident input (batch 1 only)
    if not args.no_sweep and w.batch == 1 and w.length >= (1 << 15):
        out["length_sweep"] = run_length_sweep_on(inp, y, hf, w, dev, stream, dist, world)

    # end to end through the public API from pinned host buffers, copies timed:
    # mamba_selective_scan_host (copies pipelined with the scan piece by
    # piece), and for comparison whole-tensor copies around the device call
    if not args.no_e2e:
        host = {k: v.cpu().pin_memory() for k, v in inp.items()}
        dbuf = {k: torch.empty_like(v) for k, v in inp.items()}
        y_host = torch.empty(y.shape, dtype=y.dtype).pin_memory()
        hf_host = torch.empty(hf.shape, dtype=hf.dtype).pin_memory()
        h2d = sum(v.numel() * v.element_size() for v in host.values())
        d2h = y_host.numel() * y_host.element_size() + hf_host.numel() * hf_host.element_size()
        Ke = max(3, min(K, 30 if nbytes < 2e9 else 5))

        def e2e_step():
            m.mamba_selective_scan_host(host["u"], host["delta"], host["A"], host["B"], host["C"], host["D"],
                                        y_host, hf_host, w.batch, w.length, w.channels, w.nstate, 0, dtc, stream)

        def e2e_plain_step():
            for k in host:
                dbuf[k].copy_(host[k], non_blocking=True)
            m.selective_scan(dbuf["u"], dbuf["delta"], dbuf["A"], dbuf["B"], dbuf["C"], dbuf["D"], y=y,
                             final_state=hf, stream=stream)
            y_host.copy_(y, non_blocking=True)
            hf_host.copy_(hf, non_blocking=True)

        def time_e2e(fn):
            for _ in range(2):
                fn()
            torch.cuda.synchronize()
            barrier(dist, world)
            a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            a.record(stream)
            for _ in range(Ke):
                fn()
            b.record(stream)
            torch.cuda.synchronize()
            return max_over_ranks(dist, world, a.elapsed_time(b)) / Ke

        e2e_ms = time_e2e(e2e_step)
        plain_ms = time_e2e(e2e_plain_step)
        out["e2e"] = {"value": world * tc / (e2e_ms * 1e-3), "unit": UNIT, "h2d_bytes_per_step": h2d,
                      "d2h_bytes_per_step": d2h, "ms_per_step": e2e_ms, "steps": Ke,
                      "call": "mamba_selective_scan_host (pinned host buffers, copies overlapped piecewise)",
                      "unpipelined": {"value": world * tc / (plain_ms * 1e-3), "ms_per_step": plain_ms,
                                      "call": "copies of whole tensors around mamba_selective_scan"}}
        del host, dbuf, y_host, hf_host

    # CPU oracle on every 16th channel of the headline workload (rank 0, single GPU only)
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        best, cores = oracle_strided_rate(inp, w, stride=16, budget_s=15.0)
        out["cpu_baseline"] = {"value": best["value"], "unit": UNIT, "cores": cores, "kind": "oracle",
                               "sample": f"{best['rows']} channels (every 16th) of batch row 0 x {w.length} "
                                         f"tokens of {w.name} ({best['seconds']:.1f} s, fp64)",
                               "single_thread_tiny_f32": oracle_single_thread_tiny()}
    headline = {"name": w.name, "ms": call_ms}
    del inp, y, hf
    torch.cuda.empty_cache()

    # the scan's options and Mamba-2's scalar-A scan, on the mid shape
    mid = wl.SCAN_WORKLOADS["mid_bf16"]
    if not args.no_variants:
        out["variants"] = run_variants(mid, dev, stream, dist, world, rank)
    if not args.no_ssd:
        out["ssd"] = run_ssd(args, dev, stream, dist, world, rank, hbm_peak, hbm_src, peaks)
    if not args.no_mimo:
        out["mimo"] = run_mimo(dev, stream, dist, world, rank, hbm_peak)

    # decode: 1000 single-token steps on 256 x 5120 x 16 states
    decode_res = None
    if not args.no_decode:
        decode_res = run_decode(args, dev, stream, dist, world, rank, hbm_peak, hbm_src)
        out["decode"] = decode_res

    # every configuration of the workload list
    if not args.no_configs:
        out["configs"] = run_configs(args, headline, dev, stream, dist, world, rank, hbm_peak, decode_res)

    if world > 1:
        dist.destroy_process_group()
    if rank == 0:
        print(json.dumps(out), flush=True)


def run_decode(args, dev, stream, dist, world, rank, hbm_peak, hbm_src):
    import torch

    from selective_state_space_29_b200 import mamba_ssm as m
    from selective_state_space_29_b200 import workloads as wl

    w = wl.DECODE_WORKLOADS["decode_bf16"]
    steps = args.decode_steps
    prm = wl.decode_params(w, dev, seed=rank_seed(w.seed, rank))
    chain = wl.decode_chain_inputs_bulk(w, steps, dev, seed=rank_seed(w.seed, rank))
    state = prm["state"].clone()
    y = torch.empty((steps, w.batch, w.channels), device=dev, dtype=w.torch_dtype)
    lib = m.library()
    dtc = m.dtype_code(w.torch_dtype)
    sh = stream.cuda_stream
    x, dl, B, C = chain["x"], chain["delta"], chain["B"], chain["C"]
    sx, sb = x[0].numel() * x.element_size(), B[0].numel() * B.element_size()

    def run_chain(sh):
        for s in range(steps):
            st = lib.mamba_state_update(state.data_ptr(), x.data_ptr() + s * sx, dl.data_ptr() + s * sx,
                                        prm["A"].data_ptr(), B.data_ptr() + s * sb, C.data_ptr() + s * sb,
                                        prm["D"].data_ptr(), y.data_ptr() + s * sx, w.batch, w.channels,
                                        w.nstate, dtc, sh)
            if st != 0:
                raise m.MambaError(st, "mamba_state_update")

    run_chain(sh)                    # warm-up pass over the whole chain
    torch.cuda.synchronize()
    # plain launches, one C call per step
    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    a.record(stream)
    run_chain(sh)
    b.record(stream)
    torch.cuda.synchronize()
    plain_ms = max_over_ranks(dist, world, a.elapsed_time(b)) / steps
    # the same chain captured once in a CUDA graph (no per-launch host cost)
    graph_ms = None
    try:
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g):
            run_chain(torch.cuda.current_stream().cuda_stream)
        g.replay()
        torch.cuda.synchronize()
        a.record(stream)
        g.replay()
        b.record(stream)
        torch.cuda.synchronize()
        graph_ms = max_over_ranks(dist, world, a.elapsed_time(b)) / steps
        del g
    except Exception as exc:  # the graph only removes launch overhead from the measurement
        sys.stderr.write(f"decode graph capture failed: {exc}\n")
    ms = graph_ms if graph_ms is not None else plain_ms
    nb = decode_bytes_per_step(w)
    ach = nb / (ms * 1e-3) / 1e9
    return {"workload": f"{w.name}: {w.batch} sequences x {w.channels} channels x {w.nstate} states, "
                        f"{steps} steps, fp32 state, {w.dtype} x/delta/B/C/y",
            "ms_per_step": ms, "ms_per_step_plain_launches": plain_ms,
            "updates_per_s": world * w.batch * w.channels / (ms * 1e-3),
            "roofline": {"bound": "hbm", "achieved": round(ach, 1), "peak": hbm_peak, "unit": "GB/s",
                         "frac": round(ach / hbm_peak, 4), "traffic": profiled_traffic("state_update_kernel", w.name),
                         "algorithmic_bytes_per_launch": nb, "peak_source": hbm_src,
                         "note": "the 84 MB state fits in L2; DRAM traffic per launch is in the ncu summary"},
            "gpu_launches": steps}


def ssd_bytes(w) -> int:
    """Algorithmic bytes of one scalar-A scan call: x read, y written, dt, B,
    C, the final state, A and D."""
    es = 2
    return (w.batch * w.length * w.channels * es * 2 + w.batch * w.length * w.heads * es
            + 2 * w.batch * w.length * w.nstate * es + w.batch * w.channels * w.nstate * 4
            + w.heads * 4 + w.channels * 4)


SSD_CHUNK = 64    # tokens per chunk of mamba_ssd_scan


def ssd_mma_flops(w) -> int:
    """Tensor-core FLOPs of the chunked form per call: per chunk of Q tokens
    and head, C S_in (Q x N x 64), the causal 16 x 16 blocks of C B^T (nb
    blocks of 16 x N x 16) and of M X (nb of 16 x 16 x 64), and B_w^T X
    (N x Q x 64); nb = k(k+1)/2 with k = Q/16."""
    q, p, n = SSD_CHUNK, 64, w.nstate
    nb = (q // 16) * (q // 16 + 1) // 2
    per_chunk = 2 * (q * n * p + nb * 16 * n * 16 + nb * 16 * 16 * p + n * q * p)
    chunks = -(-w.length // q)
    return w.batch * w.heads * chunks * per_chunk


def run_ssd(args, dev, stream, dist, world, rank, hbm_peak, hbm_src, peaks):
    """Mamba-2's scalar-A scan (mamba_ssd_scan) on the mid shape as 48 heads
    of 64 channels (device-timed per call, K calls), and on the long shape."""
    import torch

    from selective_state_space_29_b200 import mamba_ssm as m
    from selective_state_space_29_b200 import workloads as wl

    lib = m.library()
    sh = stream.cuda_stream
    res = {}
    for name, K in (("ssd_mid_bf16", max(args.steps, 3)), ("ssd_long_bf16", 3)):
        if args.only_ssd and name != "ssd_mid_bf16":
            continue
        w = wl.SSD_WORKLOADS[name]
        inp = wl.ssd_inputs(w, dev, seed=rank_seed(w.seed, rank))
        y = torch.empty_like(inp["x"])
        hf = torch.empty((w.batch, w.channels, w.nstate), device=dev, dtype=torch.float32)
        ptrs = [inp[k].data_ptr() for k in ("x", "dt", "A", "B", "C", "D")] + [None, y.data_ptr(), hf.data_ptr()]

        def step():
            st = lib.mamba_ssd_scan(*ptrs, w.batch, w.length, w.heads, w.headdim, w.nstate, 0, 0, m.MAMBA_BF16, sh)
            if st != 0:
                raise m.MambaError(st, "mamba_ssd_scan")

        for _ in range(max(args.warmup, 3)):
            step()
        torch.cuda.synchronize()
        barrier(dist, world)
        ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(K)]
        for i in range(K):
            ev[i][0].record(stream)
            step()
            ev[i][1].record(stream)
        torch.cuda.synchronize()
        call_ms = max_over_ranks(dist, world, statistics.mean(a.elapsed_time(b) for a, b in ev))
        nb, fl = ssd_bytes(w), ssd_mma_flops(w)
        ach = nb / (call_ms * 1e-3) / 1e9
        tpk = float(peaks.get("bf16_tflops", FALLBACK_BF16_TFLOPS))
        tfl = fl / (call_ms * 1e-3) / 1e12
        res[name] = {
            "workload": f"{w.name}: batch {w.batch}, len {w.length}, {w.heads} heads x {w.headdim} channels, "
                        f"state {w.nstate}, bf16 I/O, fp32 state",
            "ms_per_call": round(call_ms, 5), "calls": K,
            "token_channels_per_s": world * w.token_channels / (call_ms * 1e-3),
            "roofline": {"bound": "hbm", "achieved": round(ach, 1), "peak": hbm_peak, "unit": "GB/s",
                         "frac": round(ach / hbm_peak, 4), "traffic": profiled_traffic("ssd_chunk_kernel", w.name),
                         "algorithmic_bytes_per_launch": nb, "peak_source": hbm_src,
                         "tensor": {"achieved": round(tfl, 2), "peak": tpk, "unit": "TFLOP/s",
                                    "frac": round(tfl / tpk, 4), "flop_per_launch": fl,
                                    "peak_source": "measured bf16" if "bf16_tflops" in peaks else "fallback"}},
            "l2": f"inputs larger than L2 ({nb / 1e6:.0f} MB per call), no flush"}
        del inp, y, hf
    return res


def mimo_bytes(w) -> int:
    """Algorithmic bytes of one multi-input multi-output scan call: R inputs
    read and R outputs written per token and channel, Delta, the R rows of B
    and C per token, A, D and the final state."""
    es = 2 if w.dtype == "bf16" else 4
    tc = w.batch * w.length * w.channels
    return (2 * w.ranks * tc * es + tc * es + 2 * w.batch * w.length * w.ranks * w.nstate * es
            + w.channels * (w.nstate + 1) * 4 + w.batch * w.channels * w.nstate * 4)


def mimo_decode_bytes_per_step(batch, ranks, channels, nstate, es=2) -> int:
    rows = batch * channels
    return (2 * rows * nstate * 4 + (2 * ranks + 1) * rows * es + 2 * batch * ranks * nstate * es
            + channels * (nstate + 1) * 4)


def run_mimo(dev, stream, dist, world, rank, hbm_peak, reps: int = 20) -> dict:
    """The multi-input multi-output scan on the mid shape with 4 inputs and
    outputs per channel, and its single-token step on the decode shape
    (256 x 5120 x 16 states, 4 inputs and outputs per row)."""
    import torch

    from selective_state_space_29_b200 import mamba_ssm as m
    from selective_state_space_29_b200 import workloads as wl
    lib = m.library()
    w = wl.MIMO_WORKLOADS["mimo_mid_bf16"]
    inp = wl.mimo_inputs(w, dev, seed=rank_seed(w.seed, rank))
    y = torch.empty_like(inp["u"])
    hf = torch.empty((w.batch, w.channels, w.nstate), device=dev, dtype=torch.float32)
    dtc = m.dtype_code(w.torch_dtype)

    def call():
        st = lib.mamba_selective_scan_mimo(inp["u"].data_ptr(), inp["delta"].data_ptr(), inp["A"].data_ptr(),
                                           inp["B"].data_ptr(), inp["C"].data_ptr(), inp["D"].data_ptr(), None,
                                           y.data_ptr(), hf.data_ptr(), w.batch, w.length, w.ranks, w.channels,
                                           w.nstate, 0, dtc, stream.cuda_stream)
        if st != 0:
            raise m.MambaError(st, "mamba_selective_scan_mimo")

    ms = time_calls(call, stream, dist, world, reps)
    tc = w.token_channels
    res = {"scan": {"workload": f"{w.name}: batch {w.batch}, len {w.length}, {w.ranks} inputs/outputs x "
                                f"{w.channels} channels, state {w.nstate}, {w.dtype} I/O, fp32 state",
                    "ms_per_call": round(ms, 5), "token_channels_per_s": world * tc / (ms * 1e-3),
                    "outputs_per_s": world * tc * w.ranks / (ms * 1e-3),
                    **{"hbm_" + k: v for k, v in hbm_entry(mimo_bytes(w), ms, hbm_peak).items()}}}
    del inp, y, hf
    # decode step: 256 x 5120 rows, 4 inputs and outputs each, 200 steps with fresh inputs
    B_, R_, C_, N_, steps = 256, 4, 5120, 16, 200
    g = torch.Generator(device=dev).manual_seed(rank_seed(37, rank))
    A = -(torch.arange(1, N_ + 1, device=dev, dtype=torch.float32) * (1.0 + 0.1 * torch.rand((C_, 1), generator=g, device=dev))).contiguous()
    D = torch.randn(C_, generator=g, device=dev)
    state = 0.1 * torch.randn((B_, C_, N_), generator=g, device=dev)
    x = torch.randn((steps, B_, R_, C_), generator=g, device=dev).to(torch.bfloat16)
    dl = torch.exp(torch.empty((steps, B_, C_), device=dev).uniform_(math.log(1e-3), math.log(1e-1), generator=g)).to(torch.bfloat16)
    Bm = torch.randn((steps, B_, R_, N_), generator=g, device=dev).to(torch.bfloat16)
    Cm = torch.randn((steps, B_, R_, N_), generator=g, device=dev).to(torch.bfloat16)
    yd = torch.empty((steps, B_, R_, C_), device=dev, dtype=torch.bfloat16)
    sx, sd, sb = x[0].numel() * 2, dl[0].numel() * 2, Bm[0].numel() * 2

    def chain():
        for s in range(steps):
            st = lib.mamba_state_update_mimo(state.data_ptr(), x.data_ptr() + s * sx, dl.data_ptr() + s * sd,
                                             A.data_ptr(), Bm.data_ptr() + s * sb, Cm.data_ptr() + s * sb,
                                             D.data_ptr(), yd.data_ptr() + s * sx, B_, R_, C_, N_, m.MAMBA_BF16,
                                             stream.cuda_stream)
            if st != 0:
                raise m.MambaError(st, "mamba_state_update_mimo")

    ms_d = time_calls(chain, stream, dist, world, 3, warmup=1) / steps
    nb = mimo_decode_bytes_per_step(B_, R_, C_, N_)
    res["decode"] = {"workload": f"{B_} sequences x {C_} channels x {N_} states, {R_} inputs/outputs per row, "
                                 f"{steps} steps, fp32 state, bf16 x/delta/B/C/y (plain launches)",
                     "ms_per_step": round(ms_d, 5), "outputs_per_s": world * B_ * C_ * R_ / (ms_d * 1e-3),
                     **{"hbm_" + k: v for k, v in hbm_entry(nb, ms_d, hbm_peak).items()}}
    del state, x, dl, Bm, Cm, yd
    return res


def run_complex(w, dev, stream, dist, world, rank, reps: int = 20) -> dict:
    """ms per call of the complex-valued state scan on the workload's shape
    (complex diagonal A with imaginary parts pi n, complex state)."""
    import torch

    from selective_state_space_29_b200 import mamba_ssm as m
    from selective_state_space_29_b200 import workloads as wl

    lib = m.library()
    dtc = m.dtype_code(w.torch_dtype)
    tc = w.batch * w.length * w.channels
    inp = wl.scan_inputs(w, dev, seed=rank_seed(w.seed, rank))
    A_im = wl.complex_a_imag(w.channels, w.nstate, dev)
    y = torch.empty_like(inp["u"])
    hf = torch.empty((w.batch, w.channels, w.nstate, 2), device=dev, dtype=torch.float32)

    def cstep():
        st = lib.mamba_selective_scan_complex(inp["u"].data_ptr(), inp["delta"].data_ptr(), inp["A"].data_ptr(),
                                              A_im.data_ptr(), inp["B"].data_ptr(), inp["C"].data_ptr(),
                                              inp["D"].data_ptr(), None, y.data_ptr(), hf.data_ptr(), w.batch,
                                              w.length, w.channels, w.nstate, 0, dtc, stream.cuda_stream)
        if st != 0:
            raise m.MambaError(st, "mamba_selective_scan_complex")

    for _ in range(3):
        cstep()
    torch.cuda.synchronize()
    barrier(dist, world)
    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    a.record(stream)
    for _ in range(reps):
        cstep()
    b.record(stream)
    torch.cuda.synchronize()
    ms = max_over_ranks(dist, world, a.elapsed_time(b)) / reps
    del inp, A_im, y, hf
    return {"ms_per_call": round(ms, 5), "token_channels_per_s": world * tc / (ms * 1e-3),
            "nstate": w.nstate, "note": "complex diagonal A (imaginary parts pi n), complex state"}


def run_variants(w, dev, stream, dist, world, rank, reps: int = 20):
    """ms per call and token·channels/s of the scan's options on the workload's
    shape: MAMBA_SCAN_GENERAL_A, MAMBA_SCAN_EULER, MAMBA_SCAN_TRAPEZOID, and 4, 8
    and 32 states (zero-order hold, structured A)."""
    import torch

    from selective_state_space_29_b200 import mamba_ssm as m
    from selective_state_space_29_b200 import workloads as wl

    lib = m.library()
    dtc = m.dtype_code(w.torch_dtype)
    tc = w.batch * w.length * w.channels
    cases = [("general_a", w, m.MAMBA_SCAN_GENERAL_A), ("euler", w, m.MAMBA_SCAN_EULER),
             ("trapezoid", w, m.MAMBA_SCAN_TRAPEZOID)]
    cases += [(f"nstate_{n}", w.with_(nstate=n), 0) for n in (4, 8, 32)]
    res = {}
    for name, wv, flags in cases:
        inp = wl.scan_inputs(wv, dev, seed=rank_seed(wv.seed, rank))
        y = torch.empty_like(inp["u"])
        hf = torch.empty((wv.batch, wv.channels, wv.nstate), device=dev, dtype=torch.float32)

        def step():
            st = lib.mamba_selective_scan_ex(inp["u"].data_ptr(), inp["delta"].data_ptr(), inp["A"].data_ptr(),
                                             inp["B"].data_ptr(), inp["C"].data_ptr(), inp["D"].data_ptr(), None,
                                             y.data_ptr(), hf.data_ptr(), wv.batch, wv.length, wv.channels,
                                             wv.nstate, 0, flags, dtc, stream.cuda_stream)
            if st != 0:
                raise m.MambaError(st, "mamba_selective_scan_ex")

        for _ in range(3):
            step()
        torch.cuda.synchronize()
        barrier(dist, world)
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record(stream)
        for _ in range(reps):
            step()
        b.record(stream)
        torch.cuda.synchronize()
        ms = max_over_ranks(dist, world, a.elapsed_time(b)) / reps
        res[name] = {"ms_per_call": round(ms, 5), "token_channels_per_s": world * tc / (ms * 1e-3),
                     "nstate": wv.nstate}
        del inp, y, hf
    res["complex_state"] = run_complex(w, dev, stream, dist, world, rank, reps)
    res["backward"] = run_backward(w, dev, stream, dist, world, rank)
    res["note"] = (f"{w.name} shape; general A and the other discretisations take one exp2 per state "
                   f"(MUFU); nstate_* are zero-order hold with structured A")
    return res


def backward_bytes(w) -> int:
    """Algorithmic bytes of one backward call: u, delta, dy, B, C read; du,
    ddelta written (I/O dtype); dB, dC (fp32) written; A, D and their
    gradients."""
    es = 2 if w.dtype == "bf16" else 4
    tc = w.batch * w.length * w.channels
    bc = w.batch * w.length * w.nstate
    return tc * es * 5 + bc * (2 * es + 2 * 4) + w.channels * (w.nstate + 1) * 4 * 2


def run_backward(w, dev, stream, dist, world, rank, reps: int = 5):
    """ms per call of the backward (gradients of every input from dy, zero-order
    hold) on the workload's shape, with its bytes against the HBM peak."""
    import torch

    from selective_state_space_29_b200 import mamba_ssm as m
    from selective_state_space_29_b200 import workloads as wl

    lib = m.library()
    dtc = m.dtype_code(w.torch_dtype)
    tc = w.batch * w.length * w.channels
    inp = wl.scan_inputs(w, dev, seed=rank_seed(w.seed, rank))
    dy = torch.randn(inp["u"].shape, device=dev).to(inp["u"].dtype)
    f32 = dict(device=dev, dtype=torch.float32)
    outs = [torch.empty_like(inp["u"]), torch.empty_like(inp["u"]), torch.empty(inp["A"].shape, **f32),
            torch.empty(inp["B"].shape, **f32), torch.empty(inp["C"].shape, **f32), torch.empty(inp["D"].shape, **f32),
            torch.empty((w.batch, w.channels, w.nstate), **f32)]

    def bwd():
        st = lib.mamba_selective_scan_backward(
            inp["u"].data_ptr(), inp["delta"].data_ptr(), inp["A"].data_ptr(), inp["B"].data_ptr(),
            inp["C"].data_ptr(), inp["D"].data_ptr(), None, dy.data_ptr(), None, *[o.data_ptr() for o in outs],
            w.batch, w.length, w.channels, w.nstate, dtc, stream.cuda_stream)
        if st != 0:
            raise m.MambaError(st, "mamba_selective_scan_backward")

    for _ in range(2):
        bwd()
    torch.cuda.synchronize()
    barrier(dist, world)
    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    a.record(stream)
    for _ in range(reps):
        bwd()
    b.record(stream)
    torch.cuda.synchronize()
    ms = max_over_ranks(dist, world, a.elapsed_time(b)) / reps
    del inp, dy, outs
    peaks = measured_peaks()
    hbm = float(peaks.get("hbm_gbs", FALLBACK_HBM_GBS))
    nb = backward_bytes(w)
    ach = nb / (ms * 1e-3) / 1e9
    return {"ms_per_call": round(ms, 5), "token_channels_per_s": world * tc / (ms * 1e-3), "nstate": w.nstate,
            "includes": "checkpointing forward pass + reverse aggregates + reverse pass",
            "hbm": {"achieved": round(ach, 1), "peak": hbm, "unit": "GB/s", "frac": round(ach / hbm, 4),
                    "algorithmic_bytes_per_call": nb,
                    "traffic_reverse_kernel": profiled_traffic("scan_backward_kernel", w.name)}}


# --- reference arm: the fp64 oracle on the host cores ------------------------------------

def run_reference(args):
    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    if rank != 0:
        return
    import torch

    import oracle
    from selective_state_space_29_b200 import workloads as wl
    w = wl.SCAN_WORKLOADS[args.workload]
    inp = wl.scan_inputs(w, "cpu" if not torch.cuda.is_available() else "cuda")
    # each step: whole (batch row 0, channel) rows, every 16th channel, as many
    # as fit a step budget that keeps K + W steps within about three minutes
    budget = max(0.5, 180.0 / max(1, args.steps + args.warmup))
    best, cores = oracle_strided_rate(inp, w, stride=16, budget_s=budget)
    n = best["rows"]
    orc = oracle.get()
    ch = torch.arange(0, 16 * n, 16, device=inp["u"].device)
    arrs = [inp["u"][:1].index_select(2, ch), inp["delta"][:1].index_select(2, ch),
            inp["A"].index_select(0, ch), inp["B"][:1], inp["C"][:1], inp["D"].index_select(0, ch)]
    arrs = [a.to(torch.float64).cpu().numpy() for a in arrs]
    del inp
    for _ in range(args.warmup):
        orc.scan(*arrs)
    t0 = time.perf_counter()
    for _ in range(args.steps):
        orc.scan(*arrs)
    dt = (time.perf_counter() - t0) / max(1, args.steps)
    tc = n * w.length
    value = tc / dt
    sample = f"{n} channels (every 16th) of batch row 0 x {w.length} tokens of {w.name} per step"
    out = {"impl": "reference", "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world,
           "steps": args.steps, "warmup": args.warmup, "ms_per_step": dt * 1e3, "higher_is_better": True,
           "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
           "config": {"workload": f"{w.name}: batch {w.batch}, len {w.length}, channels {w.channels}, "
                                  f"state {w.nstate}, {w.dtype} I/O, fp32 state",
                      "batch": w.batch, "len": w.length, "channels": w.channels, "nstate": w.nstate},
           "cpu_baseline": {"value": value, "unit": UNIT, "cores": cores, "kind": "oracle", "sample": sample},
           "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(out), flush=True)


def run_length_sweep(args):
    """The length sweep alone (its object, one JSON line)."""
    import torch

    from selective_state_space_29_b200 import workloads as wl
    dev = torch.device("cuda", 0)
    torch.cuda.set_device(dev)
    w = wl.SCAN_WORKLOADS["long_bf16"]
    inp = wl.scan_inputs(w, dev)
    y = torch.empty_like(inp["u"])
    hf = torch.empty((w.batch, w.channels, w.nstate), device=dev, dtype=torch.float32)
    res = run_length_sweep_on(inp, y, hf, w, dev, torch.cuda.current_stream(dev), None, 1, args.steps)
    print(json.dumps({"length_sweep": res}), flush=True)


def main():
    args = parse_args()
    if args.impl == "reference":
        run_reference(args)
    elif args.only_backward:
        import torch
        from selective_state_space_29_b200 import workloads as wl
        rank, world, local = dist_setup(args.gpus)
        torch.cuda.set_device(local)
        dist = init_pg(world, local)
        res = run_backward(wl.SCAN_WORKLOADS[args.workload], torch.device("cuda", local),
                           torch.cuda.current_stream(), dist, world, rank, reps=max(1, args.steps))
        if world > 1:
            dist.destroy_process_group()
        if rank == 0:
            print(json.dumps({"backward": res}), flush=True)
    elif args.only_complex or args.only_mimo:
        import torch
        from selective_state_space_29_b200 import workloads as wl
        rank, world, local = dist_setup(args.gpus)
        torch.cuda.set_device(local)
        dist = init_pg(world, local)
        dev, st = torch.device("cuda", local), torch.cuda.current_stream()
        if args.only_complex:
            res = {"complex_state": run_complex(wl.SCAN_WORKLOADS[args.workload], dev, st, dist, world, rank,
                                                reps=max(1, args.steps))}
        else:
            peaks = measured_peaks()
            res = {"mimo": run_mimo(dev, st, dist, world, rank, float(peaks.get("hbm_gbs", FALLBACK_HBM_GBS)),
                                    reps=max(1, args.steps))}
        if world > 1:
            dist.destroy_process_group()
        if rank == 0:
            print(json.dumps(res), flush=True)
    elif args.only_ssd:
        import torch
        rank, world, local = dist_setup(args.gpus)
        torch.cuda.set_device(local)
        dist = init_pg(world, local)
        peaks = measured_peaks()
        hbm = float(peaks.get("hbm_gbs", FALLBACK_HBM_GBS))
        res = run_ssd(args, torch.device("cuda", local), torch.cuda.current_stream(), dist, world, rank, hbm,
                      "measured" if "hbm_gbs" in peaks else "fallback", peaks)
        if world > 1:
            dist.destroy_process_group()
        if rank == 0:
            print(json.dumps({"ssd": res}), flush=True)
    elif args.length_sweep:
        run_length_sweep(args)
    else:
        run_ours(args)


if __name__ == "__main__":
    main()
