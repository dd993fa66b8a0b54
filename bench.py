#!/usr/bin/env python
"""BitLinear benchmark: one JSON line on rank 0.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload 2] [--impl ours|reference]

A step is one pass of the deployed BitLinear path over one batch of the
workload: for every call, per-row int8 quantization of X, the ternary x int8
contraction and the fused dequant (a4-a6), on weights that were quantized and
packed once beforehand (a1-a3: an offline cost, timed separately and reported
under "offline").  The default workload is batch-1 decode, (K,N) = (2560,6912)
and (6912,2560) with packed trits, M = 1: its two calls are independent, so
the step is one bl_linear_group call (both weight streams in one launch of the
decode GEMV) with static weights.

Timing: inputs are resident in HBM; R replicas of every buffer rotate so the
replicas touch >= 4x the L2 size (each step's data was last touched R-1 steps
earlier, with >= 3x L2 of other data in between).  One CUDA graph issues the
step once per replica in turn; W warm-up steps, then exactly K timed steps
(whole graph replays, then a graph of the remaining replicas), bracketed by
barrier + synchronize, timed with CUDA events on the launching stream; the max
over ranks is reported.  SM clocks and throttle reasons are sampled through
NVML during the timed region.  `e2e` repeats the step through the public API's
host-buffer call (bl_linear_group_host): X moved in from page-locked host
memory and Y back every step (the packed weights stay resident, as a deployed
model's do, and rotate over the same replicas).

The line also carries, timed the same way after the main region:
  * kernels: the step's calls one launch at a time (chained with programmatic
    dependent launch), without the static-weights flag, the integer product
    alone (bl_linear_acc), and the whole forward from float32 W every call
    (bl_bitlinear_forward);
  * offline: weight quantization + packing (bl_quantize_weights_pack5);
  * prefill: the M = 4096 workload's two bl_linear calls on the int8 tensor
    cores (tensor roofline against 2 x the measured burst bf16 rate), and the
    tcgen05 GEMM kernel alone on int8 weights;
  * sweep: bl_linear at every M of the K = N = 8192 batch sweep;
  * cpu_baseline: the oracle on all host cores (one process per core) and on
    one core, on a bounded sample of the step.

Roofline (main line): the decode GEMV launch's algorithmic bytes (packed
weights + float32 X in + float32 Y out) over its measured time per launch,
against the measured HBM copy rate.

Under torchrun each rank runs its own independently seeded batch (weak
scaling, no data-path collective); only the timing reduction crosses ranks.
`--impl reference` times the CPU oracle instead (rank 0 only).
"""
from __future__ import annotations

import argparse
import hashlib
import json
import math
import os
import platform
import sys
import threading
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import workloads  # noqa: E402

METRIC = "BitLinear GMAC/s and weight-stream GB/s (% of HBM/int8 peak), M=1..4096"
UNIT = "GMAC/s"


def parse(argv=None):
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=2000)
    ap.add_argument("--warmup", type=int, default=50)
    ap.add_argument("--workload", type=int, default=2)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--e2e-steps", type=int, default=300)
    ap.add_argument("--cpu-seconds", type=float, default=8.0,
                    help="target wall time of each oracle baseline sample")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-extras", action="store_true",
                    help="skip the prefill / sweep / per-kernel objects (main line only)")
    return ap.parse_args(argv)


def dist_env():
    ws = int(os.environ.get("WORLD_SIZE", "1"))
    return int(os.environ.get("RANK", "0")), ws, int(os.environ.get("LOCAL_RANK", "0"))


# ----------------------------------------------------------------- clocks ---
class ClockSampler:
    """Polls NVML for SM clock and throttle reasons while the timed region runs."""

    REASONS = {
        "gpu_idle": 0x1, "applications_clocks_setting": 0x2, "sw_power_cap": 0x4,
        "hw_slowdown": 0x8, "sync_boost": 0x10, "sw_thermal_slowdown": 0x20,
        "hw_thermal_slowdown": 0x40, "hw_power_brake_slowdown": 0x80,
        "display_clock_setting": 0x100,
    }

    def __init__(self, device_uuid):
        self.samples, self.reasons, self.max_mhz, self.ok = [], set(), None, False
        try:
            import pynvml as nv
            nv.nvmlInit()
            self.nv = nv
            self.h = nv.nvmlDeviceGetHandleByUUID(device_uuid)
            self.max_mhz = nv.nvmlDeviceGetMaxClockInfo(self.h, nv.NVML_CLOCK_SM)
            self.ok = True
        except Exception as e:  # pragma: no cover - depends on the box
            self.err = repr(e)
        self._stop = threading.Event()

    def _poll(self):
        while not self._stop.is_set():
            self._sample_once()
            time.sleep(0.0005)

    def _sample_once(self):
        nv = self.nv
        try:
            self.samples.append(nv.nvmlDeviceGetClockInfo(self.h, nv.NVML_CLOCK_SM))
            r = nv.nvmlDeviceGetCurrentClocksEventReasons(self.h)
            for k, bit in self.REASONS.items():
                if r & bit and k != "gpu_idle":
                    self.reasons.add(k)
        except Exception:
            pass

    def __enter__(self):
        if self.ok:
            self._sample_once()
            self.t = threading.Thread(target=self._poll, daemon=True)
            self.t.start()
        return self

    def __exit__(self, *a):
        if self.ok:
            self._stop.set()
            self.t.join()
            self._sample_once()

    def summary(self):
        if not self.ok or not self.samples:
            return {"sm_mhz": None, "sm_max_mhz": self.max_mhz, "reasons": [], "samples": 0}
        return {"sm_mhz": float(np.median(self.samples)), "sm_max_mhz": self.max_mhz,
                "reasons": sorted(self.reasons), "samples": len(self.samples)}


# ------------------------------------------------------------ peaks/traffic --
def measured_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as fh:
            d = json.load(fh)
        return {"hbm_gbs": float(d["hbm_gbs"]), "bf16_tflops": float(d["bf16_tflops"]),
                "bf16_tflops_sustained": float(d.get("bf16_tflops_sustained", d["bf16_tflops"])),
                "source": "measured"}
    return {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0, "source": "fallback"}


def hbm_roofline(nbytes, ms, peaks):
    """Algorithmic bytes of one launch over its measured duration, against the
    measured HBM copy rate."""
    achieved = nbytes / (ms * 1e-3) / 1e9
    return {"bound": "hbm", "achieved": round(achieved, 1), "peak": peaks["hbm_gbs"], "unit": "GB/s",
            "frac": round(achieved / peaks["hbm_gbs"], 4),
            "peak_source": ("of measured (MEASURED_PEAKS.json hbm_gbs)" if peaks["source"] == "measured"
                            else "of fallback 6.65 TB/s")}


def tensor_roofline(macs, ms, peaks, burst=True):
    """Roofline of int8 tensor-core work: int8 operations (2 per multiply-add)
    per second over the measured duration, against 2 x the measured bf16 GEMM
    rate (the nominal dense int8 : bf16 ratio, 4.5 : 2.25 PFLOP/s).  `burst`:
    the calls were timed alone (short replays), so the burst bf16 figure
    applies; otherwise the sustained one."""
    achieved = 2.0 * macs / (ms * 1e-3) / 1e12
    key = "bf16_tflops" if burst else "bf16_tflops_sustained"
    peak = 2.0 * peaks[key]
    src = (f"of measured {'burst' if burst else 'sustained'} bf16 x 2 (MEASURED_PEAKS.json {key})"
           if peaks["source"] == "measured"
           else f"of fallback {'1.59' if burst else '1.4'} PFLOP/s bf16 x 2")
    return {"bound": "tensor", "achieved": round(achieved, 1), "peak": round(peak, 1), "unit": "TFLOP/s",
            "frac": round(achieved / peak, 4), "traffic": None, "peak_source": src}


# The sources a profiled kernel is built from: its header chain, and the lines
# of the library source that name it (its launcher and launch configuration).
KERNEL_SOURCES = {
    "wquant_kernel": (("weight_fused.cuh", "weight_quant.cuh", "act_quant.cuh", "common.cuh", "ptx.cuh"),
                      ("wquant", "kFu", "fused")),
    "gemv_pack5_kernel": (("gemv_pack5.cuh", "trit_table.cuh", "act_quant.cuh", "common.cuh", "ptx.cuh"),
                          ("gemv", "Gemv")),
    "gemm_swap_kernel": (("gemm_swap.cuh", "trit_table.cuh", "common.cuh", "ptx.cuh"),
                         ("swap", "Swap", "run_swap", "sw_")),
}


def kernel_source_hash(kernel=None):
    """Hash of the sources `kernel` is built from (all CUDA sources if it has no
    entry in KERNEL_SOURCES): a stored ncu figure is used only while it matches."""
    h = hashlib.sha256()
    d = os.path.join(ROOT, "int8_row_absmax_b200", "csrc")
    spec = KERNEL_SOURCES.get(kernel)
    if spec is None:
        for f in sorted(os.listdir(d)):
            if f.endswith((".cu", ".cuh")):
                with open(os.path.join(d, f), "rb") as fh:
                    h.update(f.encode() + fh.read())
        return h.hexdigest()[:16]
    files, keys = spec
    for f in files:
        with open(os.path.join(d, f), "rb") as fh:
            h.update(f.encode() + fh.read())
    with open(os.path.join(d, "bitlinear_lib.cu")) as fh:
        for line in fh:
            if any(k in line for k in keys):
                h.update(line.encode())
    return h.hexdigest()[:16]


def ncu_traffic(kernel: str, workload: int):
    """DRAM bytes per launch from the committed ncu summary, if it was taken on
    the current kernel sources (else None)."""
    p = os.path.join(ROOT, "profiles", "dram_traffic.json")
    if not os.path.exists(p):
        return None
    with open(p) as fh:
        d = json.load(fh)
    rec = d.get(f"{kernel}@{workload}")
    if not rec or rec.get("source_hash") != kernel_source_hash(kernel):
        return None
    return rec.get("dram_bytes_per_launch")


def packed_bytes(N, K):
    return N * math.ceil(K / 5)


def algorithmic_bytes(kind, N, K, M, fmt):
    """Bytes each kind of call must move at minimum (inputs read + outputs written)."""
    wbytes = packed_bytes(N, K) if fmt == 1 else N * K
    if kind == "wquant":          # read W once, write the codes
        return 4 * N * K + wbytes
    if kind == "linear":
        return wbytes + 4 * M * K + 4 * M * N
    if kind == "forward":         # read W and X once, write the codes and Y
        return 4 * N * K + wbytes + 4 * M * K + 4 * M * N
    raise ValueError(kind)


# ------------------------------------------------------- rank arithmetic ---
def max_over_ranks(ms: float, dist=None, device=None) -> float:
    """The timed region's duration as the max over ranks (the slowest rank)."""
    if dist is None or not dist.is_initialized() or dist.get_world_size() == 1:
        return float(ms)
    import torch
    t = torch.tensor([ms], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def whole_job_gmacs(macs_per_step_per_rank: int, steps: int, world: int, ms: float) -> float:
    """Weak scaling: every rank does its own step; value = all ranks' MACs / slowest time."""
    return macs_per_step_per_rank * steps * world / (ms * 1e-3) / 1e9


def replicas_for(nbytes_per_replica, l2, lo=2):
    """Replica count whose buffers together touch >= 4x the L2 size."""
    return max(lo, math.ceil(4 * l2 / max(1, nbytes_per_replica)))


# ------------------------------------------------------------- device side --
class Layer:
    """One call's device buffers: packed (or int8) weights quantized once, beta,
    X, Y; `clone()` makes an independent replica of the same values."""

    def __init__(self, bl, torch, p, dev, fmt, src=None):
        self.p, self.fmt, self.M, self.K, self.N, self.eps = p, fmt, p.M, p.K, p.N, p.eps
        if src is None:
            Wf = torch.from_numpy(p.W).to(dev)
            self.Wd, self.beta = (bl.quantize_weights_pack5(Wf, p.eps) if fmt == bl.PACK5
                                  else bl.quantize_weights(Wf, p.eps))
            del Wf
            self.X = torch.from_numpy(np.ascontiguousarray(p.X)).to(dev)
        else:
            self.Wd, self.beta, self.X = src.Wd.clone(), src.beta.clone(), src.X.clone()
        self.Y = torch.empty((p.M, p.N), dtype=torch.float32, device=dev)

    def nbytes(self):
        return self.Wd.numel() + self.X.numel() * 4 + self.Y.numel() * 4

    def call(self):
        return (self.X, self.Wd, self.fmt, self.N, self.K, self.beta, None, self.eps)


def time_graph(torch, stream, issue_fns, steps, warmup):
    """Capture one graph per contiguous block of `issue_fns` (one entry per step,
    in rotation) and time exactly `steps` of them after `warmup`; ms total."""
    R = len(issue_fns)

    def capture(fns):
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g, stream=stream):
            for f in fns:
                f()
        return g

    with torch.cuda.stream(stream):
        full = capture(issue_fns)
        parts = {}

        def run(n):
            for _ in range(n // R):
                full.replay()
            rem = n % R
            if rem:
                if rem not in parts:
                    parts[rem] = capture(issue_fns[:rem])
                parts[rem].replay()

        run(R)                        # first replay (uploads the graph)
        if steps % R and (steps % R) not in parts:
            parts[steps % R] = capture(issue_fns[:steps % R])
        run(warmup)
        torch.cuda.synchronize()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        run(steps)
        e1.record(stream)
    torch.cuda.synchronize()
    ms = e0.elapsed_time(e1)
    del full, parts
    return ms


def timed_calls(bl, torch, stream, layer_sets, issue, reps=None, l2=None):
    """Per-step ms of `issue(layers)` over the rotating replicas `layer_sets`
    (several replays, after one warm replay)."""
    R = len(layer_sets)
    n = reps or max(R, 64)
    return time_graph(torch, stream, [lambda ls=ls: issue(ls) for ls in layer_sets], n, R) / n


# ------------------------------------------------------------ our arm ------
def run_ours(args):
    import torch
    import torch.distributed as dist
    rank, world, local = dist_env()
    if world > 1:
        torch.cuda.set_device(local)
        dist.init_process_group("nccl", timeout=__import__("datetime").timedelta(seconds=120))
    dev = torch.device("cuda", local if world > 1 else 0)
    torch.cuda.set_device(dev)
    import int8_row_absmax_b200 as bl
    bl.load()
    peaks = measured_peaks()
    props = torch.cuda.get_device_properties(dev)
    l2 = int(getattr(props, "L2_cache_size", 126 * 2 ** 20))
    stream = torch.cuda.Stream(device=dev)

    wl = workloads.WORKLOADS[args.workload]
    fmt = bl.PACK5 if wl.fmt == workloads.FMT_PACK5 else bl.I8
    probs = list(workloads.problems(args.workload, rank=rank))
    macs_per_step = sum(p.M * p.N * p.K for p in probs)
    with torch.cuda.stream(stream):
        base = [Layer(bl, torch, p, dev, fmt) for p in probs]
        per = sum(L.nbytes() for L in base)
        R = replicas_for(per, l2)
        sets = [base] + [[Layer(bl, torch, L.p, dev, fmt, src=L) for L in base] for _ in range(R - 1)]
    torch.cuda.synchronize()

    def step(ls):
        bl.linear_group([L.call() for L in ls], static_weights=True, outs=[L.Y for L in ls])

    # one eager step per replica: launches must succeed and the device stay clean
    with torch.cuda.stream(stream):
        for ls in sets:
            step(ls)
    if bl.sync_status(dev) != "BL_OK":
        raise RuntimeError("device status not clean after the eager step")
    plans = [bl.linear_plan(L.M, L.N, L.K, fmt) for L in base]
    gemv_calls = [L for L, (path, _) in zip(base, plans) if path == bl.PATH_GEMV]
    other_launches = sum(n for path, n in plans if path != bl.PATH_GEMV)
    launches_per_step = other_launches + sum(
        math.ceil(sum(1 for L in gemv_calls if L.M == m) / 4) for m in (1, 2, 3, 4))

    K, Wm = args.steps, args.warmup
    if world > 1:
        dist.barrier()
    uuid = str(props.uuid)
    clk = ClockSampler(uuid if uuid.startswith("GPU-") else "GPU-" + uuid)
    torch.cuda.synchronize()
    with clk:
        ms_total = time_graph(torch, stream, [lambda ls=ls: step(ls) for ls in sets], K, Wm)
    if world > 1:
        dist.barrier()
    ms_max = max_over_ranks(ms_total, dist, dev)
    if bl.sync_status(dev) != "BL_OK":
        raise RuntimeError("device status not clean after the timed region")
    ms_step = ms_max / K
    value = whole_job_gmacs(macs_per_step, K, world, ms_max)

    wbytes = sum(packed_bytes(L.N, L.K) if fmt == bl.PACK5 else L.N * L.K for L in base)
    step_bytes = sum(algorithmic_bytes("linear", L.N, L.K, L.M, fmt) for L in base)
    line = {
        "metric": METRIC, "value": round(value, 2), "unit": UNIT, "n_gpus": world,
        "steps": K, "warmup": Wm, "ms_per_step": round(ms_step, 6),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": "i8 x trit -> i32, f32 scales", "data": "synthetic",
        "config": {"workload": f"{wl.id}:{wl.name}", "shapes_MKN": [list(s) for s in wl.shapes],
                   "weight_format": wl.fmt, "parallelism": f"dp{world} (independent batches)",
                   "l2_defeat": f"inputs larger than L2: {R} rotating replicas, "
                                f"{R * per / 2**20:.0f} MiB >= 4x L2 ({l2 / 2**20:.0f} MiB)",
                   "step": "bl_linear_group over the workload's calls (per-row int8 X, contraction, dequant) "
                           "on weights quantized once, static-weights flag",
                   "timing": "one CUDA graph over the replicas, CUDA events on the launching stream"},
        "macs_per_step": macs_per_step,
        "weight_stream_gbs": round(wbytes / (ms_step * 1e-3) / 1e9, 1),
        "clocks": clk.summary(),
        "gpu_launches": launches_per_step * K,
        "gpu": torch.cuda.get_device_name(dev),
    }
    if gemv_calls and len(gemv_calls) == len(base) and launches_per_step == 1:
        rl = hbm_roofline(step_bytes, ms_step, peaks)
        rl.update({"traffic": ncu_traffic("gemv_pack5_kernel", args.workload), "kernel": "gemv_pack5_kernel",
                   "call": "bl_linear_group (one launch: every call's packed weights, X in, Y out)",
                   "bytes_per_launch": step_bytes, "us_per_launch": round(ms_step * 1e3, 3)})
        line["roofline"] = rl
    else:
        line["roofline"] = tensor_roofline(macs_per_step, ms_step, peaks, burst=False)
        line["roofline"].update({"kernel": "gemm_tc_kernel", "call": "bl_linear_group"})

    if not args.no_extras:
        line["kernels"] = kernel_breakdown(bl, torch, stream, sets, base, fmt, peaks)
        line["offline"] = offline_costs(bl, torch, stream, probs, dev, fmt, l2)
        if args.workload != 4:
            line["prefill"] = prefill(bl, torch, stream, dev, peaks, rank)
        if args.workload != 5:
            line["sweep"] = sweep(bl, torch, stream, dev, peaks, l2, rank)
    # ---- end to end through the public API, host buffers -------------------
    line["e2e"] = e2e(bl, torch, sets, dev, fmt, args.e2e_steps, world, dist)
    del sets, base
    torch.cuda.empty_cache()

    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        line["cpu_baseline"] = cpu_baseline(args.workload, args.cpu_seconds)
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()
    if rank == 0:
        print(json.dumps(line), flush=True)


def kernel_breakdown(bl, torch, stream, sets, base, fmt, peaks):
    """The step's calls timed in other forms, over the same rotating replicas."""
    out = {}
    n_calls = len(base)
    macs = sum(L.M * L.N * L.K for L in base)
    step_bytes = sum(algorithmic_bytes("linear", L.N, L.K, L.M, fmt) for L in base)

    def record(name, ms, launches, nbytes=step_bytes, note=None):
        d = {"ms_per_step": round(ms, 5), "launches_per_step": launches,
             "gmacs": round(macs / (ms * 1e-3) / 1e9, 1),
             "achieved_gbs": round(nbytes / (ms * 1e-3) / 1e9, 1),
             "frac_hbm": round(nbytes / (ms * 1e-3) / 1e9 / peaks["hbm_gbs"], 4)}
        if note:
            d["note"] = note
        out[name] = d

    plans = [bl.linear_plan(L.M, L.N, L.K, fmt)[1] for L in base]
    ms = timed_calls(bl, torch, stream, sets, lambda ls: [
        bl.linear(*L.call()[:6], eps=L.eps, out=L.Y, static_weights=True) for L in ls])
    record("chained", ms, sum(plans), note="bl_linear per call, static weights: one launch each, "
                                            "consecutive launches overlap (programmatic dependent launch)")
    ms = timed_calls(bl, torch, stream, sets, lambda ls: [
        bl.linear(*L.call()[:6], eps=L.eps, out=L.Y) for L in ls])
    record("chained_nonstatic", ms, sum(plans), note="bl_linear per call without the static-weights flag: "
                                                      "each launch copies W only after the previous one ends")
    # the integer product alone on pre-quantized X
    xq = {}
    for ls in sets:
        for L in ls:
            xq[id(L)] = bl.quantize_act(L.X, L.eps)[0]
    accs = {id(L): torch.empty((L.M, L.N), dtype=torch.int32, device=L.X.device) for ls in sets for L in ls}
    lib = bl.load()

    def acc_issue(ls):
        for L in ls:
            code = lib.bl_linear_acc_ex(xq[id(L)].data_ptr(), L.M, L.K, L.Wd.data_ptr(), fmt, L.N, L.Wd.shape[1],
                                        accs[id(L)].data_ptr(), None, 0, bl.FLAG_STATIC_WEIGHTS,
                                        bl._stream(torch, L.X))
            if code:
                raise RuntimeError(bl.STATUS.get(code, code))
    ms = timed_calls(bl, torch, stream, sets, acc_issue)
    acc_bytes = sum((packed_bytes(L.N, L.K) if fmt == bl.PACK5 else L.N * L.K) + L.M * L.K + 4 * L.M * L.N
                    for L in base)
    record("linear_acc", ms, n_calls, nbytes=acc_bytes,
           note="bl_linear_acc_ex per call on int8 X_q, static weights (int32 out)")
    del xq, accs
    if bl.sync_status() != "BL_OK":
        raise RuntimeError("device status not clean after the kernel breakdown")
    return out


def offline_costs(bl, torch, stream, probs, dev, fmt, l2):
    """bl_quantize_weights_pack5 (beta, codes, packing: one launch for large
    tensors) per weight tensor, over enough fp32 copies to defeat L2, and the
    whole forward from float32 W every call (bl_bitlinear_forward)."""
    lib = bl.load()
    seen, tensors = set(), []
    for p in probs:
        if id(p.W) not in seen:
            seen.add(id(p.W))
            tensors.append(p)
    per = sum(p.W.size * 4 for p in tensors)
    R = replicas_for(per, l2)
    with torch.cuda.stream(stream):
        Ws = [[torch.from_numpy(p.W).to(dev) for p in tensors]]
        Ws += [[w.clone() for w in Ws[0]] for _ in range(R - 1)]
        outs = []
        for ws_ in Ws:
            o = []
            for p, w in zip(tensors, ws_):
                Wp = (torch.empty((p.N, bl.pack5_ldp(p.K)), dtype=torch.uint8, device=dev) if fmt == bl.PACK5
                      else torch.empty((p.N, p.K), dtype=torch.int8, device=dev))
                beta = torch.zeros(1, dtype=torch.float32, device=dev)
                wsb = bl.workspace(lib.bl_quantize_weights_workspace_size(p.N, p.K), dev)
                o.append((w, Wp, beta, wsb, p))
            outs.append(o)
    torch.cuda.synchronize()

    def issue(o):
        for w, Wp, beta, wsb, p in o:
            if fmt == bl.PACK5:
                bl.quantize_weights_pack5(w, p.eps, ws=wsb, out=Wp, beta=beta)
            else:
                bl.quantize_weights(w, p.eps, ws=wsb, out=Wp, beta=beta)
    ms = timed_calls(bl, torch, stream, outs, issue, reps=max(R, 16))
    nbytes = sum(algorithmic_bytes("wquant", p.N, p.K, 0, fmt) for p in tensors)
    res = {"weight_quant": {"call": "bl_quantize_weights_pack5" if fmt == bl.PACK5 else "bl_quantize_weights",
                            "ms_per_step": round(ms, 5), "tensors": len(tensors),
                            "achieved_gbs": round(nbytes / (ms * 1e-3) / 1e9, 1)}}
    # the forward that quantizes W every call (training-style), M <= 4 calls only
    fw = [p for p in probs if p.M <= 4]
    if fw:
        with torch.cuda.stream(stream):
            Xs = {id(p): torch.from_numpy(np.ascontiguousarray(p.X)).to(dev) for p in fw}
            Ys = {id(p): torch.empty((p.M, p.N), dtype=torch.float32, device=dev) for p in fw}
            fws = {}
            for o in outs:
                for w, Wp, beta, wsb, p in o:
                    fws[id(w)] = bl.workspace(lib.bl_bitlinear_forward_workspace_size(p.M, p.N, p.K, fmt), dev)

        def issue_fw(o):
            for w, Wp, beta, wsb, p in o:
                if id(p) in Xs:
                    bl.bitlinear_forward(Xs[id(p)], w, fmt, eps=p.eps, ws=fws[id(w)], w_out=Wp, beta=beta,
                                         out=Ys[id(p)])
        ms = timed_calls(bl, torch, stream, outs, issue_fw, reps=max(R, 16))
        fbytes = sum(algorithmic_bytes("forward", p.N, p.K, p.M, fmt) for p in fw)
        res["forward"] = {"call": "bl_bitlinear_forward (weights quantized every call)", "ms_per_step": round(ms, 5),
                          "achieved_gbs": round(fbytes / (ms * 1e-3) / 1e9, 1)}
    if bl.sync_status() != "BL_OK":
        raise RuntimeError("device status not clean after the offline timings")
    return res


def prefill(bl, torch, stream, dev, peaks, rank):
    """The M = 4096 workload: its two bl_linear calls per step (activation
    quantization, unpack, tcgen05 GEMM), and the GEMM kernel alone on int8
    weights (bl_linear_acc_ex, one launch); each call reads >= 67 MB of X."""
    probs = list(workloads.problems(4, rank=rank))
    macs = sum(p.M * p.N * p.K for p in probs)
    with torch.cuda.stream(stream):
        base = [Layer(bl, torch, p, dev, bl.PACK5) for p in probs]
        sets = [base, [Layer(bl, torch, L.p, dev, bl.PACK5, src=L) for L in base]]
        ws = {id(L): bl.workspace(bl.linear_workspace_size(L.M, L.N, L.K, bl.PACK5), dev) for ls in sets for L in ls}
    torch.cuda.synchronize()
    ms = timed_calls(bl, torch, stream, sets, lambda ls: [
        bl.linear(*L.call()[:6], eps=L.eps, out=L.Y, ws=ws[id(L)]) for L in ls], reps=8)
    out = {"workload": "4:prefill_gemm", "ms_per_step": round(ms, 5),
           "gmacs": round(macs / (ms * 1e-3) / 1e9, 1),
           "launches_per_step": sum(bl.linear_plan(L.M, L.N, L.K, bl.PACK5)[1] for L in base),
           "roofline": tensor_roofline(macs, ms, peaks, burst=True)}
    out["roofline"].update({"kernel": "gemm_tc_kernel", "call": "bl_linear x2 (act quant, unpack, GEMM)"})
    # the GEMM kernel alone: int8 weights and int8 X_q given
    lib = bl.load()
    with torch.cuda.stream(stream):
        i8 = []
        for L in base:
            Wq = bl.unpack(L.Wd, L.K)
            Xq = bl.quantize_act(L.X, L.eps)[0]
            acc = torch.empty((L.M, L.N), dtype=torch.int32, device=dev)
            i8.append((Xq, Wq, acc, L))
    torch.cuda.synchronize()

    def gemm(_):
        for Xq, Wq, acc, L in i8:
            code = lib.bl_linear_acc_ex(Xq.data_ptr(), L.M, L.K, Wq.data_ptr(), bl.I8, L.N, L.K, acc.data_ptr(),
                                        None, 0, bl.PATH_TC, bl._stream(torch, Xq))
            if code:
                raise RuntimeError(bl.STATUS.get(code, code))
    ms_g = timed_calls(bl, torch, stream, [0, 1], gemm, reps=8)
    out["gemm_alone"] = {"ms_per_step": round(ms_g, 5), "launches_per_step": 2,
                         "roofline": tensor_roofline(macs, ms_g, peaks, burst=True),
                         "call": "bl_linear_acc_ex on int8 W_q and X_q (one gemm_tc_kernel launch per call)"}
    del sets, base, i8, ws
    torch.cuda.empty_cache()
    if bl.sync_status() != "BL_OK":
        raise RuntimeError("device status not clean after the prefill timings")
    return out


def sweep(bl, torch, stream, dev, peaks, l2, rank):
    """bl_linear at each M of the K = N = 8192 sweep (one packed W, X[:M]),
    static weights, over enough replicas to defeat L2."""
    probs = list(workloads.problems(5, rank=rank))
    p0 = probs[0]
    res = []
    with torch.cuda.stream(stream):
        Wf = torch.from_numpy(p0.W).to(dev)
        Wd, beta = bl.quantize_weights_pack5(Wf, p0.eps)
        del Wf
        Xall = torch.from_numpy(np.ascontiguousarray(probs[-1].X)).to(dev)
    torch.cuda.synchronize()
    for p in probs:
        per = Wd.numel() + 8 * p.M * p.K
        R = replicas_for(per, l2)
        with torch.cuda.stream(stream):
            reps = [(Wd if r == 0 else Wd.clone(), Xall[:p.M].clone(),
                     torch.empty((p.M, p.N), dtype=torch.float32, device=dev),
                     bl.workspace(bl.linear_workspace_size(p.M, p.N, p.K, bl.PACK5), dev)) for r in range(R)]
        torch.cuda.synchronize()
        ms = timed_calls(bl, torch, stream, reps, lambda r: bl.linear(
            r[1], r[0], bl.PACK5, p.N, p.K, beta, eps=p.eps, out=r[2], ws=r[3], static_weights=True),
            reps=max(2 * R, 32))
        path, nl = bl.linear_plan(p.M, p.N, p.K, bl.PACK5)
        wb = packed_bytes(p.N, p.K)
        gbs = wb / (ms * 1e-3) / 1e9
        res.append({"M": p.M, "path": {bl.PATH_GEMV: "gemv", bl.PATH_TC: "tc", bl.PATH_SIMT: "simt"}[path],
                    "launches": nl, "us": round(ms * 1e3, 2), "gmacs": round(p.M * p.N * p.K / (ms * 1e-3) / 1e9, 1),
                    "weight_stream_gbs": round(gbs, 1), "frac_hbm_weights": round(gbs / peaks["hbm_gbs"], 4),
                    "int8_tops": round(2 * p.M * p.N * p.K / (ms * 1e-3) / 1e12, 1)})
        del reps
    del Wd, Xall
    torch.cuda.empty_cache()
    if bl.sync_status() != "BL_OK":
        raise RuntimeError("device status not clean after the sweep")
    return {"workload": "5:batch_sweep", "K": p0.K, "N": p0.N, "l2_defeat": ">= 4x L2 of rotating replicas per M",
            "points": res}


def e2e(bl, torch, sets, dev, fmt, steps, world, dist):
    """The step through the public API with host buffers: bl_linear_group_host
    copies every call's X in from page-locked host memory, runs the calls and
    copies Y back to page-locked host memory, every step; weights resident and
    rotating over the same replicas as the device-timed step (so they come from
    HBM, not L2).  The calls' rows sit back to back in one host and one device
    buffer each way, so each direction is one transfer."""
    base = sets[0]
    kt = sum(L.M * L.K for L in base)
    nt = sum(L.M * L.N for L in base)
    hx = torch.empty(kt, dtype=torch.float32).pin_memory()
    hy = torch.empty(nt, dtype=torch.float32).pin_memory()
    dx = torch.empty(kt, dtype=torch.float32, device=dev)
    dy = torch.empty(nt, dtype=torch.float32, device=dev)
    hX, hY, dX, dY, k0, n0 = [], [], [], [], 0, 0
    for L in base:          # every replica has the same shapes: one set of views
        xk, yn = L.M * L.K, L.M * L.N
        hX.append(hx[k0:k0 + xk].view(L.M, L.K))
        hX[-1].copy_(torch.from_numpy(np.ascontiguousarray(L.p.X)))
        hY.append(hy[n0:n0 + yn].view(L.M, L.N))
        dX.append(dx[k0:k0 + xk].view(L.M, L.K))
        dY.append(dy[n0:n0 + yn].view(L.M, L.N))
        k0, n0 = k0 + xk, n0 + yn
    groups = [bl.LinearGroupHost([(x, L.Wd, fmt, L.N, L.K, L.beta, None, L.eps) for x, L in zip(dX, ls)],
                                 hX, hY, static_weights=True, outs=dY) for ls in sets]
    for g in groups:
        g()
    torch.cuda.synchronize()
    t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    t0.record()
    for i in range(steps):
        groups[i % len(groups)]()
    t1.record()
    torch.cuda.synchronize()
    ms = max_over_ranks(t0.elapsed_time(t1), dist, dev)
    macs = sum(L.M * L.N * L.K for L in base)
    return {"value": round(whole_job_gmacs(macs, steps, world, ms), 2), "unit": UNIT,
            "h2d_bytes_per_step": int(kt * 4), "d2h_bytes_per_step": int(nt * 4),
            "steps": steps, "ms_per_step": round(ms / steps, 4),
            "l2_defeat": f"weights rotate over {len(groups)} replicas",
            "call": "bl_linear_group_host via the Python binding (marshalled once): X from page-locked "
                    "host memory, the calls, Y back to page-locked host memory, every step"}


# ------------------------------------------------------------ CPU oracle ----
def cpu_model():
    try:
        with open("/proc/cpuinfo") as fh:
            for line in fh:
                if line.startswith("model name"):
                    return line.split(":", 1)[1].strip()
    except OSError:
        pass
    return platform.processor() or "unknown"


def host_cores():
    try:
        return len(os.sched_getaffinity(0))
    except AttributeError:
        return os.cpu_count() or 1


def oracle_prepare(wid, rows, rank=0):
    """The step's problems with their weights quantized by the oracle, rows
    [r0, r1) of every call (a fraction of N); beta over the whole tensor."""
    import oracle
    probs = list(workloads.problems(wid, rank=rank))
    betas, out = {}, []
    for p in probs:
        if id(p.W) not in betas:
            betas[id(p.W)] = oracle.absmean_beta(p.W, p.eps)
    for p in probs:
        r0, r1 = int(round(rows[0] * p.N)), int(round(rows[1] * p.N))
        r1 = max(r1, r0 + 1) if rows[1] > rows[0] else r1
        Wq = oracle.ternarize(p.W[r0:r1], betas[id(p.W)])
        out.append((p.X, Wq, betas[id(p.W)], p.eps, p.M * (r1 - r0) * p.K))
    return out


def oracle_linear_step(prepared):
    """One step of the oracle's deployed linear over the prepared rows; MACs."""
    import oracle
    macs = 0
    for X, Wq, beta, eps, m in prepared:
        Xq, s = oracle.act_quant(X, eps)
        oracle.dequant(oracle.contract(Xq, Wq), s, beta)
        macs += m
    return macs


def _cpu_worker(wid, rows, seconds, barrier, queue):
    os.environ.setdefault("OMP_NUM_THREADS", "1")
    prepared = oracle_prepare(wid, rows)
    oracle_linear_step(prepared)                 # warm
    barrier.wait()
    t = time.perf_counter()
    macs = reps = 0
    while True:
        macs += oracle_linear_step(prepared)
        reps += 1
        if time.perf_counter() - t >= seconds:
            break
    queue.put((macs, time.perf_counter() - t, reps))


def cpu_run(wid, nproc, seconds, frac=1.0):
    """The oracle's step split by rows over `nproc` spawned processes (a
    fraction `frac` of every weight's rows in all); GMAC/s over the slowest."""
    import multiprocessing as mp
    ctx = mp.get_context("spawn")
    barrier, queue = ctx.Barrier(nproc), ctx.Queue()
    procs = []
    for i in range(nproc):
        rows = (frac * i / nproc, frac * (i + 1) / nproc)
        pr = ctx.Process(target=_cpu_worker, args=(wid, rows, seconds, barrier, queue), daemon=True)
        pr.start()
        procs.append(pr)
    res = [queue.get(timeout=600) for _ in procs]
    for pr in procs:
        pr.join(timeout=60)
    macs = sum(r[0] for r in res)
    dt = max(r[1] for r in res)
    return macs / dt / 1e9, min(r[2] for r in res), dt


def worker_limit(wid):
    """Processes whose copies of the workload's inputs fit in a quarter of RAM."""
    wl = workloads.WORKLOADS[wid]
    if wl.shared_weight:
        per = 4 * wl.shapes[0][1] * wl.shapes[0][2] + 4 * max(m * k for m, k, _ in wl.shapes)
    else:
        per = sum(4 * k * n + 4 * m * k for m, k, n in wl.shapes)
    try:
        ram = os.sysconf("SC_PAGE_SIZE") * os.sysconf("SC_PHYS_PAGES")
    except (ValueError, OSError, AttributeError):
        ram = 64 << 30
    return max(1, int(ram // 4 // max(1, 2 * per)))


def cpu_baseline(wid, seconds):
    """The oracle as committed (numpy, plain), timed on this host's cores: one
    process per core, each on its share of every weight's rows, and one core
    alone on a row slice; weights quantized beforehand (an offline step, as on
    the GPU)."""
    n = min(host_cores(), worker_limit(wid))
    allv, reps_all, dt_all = cpu_run(wid, n, seconds)
    one_frac = 1.0 / n if n > 1 else 1.0
    onev, reps_one, dt_one = cpu_run(wid, 1, seconds, frac=one_frac)
    return {"value": round(allv, 4), "unit": UNIT, "cores": n, "kind": "oracle",
            "sample": f"the step's act quant + contraction + dequant per call (oracle, numpy), every row of "
                      f"every weight split over {n} processes, >= {reps_all} step(s) each in {dt_all:.1f} s",
            "one_core": {"value": round(onev, 4), "unit": UNIT, "cores": 1,
                         "sample": f"rows [0, {one_frac:.4f} N) of every weight, {reps_one} step(s) in {dt_one:.1f} s"},
            "host": {"nproc": n, "cpu_model": cpu_model()}}


def run_reference(args):
    rank, world, _ = dist_env()
    if rank != 0:
        return
    wl = workloads.WORKLOADS[args.workload]
    # each reference step: the oracle's step on a row slice sized so the run stays short
    prepared = oracle_prepare(args.workload, (0.0, 1.0 / 64))
    t = time.perf_counter()
    oracle_linear_step(prepared)
    dt1 = time.perf_counter() - t
    budget = max(0.002, 60.0 / max(1, args.steps + args.warmup))
    frac = min(1.0, (1.0 / 64) * budget / max(dt1, 1e-6))
    prepared = oracle_prepare(args.workload, (0.0, frac))
    for _ in range(args.warmup):
        oracle_linear_step(prepared)
    t = time.perf_counter()
    macs = 0
    for _ in range(args.steps):
        macs += oracle_linear_step(prepared)
    dt = time.perf_counter() - t
    value = macs / dt / 1e9
    line = {"impl": "reference", "metric": METRIC, "value": round(value, 4), "unit": UNIT,
            "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": round(dt / max(1, args.steps) * 1e3, 3), "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "i8 x trit -> i64, f32 scales", "data": "synthetic",
            "config": {"workload": f"{wl.id}:{wl.name}", "shapes_MKN": [list(s) for s in wl.shapes],
                       "weight_format": wl.fmt, "parallelism": "cpu oracle, rank 0, one process"},
            "cpu_baseline": {"value": round(value, 4), "unit": UNIT, "cores": 1, "kind": "oracle",
                             "sample": f"each step: act quant + contraction + dequant of every call on the "
                                       f"first {frac:.4f} of each weight's rows (weights quantized beforehand)",
                             "host": {"nproc": host_cores(), "cpu_model": cpu_model()}},
            "e2e": {"value": round(value, 4), "unit": UNIT, "h2d_bytes_per_step": 0,
                    "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


def main():
    args = parse()
    if args.impl == "reference":
        run_reference(args)
    else:
        run_ours(args)


if __name__ == "__main__":
    main()
