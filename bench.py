#!/usr/bin/env python
"""BitLinear benchmark: one JSON line on rank 0.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload 2] [--impl ours|reference]

A step is one pass of the whole BitLinear hot path over one batch of the
workload: for every weight tensor, absmean beta, ternarize and pack (a1-a3,
one library call: a single streaming pass over W in one launch); for every
call, per-row int8 quantization of X, the ternary x int8 contraction and the
fused dequant (a4-a6).  The default workload is batch-1
decode: (K,N) = (2560,6912) and (6912,2560) with packed trits, M = 1.

Timing: inputs are resident in HBM; R replicas of every buffer rotate so each
rotation touches >= 4x the L2 size (no step reuses the previous step's data
from L2).  Each replica's step is captured once as a CUDA graph; W warm-up
replays, then exactly K timed replays bracketed by barrier + synchronize, timed
with CUDA events on the launching stream; the max over ranks is reported.
Per-call durations (the roofline's kernel times) come right after the timed
region from CUDA events around graphs that repeat one call of the step over the
same rotating replicas (event nodes inside a graph cost microseconds each, so
none sit inside the timed step graphs).  SM clocks and throttle reasons are
sampled through NVML during the timed region.  `e2e` repeats the step through the public Python API
with the step's inputs copied from pinned host memory and Y copied back.

Roofline: the dominant call's algorithmic bytes over its live duration against
the measured HBM copy rate; when every contraction of the step runs on the
int8 tensor cores (M >= 5), int8 operations over the live duration of the
bl_linear calls against the measured sustained bf16 GEMM rate x 2 instead (the
HBM figure then moves to `roofline_weight_path`).

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
import sys
import threading
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import workloads  # noqa: E402

METRIC = "BitLinear GMAC/s and weight-stream GB/s (% of HBM/int8 peak), M=1..4096"
UNIT = "GMAC/s"


def parse():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=2000)
    ap.add_argument("--warmup", type=int, default=50)
    ap.add_argument("--workload", type=int, default=2)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--e2e-steps", type=int, default=10)
    ap.add_argument("--cpu-seconds", type=float, default=12.0,
                    help="target CPU time of the oracle baseline sample")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--path", type=int, default=0, help="pin the linear kernel path (BL_PATH_*)")
    ap.add_argument("--concurrent", action="store_true",
                    help="issue the step's independent weight chains on separate streams")
    return ap.parse_args()


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

    def __init__(self, device_index_uuid):
        self.samples, self.reasons, self.max_mhz, self.ok = [], set(), None, False
        try:
            import pynvml as nv
            nv.nvmlInit()
            self.nv = nv
            self.h = nv.nvmlDeviceGetHandleByUUID(device_index_uuid)
            self.max_mhz = nv.nvmlDeviceGetMaxClockInfo(self.h, nv.NVML_CLOCK_SM)
            self.ok = True
        except Exception as e:  # pragma: no cover - depends on the box
            self.err = repr(e)
        self._stop = threading.Event()

    def _poll(self):
        nv = self.nv
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


def tensor_roofline(macs, ms, peaks):
    """Roofline of a step whose contractions all run on the int8 tensor cores:
    int8 operations (2 per multiply-add) per second over the live duration of
    the bl_linear calls, against the measured sustained bf16 GEMM rate times 2
    (the nominal dense int8 : bf16 ratio, 4.5 : 2.25 PFLOP/s)."""
    achieved = 2.0 * macs / (ms * 1e-3) / 1e12
    peak = 2.0 * peaks["bf16_tflops_sustained"]
    return {"bound": "tensor", "achieved": round(achieved, 1), "peak": round(peak, 1), "unit": "TFLOP/s",
            "frac": round(achieved / peak, 4), "traffic": None, "kernel": "gemm_tc_kernel", "call": "bl_linear",
            "ops": "int8: 2 per multiply-add, over whole bl_linear calls (activation quantization, "
                   "[unpack,] GEMM [, K-split reduction])",
            "peak_source": ("measured sustained bf16 x 2 (MEASURED_PEAKS.json bf16_tflops_sustained)"
                            if peaks["source"] == "measured" else "fallback 1.4 PFLOP/s bf16 sustained x 2")}


# The sources a profiled kernel is built from: its header chain, and the lines
# of the library source that name it (its launcher and launch configuration).
KERNEL_SOURCES = {
    "wquant_kernel": (("weight_fused.cuh", "weight_quant.cuh", "act_quant.cuh", "common.cuh", "ptx.cuh"),
                      ("wquant", "kFu", "fused")),
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


# ------------------------------------------------------------- the step ----
class Step:
    """Device buffers and API calls for one replica of the workload's step.

    A weight tensor used by one call runs as one BitLinear forward call (weight
    quantization, activation quantization, contraction, dequant); a tensor shared
    by several calls is quantized once, then each call runs the linear alone."""

    def __init__(self, bl, torch, probs, dev, fmt):
        self.bl, self.torch, self.fmt = bl, torch, fmt
        lib = bl.load()
        self.tensors = []          # weight tensors: (W, beta, Wout, ws, N, K)
        self.calls = []            # calls: (X, tensor index, Y, ws, M, K, N, eps)
        seen, uses = {}, {}
        for p in probs:
            uses[id(p.W)] = uses.get(id(p.W), 0) + 1
        for p in probs:
            key = id(p.W)
            if key not in seen:
                W = torch.from_numpy(p.W).to(dev)
                beta = torch.zeros(1, dtype=torch.float32, device=dev)
                if fmt == bl.PACK5:
                    Wout = torch.empty((p.N, bl.pack5_ldp(p.K)), dtype=torch.uint8, device=dev)
                else:
                    Wout = torch.empty((p.N, p.K), dtype=torch.int8, device=dev)
                fused = uses[key] == 1
                nb = (lib.bl_bitlinear_forward_workspace_size(p.M, p.N, p.K, fmt) if fused
                      else lib.bl_quantize_weights_workspace_size(p.N, p.K))
                ws = bl.workspace(nb, dev)
                seen[key] = len(self.tensors)
                self.tensors.append((W, beta, Wout, ws, p.N, p.K, fused))
            X = torch.from_numpy(np.ascontiguousarray(p.X)).to(dev)
            Y = torch.empty((p.M, p.N), dtype=torch.float32, device=dev)
            fused = self.tensors[seen[key]][6]
            lws = (self.tensors[seen[key]][3] if fused
                   else bl.workspace(bl.linear_workspace_size(p.M, p.N, p.K, fmt), dev))
            self.calls.append((X, seen[key], Y, lws, p.M, p.K, p.N, p.eps))

    def nbytes(self):
        n = 0
        for W, beta, Wout, ws, N, K, fused in self.tensors:
            n += W.numel() * 4 + Wout.numel()
        for X, ti, Y, lws, M, K, N, eps in self.calls:
            n += X.numel() * 4 + Y.numel() * 4 + (0 if self.tensors[ti][6] else lws.numel())
        return n

    def order(self):
        """(kind, index) in issue order: shared tensors' quantization, then calls."""
        out = [("wquant", ti) for ti, t in enumerate(self.tensors) if not t[6]]
        for ci, c in enumerate(self.calls):
            out.append(("forward" if self.tensors[c[1]][6] else "linear", ci))
        return out

    def run(self, only=None, path=0, streams=None):
        """Issue the step, or only entry `only` of order().  With `streams`,
        each weight tensor's chain goes on its own stream, forked from and
        joined back into the current stream."""
        bl, torch = self.bl, self.torch
        main = torch.cuda.current_stream()
        if streams:
            for st in streams:
                st.wait_stream(main)
        for k, (kind, idx) in enumerate(self.order()):
            if only is not None and only != k:
                continue
            ti = idx if kind == "wquant" else self.calls[idx][1]
            st = streams[ti % len(streams)] if streams else main
            with torch.cuda.stream(st):
                if kind == "wquant":
                    W, beta, Wout, ws, N, K, _ = self.tensors[idx]
                    if self.fmt == bl.PACK5:
                        bl.quantize_weights_pack5(W, 1e-5, ws=ws, out=Wout, beta=beta)
                    else:
                        bl.quantize_weights(W, 1e-5, ws=ws, out=Wout, beta=beta)
                else:
                    X, ti2, Y, lws, M, K, N, eps = self.calls[idx]
                    W, beta, Wout, ws, _, _, _ = self.tensors[ti2]
                    if kind == "forward":
                        bl.bitlinear_forward(X, W, self.fmt, eps=eps, ws=ws, w_out=Wout, beta=beta, out=Y)
                    else:
                        bl.linear(X, Wout, self.fmt, N, K, beta, eps=eps, ws=lws, out=Y, path=path)
        if streams:
            for st in streams:
                main.wait_stream(st)

    def labels(self):
        return self.order()


def forward_launches(bl, M, N, K, fmt, path):
    """Kernel launches of one bl_bitlinear_forward call."""
    if M <= 4 and N * K >= 2 ** 20 and K % 4 == 0 and M * K * 4 <= 48 * 1024 and path == 0:
        return 1
    q = 1 if (N * K >= 2 ** 20 and K % 4 == 0) else 2
    return q + bl.linear_plan(M, N, K, fmt, path)[1]


def algorithmic_bytes(kind, N, K, M, fmt):
    """Bytes each kind of call must move at minimum (inputs read + outputs written)."""
    wbytes = N * math.ceil(K / 5) if fmt == 1 else N * K
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

    wl = workloads.WORKLOADS[args.workload]
    fmt = bl.PACK5 if wl.fmt == workloads.FMT_PACK5 else bl.I8
    probs = list(workloads.problems(args.workload, rank=rank))
    macs_per_step = sum(p.M * p.N * p.K for p in probs)

    props = torch.cuda.get_device_properties(dev)
    l2 = int(getattr(props, "L2_cache_size", 126 * 2 ** 20))
    first = Step(bl, torch, probs, dev, fmt)
    R = max(2, math.ceil(4 * l2 / first.nbytes()))
    steps = [first] + [Step(bl, torch, probs, dev, fmt) for _ in range(R - 1)]
    torch.cuda.synchronize()

    # one eager step per replica: launches must succeed and the device stay clean
    for s in steps:
        s.run(path=args.path)
    if bl.sync_status(dev) != "BL_OK":
        raise RuntimeError("device status not clean after the eager step")

    labels = first.labels()
    stream = torch.cuda.Stream(device=dev)
    n_chains = min(len(first.tensors), 4) if args.concurrent else 0
    side = [torch.cuda.Stream(device=dev) for _ in range(n_chains)]
    graphs = []
    with torch.cuda.stream(stream):
        for s in steps:
            g = torch.cuda.CUDAGraph()
            with torch.cuda.graph(g, stream=stream):
                s.run(path=args.path, streams=side or None)
            graphs.append(g)
    torch.cuda.synchronize()

    K, Wm = args.steps, args.warmup
    with torch.cuda.stream(stream):
        for i in range(Wm):
            graphs[i % R].replay()
    torch.cuda.synchronize()
    if world > 1:
        dist.barrier()
    t0 = torch.cuda.Event(enable_timing=True)
    t1 = torch.cuda.Event(enable_timing=True)
    clk = ClockSampler(str(props.uuid) if str(props.uuid).startswith("GPU-") else "GPU-" + str(props.uuid))
    torch.cuda.synchronize()
    with clk:
        with torch.cuda.stream(stream):
            t0.record(stream)
            for i in range(K):
                graphs[(Wm + i) % R].replay()
            t1.record(stream)
        torch.cuda.synchronize()
    if world > 1:
        dist.barrier()
    ms_max = max_over_ranks(t0.elapsed_time(t1), dist, dev)
    if bl.sync_status(dev) != "BL_OK":
        raise RuntimeError("device status not clean after the timed region")

    # per-call durations: for each call of the step, one graph that issues that
    # call for every replica in turn, repeated; CUDA events around its replays
    per_call = {}
    reps = max(1, 64 // R)
    with torch.cuda.stream(stream):
        for i, lab in enumerate(labels):
            g = torch.cuda.CUDAGraph()
            with torch.cuda.graph(g, stream=stream):
                for _ in range(reps):
                    for s in steps:
                        s.run(only=i, path=args.path)
            g.replay()
            c0 = torch.cuda.Event(enable_timing=True)
            c1 = torch.cuda.Event(enable_timing=True)
            c0.record(stream)
            for _ in range(4):
                g.replay()
            c1.record(stream)
            torch.cuda.synchronize()
            per_call[lab] = [c0.elapsed_time(c1) / (4 * reps * R)]
            del g
    shapes = {}
    for kind, idx in labels:
        if kind == "wquant":
            W, beta, Wout, ws, N, Kd, _ = first.tensors[idx]
            shapes[(kind, idx)] = (N, Kd, 0, 1 if ws.numel() > 16384 else 2)
        else:
            X, ti, Y, lws, M, Kd, N, eps = first.calls[idx]
            nl = (forward_launches(bl, M, N, Kd, fmt, args.path) if kind == "forward"
                  else bl.linear_plan(M, N, Kd, fmt, args.path)[1])
            shapes[(kind, idx)] = (N, Kd, M, nl)
    kinds = {}
    for lab, v in per_call.items():
        kind = lab[0]
        N, Kd, M, nl = shapes[lab]
        d = kinds.setdefault(kind, {"ms": 0.0, "bytes": 0, "launches": 0})
        d["ms"] += float(np.mean(v))
        d["bytes"] += algorithmic_bytes(kind, N, Kd, M, fmt)
        d["launches"] += nl
    peaks = measured_peaks()
    kern_names = {"wquant": "wquant_kernel", "linear": "linear", "forward": "wquant_kernel"}
    kernels = {}
    for kind, d in kinds.items():
        gbs = d["bytes"] / (d["ms"] * 1e-3) / 1e9
        kernels[kind] = {"ms_per_step": round(d["ms"], 5), "algorithmic_bytes": d["bytes"],
                         "launches": d["launches"], "achieved_gbs": round(gbs, 1),
                         "frac_hbm": round(gbs / peaks["hbm_gbs"], 4)}
    # the dominant call of the step (the weight call is one launch for tensors
    # of 2^20 weights and more; the linear call is activation quantization plus
    # the contraction, or one fused launch for the GEMV)
    dom = max(kinds, key=lambda k: kinds[k]["ms"])
    dkind = kinds[dom]
    achieved = dkind["bytes"] / (dkind["ms"] * 1e-3) / 1e9
    roofline = {"bound": "hbm", "achieved": round(achieved, 1), "peak": peaks["hbm_gbs"],
                "unit": "GB/s", "frac": round(achieved / peaks["hbm_gbs"], 4),
                "traffic": ncu_traffic(kern_names[dom], args.workload),
                "kernel": kern_names[dom], "call": {"wquant": "bl_quantize_weights*", "linear": "bl_linear",
                                                    "forward": "bl_bitlinear_forward"}[dom],
                "call_launches": dkind["launches"] / max(
                    1, sum(1 for k, _ in labels if k == dom)),
                "peak_source": peaks["source"] + " (MEASURED_PEAKS.json hbm_gbs)"
                if peaks["source"] == "measured" else "fallback 6.65 TB/s"}

    launches_per_step = sum(d["launches"] for d in kinds.values())
    value = whole_job_gmacs(macs_per_step, K, world, ms_max)
    lin = kinds.get("linear")
    if lin is None and "forward" in kinds:
        lin = linear_alone(bl, torch, first, fmt, l2, stream, args.path)
    line = {
        "metric": METRIC, "value": round(value, 2), "unit": UNIT, "n_gpus": world,
        "steps": K, "warmup": Wm, "ms_per_step": round(ms_max / K, 6),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "i8xtrit->i32,f32",
        "data": "synthetic",
        "config": {"workload": f"{wl.id}:{wl.name}", "shapes_MKN": [list(s) for s in wl.shapes],
                   "weight_format": wl.fmt, "parallelism": f"dp{world} (independent batches)",
                   "l2_defeat": f"{R} rotating replicas, {R * first.nbytes() / 2**20:.0f} MiB >= 4x L2 "
                                f"({l2 / 2**20:.0f} MiB)",
                   "step": "per call: absmean beta, ternarize + pack W, per-row int8 X, "
                           "contraction, dequant (one bl_bitlinear_forward call per weight tensor)", "timing": "CUDA graph per replica, CUDA events",
                   "streams": (f"{n_chains} (one per independent weight chain)" if n_chains else "1")},
        "macs_per_step": macs_per_step,
        "linear_only": None if lin is None else {
            "call": "bl_linear on the step's quantized weights",
            "l2_defeat": lin.get("l2_defeat", "the step's rotating replicas"),
            "gmacs": round(macs_per_step / (lin["ms"] * 1e-3) / 1e9, 1),
            "weight_stream_gbs": round(sum(
                (p.N * math.ceil(p.K / 5) if fmt == bl.PACK5 else p.N * p.K) for p in probs)
                / (lin["ms"] * 1e-3) / 1e9, 1),
            "ms_per_step": round(lin["ms"], 5)},
        "kernels": kernels,
        "roofline": roofline,
        "clocks": clk.summary(),
        "gpu_launches": launches_per_step * K,
        "gpu": torch.cuda.get_device_name(dev),
    }
    if line["linear_only"] is not None:
        line["linear_only"]["frac_hbm"] = round(line["linear_only"]["weight_stream_gbs"] / peaks["hbm_gbs"], 4)
    # every contraction on the tensor cores: the step is bound by them, not by HBM
    if lin is not None and all(bl.linear_plan(c[4], c[6], c[5], fmt, args.path)[0] == bl.PATH_TC
                               for c in first.calls):
        line["roofline_weight_path"] = roofline
        line["roofline"] = tensor_roofline(macs_per_step, lin["ms"], peaks)

    # ---- end to end through the public API, host buffers -------------------
    line["e2e"] = e2e(bl, torch, probs, dev, fmt, args.e2e_steps, world)
    for g in graphs:
        del g
    graphs.clear()

    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        line["cpu_baseline"] = cpu_baseline(args.workload, args.cpu_seconds)
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()
    if rank == 0:
        print(json.dumps(line), flush=True)


def linear_alone(bl, torch, step, fmt, l2, stream, path):
    """bl_linear per call of the step on its quantized weights (the contraction
    side of the forward, SURVEY's GEMV unit), over enough copies of the packed
    weights and X to defeat L2; CUDA events around graph replays."""
    per = sum(step.tensors[c[1]][2].numel() + c[0].numel() * 4 for c in step.calls)
    R = max(2, math.ceil(4 * l2 / per))
    reps = []
    for _ in range(R):
        reps.append([(c[0].clone(), step.tensors[c[1]][2].clone(), step.tensors[c[1]][1], c[2].clone(),
                      bl.workspace(bl.linear_workspace_size(c[4], c[6], c[5], fmt), c[0].device), c)
                     for c in step.calls])
    torch.cuda.synchronize()

    def issue():
        for r in reps:
            for X, Wd, beta, Y, lws, c in r:
                bl.linear(X, Wd, fmt, c[6], c[5], beta, eps=c[7], ws=lws, out=Y, path=path)
    with torch.cuda.stream(stream):
        issue()
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g, stream=stream):
            issue()
        g.replay()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        for _ in range(5):
            g.replay()
        e1.record(stream)
    torch.cuda.synchronize()
    ms = e0.elapsed_time(e1) / (5 * R)
    del g
    return {"ms": ms, "l2_defeat": f"{R} copies of packed W and X, {R * per / 2**20:.0f} MiB >= 4x L2"}


def e2e(bl, torch, probs, dev, fmt, steps, world):
    """The step through the public API with pinned host inputs copied in and Y
    copied out: one bl_bitlinear_forward per single-use weight tensor, else
    quantize once and run the linear per call."""
    uses = {}
    for p in probs:
        uses[id(p.W)] = uses.get(id(p.W), 0) + 1
    host_W, host_X, seen = [], [], {}
    for p in probs:
        if id(p.W) not in seen:
            seen[id(p.W)] = len(host_W)
            host_W.append(torch.from_numpy(p.W).pin_memory())
        host_X.append(torch.from_numpy(np.ascontiguousarray(p.X)).pin_memory())
    dW = [torch.empty_like(h, device=dev) for h in host_W]
    dX = [torch.empty_like(h, device=dev) for h in host_X]
    hY = [torch.empty((p.M, p.N), dtype=torch.float32).pin_memory() for p in probs]
    lib = bl.load()
    ws = {}
    for j, p in enumerate(probs):
        i = seen[id(p.W)]
        if uses[id(p.W)] == 1:
            ws[i] = bl.workspace(lib.bl_bitlinear_forward_workspace_size(p.M, p.N, p.K, fmt), dev)
        elif i not in ws:
            ws[i] = bl.workspace(lib.bl_quantize_weights_workspace_size(p.N, p.K), dev)
    h2d = sum(h.numel() * 4 for h in host_W) + sum(h.numel() * 4 for h in host_X)
    d2h = sum(h.numel() * 4 for h in hY)

    def one():
        for h, d in zip(host_W, dW):
            d.copy_(h, non_blocking=True)
        for h, d in zip(host_X, dX):
            d.copy_(h, non_blocking=True)
        packed = {}
        for i, W in enumerate(dW):
            if i in ws and ws[i].numel() and any(uses[id(p.W)] > 1 and seen[id(p.W)] == i for p in probs):
                if fmt == bl.PACK5:
                    packed[i] = bl.quantize_weights_pack5(W, 1e-5, ws=ws[i])
                else:
                    packed[i] = bl.quantize_weights(W, 1e-5, ws=ws[i])
        for j, p in enumerate(probs):
            i = seen[id(p.W)]
            if uses[id(p.W)] == 1:
                Y = bl.bitlinear_forward(dX[j], dW[i], fmt, eps=p.eps, ws=ws[i])[0]
            else:
                Wd, beta = packed[i]
                Y = bl.linear(dX[j], Wd, fmt, p.N, p.K, beta, eps=p.eps)
            hY[j].copy_(Y, non_blocking=True)

    one()
    torch.cuda.synchronize()
    t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    t0.record()
    for _ in range(steps):
        one()
    t1.record()
    torch.cuda.synchronize()
    import torch.distributed as dist
    ms = max_over_ranks(t0.elapsed_time(t1), dist, dev)
    macs = sum(p.M * p.N * p.K for p in probs)
    return {"value": round(whole_job_gmacs(macs, steps, world, ms), 2), "unit": UNIT,
            "h2d_bytes_per_step": int(h2d), "d2h_bytes_per_step": int(d2h),
            "steps": steps, "ms_per_step": round(ms / steps, 4)}


# ------------------------------------------------------------ CPU oracle ----
def oracle_step(probs, rows_frac=1.0):
    """The oracle on (a row slice of) the step's problems; returns MACs done."""
    import oracle
    macs, done = 0, {}
    for p in probs:
        n = max(1, int(round(p.N * rows_frac)))
        W = p.W[:n]
        key = id(p.W)
        if key not in done:
            beta = oracle.absmean_beta(W, p.eps)
            Wq = oracle.ternarize(W, beta)
            if p.fmt == workloads.FMT_PACK5:
                oracle.unpack5(oracle.pack5(Wq), p.K)
            done[key] = (beta, Wq)
        beta, Wq = done[key]
        Xq, s = oracle.act_quant(p.X, p.eps)
        oracle.dequant(oracle.contract(Xq, Wq), s, beta)
        macs += p.M * n * p.K
    return macs


def cpu_sample_fraction(wid, seconds):
    """Row fraction of the step the oracle finishes in about `seconds`."""
    probs = list(workloads.problems(wid))
    frac = 1.0 / 64
    t = time.perf_counter()
    oracle_step(probs, frac)
    dt = time.perf_counter() - t
    return probs, min(1.0, frac * seconds / max(dt, 1e-3))


def cpu_baseline(wid, seconds):
    """The oracle as committed, single-threaded numpy, on a bounded sample of the
    step: a row slice of every weight when a whole step is too long, else whole
    steps repeated until about `seconds` of CPU time."""
    probs, frac = cpu_sample_fraction(wid, seconds)
    t = time.perf_counter()
    macs, reps = 0, 0
    while True:
        macs += oracle_step(probs, frac)
        reps += 1
        if frac < 1.0 or time.perf_counter() - t >= seconds:
            break
    dt = time.perf_counter() - t
    what = (f"{reps} whole step(s)" if frac >= 1.0 else
            f"the step on the first {frac:.4f} of each weight's rows (beta over that slice)")
    return {"value": round(macs / dt / 1e9, 4), "unit": UNIT, "cores": 1, "kind": "oracle",
            "sample": f"{what}, numpy oracle as committed, {dt:.1f} s"}


def run_reference(args):
    rank, world, _ = dist_env()
    if rank != 0:
        return
    wl = workloads.WORKLOADS[args.workload]
    # each reference step: the oracle's whole step on a row slice sized so the run stays short
    probs, frac = cpu_sample_fraction(args.workload, max(0.05, 60.0 / max(1, args.steps + args.warmup)))
    for _ in range(args.warmup):
        oracle_step(probs, frac)
    t = time.perf_counter()
    macs = 0
    for _ in range(args.steps):
        macs += oracle_step(probs, frac)
    dt = time.perf_counter() - t
    value = macs / dt / 1e9
    line = {"impl": "reference", "metric": METRIC, "value": round(value, 4), "unit": UNIT,
            "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": round(dt / max(1, args.steps) * 1e3, 3), "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "i8xtrit->i64,f32", "data": "synthetic",
            "config": {"workload": f"{wl.id}:{wl.name}", "shapes_MKN": [list(s) for s in wl.shapes],
                       "weight_format": wl.fmt, "parallelism": "cpu oracle, rank 0"},
            "cpu_baseline": {"value": round(value, 4), "unit": UNIT, "cores": 1, "kind": "oracle",
                             "sample": f"each step: the whole step on the first {frac:.4f} of each "
                                       f"weight's rows"},
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
