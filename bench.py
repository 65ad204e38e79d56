"""Benchmark of the SVDQ W4A4 linear layer (nvfp4, group 16, rank 32).

One step = one forward of the layer on the fused-QKV projection of a DiT at
1024x1024 (4096 image + 512 text tokens): M=4608, K=3072, N=9216, rank 32,
i.e. svdq_quantize_act followed by svdq_gemm_w4a4, inputs resident in HBM,
L2 flushed (256 MiB write) before every step.  The weight side is packed
once before timing (offline in the layer's life cycle).

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl {cuda,reference}]

Multi-GPU (torchrun, one rank per GPU): every rank runs its own batch of
tokens through its own replica of the packed weight (weak scaling, no
collective on the data path); the step time is the max over ranks.
--impl reference times the CPU oracle on the host cores on a bounded sample
of rows of the same workload.
"""
from __future__ import annotations

import argparse
import json
import os
import statistics
import subprocess
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

METRIC = "SVDQ W4A4 linear TFLOPS (2MNK) and % of B200 dense FP4 tensor peak"

# DRAM bytes (read + write) per launch from one ncu capture of the kernels as
# they are now (profiles/gemm_nvfp4_pair_qkv.md, profiles/quantize_act_nvfp4_qkv.md).
# Set an entry to None whenever its kernel changes until it is profiled again.
PROFILED_DRAM_BYTES = {
    "gemm_nvfp4_pair_kernel": 25369344 + 32259072,
    "quantize_act_kernel": 28766208 + 0,
}
UNIT = "TFLOPS"
FP4_OVER_BF16 = 4.0        # nominal dense FP4 : BF16 tensor throughput on B200 (9 : 2.25 PFLOP/s)


def load_peaks() -> dict:
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            p = json.load(f)
        return {"hbm_gbs": float(p["hbm_gbs"]), "bf16_tflops": float(p["bf16_tflops"]),
                "bf16_tflops_sustained": float(p.get("bf16_tflops_sustained", p["bf16_tflops"])),
                "source": "measured"}
    except (OSError, KeyError, ValueError):
        return {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0, "source": "fallback"}


# ------------------------------------------------------------------ ranks
def dist_env():
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return world, rank, local


def max_over_ranks(value: float, world: int, device=None) -> float:
    """Max of a per-rank float over all ranks (identity when world == 1)."""
    if world == 1:
        return value
    import torch
    import torch.distributed as dist

    t = torch.tensor([value], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def aggregate(per_rank_flops: float, world: int, t_max_s: float) -> float:
    """Whole-job throughput: the work of all ranks over the slowest rank's time."""
    return per_rank_flops * world / t_max_s / 1e12


# ------------------------------------------------------------------ clocks
# Polls one GPU's SM clock, power and clock-event reasons through NVML every
# millisecond and prints "t,sm_mhz,power_w,reason_bits" lines (t: the
# system-wide monotonic clock).  Read-only queries; run as its own process so
# that the bench's Python launch loop cannot starve it of the GIL.
SAMPLER_SRC = r"""
import sys, time
import pynvml
pynvml.nvmlInit()
h = None
if sys.argv[1]:
    try:
        h = pynvml.nvmlDeviceGetHandleByUUID(sys.argv[1])
    except Exception:
        h = None
if h is None:
    h = pynvml.nvmlDeviceGetHandleByIndex(int(sys.argv[2]))
print("max,%d" % pynvml.nvmlDeviceGetMaxClockInfo(h, pynvml.NVML_CLOCK_SM), flush=True)
get_r = getattr(pynvml, "nvmlDeviceGetCurrentClocksEventReasons", None) or pynvml.nvmlDeviceGetCurrentClocksThrottleReasons
while True:
    t = time.monotonic()
    sm = pynvml.nvmlDeviceGetClockInfo(h, pynvml.NVML_CLOCK_SM)
    try:
        pw = pynvml.nvmlDeviceGetPowerUsage(h) / 1000.0
    except Exception:
        pw = 0.0
    try:
        rs = int(get_r(h))
    except Exception:
        rs = 0
    print("%.6f,%d,%.1f,%d" % (t, sm, pw, rs), flush=True)
    time.sleep(0.001)
"""


class ClockSampler:
    """SM clock, power and clock-event (throttle) reasons of one GPU while the
    timed region runs: a child process polls NVML every millisecond (see
    SAMPLER_SRC); only samples between begin() and end() count.  Without NVML
    it falls back to nvidia-smi at 100 ms."""

    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")
    # NVML clock-event reason bits
    REASON_BITS = (("sw_power_cap", 0x4), ("hw_slowdown", 0x8), ("sw_thermal_slowdown", 0x20),
                   ("hw_thermal_slowdown", 0x40), ("hw_power_brake_slowdown", 0x80))

    def __init__(self, gpu_index: int, torch_device=None):
        self.gpu = gpu_index
        self.torch_device = torch_device
        self.proc = None
        self.mode = None
        self.lines = []
        self._t = None
        self._ready = threading.Event()
        self.max_mhz = None
        self.t_begin = self.t_end = None

    def _nvml_index_and_uuid(self):
        idx = self.gpu
        vis = os.environ.get("CUDA_VISIBLE_DEVICES", "")
        ids = [v.strip() for v in vis.split(",") if v.strip()]
        if ids and all(v.isdigit() for v in ids) and self.gpu < len(ids):
            idx = int(ids[self.gpu])
        uuid = ""
        if self.torch_device is not None:
            try:
                import torch

                u = str(torch.cuda.get_device_properties(self.torch_device).uuid)
                uuid = u if u.startswith("GPU-") else "GPU-" + u
            except Exception:
                uuid = ""
        return idx, uuid

    def start(self):
        idx, uuid = self._nvml_index_and_uuid()
        try:
            self.proc = subprocess.Popen([sys.executable, "-c", SAMPLER_SRC, uuid, str(idx)],
                                         stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            self.mode = "nvml"
            self._t = threading.Thread(target=self._read, daemon=True)
            self._t.start()
            self._ready.wait(timeout=20.0)
            if self.max_mhz is not None:
                return
            self._kill()
        except OSError:
            self.proc = None
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.gpu), f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                 "-lms", "100"], stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            self.mode = "smi"
            self.lines = []
            self._t = threading.Thread(target=self._read, daemon=True)
            self._t.start()
        except OSError:
            self.proc = None
            self.mode = None

    def _read(self):
        proc = self.proc
        for line in proc.stdout:
            line = line.strip()
            if self.mode == "nvml" and line.startswith("max,"):
                self.max_mhz = float(line.split(",")[1])
                self._ready.set()
                continue
            self.lines.append((time.monotonic(), line))
        self._ready.set()      # the poller ended (or never started): stop waiting for it

    def _kill(self):
        if self.proc is None:
            return
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        if self._t:
            self._t.join(timeout=2)

    def begin(self):
        self.t_begin = time.monotonic()

    def end(self):
        self.t_end = time.monotonic()

    def _in_region(self, t):
        return (self.t_begin is None or t >= self.t_begin) and (self.t_end is None or t <= self.t_end)

    def stop(self) -> dict:
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["no clock sampler available"]}
        self._kill()
        if self.mode == "nvml":
            rows = []
            for _, ln in self.lines:
                parts = ln.split(",")
                if len(parts) != 4:
                    continue
                try:
                    t, sm, pw, rs = float(parts[0]), float(parts[1]), float(parts[2]), int(parts[3])
                except ValueError:
                    continue
                if self._in_region(t):
                    rows.append((sm, pw, rs))
            if not rows:
                return {"sm_mhz": None, "sm_max_mhz": self.max_mhz, "reasons": ["no samples in the timed region"]}
            reasons = sorted({name for _, _, bits in rows for name, bit in self.REASON_BITS if bits & bit})
            return {"sm_mhz": statistics.median(r[0] for r in rows), "sm_max_mhz": self.max_mhz,
                    "reasons": reasons, "samples": len(rows), "power_w_max": max(r[1] for r in rows),
                    "source": "NVML every 1 ms during the timed region"}
        sm, smax, power, reasons = [], [], [], set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for _, ln in self.lines:
            parts = [p.strip() for p in ln.split(",")]
            if len(parts) < 9:
                continue
            try:
                sm.append(float(parts[1]))
                smax.append(float(parts[2]))
                power.append(float(parts[3]))
            except ValueError:
                continue
            for name, flag in zip(names, parts[5:9]):
                if flag.lower() == "active":
                    reasons.add(name)
        if not sm:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["no samples"]}
        loaded = [s for s, p in zip(sm, power) if p > 0.3 * max(power)] or sm
        return {"sm_mhz": statistics.median(loaded), "sm_max_mhz": max(smax), "reasons": sorted(reasons),
                "samples": len(sm), "power_w_max": max(power), "source": "nvidia-smi every 100 ms"}


# ------------------------------------------------------------------ CUDA arm
def run_cuda(args) -> dict | None:
    import torch

    from bit_w4a4_quantized_token_b200 import _lib, layer
    from bit_w4a4_quantized_token_b200 import workloads as W

    world, rank, local = dist_env()
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    if world > 1:
        import datetime

        import torch.distributed as dist

        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120), device_id=dev)

    case = W.QKV
    M, K, N, r = case.M, case.K, case.N, case.rank
    inp = W.make_inputs(case)
    d = {k: v.to(dev) for k, v in inp.items()}
    stream = torch.cuda.current_stream(dev)
    packed = layer.pack_weight(d["R"], d["lam"], d["L_down"], d["L_up"], d["b"], precision="nvfp4")
    q = layer.alloc_act(packed, M, dev)
    y = torch.empty(M, N, dtype=torch.bfloat16, device=dev)
    # static activation tensor scale, calibrated once (the amax pre-pass)
    layer.quantize_act(d["x"], packed, out=q)
    if args.dynamic_scale:
        compute_scale = 1
    else:
        compute_scale = 0
    flush = torch.empty(256 << 20, dtype=torch.uint8, device=dev)
    x = d["x"]

    def step():
        _lib.svdq_quantize_act("nvfp4", 16, x, M, K, packed.inv_lambda, q.x_tensor_scale, compute_scale,
                               packed.w_tensor_scale, packed.L_down_t, r, q.x_codes, q.x_scales, q.lowrank_act,
                               q.workspace, stream=stream)

    def gemm():
        _lib.svdq_gemm_w4a4("nvfp4", 16, q.x_codes, q.x_scales, q.x_tensor_scale, M, packed.w_codes,
                            packed.w_scales, packed.w_tensor_scale, N, K, q.lowrank_act, packed.L_up_t, r,
                            packed.bias, y, stream=stream)

    for _ in range(args.warmup):
        flush.fill_(1)
        step()
        gemm()
    torch.cuda.synchronize(dev)
    st, site = _lib.svdq_device_status(clear=True)
    if st != 0:
        raise RuntimeError(f"device status {st} at site {site} during warm-up")

    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(3)] for _ in range(args.steps)]
    sampler = ClockSampler(local, dev)
    sampler.start()
    time.sleep(0.05)
    if world > 1:
        import torch.distributed as dist

        dist.barrier()
    torch.cuda.synchronize(dev)
    sampler.begin()
    for i in range(args.steps):
        flush.fill_(i & 0xFF)
        evs[i][0].record(stream)
        step()
        evs[i][1].record(stream)
        gemm()
        evs[i][2].record(stream)
    torch.cuda.synchronize(dev)
    sampler.end()
    if world > 1:
        dist.barrier()
    clocks = sampler.stop()
    st, site = _lib.svdq_device_status(clear=True)
    if st != 0:
        raise RuntimeError(f"device status {st} at site {site} in the timed region")
    t_quant = sum(e[0].elapsed_time(e[1]) for e in evs) / args.steps / 1e3
    t_gemm = sum(e[1].elapsed_time(e[2]) for e in evs) / args.steps / 1e3
    t_step = max_over_ranks(t_quant + t_gemm, world, dev)
    t_gemm_max = max_over_ranks(t_gemm, world, dev)
    t_quant_max = max_over_ranks(t_quant, world, dev)

    # end to end through the public API: pinned host x -> device, forward, y -> pinned host
    x_host = inp["x"].pin_memory()
    y_host = torch.empty(M, N, dtype=torch.bfloat16).pin_memory()
    x_dev = torch.empty_like(x)
    e2e_steps = max(1, min(args.steps, 20))
    for _ in range(2):
        x_dev.copy_(x_host, non_blocking=True)
        layer.gemm(layer.quantize_act(x_dev, packed, out=q, x_tensor_scale=q.x_tensor_scale), packed, y=y)
        y_host.copy_(y, non_blocking=True)
    torch.cuda.synchronize(dev)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    if world > 1:
        dist.barrier()
    e0.record(stream)
    for _ in range(e2e_steps):
        x_dev.copy_(x_host, non_blocking=True)
        _lib.svdq_quantize_act("nvfp4", 16, x_dev, M, K, packed.inv_lambda, q.x_tensor_scale, compute_scale,
                               packed.w_tensor_scale, packed.L_down_t, r, q.x_codes, q.x_scales, q.lowrank_act,
                               q.workspace, stream=stream)
        gemm()
        y_host.copy_(y, non_blocking=True)
    e1.record(stream)
    torch.cuda.synchronize(dev)
    t_e2e = max_over_ranks(e0.elapsed_time(e1) / e2e_steps / 1e3, world, dev)
    # the int4 W4A4 variant on the same QKV shape (group 64, bf16 scales): reported beside the headline
    int4 = time_int4(args, dev, stream, flush)
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()
    if rank != 0:
        return None

    flops = case.flops
    peaks = load_peaks()
    fp4_peak = peaks["bf16_tflops"] * FP4_OVER_BF16
    gemm_tflops = flops / t_gemm_max / 1e12
    quant_bytes = M * K * 2 + M * K // 2 + M * K // 16 + 4 * M * r + K * 4
    launches = (2 if not args.dynamic_scale else 4) * args.steps   # quantize_act + gemm per step
    extra = {"int4_qkv": int4}
    return {
        "metric": METRIC,
        "value": round(aggregate(flops, world, t_step), 3),
        "unit": UNIT,
        "n_gpus": world,
        "steps": args.steps,
        "warmup": args.warmup,
        "ms_per_step": round(t_step * 1e3, 5),
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": "nvfp4 (e2m1 x e2m1, ue4m3 group scales) -> fp32 accumulate -> bf16",
        "data": "synthetic (seeded DiT-shaped activations with 1% outlier channels; random-init weights)",
        "config": {"workload": "DiT fused-QKV projection, 1024^2 (4096 image + 512 text tokens)",
                   "M": M, "K": K, "N": N, "rank": r, "group_size": 16, "precision": "nvfp4",
                   "x_tensor_scale": "dynamic (amax pre-pass)" if args.dynamic_scale else "static (calibrated)",
                   "l2": "flushed before every step (256 MiB write, outside the timed events)",
                   "step": "svdq_quantize_act + svdq_gemm_w4a4", "parallelism": f"replicas x{world} (tokens)"},
        "breakdown_us": {"quantize_act": round(t_quant_max * 1e6, 2), "gemm_w4a4": round(t_gemm_max * 1e6, 2)},
        "roofline": {"bound": "tensor", "kernel": "gemm_nvfp4_pair_kernel", "achieved": round(gemm_tflops, 2),
                     "peak": round(fp4_peak, 1), "unit": "TFLOP/s", "frac": round(gemm_tflops / fp4_peak, 4),
                     "peak_source": f"{peaks['source']} bf16 burst {peaks['bf16_tflops']} x {FP4_OVER_BF16} (nominal FP4:BF16)",
                     "traffic": PROFILED_DRAM_BYTES.get("gemm_nvfp4_pair_kernel")},
        "quantizer_roofline": {"bound": "hbm", "kernel": "quantize_act_kernel",
                               "achieved": round(quant_bytes / t_quant_max / 1e9, 1), "peak": peaks["hbm_gbs"],
                               "unit": "GB/s", "frac": round(quant_bytes / t_quant_max / 1e9 / peaks["hbm_gbs"], 4),
                               "traffic": PROFILED_DRAM_BYTES.get("quantize_act_kernel")},
        "e2e": {"value": round(aggregate(flops, world, t_e2e), 3), "unit": UNIT,
                "h2d_bytes_per_step": M * K * 2, "d2h_bytes_per_step": M * N * 2},
        "gpu_launches": launches,
        "clocks": clocks,
        "extra": extra,
    }


def time_int4(args, dev, stream, flush) -> dict:
    """Device time of the int4 W4A4 layer (quantize + GEMM) on the QKV shape."""
    import torch

    from bit_w4a4_quantized_token_b200 import _lib, layer
    from bit_w4a4_quantized_token_b200 import workloads as W

    case = W.INT4_QKV
    M, K, N, r = case.M, case.K, case.N, case.rank
    inp = W.make_inputs(case)
    d = {k: v.to(dev) for k, v in inp.items()}
    packed = layer.pack_weight(d["R"], d["lam"], d["L_down"], d["L_up"], d["b"], precision="int4")
    q = layer.alloc_act(packed, M, dev)
    y = torch.empty(M, N, dtype=torch.bfloat16, device=dev)
    steps = max(3, min(args.steps, 10))
    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(3)] for _ in range(steps)]
    for i in range(args.warmup + steps):
        flush.fill_(i & 0xFF)
        j = i - args.warmup
        if j >= 0:
            evs[j][0].record(stream)
        layer.quantize_act(d["x"], packed, out=q, stream=stream)
        if j >= 0:
            evs[j][1].record(stream)
        layer.gemm(q, packed, y=y, stream=stream)
        if j >= 0:
            evs[j][2].record(stream)
    torch.cuda.synchronize(dev)
    st, site = _lib.svdq_device_status(clear=True)
    if st != 0:
        raise RuntimeError(f"device status {st} at site {site} in the int4 leg")
    tq = sum(e[0].elapsed_time(e[1]) for e in evs) / steps / 1e3
    tg = sum(e[1].elapsed_time(e[2]) for e in evs) / steps / 1e3
    return {"workload": "int4 W4A4 QKV projection M=4608 K=3072 N=9216 rank 32 group 64",
            "value": round(case.flops / (tq + tg) / 1e12, 2), "unit": "TOPS",
            "breakdown_us": {"quantize_act": round(tq * 1e6, 2), "gemm_w4a4": round(tg * 1e6, 2)}}


# ------------------------------------------------------------------ CPU oracle
def oracle_sample(target_s: float = 10.0):
    """Times the CPU oracle on a bounded sample of rows of the same workload."""
    import numpy as np

    from bit_w4a4_quantized_token_b200 import workloads as W
    from oracle import oracle as O

    case = W.QKV
    inp = W.make_inputs(case)
    x, lam = W.bits(inp["x"]), inp["lam"].numpy()
    Ld, Lu, b = W.bits(inp["L_down"]), W.bits(inp["L_up"]), W.bits(inp["b"])
    R = W.bits(inp["R"])
    S_w = O.nvfp4_tensor_scale(R, None)
    wc, ws = O.nvfp4_quantize(R, None, S_w)
    wd = O.nvfp4_dequant(wc, ws, S_w)          # weight packing is offline: not timed
    S_x = O.nvfp4_tensor_scale(x, lam)         # static scale, as in the CUDA arm

    def run(rows: int) -> float:
        xs = np.ascontiguousarray(x[:rows])
        t0 = time.perf_counter()
        xc, xsc = O.nvfp4_quantize(xs, lam, S_x)
        L = O.lowrank_down(xs, lam, Ld)
        xd = O.nvfp4_dequant(xc, xsc, S_x)
        O.nvfp4_linear(xd, wd, L, Lu, b)
        return time.perf_counter() - t0

    t64 = run(64)
    rows = int(min(case.M, max(64, 64 * round(target_s / max(t64, 1e-3)))))
    t = run(rows)
    tflops = 2 * rows * case.N * case.K / t / 1e12
    return case, rows, t, tflops, O.num_threads()


def cpu_baseline_obj(target_s: float = 10.0) -> dict:
    case, rows, t, tflops, cores = oracle_sample(target_s)
    return {"value": round(tflops, 6), "unit": UNIT, "cores": cores, "kind": "oracle",
            "sample": f"{rows} of {case.M} token rows of the QKV workload (quantize + rank-r + fp64 GEMM + bias), "
                      f"{t:.1f} s on {cores} threads"}


def run_reference(args) -> dict | None:
    world, rank, _ = dist_env()
    if rank != 0:
        return None
    cb = cpu_baseline_obj(target_s=max(3.0, min(20.0, 4.0 * args.steps)))
    from bit_w4a4_quantized_token_b200 import workloads as W

    case = W.QKV
    v = cb["value"]
    return {
        "impl": "reference", "metric": METRIC, "value": v, "unit": UNIT, "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": round(case.flops / (v * 1e12) * 1e3, 3) if v else None,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic", "config": {"workload": "DiT fused-QKV projection, 1024^2 (4096 image + 512 text tokens)",
                                        "M": case.M, "K": case.K, "N": case.N, "rank": case.rank,
                                        "group_size": 16, "precision": "nvfp4"},
        "cpu_baseline": cb,
        "e2e": {"value": v, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=50)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["cuda", "reference"], default="cuda")
    ap.add_argument("--dynamic-scale", action="store_true", help="derive S_x by the amax pre-pass every step")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    args = ap.parse_args()
    if args.warmup < 3:
        args.warmup = 3
    if args.impl == "reference":
        out = run_reference(args)
    else:
        # the CPU baseline runs first, before any CUDA work, on rank 0 at N=1 only
        world, rank, _ = dist_env()
        cb = None
        if world == 1 and not args.no_cpu_baseline:
            cb = cpu_baseline_obj(target_s=10.0)
        out = run_cuda(args)
        if out is not None:
            out["cpu_baseline"] = cb
    if out is not None:
        print(json.dumps(out), flush=True)


if __name__ == "__main__":
    main()
