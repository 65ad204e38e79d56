"""Benchmark of the SVDQ W4A4 linear layer (nvfp4, group 16, rank 32).

One step = one forward of the layer: svdq_quantize_act followed by
svdq_gemm_w4a4, inputs resident in HBM, L2 flushed (256 MiB write) before
every step outside the timed events.  The headline workload is the fused-QKV
projection of a DiT at 1024x1024 (4096 image + 512 text tokens): M=4608,
K=3072, N=9216, rank 32.  The weight side is packed once before timing
(offline in the layer's life cycle).  Each step is replayed from a CUDA graph
of the two launches, so host launch overhead stays out of the device time.
The other DiT shapes (MLP fc1 / fc2, the batch-4 attention out-projection over
ranks 0..128, the int4 variant) are reported under "extra" with the same
measurements.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl {cuda,reference}]
                    [--config NAME] [--no-extra] [--dynamic-scale] [--no-cpu-baseline]

Multi-GPU (torchrun, one rank per GPU): every rank runs its own batch of
tokens through its own replica of the packed weight (weak scaling, no
collective on the data path); the step time is the max over ranks.
--impl reference times the CPU oracle on the host cores: each step is the
oracle on a bounded sample of rows of the same workload.
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
UNIT = "TFLOPS"
FP4_OVER_BF16 = 4.0        # nominal dense FP4 : BF16 tensor throughput on B200 (9 : 2.25 PFLOP/s)
# dense block-scaled FP4 work one SM retires per clock: an M128 N256 K64
# kind::mxf4nvf4 MMA (4.19 MFLOP) every 128 cycles, measured on this B200
FP4_FLOP_PER_CLK_SM = 32768
# DRAM bytes per launch taken from ncu captures, with the hash of the kernel
# sources they were taken on; a value whose sources changed since is not used
TRAFFIC_FILE = os.path.join(ROOT, "profiles", "dram_traffic.json")


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
                    "source": "NVML every 1 ms during the timed graphs"}
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


# ------------------------------------------------------------------ helpers
def cpu_model() -> str:
    try:
        with open("/proc/cpuinfo") as f:
            for line in f:
                if line.startswith("model name"):
                    return line.split(":", 1)[1].strip()
    except OSError:
        pass
    import platform

    return platform.processor() or "unknown"


def workload_config(case, dynamic_scale: bool, world: int) -> dict:
    """The `config` object of both arms (identical for the same workload)."""
    names = {"qkv": "DiT fused-QKV projection, 1024^2 (4096 image + 512 text tokens)",
             "fc1": "DiT MLP fc1, 1024^2 (4096 image + 512 text tokens)",
             "fc2": "DiT MLP fc2, 1024^2 (4096 image + 512 text tokens), GELU input",
             "int4_qkv": "DiT fused-QKV projection, int4 W4A4 variant"}
    name = names.get(case.name, f"batch-4 DiT attention out-projection, rank {case.rank}"
                     if case.name.startswith("outproj") else case.name)
    return {"workload": name, "M": case.M, "K": case.K, "N": case.N, "rank": case.rank,
            "group_size": case.group_size, "precision": case.precision,
            "x_tensor_scale": "dynamic (amax pre-pass)" if dynamic_scale else "static (calibrated)",
            "l2": (f"inputs larger than L2: {input_sets(case)} rotating input sets of "
                   f"{set_bytes_estimate(case) / 1e6:.0f} MB (x, packed weight, activation buffers, y), step i on "
                   f"set i mod {input_sets(case)}, steps back to back in one CUDA graph; the L2 flushed "
                   "(256 MiB write) once before it, outside the events"),
            "step": "svdq_quantize_act + svdq_gemm_w4a4", "parallelism": f"replicas x{world} (tokens)"}


def set_bytes_estimate(case) -> int:
    """Device bytes of one input set of the step: x, y, the activation codes
    and scales, the packed weight (nvfp4 scales with their GEMM-ready copy)."""
    M, K, N, r = case.M, case.K, case.N, case.rank
    if case.precision == "nvfp4":
        wsc = N * K // 16 + ((N + 255) // 256) * ((K + 255) // 256) * 16384
        return 2 * M * K + 2 * M * N + M * K // 2 + M * K // 16 + N * K // 2 + wsc + 4 * M * r + 6 * N * r
    return 2 * M * K + 2 * M * N + M * K // 2 + 2 * M * K // 64 + N * K // 2 + 2 * N * K // 64 + 4 * M * r + 6 * N * r


def input_sets(case) -> int:
    """Input sets to rotate through so that, in each of the step, quantizer
    and GEMM graphs, a set is reused only after at least twice the L2 (126 MB)
    of other sets' data has gone through it."""
    least = min(quant_bytes(case), gemm_bytes(case))
    return max(3, 1 + -(-(256 << 20) // least))


def quant_bytes(case) -> int:
    """Algorithmic HBM bytes of the activation quantizer: x read once; codes,
    group scales and the rank-r activations (hi and lo bf16 planes) written once."""
    M, K, r = case.M, case.K, case.rank
    if case.precision == "nvfp4":
        return M * K * 2 + M * K // 2 + M * K // 16 + 4 * M * r
    return M * K * 2 + M * K // 2 + 2 * M * K // 64 + 4 * M * r


def gemm_bytes(case) -> int:
    """Algorithmic HBM bytes of the GEMM: both operands' codes and scales read
    once, the rank-r operands and bias read once, y written once."""
    M, K, N, r = case.M, case.K, case.N, case.rank
    sc = (M + N) * K // 16 if case.precision == "nvfp4" else 2 * (M + N) * K // 64
    return (M + N) * K // 2 + sc + 4 * M * r + 2 * N * r + 2 * N + 2 * M * N


def profiled_traffic(kernel: str):
    """(bytes per launch, note) from the committed ncu summary when the kernel's
    sources are unchanged since it was taken, else (None, why)."""
    import hashlib

    try:
        with open(TRAFFIC_FILE) as f:
            entry = json.load(f)["kernels"][kernel]
    except (OSError, KeyError, ValueError):
        return None, "no ncu capture recorded for this kernel"
    h = hashlib.sha256()
    for rel in entry["source_files"]:
        try:
            with open(os.path.join(ROOT, rel), "rb") as f:
                h.update(f.read())
        except OSError:
            return None, f"source {rel} missing"
    if h.hexdigest() != entry["source_sha256"]:
        return None, "kernel sources changed since the ncu capture"
    return int(entry["dram_bytes_per_launch"]), f"ncu capture on the {entry['workload']} workload"


def fp4_peaks(peaks: dict, sm_mhz) -> dict:
    """The FP4 roofline: measured bf16 burst x the nominal FP4:BF16 ratio, and
    the MMA rate at the SM clock sampled during the run."""
    out = {"peak": peaks["bf16_tflops"] * FP4_OVER_BF16,
           "peak_source": f"{peaks['source']} bf16 burst {peaks['bf16_tflops']} x {FP4_OVER_BF16} (nominal FP4:BF16)"}
    if sm_mhz:
        out["peak_at_clock"] = 148 * FP4_FLOP_PER_CLK_SM * sm_mhz * 1e6 / 1e12
    return out


# ------------------------------------------------------------------ CUDA arm
class Shape:
    """One workload on the device: `sets` copies of the step's inputs (x and
    the packed weight, each with its own activation buffers and y), and CUDA
    graphs of the step that rotate through them."""

    def __init__(self, case, dev, stream, dynamic_scale=False, sets=1):
        import torch

        from bit_w4a4_quantized_token_b200 import _lib, layer
        from bit_w4a4_quantized_token_b200 import workloads as W

        self.case, self.dev, self.stream = case, dev, stream
        inp = W.make_inputs(case)
        self.x_host = inp["x"]
        d = {k: v.to(dev) for k, v in inp.items()}
        r = case.rank
        self.packeds, self.xs, self.qs, self.ys = [], [], [], []
        for k in range(sets):
            p = layer.pack_weight(d["R"], d["lam"], d["L_down"] if r else None, d["L_up"] if r else None,
                                  d["b"], precision=case.precision)
            x = d["x"] if k == 0 else d["x"].clone()
            q = layer.alloc_act(p, case.M, dev)
            # static activation tensor scale, calibrated once (the amax pre-pass)
            layer.quantize_act(x, p, out=q)
            self.packeds.append(p)
            self.xs.append(x)
            self.qs.append(q)
            self.ys.append(torch.empty(case.M, case.N, dtype=torch.bfloat16, device=dev))
        self.packed, self.x, self.q, self.y = self.packeds[0], self.xs[0], self.qs[0], self.ys[0]
        self.sets = sets
        self.compute_scale = 1 if dynamic_scale else 0
        self._lib = _lib
        torch.cuda.synchronize(dev)

    def set_bytes(self) -> int:
        """Device bytes one step touches in its own set: x, the packed weight,
        the activation buffers and y."""
        p, q = self.packed, self.q
        ts = [self.x, p.w_codes, p.w_scales, p.inv_lambda, p.L_down_t, p.L_up_t, p.bias,
              q.x_codes, q.x_scales, q.lowrank_act, q.workspace, self.y]
        return sum(int(v.numel()) * v.element_size() for v in ts if v is not None)

    def quant(self, x=None, k=0):
        c, p, q = self.case, self.packeds[k], self.qs[k]
        self._lib.svdq_quantize_act(c.precision, c.group_size, self.xs[k] if x is None else x, c.M, c.K,
                                    p.inv_lambda, q.x_tensor_scale, self.compute_scale, p.w_tensor_scale, p.L_down_t,
                                    c.rank, q.x_codes, q.x_scales, q.lowrank_act, q.workspace, stream=self.stream)

    def gemm(self, y=None, k=0):
        c, p, q = self.case, self.packeds[k], self.qs[k]
        self._lib.svdq_gemm_w4a4(c.precision, c.group_size, q.x_codes, q.x_scales, q.x_tensor_scale, c.M, p.w_codes,
                                 p.w_scales, p.w_tensor_scale, c.N, c.K, q.lowrank_act, p.L_up_t, c.rank, p.bias,
                                 self.ys[k] if y is None else y, stream=self.stream)

    def graphs(self, steps=1):
        """CUDA graphs of `steps` consecutive steps (step i on set i mod sets),
        of the step and of each kernel alone."""
        import torch

        gs = {}
        for name, parts in (("step", ("quant", "gemm")), ("quant", ("quant",)), ("gemm", ("gemm",))):
            g = torch.cuda.CUDAGraph()
            with torch.cuda.graph(g, stream=self.stream):
                for i in range(steps):
                    for part in parts:
                        getattr(self, part)(k=i % self.sets)
            gs[name] = g
        return gs


def time_qkv_fusion(dev, stream, flush, steps: int) -> dict:
    """The QKV projection with the attention-input RMSNorm + RoPE (24 heads of
    128): fused into the GEMM epilogue against the unfused path (the plain
    GEMM, then the separate norm + rotary pass over its bf16 output)."""
    import torch

    from bit_w4a4_quantized_token_b200 import _lib
    from bit_w4a4_quantized_token_b200 import workloads as W

    case = W.QKV
    heads = case.N // (3 * W.QKV_HEAD_DIM)
    sets = input_sets(case)
    with torch.cuda.stream(stream):
        sh = Shape(case, dev, stream, sets=sets)
        ex = W.qkv_inputs(case.M, heads)
        d = {k: (v.to(dev) if isinstance(v, torch.Tensor) else v) for k, v in ex.items()}

    def fused(k=0):
        p, q = sh.packeds[k], sh.qs[k]
        _lib.svdq_gemm_w4a4_qkv_norm_rope("nvfp4", 16, q.x_codes, q.x_scales, q.x_tensor_scale, case.M, p.w_codes,
                                          p.w_scales, p.w_tensor_scale, case.N, case.K, q.lowrank_act, p.L_up_t,
                                          case.rank, p.bias, heads, W.QKV_HEAD_DIM, d["norm_q"], d["norm_k"],
                                          W.QKV_EPS, d["cos"], d["sin"], sh.ys[k], stream=stream)

    def norm_rope(k=0):
        _lib.svdq_qkv_norm_rope(sh.ys[k], sh.ys[k], case.M, heads, W.QKV_HEAD_DIM, d["norm_q"], d["norm_k"], W.QKV_EPS,
                                d["cos"], d["sin"], stream=stream)

    gs = {}
    for name, fns in (("fused", (sh.quant, fused)), ("unfused", (sh.quant, sh.gemm, norm_rope))):
        with torch.cuda.stream(stream):
            for i in range(3):
                for fn in fns:
                    fn(k=i % sets)
        torch.cuda.synchronize(dev)
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g, stream=stream):
            for i in range(steps):
                for fn in fns:
                    fn(k=i % sets)
        g.replay()
        gs[name] = g
    res = {}
    for name, g in gs.items():
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        with torch.cuda.stream(stream):
            flush.fill_(len(res))
        torch.cuda.synchronize(dev)
        with torch.cuda.stream(stream):
            e0.record(stream)
            g.replay()
            e1.record(stream)
        torch.cuda.synchronize(dev)
        res[name] = e0.elapsed_time(e1) / steps / 1e3
    st, site = _lib.svdq_device_status(clear=True)
    if st != 0:
        raise RuntimeError(f"device status {st} at site {site} in the QKV fusion leg")
    del gs, sh
    return {"workload": "DiT fused-QKV projection + per-head RMSNorm + RoPE (24 heads x 128), M=4608 K=3072 N=9216 "
                        "rank 32",
            "step_us": {"fused": round(res["fused"] * 1e6, 2), "unfused": round(res["unfused"] * 1e6, 2)},
            "speedup": round(res["unfused"] / res["fused"], 3),
            "value": round(case.flops / res["fused"] / 1e12, 2), "unit": UNIT,
            "unfused_step": "svdq_quantize_act + svdq_gemm_w4a4 + svdq_qkv_norm_rope (in place)",
            "fused_step": "svdq_quantize_act + svdq_gemm_w4a4_qkv_norm_rope",
            "timing": f"{steps} steps back to back in one CUDA graph, {sets} rotating input sets"}


FLUSHED_TIMING = ("single steps, each replayed after a 256 MiB L2 flush (outside the events; the event pair "
                  "then also holds the ~6 us any kernel launched right after the flush takes)")


def _graph_time(fns, stream, dev, flush, steps: int) -> float:
    """Seconds per replay of one CUDA graph of `fns` (L2 flushed before each
    replay, outside the events on the launching stream)."""
    import torch

    with torch.cuda.stream(stream):
        for i in range(3):
            flush.fill_(i)
            for fn in fns:
                fn()
    torch.cuda.synchronize(dev)
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=stream):
        for fn in fns:
            fn()
    evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(steps)]
    torch.cuda.synchronize(dev)
    with torch.cuda.stream(stream):
        for i in range(steps):
            flush.fill_(i & 0xFF)
            evs[i][0].record(stream)
            g.replay()
            evs[i][1].record(stream)
    torch.cuda.synchronize(dev)
    del g
    return sum(a.elapsed_time(b) for a, b in evs) / steps / 1e3


def time_gelu_mlp(dev, stream, flush, steps: int) -> dict:
    """The DiT MLP block (3072 -> 12288 -> GELU -> 3072, rank 32, 4608 tokens):
    fc1's GEMM with the fused GELU + fc2-activation epilogue against the
    unfused path (fc1 GEMM -> bf16 -> GELU pass -> fc2's quantizer)."""
    import torch

    from bit_w4a4_quantized_token_b200 import _lib, layer
    from bit_w4a4_quantized_token_b200 import workloads as W

    c1, c2 = W.FC1, W.FC2
    M, Hd = c1.M, c1.N
    with torch.cuda.stream(stream):
        s1, s2 = Shape(c1, dev, stream), Shape(c2, dev, stream)
        p1, q1, p2 = s1.packed, s1.q, s2.packed
        y1 = torch.empty(M, Hd, dtype=torch.bfloat16, device=dev)
        h = torch.empty_like(y1)
        y2 = torch.empty(M, c2.N, dtype=torch.bfloat16, device=dev)
        # fc2's static activation scale: the amax pre-pass on this h, once
        layer.gemm(q1, p1, y1, stream=stream)
        _lib.svdq_gelu(y1, h, M * Hd, 0, stream=stream)
        qu = layer.quantize_act(h, p2, stream=stream)
        qf = layer.alloc_act(p2, M, dev)
        qf.x_tensor_scale.copy_(qu.x_tensor_scale)
        ws = torch.zeros(_lib.svdq_gelu_mlp_workspace_bytes(M, c2.rank) // 4, dtype=torch.float32, device=dev)
    torch.cuda.synchronize(dev)

    def fused_fc1():
        _lib.svdq_gemm_w4a4_gelu_quant("nvfp4", 16, q1.x_codes, q1.x_scales, q1.x_tensor_scale, M, p1.w_codes,
                                       p1.w_scales, p1.w_tensor_scale, Hd, c1.K, q1.lowrank_act, p1.L_up_t, c1.rank,
                                       p1.bias, 0, p2.inv_lambda, p2.L_down_t, c2.rank, qf.x_tensor_scale,
                                       p2.w_tensor_scale, qf.x_codes, qf.x_scales, qf.lowrank_act, ws, stream=stream)

    def fc2_fused():
        layer.gemm(qf, p2, y2, stream=stream)

    def fc1_plain():
        layer.gemm(q1, p1, y1, stream=stream)

    def gelu():
        _lib.svdq_gelu(y1, h, M * Hd, 0, stream=stream)

    def quant2():   # static scale (compute flag 0)
        _lib.svdq_quantize_act("nvfp4", 16, h, M, Hd, p2.inv_lambda, qu.x_tensor_scale, 0, p2.w_tensor_scale,
                               p2.L_down_t, c2.rank, qu.x_codes, qu.x_scales, qu.lowrank_act, qu.workspace,
                               stream=stream)

    def fc2_unfused():
        layer.gemm(qu, p2, y2, stream=stream)

    def fc1_gelu():   # fc1 with only the GELU in its epilogue, storing h
        _lib.svdq_gemm_w4a4_gelu("nvfp4", 16, q1.x_codes, q1.x_scales, q1.x_tensor_scale, M, p1.w_codes, p1.w_scales,
                                 p1.w_tensor_scale, Hd, c1.K, q1.lowrank_act, p1.L_up_t, c1.rank, p1.bias, 0, h,
                                 stream=stream)

    t_f = _graph_time([s1.quant, fused_fc1, fc2_fused], stream, dev, flush, steps)
    t_u = _graph_time([s1.quant, fc1_plain, gelu, quant2, fc2_unfused], stream, dev, flush, steps)
    t_g = _graph_time([s1.quant, fc1_gelu, quant2, fc2_unfused], stream, dev, flush, steps)
    t_f1 = _graph_time([fused_fc1], stream, dev, flush, steps)
    t_p1 = _graph_time([fc1_plain], stream, dev, flush, steps)
    t_g1 = _graph_time([fc1_gelu], stream, dev, flush, steps)
    st, site = _lib.svdq_device_status(clear=True)
    if st != 0:
        raise RuntimeError(f"device status {st} at site {site} in the GELU MLP leg")
    flops = c1.flops + c2.flops
    return {"workload": "DiT MLP 3072 -> 12288 -> GELU -> 3072, rank 32 both layers, M=4608",
            "step_us": {"fused": round(t_f * 1e6, 2), "unfused": round(t_u * 1e6, 2),
                        "gelu_epilogue": round(t_g * 1e6, 2)},
            "speedup": round(t_u / t_f, 3),
            "speedup_gelu_epilogue": round(t_u / t_g, 3),
            "fc1_us": {"gelu_quant_epilogue": round(t_f1 * 1e6, 2), "plain_epilogue": round(t_p1 * 1e6, 2),
                       "gelu_epilogue": round(t_g1 * 1e6, 2)},
            "value": round(flops / t_f / 1e12, 2), "unit": UNIT,
            "fused_step": "quantize_act(fc1) + gemm_w4a4_gelu_quant(fc1) + gemm_w4a4(fc2)",
            "unfused_step": "quantize_act(fc1) + gemm_w4a4(fc1) + gelu + quantize_act(fc2) + gemm_w4a4(fc2)",
            "gelu_epilogue_step": "quantize_act(fc1) + gemm_w4a4_gelu(fc1) + quantize_act(fc2) + gemm_w4a4(fc2)",
            "timing": FLUSHED_TIMING}


def time_w4a16(dev, stream, flush, steps: int, peaks: dict) -> dict:
    """The weight-only int4 GEMM (awq_w4a16, int4 group 64) at the QKV
    projection shape: bf16 x, packed int4 weight, fp16 tensor-core MMA."""
    import torch

    from bit_w4a4_quantized_token_b200 import _lib, layer
    from bit_w4a4_quantized_token_b200 import workloads as W

    case = W.QKV
    with torch.cuda.stream(stream):
        inp = W.make_inputs(case)
        x, Wt, b = inp["x"].to(dev), inp["R"].to(dev), inp["b"].to(dev)
        ones = torch.ones(case.K, dtype=torch.float32, device=dev)
        p = layer.pack_weight(Wt, ones, None, None, b, precision="int4", stream=stream)
        y = torch.empty(case.M, case.N, dtype=torch.bfloat16, device=dev)

    def run():
        _lib.svdq_gemm_w4a16(x, case.M, p.w_codes, p.w_scales, case.N, case.K, p.bias, y, stream=stream)

    t = _graph_time([run], stream, dev, flush, steps)
    st, site = _lib.svdq_device_status(clear=True)
    if st != 0:
        raise RuntimeError(f"device status {st} at site {site} in the W4A16 leg")
    tf = case.flops / t / 1e12
    nbytes = case.M * case.K * 2 + case.N * case.K // 2 + case.N * (case.K // 64) * 2 + case.M * case.N * 2
    return {"workload": "awq_w4a16 weight-only int4 g64 GEMM at the QKV shape, M=4608 K=3072 N=9216",
            "value": round(tf, 2), "unit": "TFLOP/s", "us": round(t * 1e6, 2), "timing": FLUSHED_TIMING,
            "roofline": {"bound": "tensor", "achieved": round(tf, 2), "peak": peaks["bf16_tflops"],
                         "unit": "TFLOP/s", "frac": round(tf / peaks["bf16_tflops"], 4),
                         "peak_source": f"{peaks['source']} bf16 burst (fp16 has the same nominal rate)",
                         "hbm_frac": round(nbytes / t / 1e9 / peaks["hbm_gbs"], 4), "algorithmic_bytes": nbytes}}


def time_svd_split(dev, stream, flush, steps: int) -> dict:
    """The offline split of the QKV weight (9216 x 3072) at rank 32: randomized
    range finder with 8 oversamples and 2 power iterations."""
    import torch

    from bit_w4a4_quantized_token_b200 import _lib
    from bit_w4a4_quantized_token_b200 import workloads as W

    N, K, r, p = W.QKV.N, W.QKV.K, 32, 8
    with torch.cuda.stream(stream):
        d = {k: (v.to(dev) if isinstance(v, torch.Tensor) else v) for k, v in W.svd_split_inputs(N, K, r, p).items()}
        R = torch.empty(N, K, dtype=torch.bfloat16, device=dev)
        Ld = torch.empty(K, r, dtype=torch.bfloat16, device=dev)
        Lu = torch.empty(r, N, dtype=torch.bfloat16, device=dev)
        sv = torch.empty(r + p, dtype=torch.float32, device=dev)
        ws = torch.empty(_lib.svdq_svd_split_workspace_bytes(N, K, r, p), dtype=torch.uint8, device=dev)

    def run():
        _lib.svdq_svd_split(d["W"], d["lam"], N, K, r, d["omega"], p, 2, R, Ld, Lu, sv, ws, ws.numel(),
                            stream=stream)

    with torch.cuda.stream(stream):
        run()
        torch.cuda.synchronize(dev)
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        for _ in range(steps):
            run()
        e1.record(stream)
    torch.cuda.synchronize(dev)
    t = e0.elapsed_time(e1) / steps / 1e3
    st, site = _lib.svdq_device_status(clear=True)
    if st != 0:
        raise RuntimeError(f"device status {st} at site {site} in the SVD split leg")
    return {"workload": f"offline SVD split of a {N} x {K} weight, rank {r}, oversample {p}, 2 power iterations",
            "ms": round(t * 1e3, 3)}


def time_graphs(shape, gs, steps, flush, sampler=None):
    """Device time per step of each graph: `steps` steps back to back in one
    graph replay, step i reading input set i mod sets, so that (with enough
    sets) every step's x and weight come from HBM; CUDA events on the
    launching stream around the replay; the L2 is flushed once before it,
    outside the events."""
    import torch

    st = shape.stream
    res = {}
    for name in ("step", "quant", "gemm"):
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        with torch.cuda.stream(st):
            flush.fill_(len(res))
        torch.cuda.synchronize(shape.dev)
        if sampler is not None and name == "step":
            sampler.begin()
        with torch.cuda.stream(st):
            e0.record(st)
            gs[name].replay()
            e1.record(st)
        torch.cuda.synchronize(shape.dev)
        if sampler is not None and name == "step":
            sampler.end()
        res[name] = e0.elapsed_time(e1) / steps / 1e3
    return res


def time_sustained(shape, flush, steps: int) -> dict:
    """The headline step for long enough (~40 ms back to back) that the SM
    clock settles under the board's power cap; the headline's `--steps` steps
    are a few milliseconds, most of them before it does."""
    import torch

    st = shape.stream
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=st):
        for i in range(steps):
            shape.quant(k=i % shape.sets)
            shape.gemm(k=i % shape.sets)
    g.replay()
    with torch.cuda.stream(st):
        flush.fill_(5)
    torch.cuda.synchronize(shape.dev)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    with torch.cuda.stream(st):
        e0.record(st)
        g.replay()
        e1.record(st)
    torch.cuda.synchronize(shape.dev)
    t = e0.elapsed_time(e1) / steps / 1e3
    del g
    return {"workload": workload_config(shape.case, False, 1)["workload"], "steps": steps,
            "step_us": round(t * 1e6, 2), "value": round(shape.case.flops / t / 1e12, 2), "unit": UNIT,
            "timing": f"{steps} steps back to back in one CUDA graph, rotating input sets as the headline"}


def time_graphs_flushed(shape, gs1, steps, flush):
    """The same per step with a 256 MiB L2 flush before every single-step
    replay (outside the events).  Each event pair then also holds the ~6 us a
    kernel launched right after the flush kernel takes even when it does
    nothing (B200: a kernel that returns at once measures 6.1 us this way)."""
    import torch

    st = shape.stream
    res = {}
    for name in ("step", "quant", "gemm"):
        evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(steps)]
        torch.cuda.synchronize(shape.dev)
        with torch.cuda.stream(st):
            for i in range(steps):
                flush.fill_(i & 0xFF)
                evs[i][0].record(st)
                gs1[name].replay()
                evs[i][1].record(st)
        torch.cuda.synchronize(shape.dev)
        res[name] = sum(a.elapsed_time(b) for a, b in evs) / steps / 1e3
    return res


def shape_report(case, t: dict, peaks: dict, sm_mhz, world: int) -> dict:
    flops = case.flops
    fp = fp4_peaks(peaks, sm_mhz)
    gemm_tf = flops / t["gemm"] / 1e12
    qb = quant_bytes(case)
    out = {"workload": workload_config(case, False, world)["workload"],
           "M": case.M, "K": case.K, "N": case.N, "rank": case.rank, "precision": case.precision,
           "value": round(aggregate(flops, world, t["step"]), 2), "unit": UNIT if case.precision == "nvfp4" else "TOPS",
           "breakdown_us": {"step": round(t["step"] * 1e6, 2), "quantize_act": round(t["quant"] * 1e6, 2),
                            "gemm_w4a4": round(t["gemm"] * 1e6, 2)},
           "quantizer_roofline": {"bound": "hbm", "achieved": round(qb / t["quant"] / 1e9, 1),
                                  "peak": peaks["hbm_gbs"], "unit": "GB/s",
                                  "frac": round(qb / t["quant"] / 1e9 / peaks["hbm_gbs"], 4), "bytes": qb}}
    if case.precision == "nvfp4":
        g = {"bound": "tensor", "achieved": round(gemm_tf, 2), "peak": round(fp["peak"], 1), "unit": "TFLOP/s",
             "frac": round(gemm_tf / fp["peak"], 4)}
        if "peak_at_clock" in fp:
            g["frac_at_clock"] = round(gemm_tf / fp["peak_at_clock"], 4)
        out["roofline"] = g
    else:
        # int4: codes times group scales expanded into fp16, fp16 x fp16 MMAs
        out["roofline"] = {"bound": "tensor", "achieved": round(gemm_tf, 2), "peak": peaks["bf16_tflops"],
                           "unit": "TFLOP/s", "frac": round(gemm_tf / peaks["bf16_tflops"], 4),
                           "peak_source": f"{peaks['source']} bf16 burst (fp16 has the same nominal rate)"}
    if case.rank:
        out["lowrank_flops_not_counted"] = 2 * case.M * case.rank * (case.K + 2 * case.N)
    return out


def run_cuda(args) -> dict | None:
    import torch

    from bit_w4a4_quantized_token_b200 import _lib
    from bit_w4a4_quantized_token_b200 import workloads as W

    world, rank, local = dist_env()
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    if world > 1:
        import datetime

        import torch.distributed as dist

        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120), device_id=dev)

    case = W.BY_NAME[args.config]
    stream = torch.cuda.Stream(dev)
    flush = torch.empty(256 << 20, dtype=torch.uint8, device=dev)
    with torch.cuda.stream(stream):
        sh = Shape(case, dev, stream, args.dynamic_scale, sets=input_sets(case))
        for i in range(args.warmup):
            sh.quant(k=i % sh.sets)
            sh.gemm(k=i % sh.sets)
    torch.cuda.synchronize(dev)
    st, site = _lib.svdq_device_status(clear=True)
    if st != 0:
        raise RuntimeError(f"device status {st} at site {site} during warm-up")
    gs = sh.graphs(args.steps)
    for g in gs.values():   # warm the graphs too
        g.replay()
    gs1 = sh.graphs(1)
    for g in gs1.values():
        g.replay()
    torch.cuda.synchronize(dev)
    flushed_steps = min(args.steps, 20)

    sampler = ClockSampler(local, dev)
    sampler.start()
    time.sleep(0.05)
    if world > 1:
        dist.barrier()
    # clocks are taken over all the timed graphs (back to back, then one step
    # per flush): the step graph alone lasts only a few milliseconds
    sampler.begin()
    t = time_graphs(sh, gs, args.steps, flush)
    t_fl = time_graphs_flushed(sh, gs1, flushed_steps, flush)
    sampler.end()
    if world > 1:
        dist.barrier()
    clocks = sampler.stop()
    st, site = _lib.svdq_device_status(clear=True)
    if st != 0:
        raise RuntimeError(f"device status {st} at site {site} in the timed region")
    t = {k: max_over_ranks(v, world, dev) for k, v in t.items()}
    t_fl = {k: max_over_ranks(v, world, dev) for k, v in t_fl.items()}

    # end to end through the public API: every step copies its x from pinned
    # host memory to the device, runs the quantizer and the GEMM, and copies
    # y back to pinned host memory.  Steps are pipelined over three streams
    # (input copies, compute, output copies) with two device buffers of x and
    # of y, so that step i's copies overlap the neighbouring steps' work, as a
    # serving loop would run them; the copy engines of both directions work
    # at once.
    x_host = sh.x_host.pin_memory()
    y_host = [torch.empty(case.M, case.N, dtype=torch.bfloat16).pin_memory() for _ in range(2)]
    xd = [sh.x, torch.empty_like(sh.x)]
    yd = [sh.y, torch.empty_like(sh.y)]
    s_in, s_out = torch.cuda.Stream(dev), torch.cuda.Stream(dev)
    x_ready, x_free, y_ready, y_free = ([torch.cuda.Event() for _ in range(2)] for _ in range(4))

    def e2e_step(i):
        b = i % 2
        if i >= 2:
            s_in.wait_event(x_free[b])
        with torch.cuda.stream(s_in):
            xd[b].copy_(x_host, non_blocking=True)
            x_ready[b].record(s_in)
        stream.wait_event(x_ready[b])
        with torch.cuda.stream(stream):
            sh.quant(x=xd[b])
            x_free[b].record(stream)
            if i >= 2:
                stream.wait_event(y_free[b])
            sh.gemm(y=yd[b])
            y_ready[b].record(stream)
        s_out.wait_event(y_ready[b])
        with torch.cuda.stream(s_out):
            y_host[b].copy_(yd[b], non_blocking=True)
            y_free[b].record(s_out)

    e2e_steps = max(2, min(args.steps, 20))
    for i in range(2):
        e2e_step(i)
    torch.cuda.synchronize(dev)
    if world > 1:
        dist.barrier()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(s_in)
    for i in range(2, 2 + e2e_steps):
        e2e_step(i)
    s_out.wait_stream(s_in)
    s_out.wait_stream(stream)
    e1.record(s_out)
    torch.cuda.synchronize(dev)
    t_e2e = max_over_ranks(e0.elapsed_time(e1) / e2e_steps / 1e3, world, dev)
    del gs

    peaks = load_peaks()
    report = shape_report(case, t, peaks, clocks.get("sm_mhz"), world)
    report["breakdown_us"]["flushed_per_step"] = {k: round(v * 1e6, 2) for k, v in t_fl.items()}
    extra = {}
    if world == 1 and not args.no_extra:
        names = ["qkv", "fc1", "fc2"] + [f"outproj_r{r}" for r in (0, 16, 32, 64, 128)] + ["int4_qkv"]
        for name in names:
            if name == case.name:
                continue
            c = W.BY_NAME[name]
            n2 = max(6, min(args.steps, 20))
            with torch.cuda.stream(stream):
                s2 = Shape(c, dev, stream, sets=input_sets(c))
                for i in range(3):
                    s2.quant(k=i % s2.sets)
                    s2.gemm(k=i % s2.sets)
            g2 = s2.graphs(n2)
            for g in g2.values():
                g.replay()
            t2 = time_graphs(s2, g2, n2, flush)
            st, site = _lib.svdq_device_status(clear=True)
            if st != 0:
                raise RuntimeError(f"device status {st} at site {site} on {name}")
            extra[name] = shape_report(c, t2, peaks, clocks.get("sm_mhz"), world)
            del g2, s2
            torch.cuda.empty_cache()
        extra["qkv_norm_rope"] = time_qkv_fusion(dev, stream, flush, max(3, min(args.steps, 10)))
        torch.cuda.empty_cache()
        extra["gelu_mlp"] = time_gelu_mlp(dev, stream, flush, max(3, min(args.steps, 10)))
        torch.cuda.empty_cache()
        extra["w4a16_qkv"] = time_w4a16(dev, stream, flush, max(3, min(args.steps, 10)), peaks)
        torch.cuda.empty_cache()
        extra["svd_split_qkv"] = time_svd_split(dev, stream, flush, 3)
        torch.cuda.empty_cache()
        extra[f"{case.name}_sustained"] = time_sustained(sh, flush, 400)
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()
    if rank != 0:
        return None

    traffic, traffic_note = profiled_traffic("gemm_nvfp4_pair_kernel")
    qtraffic, qtraffic_note = profiled_traffic("quantize_act_kernel")
    roofline = dict(report["roofline"], kernel="gemm_nvfp4_pair_kernel",
                    peak_source=fp4_peaks(peaks, None)["peak_source"], traffic=traffic, traffic_note=traffic_note,
                    algorithmic_bytes=gemm_bytes(case))
    if "frac_at_clock" in roofline:
        roofline["peak_at_clock_note"] = (f"148 SMs x {FP4_FLOP_PER_CLK_SM} FLOP/clk x the sampled "
                                          f"{clocks.get('sm_mhz')} MHz; the 60 % target is judged against `peak`")
    qroof = dict(report["quantizer_roofline"], kernel="quantize_act_kernel", traffic=qtraffic,
                 traffic_note=qtraffic_note)
    # our kernels launched in the timed passes of this workload: the step graph
    # (quantizer, GEMM) and the quantizer and GEMM graphs alone, back to back
    # (`steps` steps each) and single steps after a flush; the end-to-end steps
    n_quant = 1 + (2 if args.dynamic_scale else 0)   # + the amax pre-pass and its finalisation
    launches = 2 * (n_quant + 1) * (args.steps + flushed_steps) + (n_quant + 1) * e2e_steps
    return {
        "metric": METRIC,
        "value": report["value"],
        "unit": UNIT,
        "n_gpus": world,
        "steps": args.steps,
        "warmup": args.warmup,
        "ms_per_step": round(t["step"] * 1e3, 5),
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": "nvfp4 (e2m1 x e2m1, ue4m3 group scales) -> fp32 accumulate -> bf16"
                 if case.precision == "nvfp4" else "int4 codes x bf16 group scales -> fp16 x fp16 -> fp32 -> bf16",
        "data": "synthetic (seeded DiT-shaped activations with 1% outlier channels; random-init weights)",
        "config": workload_config(case, args.dynamic_scale, world),
        "breakdown_us": report["breakdown_us"],
        "roofline": roofline,
        "quantizer_roofline": qroof,
        "e2e": {"value": round(aggregate(case.flops, world, t_e2e), 3), "unit": UNIT,
                "h2d_bytes_per_step": case.M * case.K * 2, "d2h_bytes_per_step": case.M * case.N * 2},
        "gpu_launches": launches,
        "clocks": clocks,
        "extra": extra,
    }


# ------------------------------------------------------------------ CPU oracle
def oracle_setup(case):
    """Inputs of the workload and the offline (untimed) weight side, for the oracle."""
    from bit_w4a4_quantized_token_b200 import workloads as W
    from oracle import oracle as O

    inp = W.make_inputs(case)
    x, lam = W.bits(inp["x"]), inp["lam"].numpy()
    Ld, Lu, b = W.bits(inp["L_down"]), W.bits(inp["L_up"]), W.bits(inp["b"])
    R = W.bits(inp["R"])
    S_w = O.nvfp4_tensor_scale(R, None)
    wc, ws = O.nvfp4_quantize(R, None, S_w)
    wd = O.nvfp4_dequant(wc, ws, S_w)          # weight packing is offline: not timed
    S_x = O.nvfp4_tensor_scale(x, lam)         # static scale, as in the CUDA arm
    return {"x": x, "lam": lam, "Ld": Ld, "Lu": Lu, "b": b, "wd": wd, "S_x": S_x}


def oracle_pass(o, rows: int, start: int = 0) -> float:
    """One oracle forward on `rows` token rows (quantize + rank-r + fp64 GEMM + bias); seconds."""
    import numpy as np

    from oracle import oracle as O

    xs = np.ascontiguousarray(o["x"][start:start + rows])
    t0 = time.perf_counter()
    xc, xsc = O.nvfp4_quantize(xs, o["lam"], o["S_x"])
    L = O.lowrank_down(xs, o["lam"], o["Ld"])
    xd = O.nvfp4_dequant(xc, xsc, o["S_x"])
    O.nvfp4_linear(xd, o["wd"], L, o["Lu"], o["b"])
    return time.perf_counter() - t0


def rows_for(o, case, seconds: float) -> int:
    t64 = oracle_pass(o, 64)
    return int(min(case.M, max(64, 64 * round(seconds / max(t64, 1e-3)))))


def cpu_baseline_obj(case, target_s: float = 10.0) -> dict:
    from oracle import oracle as O

    o = oracle_setup(case)
    rows = rows_for(o, case, target_s)
    t = oracle_pass(o, rows)
    cores = O.num_threads()
    return {"value": round(2 * rows * case.N * case.K / t / 1e12, 6), "unit": UNIT, "cores": cores,
            "cpu": cpu_model(), "kind": "oracle",
            "sample": f"{rows} of {case.M} token rows of the {case.name} workload (quantize + rank-r + fp64 GEMM "
                      f"+ bias), {t:.1f} s on {cores} threads"}


def run_reference(args) -> dict | None:
    """The oracle as it stands, timed on the host cores: `warmup` untimed and
    `steps` timed passes, each over the same bounded sample of rows."""
    from bit_w4a4_quantized_token_b200 import workloads as W
    from oracle import oracle as O

    world, rank, _ = dist_env()
    if rank != 0:
        return None
    case = W.BY_NAME[args.config]
    o = oracle_setup(case)
    # size one pass so that warm-up + timed passes take about two minutes
    per_pass = max(1.0, min(10.0, 120.0 / (args.steps + args.warmup)))
    rows = rows_for(o, case, per_pass)
    for i in range(args.warmup):
        oracle_pass(o, rows, start=(i * rows) % max(1, case.M - rows + 1))
    ts = [oracle_pass(o, rows, start=(i * rows) % max(1, case.M - rows + 1)) for i in range(args.steps)]
    t = sum(ts) / len(ts)
    v = 2 * rows * case.N * case.K / t / 1e12
    cores = O.num_threads()
    cb = {"value": round(v, 6), "unit": UNIT, "cores": cores, "cpu": cpu_model(), "kind": "oracle",
          "sample": f"{rows} of {case.M} token rows of the {case.name} workload per step "
                    f"(quantize + rank-r + fp64 GEMM + bias), {args.steps} timed + {args.warmup} warm-up passes, "
                    f"{t:.2f} s per pass on {cores} threads"}
    return {
        "impl": "reference", "metric": METRIC, "value": round(v, 6), "unit": UNIT, "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(t * 1e3, 3),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic (seeded DiT-shaped activations with 1% outlier channels; random-init weights)",
        "config": workload_config(case, args.dynamic_scale, world),
        "cpu_baseline": cb,
        "e2e": {"value": round(v, 6), "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }


def run_leg(args) -> dict:
    """One extra leg on cuda:0 (one GPU), e.g. to capture its kernels with ncu."""
    import torch

    dev = torch.device("cuda", 0)
    torch.cuda.set_device(dev)
    stream = torch.cuda.Stream(dev)
    flush = torch.empty(256 << 20, dtype=torch.uint8, device=dev)
    steps = max(3, args.steps)
    if args.leg == "qkv_norm_rope":
        return time_qkv_fusion(dev, stream, flush, steps)
    if args.leg == "gelu_mlp":
        return time_gelu_mlp(dev, stream, flush, steps)
    if args.leg == "w4a16_qkv":
        return time_w4a16(dev, stream, flush, steps, load_peaks())
    return time_svd_split(dev, stream, flush, steps)


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=50)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["cuda", "reference"], default="cuda")
    ap.add_argument("--config", default="qkv",
                    choices=["qkv", "fc1", "fc2", "outproj_r0", "outproj_r16", "outproj_r32", "outproj_r64",
                             "outproj_r128", "int4_qkv"], help="the headline workload (default: the QKV projection)")
    ap.add_argument("--no-extra", action="store_true", help="skip the other DiT shapes")
    ap.add_argument("--dynamic-scale", action="store_true", help="derive S_x by the amax pre-pass every step")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--leg", choices=["qkv_norm_rope", "gelu_mlp", "w4a16_qkv", "svd_split_qkv"],
                    help="time one of the extra legs alone and print its JSON (for profiling)")
    args = ap.parse_args()
    if args.warmup < 3:
        args.warmup = 3
    if args.leg:
        print(json.dumps(run_leg(args)), flush=True)
        return
    if args.impl == "reference":
        out = run_reference(args)
    else:
        # the CPU baseline runs first, before any CUDA work, on rank 0 at N=1 only
        world, rank, _ = dist_env()
        cb = None
        if world == 1 and not args.no_cpu_baseline:
            from bit_w4a4_quantized_token_b200 import workloads as W

            cb = cpu_baseline_obj(W.BY_NAME[args.config] if args.config != "int4_qkv" else W.QKV, target_s=10.0)
        out = run_cuda(args)
        if out is not None:
            out["cpu_baseline"] = cb
    if out is not None:
        print(json.dumps(out), flush=True)


if __name__ == "__main__":
    main()
