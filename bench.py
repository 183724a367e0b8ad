"""Benchmark of the MoE layer forward on B200: tokens/s of whole layer steps.

    python bench.py [--gpus N] [--steps K] [--warmup W]
                    [--workload all|decode|prefill|skewed|fp8|tiny|mx|prefill_shared]
                    [--impl ours|reference] [--schedule ...] [--pair ...] [--swap-ab ...] [--shape K=V,...]

One step = one pass of the whole layer (router softmax top-k, permute, grouped
gate/up GEMM + SwiGLU, grouped down GEMM, combine) over one batch of seeded
synthetic inputs already resident in HBM.  L2 is flushed (a 512 MiB write, then a 256 MiB read)
before every step, outside that step's CUDA-event pair.  Prints one JSON line.

With no --workload (``all``) every workload is timed in turn, K steps each, and the
line printed is the headline workload's -- Skewed (T=8192, H=4096, E=64, top-6,
I=1408), the largest configuration and the only compute-bound one -- with the
other four workloads' lines, each complete, under its ``workloads`` key, together
with two variants of the layer: ``mx`` (FP4 e2m1 weights and e4m3 activations with
per-32 power-of-two scales, on the FP8 workload's shapes) and ``prefill_shared`` (the
Prefill workload with a shared expert of 2 x I columns).

Multi-GPU: the layer does not shard on one node in this design, so N GPUs run N
independent replicas (one process per GPU, launched by torchrun); the time is the
max over ranks and ``value`` counts the tokens of all ranks.

``--impl reference`` times the CPU oracle (the only reference there is) on the
host cores, rank 0 only, each step a bounded sample of the same workload.
"""
from __future__ import annotations

import argparse
import datetime as _dt
import hashlib
import json
import math
import os
import statistics
import subprocess
import sys
import threading
import time

import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

from routed_grouped_gemm_softmax_b200.inputs import (CONFIGS, EXTRA_WORKLOADS, make_fp8_weights,  # noqa: E402
                                                     make_inputs, make_mx_weights, make_shared_weights, pack_e2m1)

METRIC = "MoE-layer tokens/s at 1 B200; % of BF16/FP8 TC peak or % of HBM BW"
HEADLINE = "skewed"                                   # the largest configuration
ALL_ORDER = ["tiny", "decode", "prefill", "fp8", "mx", "prefill_shared", HEADLINE]   # the headline is timed last
WORKLOADS = dict(CONFIGS, **EXTRA_WORKLOADS)
GEMM_TRACE_CTAS = 1024


def schedule_stats(trace, mode):
    """Per GEMM: the span from the first CTA start to the last CTA end, and how busy the
    CTAs were over it (busy = that CTA's own start-to-end time)."""
    out = {"mode": mode}
    for k, name in enumerate(("gemm_gate_up", "gemm_down")):
        spans = [(trace[2 * (k * GEMM_TRACE_CTAS + c)], trace[2 * (k * GEMM_TRACE_CTAS + c) + 1])
                 for c in range(GEMM_TRACE_CTAS)]
        spans = [(a, b) for a, b in spans if b > a > 0]
        if not spans:
            continue
        t0, t1 = min(a for a, _ in spans), max(b for _, b in spans)
        busy = sorted((b - a) / (t1 - t0) for a, b in spans)
        out[name] = {"ctas": len(spans), "span_us": round((t1 - t0) / 1e3, 1),
                     "busy_mean": round(sum(busy) / len(busy), 3), "busy_min": round(busy[0], 3),
                     "busy_median": round(busy[len(busy) // 2], 3)}
    return out


def kernels_per_forward(cfg, plan=None) -> int:
    """Library kernels one forward launches (plan: the library's MOE_PLAN bits for the
    run's settings, when known; the layer GEMM is one launch for both expert GEMMs)."""
    A = cfg.T * cfg.top_k
    if cfg.T > 32:
        route = 3 + 3      # transpose/norms, tensor-core logits, certify; count, scan, scatter
    elif cfg.E % 8 == 0 and cfg.H % 128 == 0 and A <= 4096 and (A + 31) // 32 * cfg.E <= 16384:
        route = 2          # logits, top-k + grouping
    else:
        route = 2 + 3      # logits, top-k; count, scan, scatter
    # small batches combine inside the down GEMM (bf16 up to 32 tokens, fp8 up to 64)
    combine = 0 if cfg.T <= (64 if cfg.dtype == "fp8" else 32) else 1
    # fp8 / MX: quantise per token, then gather; bf16: the gather kernel, or (up to 16
    # rows per expert) the gate/up GEMM gathers x rows itself
    rows = 2 if cfg.dtype in ("fp8", "mx") else (0 if A <= 16 * cfg.E else 1)
    if cfg.dtype == "mx":
        combine = 1   # the MX down GEMM has no fused combine
    gemms = 1 if cfg.dtype == "bf16" else 2   # bf16: both expert GEMMs in one launch (the layer kernel)
    if plan is not None and plan >= 0:
        combine = 0 if plan & 4 else 1       # MOE_PLAN_FUSED_COMBINE
        gemms = 1 if plan & 8 else 2         # MOE_PLAN_LAYER_GEMM
        if cfg.dtype == "bf16":
            rows = 0 if plan & 16 else 1     # MOE_PLAN_DIRECT_A, else the gather kernel
    return route + rows + gemms + combine
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}
B200_SMS, FP32_LANES_PER_SM = 148, 128   # CUDA-core fp32 FMA lanes of one B200


def alu_peak_tflops(sm_max_mhz: float) -> float:
    """CUDA-core fp32 peak: every lane retiring one FMA (2 FLOPs) per cycle at the max SM clock."""
    return B200_SMS * FP32_LANES_PER_SM * 2 * sm_max_mhz * 1e6 / 1e12
FLUSH_BYTES = 512 << 20
L2_BYTES = 126 << 20      # the B200's L2
EVICT_FLOATS = 64 << 20   # 256 MiB read after the write, so the flush leaves no dirty lines


def parse():
    p = argparse.ArgumentParser()
    p.add_argument("--gpus", type=int, default=1)
    p.add_argument("--steps", type=int, default=400)
    p.add_argument("--warmup", type=int, default=20)
    p.add_argument("--workload", default="all", choices=["all"] + sorted(WORKLOADS))
    p.add_argument("--impl", default="ours", choices=["ours", "reference"])
    p.add_argument("--no-e2e", action="store_true")
    p.add_argument("--no-cpu-baseline", action="store_true")
    p.add_argument("--cpu-budget", type=float, default=None,
                   help="seconds of oracle work behind each cpu_baseline (default 20, or 12 per "
                        "workload when all workloads run)")
    p.add_argument("--schedule", default="queue", choices=["queue", "static_items", "static_experts"],
                   help="how the GEMM CTAs get work items: the atomic queue (the design), or a static "
                        "split of the items or of the experts (ablations)")
    p.add_argument("--pair", default="auto", choices=["auto", "always", "never"],
                   help="the bf16 GEMMs on CTA pairs (tcgen05 cta_group::2): automatic choice or forced")
    p.add_argument("--swap-ab", default="auto", choices=["auto", "always", "never"],
                   help="the fp8 gate/up GEMM with swapped MMA operands: automatic choice or forced")
    p.add_argument("--layer-gemm", default="auto", choices=["auto", "always", "never"],
                   help="both bf16 expert GEMMs in one persistent launch: automatic choice or forced")
    p.add_argument("--direct-a", default="auto", choices=["auto", "always", "never"],
                   help="bf16 gate/up A rows gathered straight from x by the GEMM, or from a sorted "
                        "copy of x made by a gather kernel: automatic choice or forced")
    p.add_argument("--fused-combine", default="auto", choices=["auto", "always", "never"],
                   help="the bf16 combine inside the down GEMM's epilogue: automatic choice or forced")
    p.add_argument("--tile-sweep", action="store_true",
                   help="instead of the bench line: time the kernel variants (tile shapes, one or two GEMM "
                        "launches, combine placement, fp8 operand order) over M buckets of average rows per "
                        "expert, one JSON line per bucket (the data behind the library's tile table)")
    p.add_argument("--shape", default="",
                   help="override config fields, e.g. T=1024,E=64 (reduced cases for profiler captures)")
    return p.parse_args()


def workload_config(args, name=None):
    name = name or (HEADLINE if args.workload == "all" else args.workload)
    cfg = WORKLOADS[name]
    if args.shape:
        kw = {}
        for item in args.shape.split(","):
            key, val = item.split("=")
            kw[key.strip()] = int(val)
        cfg = cfg.replace(name=f"{cfg.name}[{args.shape}]", **kw)
    return cfg


# ------------------------------------------------------------------ helpers

def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            d = json.load(f)
        p = {k: float(d[k]) for k in FALLBACK_PEAKS}
        p["sm_max_mhz"] = float(d.get("sm_max_mhz", 1965.0))
        return p, "measured"
    except (OSError, KeyError, ValueError):
        return dict(FALLBACK_PEAKS, sm_max_mhz=1965.0), "fallback"


STAGE_SOURCES = {
    "route": ["route.cu", "route_certified.cu", "route_common.cuh", "fp8.cu", "fp8_common.cuh", "sm100_ptx.cuh",
              "moe_internal.h"],
    "gemm_gate_up": ["grouped_gemm.cu", "grouped_gemm_2cta.cu", "fp8.cu", "fp8_swapab.cu", "fp8_common.cuh",
                     "mx.cu", "sm100_ptx.cuh", "moe_internal.h"],
    "gemm_down": ["grouped_gemm.cu", "grouped_gemm_2cta.cu", "fp8.cu", "fp8_common.cuh", "mx.cu", "combine.cuh",
                  "sm100_ptx.cuh", "moe_internal.h"],
    "combine": ["combine.cu", "combine.cuh"],
    "gemm_layer": ["grouped_gemm.cu", "grouped_gemm_2cta.cu", "combine.cuh", "sm100_ptx.cuh", "moe_internal.h"],
}


def kernel_sources_hash(stage: str) -> str:
    """Hash of the CUDA sources a stage's kernel is built from."""
    h = hashlib.sha256()
    csrc = os.path.join(ROOT, "routed_grouped_gemm_softmax_b200", "csrc")
    for name in STAGE_SOURCES.get(stage, sorted(os.listdir(csrc))):
        with open(os.path.join(csrc, name), "rb") as f:
            h.update(name.encode() + f.read())
    return h.hexdigest()[:16]


def recorded_traffic(workload: str, stage: str):
    """DRAM bytes per launch of `stage` from the committed ncu capture summary, or None
    when there is none or the kernel sources changed since it was taken."""
    path = os.path.join(ROOT, "profiles", "traffic.json")
    try:
        with open(path) as f:
            d = json.load(f)
    except (OSError, ValueError):
        return None
    rec = d.get(workload, {}).get(stage)
    if not rec or rec.get("sources") != kernel_sources_hash(stage):
        return None
    return rec.get("dram_bytes_per_launch")


class ClockSampler:
    """SM clock and clock-event (throttle) reasons of this GPU while the timed region
    runs: NVML polled every 2 ms from a background thread (the timed region can be a
    few milliseconds long), or nvidia-smi every 50 ms where NVML is missing.  Reads
    only; changes no setting."""
    Q = ("timestamp,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
         "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
         "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")
    NAMES = ("hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap")

    def __init__(self, device: int):
        self.proc = None
        self.lines = []
        self.samples = []  # NVML: (unix time, SM MHz, reason bitmask)
        self.nv = self.handle = self.thread = None
        self.max_mhz = None
        self.stop_flag = threading.Event()
        try:
            p = torch.cuda.get_device_properties(device)
            bus = f"{p.pci_domain_id:08X}:{p.pci_bus_id:02X}:{p.pci_device_id:02X}.0"
        except Exception:
            bus = None
        try:
            import pynvml
            pynvml.nvmlInit()
            self.handle = (pynvml.nvmlDeviceGetHandleByPciBusId(bus) if bus else
                           pynvml.nvmlDeviceGetHandleByIndex(device))
            self.max_mhz = float(pynvml.nvmlDeviceGetMaxClockInfo(self.handle, pynvml.NVML_CLOCK_SM))
            self.nv = pynvml
            self.bits = (pynvml.nvmlClocksEventReasonHwSlowdown, pynvml.nvmlClocksEventReasonHwThermalSlowdown,
                         pynvml.nvmlClocksEventReasonSwThermalSlowdown, pynvml.nvmlClocksEventReasonSwPowerCap)
        except Exception:
            self.nv = self.handle = None
        self.cmd = ["nvidia-smi", f"--query-gpu={self.Q}", "--format=csv,noheader,nounits",
                    "-lms", "50", *(["-i", bus] if bus else [])]

    def _poll(self):
        nv, h = self.nv, self.handle
        while not self.stop_flag.is_set():
            try:
                self.samples.append((time.time(), float(nv.nvmlDeviceGetClockInfo(h, nv.NVML_CLOCK_SM)),
                                     int(nv.nvmlDeviceGetCurrentClocksEventReasons(h))))
            except Exception:
                pass
            time.sleep(0.002)

    def start(self):
        if self.nv is not None:
            self.thread = threading.Thread(target=self._poll, daemon=True)
            self.thread.start()
            return
        try:
            self.proc = subprocess.Popen(self.cmd, stdout=subprocess.PIPE, stderr=subprocess.DEVNULL,
                                         text=True)
        except OSError:
            self.proc = None

    def stop(self):
        if self.thread is not None:
            self.stop_flag.set()
            self.thread.join(timeout=5)
            return
        if self.proc is None:
            return
        self.proc.terminate()
        try:
            out, _ = self.proc.communicate(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
            out, _ = self.proc.communicate()
        self.lines = [ln for ln in out.splitlines() if ln.strip()]

    def summary(self, t0: float, t1: float):
        sm, mx, reasons = [], self.max_mhz, set()
        if self.thread is not None:
            for ts, mhz, bits in self.samples:
                if t0 <= ts <= t1:
                    sm.append(mhz)
                    reasons.update(n for n, b in zip(self.NAMES, self.bits) if bits & b)
            return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": mx,
                    "reasons": sorted(reasons), "samples": len(sm), "source": "nvml, 2 ms"}
        for ln in self.lines:
            f = [x.strip() for x in ln.split(",")]
            if len(f) < 9:
                continue
            try:
                ts = _dt.datetime.strptime(f[0], "%Y/%m/%d %H:%M:%S.%f").timestamp()
            except ValueError:
                continue
            if not (t0 - 0.05 <= ts <= t1 + 0.05):
                continue
            try:
                sm.append(float(f[1]))
                mx = float(f[2])
            except ValueError:
                continue
            for n, v in zip(self.NAMES, f[5:9]):
                if v.lower() == "active":
                    reasons.add(n)
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": mx,
                "reasons": sorted(reasons), "samples": len(sm), "source": "nvidia-smi, 50 ms"}


def rank_env():
    """(world size, rank, local rank) from the launcher's environment."""
    return (int(os.environ.get("WORLD_SIZE", "1")), int(os.environ.get("RANK", "0")),
            int(os.environ.get("LOCAL_RANK", "0")))


def dist_setup(backend: str = "nccl"):
    """One process per GPU: the process group the replicas use for their barrier and
    the max over ranks (NCCL on the GPUs; gloo for the CPU tests of this logic)."""
    world, rank, local = rank_env()
    if world > 1:
        import torch.distributed as dist
        if backend == "nccl":
            torch.cuda.set_device(local)
            dist.init_process_group("nccl", timeout=_dt.timedelta(seconds=300),
                                    device_id=torch.device("cuda", local))
        else:
            dist.init_process_group(backend, timeout=_dt.timedelta(seconds=60))
    return world, rank, local


def dist_teardown(world):
    if world > 1:
        import torch.distributed as dist
        dist.destroy_process_group()


def barrier(world):
    if world > 1:
        import torch.distributed as dist
        dist.barrier()


def max_over_ranks(v: float, world: int) -> float:
    if world == 1:
        return v
    import torch.distributed as dist
    t = torch.tensor([v], dtype=torch.float64, device="cuda" if dist.get_backend() == "nccl" else "cpu")
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def throughput(tokens_per_rank: int, world: int, steps: int, total_ms: float) -> float:
    """Whole-job tokens/s: the tokens every replica processed over the slowest rank's time."""
    return tokens_per_rank * world * steps / (total_ms * 1e-3)


# ----------------------------------------------------------- per-stage bytes

def _weight_bytes(cfg, N, K):
    """Bytes of one expert's [N, K] weight matrix: bf16; e4m3 + an fp32 scale per 128x128
    block (fp8); packed e2m1 (half a byte) + an e8m0 scale per 32 along K (MX)."""
    if cfg.dtype == "fp8":
        return N * K + (N // 128) * (K // 128) * 4
    if cfg.dtype == "mx":
        return N * K // 2 + N * K // 32
    return N * K * 2


def _act_bytes(cfg, n):
    """Bytes of n activation values as the GEMMs read or write them: bf16; e4m3 + an fp32
    scale per 128 (fp8); e4m3 + an e8m0 scale per 32 (MX)."""
    if cfg.dtype == "fp8":
        return n + n // 128 * 4
    if cfg.dtype == "mx":
        return n + n // 32
    return 2 * n


def stage_work(cfg, counts):
    """Algorithmic bytes and FLOPs of each stage for the realised routing (counts[e] =
    rows of expert e).  Weight bytes count only the touched experts, in the workload's
    storage (_weight_bytes); a shared expert of shared_mult * I columns adds its weights,
    its T rows of x and h and its FLOPs."""
    T, H, I, E, k = cfg.T, cfg.H, cfg.I, cfg.E, cfg.top_k
    A = T * k
    D = int(sum(1 for c in counts if c > 0))
    SI = cfg.shared_mult * I
    return {
        # T <= 32: every logit is an fp32 FMA chain on the CUDA cores; above, the logits run
        # on the tensor cores and only the candidates' chains on the CUDA cores
        "route": {"bytes": T * H * 2 + H * E * 2 + A * 8, "flops": 2.0 * T * H * E, "alu": T <= 32},
        "gemm_gate_up": {"bytes": D * 2 * _weight_bytes(cfg, I, H) + _act_bytes(cfg, A * H) + _act_bytes(cfg, A * I)
                                  + (2 * SI * H * 2 + T * H * 2 + T * SI * 2 if SI else 0),
                         "flops": 2.0 * A * H * 2 * I + 2.0 * T * H * 2 * SI},
        "gemm_down": {"bytes": D * _weight_bytes(cfg, H, I) + _act_bytes(cfg, A * I) + A * H * 2
                               + (H * SI * 2 + T * SI * 2 + cfg.shared_mult * T * H * 2 if SI else 0),
                      "flops": 2.0 * A * I * H + 2.0 * T * SI * H},
        "combine": {"bytes": (A + cfg.shared_mult * T) * H * 2 + A * 4 + T * H * 2, "flops": 2.0 * A * H},
        "_D": D,
    }


def layer_work(cfg, counts):
    """The whole layer's algorithmic bytes and FLOPs: the touched experts' weights (with
    their scales where quantised) and a shared expert's, x, out, router_w and the chosen
    indices and gates; the router and expert FLOPs.  The expert-ordered copy of x, h and
    y are the implementation's own traffic, counted apart in `implementation_bytes`
    (each written once and read once)."""
    T, H, I, E, k = cfg.T, cfg.H, cfg.I, cfg.E, cfg.top_k
    A = T * k
    D = int(sum(1 for c in counts if c > 0))
    SI, m = cfg.shared_mult * I, cfg.shared_mult
    per_expert = 2 * _weight_bytes(cfg, I, H) + _weight_bytes(cfg, H, I)
    inter = 2 * _act_bytes(cfg, A * H) + 2 * _act_bytes(cfg, A * I) + 2 * (A * H * 2)
    inter += 2 * (m * T * I * 2) + 2 * (m * T * H * 2)  # a shared expert's h and y rows
    return {"bytes": D * per_expert + 3 * SI * H * 2 + 2 * T * H * 2 + H * E * 2 + A * 8,
            "flops": 2.0 * A * H * 2 * I + 2.0 * A * I * H + 2.0 * T * H * E + 2.0 * T * H * 3 * SI,
            "implementation_bytes": inter}


def layer_roofline(cfg, counts, ms, peaks, peaks_kind, sustained):
    """The layer per step against its binding roofline: HBM when its algorithmic bytes
    take longer at the measured bandwidth than its FLOPs at the measured tensor peak."""
    w = layer_work(cfg, counts)
    fp8 = cfg.dtype in ("fp8", "mx")  # e4m3 x e4m3 and e2m1 x e4m3 MMAs run at the fp8 rate
    pk_tf = peaks["bf16_tflops_sustained" if sustained else "bf16_tflops"] * (2.0 if fp8 else 1.0)
    t = ms * 1e-3
    if w["bytes"] / (peaks["hbm_gbs"] * 1e9) >= w["flops"] / (pk_tf * 1e12):
        achieved, peak, unit, bound = w["bytes"] / t / 1e9, peaks["hbm_gbs"], "GB/s", "hbm"
    else:
        achieved, peak, unit, bound = w["flops"] / t / 1e12, pk_tf, "TFLOP/s", "tensor"
    return {"bound": bound, "achieved": round(achieved, 1), "peak": peak, "unit": unit,
            "frac": round(achieved / peak, 4), "algorithmic_bytes": w["bytes"], "algorithmic_flops": w["flops"],
            "implementation_bytes": w["implementation_bytes"], "peak_source": peaks_kind, "ms": round(ms, 5)}


def roofline_for(stage, work, ms, peaks, peaks_kind, sustained, workload, fp8=False):
    w = work[stage]
    t = ms * 1e-3
    bw_time = w["bytes"] / (peaks["hbm_gbs"] * 1e9)
    # fp8 tensor peak = measured bf16 peak x the nominal fp8/bf16 ratio (4.5 / 2.25 PF)
    pk_tf = peaks["bf16_tflops_sustained" if sustained else "bf16_tflops"] * (2.0 if fp8 else 1.0)
    tc_time = w["flops"] / (pk_tf * 1e12)
    if w.get("alu"):
        achieved = w["flops"] / t / 1e12
        r = {"bound": "alu", "achieved": round(achieved, 3),
             "peak": round(alu_peak_tflops(peaks.get("sm_max_mhz", 1965.0)), 1), "unit": "TFLOP/s"}
    elif bw_time >= tc_time:
        achieved = w["bytes"] / t / 1e9
        r = {"bound": "hbm", "achieved": round(achieved, 1), "peak": peaks["hbm_gbs"], "unit": "GB/s"}
    else:
        achieved = w["flops"] / t / 1e12
        r = {"bound": "tensor", "achieved": round(achieved, 1), "peak": pk_tf, "unit": "TFLOP/s"}
    r["frac"] = round(achieved / r["peak"], 4)
    r["traffic"] = recorded_traffic(workload, stage)
    r["kernel"] = stage
    r["algorithmic_bytes"] = w["bytes"]
    r["algorithmic_flops"] = w["flops"]
    if r["bound"] == "alu":
        r["peak_source"] = "148 SMs x 128 fp32 lanes x 2 FLOPs x the max SM clock"
    else:
        r["peak_source"] = f"{peaks_kind}" + ("" if r["bound"] == "hbm" else (" sustained" if sustained else " burst")
                                              + (" bf16 x 2 (nominal fp8/bf16 ratio)" if fp8 else ""))
    r["ms"] = round(ms, 4)
    return r


# ------------------------------------------------------------- CPU oracle leg

def host_inputs(cfg, inp=None, wq=None, shared=None):
    """The workload's tensors as host numpy arrays (bf16 bit patterns; quantised codes
    and scales for fp8 / MX), drawn on the GPU when one is present (data preparation
    only; nothing of the layer runs there).  wq: the fp8 or MX weights already drawn."""
    import types

    import numpy as np
    dev = "cuda" if torch.cuda.is_available() else "cpu"
    if inp is None:
        inp = make_inputs(cfg, device=dev, weights=cfg.dtype == "bf16")

    def bits(t):
        return t.detach().cpu().contiguous().view(torch.int16).numpy().view(np.uint16)
    ns = types.SimpleNamespace(
        x=bits(inp.x), router_w=bits(inp.router_w),
        bias=None if inp.bias is None else inp.bias.detach().cpu().float().numpy(), fp8=None, mx=None,
        shared=None)
    if cfg.dtype == "fp8":
        if wq is None:
            wq = make_fp8_weights(cfg, device=inp.x.device)
        ns.fp8 = {k: v.detach().cpu().numpy() for k, v in wq.items()}
    elif cfg.dtype == "mx":
        if wq is None:
            wq = make_mx_weights(cfg, device=inp.x.device)
        ns.mx = {k: v.detach().cpu().numpy() for k, v in wq.items()}
    else:
        ns.w_gate, ns.w_up, ns.w_down = bits(inp.w_gate), bits(inp.w_up), bits(inp.w_down)
    if cfg.shared_mult:
        if shared is None:
            shared = make_shared_weights(cfg, cfg.shared_mult * cfg.I, device=inp.x.device)
        ns.shared = [bits(t) for t in shared]
    return ns


def oracle_step_timer(cfg, h):
    """Returns f(n) -> (route seconds, FFN seconds) for one oracle pass: the routing of
    all T tokens plus the expert FFN/combine of n sampled tokens; and the threads used."""
    import numpy as np

    import oracle
    threads = oracle.default_threads()
    rng = np.random.default_rng(cfg.seed)

    def run(n):
        t0 = time.perf_counter()
        idx, gate = oracle.route(h.x, h.router_w, h.bias, cfg.top_k, nthreads=threads)
        t1 = time.perf_counter()
        tok = np.sort(rng.choice(cfg.T, size=n, replace=False)).astype(np.int32)
        if h.fp8 is not None:
            f = h.fp8
            oracle.combine_ffn_fp8(h.x, idx, gate, f["w_gate_q"], f["w_gate_s"], f["w_up_q"], f["w_up_s"],
                                   f["w_down_q"], f["w_down_s"], tokens=tok, nthreads=threads)
        elif h.mx is not None:
            f = h.mx
            oracle.get().combine_ffn_mx(h.x, idx, gate, f["w_gate_q"], f["w_gate_x"], f["w_up_q"], f["w_up_x"],
                                        f["w_down_q"], f["w_down_x"], tokens=tok, nthreads=threads)
        else:
            oracle.combine_ffn(h.x, idx, gate, h.w_gate, h.w_up, h.w_down, tokens=tok, nthreads=threads)
        if h.shared is not None:
            oracle.shared_ffn(h.x, *h.shared, tokens=tok, nthreads=threads)
        t2 = time.perf_counter()
        return t1 - t0, t2 - t1
    return run, threads


def cpu_baseline(cfg, h, budget_s=20.0):
    run, threads = oracle_step_timer(cfg, h)
    n = min(cfg.T, max(threads, 1))
    tr, tf = run(n)
    per_tok = tf / n
    # layer tokens/s estimate: routing all T tokens + FFN of all T at the measured per-token rate
    n_tot, t_route, t_ffn, reps = 0, 0.0, 0.0, 0
    t_start = time.perf_counter()
    while time.perf_counter() - t_start < budget_s:
        m = min(cfg.T, max(n, int(max(1.0, budget_s / 4) / max(per_tok, 1e-9))))
        a, b = run(m)
        t_route += a
        t_ffn += b
        n_tot += m
        reps += 1
    est = cfg.T / (t_route / reps + (t_ffn / n_tot) * cfg.T)
    return {"value": round(est, 3), "unit": "tokens/s", "cores": threads, "kind": "oracle",
            "sample": f"{reps} passes of: router+top-k over all {cfg.T} tokens, expert FFN + "
                      f"combine of {n_tot // reps} sampled tokens (fp64 CPU oracle); "
                      f"tokens/s = T / (route time + per-token FFN time * T)"}


def run_reference(args, world, rank):
    if rank != 0:
        return
    cfg = workload_config(args)
    run, threads = oracle_step_timer(cfg, host_inputs(cfg))
    tr, tf = run(min(cfg.T, threads))
    per_tok = tf / min(cfg.T, threads)
    budget = 150.0 / max(args.steps + args.warmup, 1)
    n = int(min(cfg.T, max(1, (budget - tr) / max(per_tok, 1e-9))))
    for _ in range(args.warmup):
        run(n)
    tot_r = tot_f = 0.0
    for _ in range(args.steps):
        a, b = run(n)
        tot_r += a
        tot_f += b
    step_s = tot_r / args.steps + tot_f / args.steps * cfg.T / n
    value = cfg.T / step_s
    sample = (f"each step: router+top-k over all {cfg.T} tokens + expert FFN/combine of {n} sampled "
              f"tokens, scaled to the full batch (fp64 CPU oracle, {threads} threads)")
    line = {"metric": METRIC, "value": round(value, 3), "unit": "tokens/s", "n_gpus": args.gpus,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(step_s * 1e3, 3),
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
            "data": "synthetic", "impl": "reference",
            "config": config_block(cfg, world),
            "cpu_baseline": {"value": round(value, 3), "unit": "tokens/s", "cores": threads,
                             "kind": "oracle", "sample": sample},
            "e2e": {"value": round(value, 3), "unit": "tokens/s", "h2d_bytes_per_step": 0,
                    "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


def config_block(cfg, world):
    return {"workload": cfg.name, "T": cfg.T, "H": cfg.H, "I": cfg.I, "E": cfg.E, "top_k": cfg.top_k,
            "weights": {"fp8": "e4m3 + fp32 128x128 block scales",
                        "mx": "e2m1 (packed 2 per byte) + e8m0 scale per 32 along K"}.get(cfg.dtype, "bf16"),
            "shared_expert_I": cfg.shared_mult * cfg.I if cfg.shared_mult else None,
            "seed": cfg.seed, "router_bias": "zipf(1.2)" if cfg.zipf_s else None,
            "global_batch": cfg.T * world, "parallelism": f"replicas{world}",
            "l2": "flushed before every step: 512 MiB write then 256 MiB read, outside the step's events",
            "launch": "timed steps: K moe_forward calls captured in one CUDA graph, an event pair per step; "
                      "stage times from a second graph with events between the stages; e2e: direct calls with the copies of neighbouring steps overlapped (e2e.overlap)"}


# ---------------------------------------------------------------- our arm

def run_one(args, cfg, world, rank, local):
    """Times `cfg` (K graph-captured steps after W warm-ups) and returns its JSON line
    (on every rank; rank 0 prints it)."""
    from routed_grouped_gemm_softmax_b200 import api

    dev = torch.device("cuda", local)
    torch.cuda.set_device(dev)
    fp8 = cfg.dtype in ("fp8", "mx")   # quantised: the tensor peak is the fp8 rate
    inp = make_inputs(cfg, device=dev, weights=cfg.dtype == "bf16")
    x, rw, bias = inp.x, inp.router_w, inp.bias
    k = cfg.top_k
    w8 = shared = None
    if cfg.dtype == "fp8":
        w8 = make_fp8_weights(cfg, device=dev)
        wq = (w8["w_gate_q"], w8["w_gate_s"], w8["w_up_q"], w8["w_up_s"], w8["w_down_q"], w8["w_down_s"])
        forward = lambda xx, st, oo=None: api.moe_forward_fp8(xx, rw, bias, *wq, k, out=out if oo is None else oo,
                                                              ws=ws, stream=st)
        ws = api.workspace(cfg.T, cfg.H, cfg.I, cfg.E, k, dev, api.DTYPE_FP8)
    elif cfg.dtype == "mx":
        w8 = make_mx_weights(cfg, device=dev)
        wq = (pack_e2m1(w8["w_gate_q"]), w8["w_gate_x"], pack_e2m1(w8["w_up_q"]), w8["w_up_x"],
              pack_e2m1(w8["w_down_q"]), w8["w_down_x"])
        forward = lambda xx, st, oo=None: api.moe_forward_mx(xx, rw, bias, *wq, k, out=out if oo is None else oo,
                                                             ws=ws, stream=st)
        ws = api.workspace(cfg.T, cfg.H, cfg.I, cfg.E, k, dev, api.DTYPE_MX)
    elif cfg.shared_mult:
        wg, wu, wd = inp.w_gate, inp.w_up, inp.w_down
        shared = make_shared_weights(cfg, cfg.shared_mult * cfg.I, device=dev)
        forward = lambda xx, st, oo=None: api.moe_forward_shared(xx, rw, bias, wg, wu, wd, *shared, k,
                                                                 out=out if oo is None else oo, ws=ws, stream=st)
        ws = torch.empty(api.moe_workspace_size_shared(cfg.T, cfg.H, cfg.I, cfg.E, k, cfg.shared_mult * cfg.I),
                         dtype=torch.uint8, device=dev)
    else:
        wg, wu, wd = inp.w_gate, inp.w_up, inp.w_down
        forward = lambda xx, st, oo=None: api.moe_forward(xx, rw, bias, wg, wu, wd, k, out=out if oo is None else oo,
                                                          ws=ws, stream=st)
        ws = api.workspace(cfg.T, cfg.H, cfg.I, cfg.E, k, dev, api.DTYPE_BF16)
    out = torch.empty(cfg.T, cfg.H, dtype=torch.bfloat16, device=dev)
    flush_buf = torch.empty(FLUSH_BYTES, dtype=torch.uint8, device=dev)
    evict_buf = torch.ones(EVICT_FLOATS, dtype=torch.float32, device=dev)
    evict_out = torch.empty((), dtype=torch.float32, device=dev)

    class _Flush:
        """L2 flush between steps: write 512 MiB, then read 256 MiB of other data so that
        the write-backs of the flush happen here and not inside the next timed step."""
        @staticmethod
        def fill_(v):
            flush_buf.fill_(v)
            torch.sum(evict_buf, dim=0, out=evict_out)
    flush = _Flush()
    stream = torch.cuda.current_stream(dev)

    def step():
        forward(x, stream)

    # events: a start/end pair per timed step, and (in a second, untimed graph) the six
    # stage marks of every step for the breakdown -- an event between two kernels costs
    # the step a few microseconds, so the headline time carries only the outer pair
    ev_step = [[torch.cuda.Event(enable_timing=True) for _ in range(2)] for _ in range(args.steps)]
    ev = [[torch.cuda.Event(enable_timing=True) for _ in range(6)] for _ in range(args.steps)]
    for s in ev + ev_step:
        for e in s:
            e.record(stream)
    api.set_claim_order(False if args.schedule == "queue" else args.schedule)
    api.set_pair_mma(args.pair)
    api.set_fp8_swap_ab(args.swap_ab)
    api.set_fused_combine(args.fused_combine)
    api.set_layer_gemm(args.layer_gemm)
    api.set_direct_a(args.direct_a)
    for _ in range(max(args.warmup, 3)):
        flush.fill_(1)
        step()
    torch.cuda.synchronize()
    status = api.moe_get_device_status(ws)
    if status != api.MOE_OK:
        raise RuntimeError(f"device status {status} after warm-up")

    # The timed region is one CUDA graph holding the K steps: before each step an L2
    # flush (outside that step's events), then the step between its two events.
    cap = torch.cuda.Stream(dev)
    cap.wait_stream(stream)
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.stream(cap):
        with torch.cuda.graph(graph, stream=cap):
            for i in range(args.steps):
                flush.fill_(1)
                api.set_stage_events([ev_step[i][0], None, None, None, None, ev_step[i][1]])
                forward(x, cap)
    # the stage breakdown: the same steps with the library's six stage marks, and the
    # GEMM CTAs' busy spans (the last step's remain in the trace buffer)
    trace = torch.zeros(4 * GEMM_TRACE_CTAS, dtype=torch.int64, device=dev)
    graph_stages = torch.cuda.CUDAGraph()
    with torch.cuda.stream(cap):
        with torch.cuda.graph(graph_stages, stream=cap):
            for i in range(args.steps):
                flush.fill_(1)
                api.set_stage_events(ev[i])
                api.set_gemm_trace(trace)
                forward(x, cap)
    api.set_stage_events(None)
    api.set_gemm_trace(None)
    stream.wait_stream(cap)
    graph_stages.replay()
    torch.cuda.synchronize()
    sched = schedule_stats(trace.cpu().tolist(), args.schedule)
    graph.replay()  # one untimed replay so the timed one starts warm
    torch.cuda.synchronize()

    sampler = ClockSampler(local)
    sampler.start()
    time.sleep(0.2)
    barrier(world)
    torch.cuda.synchronize()
    t_wall0 = time.time()
    graph.replay()
    torch.cuda.synchronize()
    barrier(world)
    t_wall1 = time.time()
    time.sleep(0.1)
    sampler.stop()
    status = api.moe_get_device_status(ws)
    if status != api.MOE_OK:
        raise RuntimeError(f"device status {status} after the timed steps")
    del graph, graph_stages

    step_ms = [ev_step[i][0].elapsed_time(ev_step[i][1]) for i in range(args.steps)]
    stage_ms = {name: statistics.mean(ev[i][j].elapsed_time(ev[i][j + 1]) for i in range(args.steps))
                for j, name in enumerate(api.STAGES)}
    total_ms = max_over_ranks(sum(step_ms), world)
    ms_per_step = total_ms / args.steps
    value = throughput(cfg.T, world, args.steps, total_ms)

    # routing of this workload (for the touched-expert weight bytes)
    idx, _ = api.moe_route(x, rw, bias, k)
    counts = torch.bincount(idx.view(-1).long(), minlength=cfg.E).tolist()
    work = stage_work(cfg, counts)
    peaks, peaks_kind = load_peaks()
    plan = api.forward_plan(cfg.T, cfg.H, cfg.I, cfg.E, k, {"fp8": api.DTYPE_FP8, "mx": api.DTYPE_MX}.get(
        cfg.dtype, api.DTYPE_BF16))
    kernels = ["route", "gemm_gate_up", "gemm_down", "combine"]
    if plan >= 0 and plan & api.PLAN_LAYER_GEMM:
        # both expert GEMMs run as one launch (the stage marks around it are 2 and 4)
        work["gemm_layer"] = {"bytes": work["gemm_gate_up"]["bytes"] + work["gemm_down"]["bytes"],
                              "flops": work["gemm_gate_up"]["flops"] + work["gemm_down"]["flops"]}
        stage_ms["gemm_layer"] = stage_ms["gemm_gate_up"] + stage_ms["gemm_down"]
        kernels = ["route", "gemm_layer", "combine"]
    dominant = max(kernels, key=lambda s: stage_ms[s])
    sustained = total_ms > 1000.0
    roof = roofline_for(dominant, work, stage_ms[dominant], peaks, peaks_kind, sustained, cfg.name, fp8)
    try:  # an extra view of the same step; never allowed to cost the bench line
        layer_roof = layer_roofline(cfg, counts, ms_per_step, peaks, peaks_kind, sustained)
    except Exception as exc:
        layer_roof = {"error": repr(exc)}
    stages = {s: {"ms": round(stage_ms[s], 4)} for s in list(api.STAGES) + kernels}
    for s in kernels:
        r = roofline_for(s, work, stage_ms[s], peaks, peaks_kind, sustained, cfg.name, fp8)
        stages[s].update({"bound": r["bound"], "achieved": r["achieved"], "unit": r["unit"], "frac": r["frac"]})

    # End to end through the public API with host buffers: every step copies its x from
    # pinned host memory and reads its output back.  Two buffer slots and a copy stream
    # each way let step i+1's upload and step i-1's read-back run under step i's forward,
    # as a serving loop would; the timed region spans all copies of all steps.  L2 is
    # flushed (inside the region) before each forward whose weights would otherwise stay
    # in it.
    e2e = None
    if not args.no_e2e:
        x_host = x.cpu().pin_memory()
        nslot = 2
        x_dev = [torch.empty_like(x) for _ in range(nslot)]
        out_dev = [torch.empty_like(out) for _ in range(nslot)]
        out_host = [torch.empty(cfg.T, cfg.H, dtype=torch.bfloat16).pin_memory() for _ in range(nslot)]
        s_in, s_out = torch.cuda.Stream(device=dev), torch.cuda.Stream(device=dev)
        ev_in = [torch.cuda.Event() for _ in range(nslot)]
        ev_comp = [torch.cuda.Event() for _ in range(nslot)]
        ev_out = [torch.cuda.Event() for _ in range(nslot)]
        weight_bytes = work["gemm_gate_up"]["bytes"] + work["gemm_down"]["bytes"]
        flush_each = weight_bytes < 2 * L2_BYTES
        n_e2e = max(nslot, min(args.steps, 200))
        t0e, t1e = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        barrier(world)
        torch.cuda.synchronize()
        t0e.record(stream)
        s_in.wait_stream(stream)
        s_out.wait_stream(stream)
        for i in range(n_e2e):
            j = i % nslot
            with torch.cuda.stream(s_in):
                if i >= nslot:
                    s_in.wait_event(ev_comp[j])  # the forward that read this slot is done
                x_dev[j].copy_(x_host, non_blocking=True)
                ev_in[j].record(s_in)
            stream.wait_event(ev_in[j])
            if i >= nslot:
                stream.wait_event(ev_out[j])  # this slot's previous output was read back
            if flush_each:
                with torch.cuda.stream(stream):
                    flush.fill_(1)
            forward(x_dev[j], stream, out_dev[j])
            ev_comp[j].record(stream)
            with torch.cuda.stream(s_out):
                s_out.wait_event(ev_comp[j])
                out_host[j].copy_(out_dev[j], non_blocking=True)
                ev_out[j].record(s_out)
        stream.wait_stream(s_in)
        stream.wait_stream(s_out)
        t1e.record(stream)
        torch.cuda.synchronize()
        # every step computed the same layer on the same x: the last read-back must equal
        # the timed steps' output bit for bit
        if not torch.equal(out_host[(n_e2e - 1) % nslot].view(torch.int16), out.cpu().view(torch.int16)):
            raise RuntimeError("end-to-end output differs from the timed steps' output")
        e2e_ms = max_over_ranks(t0e.elapsed_time(t1e), world) / n_e2e
        e2e = {"value": round(throughput(cfg.T, world, 1, e2e_ms), 3), "unit": "tokens/s",
               "h2d_bytes_per_step": x.numel() * 2, "d2h_bytes_per_step": out.numel() * 2,
               "ms_per_step": round(e2e_ms, 4), "steps": n_e2e,
               "overlap": "two buffer slots; step i+1's upload and step i-1's read-back on their own streams "
                          "under step i's forward",
               "l2": "flushed before each forward inside the region" if flush_each
                     else "not flushed: the touched weights are over twice the L2"}

    clocks = sampler.summary(t_wall0, t_wall1)
    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        budget = args.cpu_budget if args.cpu_budget else (12.0 if args.workload == "all" else 20.0)
        cpu = cpu_baseline(cfg, host_inputs(cfg, inp, w8, shared), budget_s=budget)

    line = None
    if rank == 0:
        line = {"metric": METRIC, "value": round(value, 3), "unit": "tokens/s", "n_gpus": world,
                "steps": args.steps, "warmup": max(args.warmup, 3), "ms_per_step": round(ms_per_step, 5),
                "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
                "dtype": {"fp8": "e4m3", "mx": "e2m1 x e4m3 (mx)"}.get(cfg.dtype, "bf16"),
                "data": "synthetic", "config": config_block(cfg, world),
                "roofline": roof, "layer_roofline": layer_roof, "stages": stages, "experts_touched": work["_D"],
                "e2e": e2e, "gpu_launches": kernels_per_forward(cfg, plan) * args.steps, "schedule": sched,
                "plan": plan,
                "clocks": clocks, "cpu_baseline": cpu,
                "p99_ms_per_step": round(sorted(step_ms)[min(len(step_ms) - 1, math.ceil(0.99 * len(step_ms)) - 1)], 5)}
    torch.cuda.synchronize()
    return line


def run_and_release(args, cfg, world, rank, local):
    """run_one, then hand this workload's device memory back before the next is drawn."""
    import gc
    line = run_one(args, cfg, world, rank, local)
    gc.collect()
    torch.cuda.empty_cache()
    return line


def tile_sweep(args):
    """Times the kernel variants the tile table chooses between, per M bucket r (average
    rows per expert) of H=2048, I=1024, E=64, top-8 with T = r*E/k: CUDA events around
    the two GEMM stages and the whole step, L2 flushed before every step, median over
    --steps steps.  bf16: 128-row or pair tiles, one or two GEMM launches, combine
    inside the down GEMM or not, A rows gathered by the GEMM or copied first; fp8:
    plain or swapped gate/up operands."""
    from routed_grouped_gemm_softmax_b200 import api
    dev = torch.device("cuda", 0)
    torch.cuda.set_device(dev)
    flush = torch.empty(FLUSH_BYTES, dtype=torch.uint8, device=dev)
    steps = max(args.steps, 5) if args.steps != 400 else 30

    def time_stages(forward):
        ev = [[torch.cuda.Event(enable_timing=True) for _ in range(6)] for _ in range(steps)]
        for s_ in ev:
            for e in s_:
                e.record()
        for _ in range(max(args.warmup, 3)):
            flush.fill_(1)
            forward()
        torch.cuda.synchronize()
        try:
            for i in range(steps):
                flush.fill_(1)
                api.set_stage_events(ev[i])
                forward()
        finally:
            api.set_stage_events(None)
        torch.cuda.synchronize()
        med = lambda a, b: round(statistics.median(ev[i][a].elapsed_time(ev[i][b]) for i in range(steps)) * 1e3, 1)
        return {"gemm_gate_up_us": med(2, 3), "gemm_down_us": med(3, 4), "step_us": med(0, 5)}

    H, I, E, k = 2048, 1024, 64, 8
    variants = {"tiles128": ("never", "never", "never", "auto"), "tiles128_layer": ("never", "always", "never", "auto"),
                "tiles128_layer_combine_in_down": ("never", "always", "always", "auto"),
                "pairs": ("always", "never", "never", "auto"), "pairs_layer": ("always", "always", "never", "auto"),
                "table": ("auto", "auto", "auto", "auto"), "table_direct_a": ("auto", "auto", "auto", "always"),
                "table_sorted_copy": ("auto", "auto", "auto", "never")}
    for r in [1, 2, 4, 8, 16, 32, 64, 96, 128, 192, 256, 384, 512, 768, 1024, 2048, 4096]:
        T = max(1, r * E // k)
        cfg = CONFIGS["prefill"].replace(name=f"bucket{r}", T=T, H=H, I=I, E=E, top_k=k, seed=100 + r)
        inp = make_inputs(cfg, device=dev)
        ws = api.workspace(T, H, I, E, k, dev)
        o = torch.empty(T, H, dtype=torch.bfloat16, device=dev)
        f = lambda: api.moe_forward(inp.x, inp.router_w, None, inp.w_gate, inp.w_up, inp.w_down, k, out=o, ws=ws)
        row = {"sweep": "bf16", "rows_per_expert": r, "T": T, "H": H, "I": I, "E": E, "top_k": k}
        for name, (pm, lg, fc, da) in variants.items():
            api.set_pair_mma(pm)
            api.set_layer_gemm(lg)
            api.set_fused_combine(fc)
            api.set_direct_a(da)
            row[name] = time_stages(f)
        api.set_pair_mma("auto")
        api.set_layer_gemm("auto")
        api.set_fused_combine("auto")
        api.set_direct_a("auto")
        row["table_plan"] = api.forward_plan(T, H, I, E, k)
        print(json.dumps(row), flush=True)
        del inp, ws, o, f
        torch.cuda.empty_cache()
    for r in [1, 4, 16, 32, 48, 64, 96, 128, 256, 512, 1024]:
        T = max(1, r * E // k)
        cfg = CONFIGS["fp8"].replace(name=f"bucket8_{r}", T=T, H=H, I=I, E=E, top_k=k, seed=200 + r)
        inp = make_inputs(cfg, device=dev, weights=False)
        w = make_fp8_weights(cfg, device=dev)
        wq = (w["w_gate_q"], w["w_gate_s"], w["w_up_q"], w["w_up_s"], w["w_down_q"], w["w_down_s"])
        ws = api.workspace(T, H, I, E, k, dev, api.DTYPE_FP8)
        o = torch.empty(T, H, dtype=torch.bfloat16, device=dev)
        f = lambda: api.moe_forward_fp8(inp.x, inp.router_w, None, *wq, k, out=o, ws=ws)
        row = {"sweep": "fp8", "rows_per_expert": r, "T": T, "H": H, "I": I, "E": E, "top_k": k}
        for mode in ("never", "always", "auto"):
            api.set_fp8_swap_ab(mode)
            row["swap_" + mode] = time_stages(f)
        api.set_fp8_swap_ab("auto")
        print(json.dumps(row), flush=True)
        del inp, w, wq, ws, o, f
        torch.cuda.empty_cache()


def main():
    args = parse()
    if args.tile_sweep:
        tile_sweep(args)
        return
    if args.impl == "reference":
        # rank 0 alone times the oracle on the host cores; the other ranks have no work
        # and open no process group
        world, rank, _ = rank_env()
        run_reference(args, world, rank)
        return
    world, rank, local = dist_setup()
    torch.cuda.set_device(torch.device("cuda", local))
    if args.workload != "all":
        line = run_one(args, workload_config(args), world, rank, local)
    else:
        # every workload in turn, the headline last; one line: the headline's, with the
        # others' complete lines under "workloads"
        lines = {name: run_and_release(args, workload_config(args, name), world, rank, local)
                 for name in ALL_ORDER}
        line = lines[HEADLINE]
        if line is not None:
            line["workloads"] = {n: lines[n] for n in ALL_ORDER if n != HEADLINE}
            line["headline"] = (f"{HEADLINE}: the largest configuration (the metric names none); "
                                f"the other workloads under 'workloads'")
    if rank == 0:
        print(json.dumps(line), flush=True)
    dist_teardown(world)


if __name__ == "__main__":
    main()
