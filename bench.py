#!/usr/bin/env python
"""Benchmark of the MoE expert-FFN layer (libmoe_b200) on B200.

One step = one whole layer call (route, permute + gather, grouped GEMM
gate/up + SwiGLU, grouped GEMM down, finalize) over one batch of synthetic
tokens, through the C ABI (moe_forward). The headline workload is the
largest single-GPU one, the Qwen3-30B-A3B-shaped prefill layer: T=8192,
H=2048, I=768, E=128, top_k=8, bf16 weights. The same run also times the
other graded workloads (Qwen3 decode, the skewed Zipf layer and the W4A16
decode layer) and, ungraded, the MXFP8, MXFP4 and shared-expert decode
layers, and reports them under "workloads". Every workload reads more than
the 126 MB L2 per step (its expert weights), so no flush is needed between
steps. For a bf16 decode batch moe_forward is one persistent kernel (after a
one-warp counter reset); its roofline is taken over the timed region.

  python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME]
                  [--extra all|none|NAME,...] [--impl ours|reference]

With --gpus N > 1 (one process per GPU under torchrun; started without
torchrun, bench.py relaunches itself under torchrun) every rank runs its own
replica on its own token batch (token-sharded data parallel: the layer needs
no exchange between ranks), and value = all ranks' tokens / the slowest
rank's time.

--impl reference times the CPU oracle (the plain C reference in oracle/) on
the host cores, on the headline workload, metric and unit.
"""

from __future__ import annotations

import argparse
import hashlib
import json
import os
import re
import socket
import statistics
import subprocess
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

METRIC = "MoE-layer tokens/s on 1 B200; fraction of HBM / bf16 tensor-core roofline"
UNIT = "tokens/s"
HEADLINE = "qwen3_prefill"
EXTRA = ["qwen3_decode", "skewed", "w4a16_decode"]
# the layer's targets: decode layers against 8 TB/s of activated weight bytes,
# prefill-like layers against 2.25 PFLOP/s dense bf16
TARGETS = {"qwen3_decode": ("hbm", 0.70), "w4a16_decode": ("hbm", 0.70),
           "qwen3_prefill": ("tensor", 0.60), "skewed": ("tensor", 0.60), "tiny": (None, None)}
# measured beside the graded workloads (no target of their own): MXFP8
# weights on the block-scaled MMA, and shared experts
UNGRADED = ["mxfp8_decode", "mxfp4_decode", "shared_decode"]
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}
NORTH_STAR_HBM_GBS = 8000.0       # the roofline literals the layer's target is stated against
NORTH_STAR_BF16_TFLOPS = 2250.0
PROFILE_DIR = os.path.join(ROOT, "profiles")
# Kernel sources whose change invalidates stored counters. A profile summary
# may name the files its kernel is built from ("kernel_sources: a.cu b.cuh",
# paths under csrc/); its counters then stand while those files are
# unchanged. Without that line every file below counts.
CSRC_DIR = "mixture_experts_expert_top_b200/csrc"
KERNEL_SOURCES = ["mixture_experts_expert_top_b200/csrc/gemm_sm100.cu",
                  "mixture_experts_expert_top_b200/csrc/fused_decode_sm100.cu",
                  "mixture_experts_expert_top_b200/csrc/route_dev.cuh",
                  "mixture_experts_expert_top_b200/csrc/gemm_prefill_sm100.cu",
                  "mixture_experts_expert_top_b200/csrc/gemm_wm_pair_sm100.cu",
                  "mixture_experts_expert_top_b200/csrc/gemm_mxfp8_sm100.cu",
                  "mixture_experts_expert_top_b200/csrc/gemm_int4_warp_sm100.cu",
                  "mixture_experts_expert_top_b200/csrc/gemm_common.cuh",
                  "mixture_experts_expert_top_b200/csrc/common.cuh",
                  "mixture_experts_expert_top_b200/csrc/launch_util.cuh"]


# ----------------------------------------------------------------- helpers --

def parse_args(argv=None):
    ap = argparse.ArgumentParser(description=__doc__.split("\n")[0])
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=1000)
    ap.add_argument("--warmup", type=int, default=10)
    ap.add_argument("--workload", default=HEADLINE)
    ap.add_argument("--extra", default="all",
                    help="other workloads timed in the same run: all, none, or a comma list")
    ap.add_argument("--set", action="append", default=[], metavar="KEY=VALUE",
                    help="override a field (T, H, I, E, k) of the headline workload, e.g. for a profiling case")
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--seed", type=int, default=0)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--cpu-budget-s", type=float, default=12.0, help="CPU seconds for the oracle baseline")
    ap.add_argument("--ref-budget-s", type=float, default=120.0, help="total seconds for --impl reference")
    a = ap.parse_args(argv)
    if a.warmup < 3:
        ap.error("--warmup must be >= 3")
    if a.steps < 1:
        ap.error("--steps must be >= 1")
    if a.gpus < 1:
        ap.error("--gpus must be >= 1")
    return a


def extra_workloads(args):
    if args.set or args.extra == "none":
        return []
    names = EXTRA + UNGRADED if args.extra == "all" else [n for n in args.extra.split(",") if n]
    return [n for n in names if n != args.workload]


def dist_env():
    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    local = int(os.environ.get("LOCAL_RANK", str(rank)))
    return rank, world, local


def max_over_ranks(x: float) -> float:
    """Max of a float over all ranks (identity without a process group)."""
    import torch
    import torch.distributed as dist
    if not (dist.is_available() and dist.is_initialized()) or dist.get_world_size() == 1:
        return float(x)
    dev = "cuda" if dist.get_backend() == "nccl" else "cpu"
    t = torch.tensor([float(x)], dtype=torch.float64, device=dev)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def barrier():
    import torch.distributed as dist
    if dist.is_available() and dist.is_initialized():
        dist.barrier()


def read_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            p = json.load(f)
        return {k: float(p[k]) for k in ("hbm_gbs", "bf16_tflops", "bf16_tflops_sustained")}, "measured"
    except (OSError, KeyError, ValueError):
        return dict(FALLBACK_PEAKS), "fallback"


def host_cpu_model() -> str:
    try:
        with open("/proc/cpuinfo") as f:
            for line in f:
                if line.startswith("model name"):
                    return line.split(":", 1)[1].strip()
    except OSError:
        pass
    import platform
    return platform.processor() or "unknown"


def kernel_source_hash(files=None) -> str:
    """First 16 hex digits of the SHA-256 of the given source files' bytes,
    in order (default: KERNEL_SOURCES)."""
    h = hashlib.sha256()
    for rel in (files if files is not None else KERNEL_SOURCES):
        with open(os.path.join(ROOT, rel), "rb") as f:
            h.update(f.read())
    return h.hexdigest()[:16]


def profiled_traffic(kernel: str, workload: str):
    """DRAM bytes per launch of `kernel` on `workload` from the committed ncu
    summary, if it was taken on the current kernel source; else None."""
    path = os.path.join(PROFILE_DIR, f"{kernel}_{workload}.md")
    try:
        text = open(path).read()
    except OSError:
        return None
    m_hash = re.search(r"kernel_source_sha256_16:\s*([0-9a-f]{16})", text)
    m_tr = re.search(r"dram_bytes_per_launch:\s*([0-9.eE+]+)", text)
    m_src = re.search(r"kernel_sources:[ \t]*(\S.*)", text)
    files = [f"{CSRC_DIR}/{n}" for n in m_src.group(1).split()] if m_src else None
    try:
        current = kernel_source_hash(files)
    except OSError:
        return None
    if not m_hash or not m_tr or m_hash.group(1) != current:
        return None
    return float(m_tr.group(1))


class ClockSampler:
    """SM clock, power and clock-event reasons of one GPU, polled through NVML
    every couple of milliseconds in a background thread (so that even a timed
    region of a few milliseconds holds samples); falls back to nvidia-smi
    polling when NVML is not importable."""

    REASONS = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]

    def __init__(self, uuid: str, index: int, period_s: float = 0.002):
        self.uuid, self.index, self.period_s = uuid, index, period_s
        self.samples = []          # (time, sm_mhz, power_w, reasons)
        self.sm_max = None
        self.source = None
        self._stop = threading.Event()
        self._thread = None
        self._proc = None
        self.t0 = self.t1 = None

    def start(self):
        try:
            import pynvml as nv
            nv.nvmlInit()
            try:
                h = nv.nvmlDeviceGetHandleByUUID(self.uuid)
            except Exception:      # noqa: BLE001 - UUID form not accepted: fall back to the index
                h = nv.nvmlDeviceGetHandleByIndex(self.index)
            self.sm_max = float(nv.nvmlDeviceGetMaxClockInfo(h, nv.NVML_CLOCK_SM))
            get_reasons = getattr(nv, "nvmlDeviceGetCurrentClocksEventReasons",
                                  getattr(nv, "nvmlDeviceGetCurrentClocksThrottleReasons", None))
            bits = {"hw_slowdown": 0x8, "hw_thermal_slowdown": 0x40, "sw_thermal_slowdown": 0x20,
                    "sw_power_cap": 0x4}
            self.source = "nvml"

            def loop():
                while not self._stop.is_set():
                    try:
                        t = time.time()
                        sm = float(nv.nvmlDeviceGetClockInfo(h, nv.NVML_CLOCK_SM))
                        pw = nv.nvmlDeviceGetPowerUsage(h) / 1000.0
                        r = int(get_reasons(h)) if get_reasons else 0
                        self.samples.append((t, sm, pw, [n for n, b in bits.items() if r & b]))
                    except Exception:  # noqa: BLE001 - a failed poll is skipped
                        pass
                    self._stop.wait(self.period_s)

            self._thread = threading.Thread(target=loop, daemon=True)
            self._thread.start()
            return
        except Exception:          # noqa: BLE001 - no NVML: nvidia-smi below
            pass
        fields = ["clocks.sm", "clocks.max.sm", "power.draw", "clocks_event_reasons.hw_slowdown",
                  "clocks_event_reasons.hw_thermal_slowdown", "clocks_event_reasons.sw_thermal_slowdown",
                  "clocks_event_reasons.sw_power_cap"]
        try:
            self._proc = subprocess.Popen(
                ["nvidia-smi", "-i", self.uuid, f"--query-gpu={','.join(fields)}", "--format=csv,noheader,nounits",
                 "-lms", "20"], stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except OSError:
            self._proc = None
            return
        self.source = "nvidia-smi"

        def read():
            for line in self._proc.stdout:
                p = [x.strip() for x in line.split(",")]
                if len(p) != 7 or not _isnum(p[0]):
                    continue
                self.sm_max = float(p[1]) if _isnum(p[1]) else self.sm_max
                self.samples.append((time.time(), float(p[0]), float(p[2]) if _isnum(p[2]) else None,
                                     [n for n, v in zip(self.REASONS, p[3:]) if v.lower().startswith("active")]))

        self._thread = threading.Thread(target=read, daemon=True)
        self._thread.start()

    def mark_begin(self):
        self.t0 = time.time()

    def mark_end(self):
        self.t1 = time.time()

    def stop(self):
        time.sleep(0.01)
        self._stop.set()
        if self._proc is not None:
            self._proc.terminate()
            try:
                self._proc.wait(timeout=5)
            except subprocess.TimeoutExpired:
                self._proc.kill()
        if self._thread is not None:
            self._thread.join(timeout=5)

    def summary(self, t0=None, t1=None):
        """Samples inside [t0, t1] (default: the marked region)."""
        t0 = self.t0 if t0 is None else t0
        t1 = self.t1 if t1 is None else t1
        inside = [s for s in list(self.samples) if t0 is not None and t1 is not None and t0 <= s[0] <= t1]
        sm = [s[1] for s in inside]
        pw = [s[2] for s in inside if s[2] is not None]
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": self.sm_max,
                "reasons": sorted({r for s in inside for r in s[3]}), "samples_inside_timed_region": len(inside),
                "power_w_max": max(pw) if pw else None, "source": self.source}


def _isnum(s):
    try:
        float(s)
        return True
    except ValueError:
        return False


def free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


# -------------------------------------------------------- workload accounting --

def weight_row_bytes(fmt, K):
    """Bytes of one weight row of K elements with its scales."""
    if fmt == "bf16":
        return 2 * K
    if fmt == "int4_g128":
        return K // 2 + (K // 128) * 2
    if fmt == "mxfp4":
        return K // 2 + K // 32                 # E2M1 codes (two per byte) + E8M0 scales
    return K + K // 32                          # mxfp8: E4M3 codes + E8M0 scales


def work_per_step(cfg, counts):
    """Algorithmic bytes and FLOPs of each kernel for one step, from the real
    per-expert counts (experts with no rows read no weights; shared experts
    count as experts, their slots as pairs)."""
    T, H, I, k = cfg.T, cfg.H, cfg.I, cfg.k
    S = getattr(cfg, "n_shared", 0)
    E = cfg.E + S
    P = T * (k + S)
    active = int(sum(1 for c in counts if c > 0))
    w_gu = active * 2 * I * weight_row_bytes(cfg.fmt, H)
    w_d = active * H * weight_row_bytes(cfg.fmt, I)
    # token operand bytes per element: bf16, or MX codes + scales
    xb = (lambda K: K + K // 32) if cfg.fmt in ("mxfp8", "mxfp4") else (lambda K: 2 * K)
    return {
        "active_experts": active,
        "weight_bytes": w_gu + w_d,
        "gemm_swiglu": {"bytes": w_gu + P * xb(H) + P * xb(I) + (E + 1) * 4, "flops": 2 * P * 2 * I * H},
        "gemm_down": {"bytes": w_d + P * xb(I) + P * H * 2 + (E + 1) * 4, "flops": 2 * P * H * I},
        "route": {"bytes": T * cfg.E * 4 + P * 8, "flops": 0},
        "permute": {"bytes": P * 4 * 3 + (2 * E + 1) * 4 + T * H * 2 + P * H * 2, "flops": 0},
        "quantize": {"bytes": T * H * 2 + T * xb(H), "flops": 0},
        "finalize": {"bytes": P * H * 2 + T * H * 2 + P * 8, "flops": 0},
        # the persistent decode kernel: the bytes the layer must move (weights,
        # hidden, logits, out); act and y stay on chip or in L2
        "fused": {"bytes": w_gu + w_d + T * H * 2 + T * cfg.E * 4 + T * H * 2, "flops": 2 * P * 3 * H * I},
        "layer_flops": 2 * P * 3 * H * I,
    }


def launches_per_step(cfg) -> int:
    """Kernels one moe_forward call enqueues for this workload (the library's own count)."""
    import mixture_experts_expert_top_b200 as moe
    return moe.moe_forward_kernel_count(moe.Shape.of(cfg.T, cfg.H, cfg.I, cfg.E, cfg.k, cfg.fmt,
                                                     n_shared=getattr(cfg, "n_shared", 0)))


def get_workload(name, sets=()):
    import moe_synth
    cfg = moe_synth.get_config(name)
    over = {}
    for kv in sets:
        k, v = kv.split("=", 1)
        if k not in ("T", "H", "I", "E", "k"):
            raise SystemExit(f"--set: unknown field {k}")
        over[k] = int(v)
    if over:
        cfg = cfg.with_(**over, name=cfg.name + "+" + ",".join(f"{k}={v}" for k, v in sorted(over.items())))
    return cfg


def config_of(cfg, world):
    """The `config` object of the JSON line (the same for both arms)."""
    return {"workload": cfg.describe(), "T": cfg.T, "H": cfg.H, "I": cfg.I, "E": cfg.E, "top_k": cfg.k,
            "weights": cfg.fmt, "global_batch": world * cfg.T,
            "parallelism": "replicas (token-sharded, no collective)" if world > 1 else "single GPU",
            "l2": f"inputs larger than L2: {expert_weight_bytes(cfg) / 1e9:.3f} GB of expert weights, of which "
                  "each step reads its activated experts' (> 126 MB); no flush"}


def expert_weight_bytes(cfg):
    """Bytes of all E experts' weights (and scales) of a workload."""
    return cfg.E * (2 * cfg.I * weight_row_bytes(cfg.fmt, cfg.H) + cfg.H * weight_row_bytes(cfg.fmt, cfg.I))


def layer_fractions(cfg, work, layer_s, peaks):
    bound, target = TARGETS.get(cfg.name.split("+")[0], (None, None))
    f = {"active_experts": work["active_experts"], "weight_bytes": work["weight_bytes"],
         "flops": work["layer_flops"],
         "hbm_frac_of_8TBps": work["weight_bytes"] / layer_s / (NORTH_STAR_HBM_GBS * 1e9),
         "hbm_frac_of_measured": work["weight_bytes"] / layer_s / (peaks["hbm_gbs"] * 1e9),
         "tensor_frac_of_2250TF": work["layer_flops"] / layer_s / (NORTH_STAR_BF16_TFLOPS * 1e12),
         "tensor_frac_of_measured_burst": work["layer_flops"] / layer_s / (peaks["bf16_tflops"] * 1e12)}
    if bound:
        got = f["hbm_frac_of_8TBps"] if bound == "hbm" else f["tensor_frac_of_2250TF"]
        f["target"] = {"bound": bound, "frac": target, "achieved": got, "met": got >= target}
    return f


# ------------------------------------------------------------------ our arm --

def measure(cfg, args, dev, world, rank, sampler, headline):
    """Time one workload: K whole-layer steps (the value), a per-step pass
    (median and minimum), a CUDA-graph replay for decode batches, a per-stage
    pass (the roofline of the dominant kernel) and K steps end to end through
    moe_forward_host."""
    import torch

    import moe_synth
    import mixture_experts_expert_top_b200 as moe

    inp = moe_synth.gen_inputs(cfg, seed=args.seed)
    if rank:   # weights are the same on every rank (replicas); each rank draws its own tokens
        inp["hidden"] = moe_synth.gen_hidden(cfg, seed=args.seed + rank)
        inp["logits"] = moe_synth.gen_logits(cfg, seed=args.seed + rank)
    d = {n: t.to(dev) for n, t in inp.items()}
    S = cfg.n_shared
    shape = moe.Shape.of(cfg.T, cfg.H, cfg.I, cfg.E, cfg.k, cfg.fmt, n_shared=S)
    ws = torch.empty(moe.moe_workspace_size(shape), dtype=torch.uint8, device=dev)
    out = torch.empty(cfg.T, cfg.H, dtype=torch.bfloat16, device=dev)
    stream = torch.cuda.current_stream(dev)
    scales = (d.get("w_gu_scales"), d.get("w_d_scales"))
    K, W = args.steps, args.warmup

    def step(s=stream):
        moe.moe_forward(d["hidden"], d["logits"], d["w_gu"], scales[0], d["w_d"], scales[1], shape, out, ws, s)

    def ev():
        return torch.cuda.Event(enable_timing=True)

    # ---- value: exactly K steps, barrier + synchronize on both sides --------
    for _ in range(W):
        step()
    torch.cuda.synchronize()
    barrier()
    torch.cuda.synchronize()
    a, b = ev(), ev()
    sampler.mark_begin()
    a.record(stream)
    for _ in range(K):
        step()
    b.record(stream)
    torch.cuda.synchronize()
    sampler.mark_end()
    barrier()
    clocks = sampler.summary()
    ms_max = max_over_ranks(a.elapsed_time(b))
    value = world * cfg.T * K / (ms_max / 1e3)

    # ---- per-step distribution: at least 50 steps, each between events -----
    n_it = max(50, min(K, 500))
    evs = [ev() for _ in range(n_it + 1)]
    evs[0].record(stream)
    for i in range(n_it):
        step()
        evs[i + 1].record(stream)
    torch.cuda.synchronize()
    per = [evs[i].elapsed_time(evs[i + 1]) for i in range(n_it)]
    step_ms = {"median": statistics.median(per), "min": min(per), "n": n_it,
               "note": "an event between steps keeps the next step from starting early"}

    # ---- CUDA-graph replay of one captured step (decode batches) ------------
    graph = None
    if cfg.T <= 256:
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g):
            step(torch.cuda.current_stream(dev))
        for _ in range(W):
            g.replay()
        torch.cuda.synchronize()
        ga, gb = ev(), ev()
        ga.record(stream)
        for _ in range(K):
            g.replay()
        gb.record(stream)
        torch.cuda.synchronize()
        gms = max_over_ranks(ga.elapsed_time(gb))
        graph = {"ms_per_step": gms / K, "value": world * cfg.T * K / (gms / 1e3), "steps": K}
        del g

    # ---- per-stage pass: one C-ABI call per stage, events between ------------
    P = cfg.P
    Kslots, Et = cfg.k + S, cfg.E + S
    i32 = dict(dtype=torch.int32, device=dev)
    ids = torch.empty(cfg.T, Kslots, **i32)
    wts = torch.empty(cfg.T, Kslots, dtype=torch.float32, device=dev)
    counts = torch.empty(Et, **i32)
    offsets = torch.empty(Et + 1, **i32)
    perm = torch.empty(P, **i32)
    inv = torch.empty(P, **i32)
    # the same gate/up kernel as moe_forward: rows read through perm, or a gathered copy
    in_gemm = moe.moe_forward_gathers_in_gemm(shape)
    hp = None if in_gemm else torch.empty(P, cfg.H, dtype=torch.bfloat16, device=dev)
    act = torch.empty(P, cfg.I, dtype=torch.bfloat16, device=dev)
    y = torch.empty(P, cfg.H, dtype=torch.bfloat16, device=dev)
    pws = torch.empty(max(1, moe.moe_permute_workspace_size(shape)), dtype=torch.uint8, device=dev)
    if cfg.fmt in ("mxfp8", "mxfp4"):
        # the MXFP8 layer: hidden quantised once per token, gate/up reads its
        # rows through perm and writes act quantised, down reads act's codes
        u8 = dict(dtype=torch.uint8, device=dev)
        hq, hs = torch.empty(cfg.T, cfg.H, **u8), torch.empty(cfg.T, cfg.H // 32, **u8)
        aq, as_ = torch.empty(P, cfg.I, **u8), torch.empty(P, cfg.I // 32, **u8)
        stages = ["route", "permute", "quantize", "gemm_swiglu", "gemm_down", "finalize"]
        calls = [
            lambda: moe.moe_route(d["logits"], shape, ids, wts, stream),
            lambda: moe.moe_permute(ids, shape, counts, offsets, perm, inv, None, None, pws, stream),
            lambda: moe.moe_mx_quantize(d["hidden"], cfg.T, cfg.H, hq, hs, stream),
            lambda: moe.moe_grouped_gemm_swiglu_mx(hq, hs, perm, offsets, d["w_gu"], scales[0], shape, aq, as_,
                                                   stream),
            lambda: moe.moe_grouped_gemm_down_mx(aq, as_, offsets, d["w_d"], scales[1], shape, y, stream),
            lambda: moe.moe_finalize(y, wts, inv, shape, out, stream),
        ]
    else:
        stages = ["route", "permute", "gemm_swiglu", "gemm_down", "finalize"]
        calls = [
            lambda: moe.moe_route(d["logits"], shape, ids, wts, stream),
            (lambda: moe.moe_permute(ids, shape, counts, offsets, perm, inv, None, None, pws, stream)) if in_gemm else
            (lambda: moe.moe_permute(ids, shape, counts, offsets, perm, inv, d["hidden"], hp, pws, stream)),
            (lambda: moe.moe_grouped_gemm_swiglu(d["hidden"], perm, offsets, d["w_gu"], scales[0], shape, act,
                                                 stream))
            if in_gemm else
            (lambda: moe.moe_grouped_gemm_swiglu(hp, None, offsets, d["w_gu"], scales[0], shape, act, stream)),
            lambda: moe.moe_grouped_gemm_down(act, offsets, d["w_d"], scales[1], shape, y, stream),
            lambda: moe.moe_finalize(y, wts, inv, shape, out, stream),
        ]
    fused = moe.moe_forward_is_fused(shape)
    if fused:
        # moe_forward runs the layer as one persistent kernel: time it too
        stages.append("fused")
        calls.append(lambda: moe.moe_forward_fused(d["hidden"], d["logits"], d["w_gu"], d["w_d"], shape, out, ws,
                                                   stream))
    for _ in range(W):
        for c in calls:
            c()
    torch.cuda.synchronize()
    n_rep = max(20, min(K, 200))
    se = [[ev() for _ in range(len(calls) + 1)] for _ in range(n_rep)]
    for r in range(n_rep):
        se[r][0].record(stream)
        for i, c in enumerate(calls):
            c()
            se[r][i + 1].record(stream)
    torch.cuda.synchronize()
    # median over repetitions: robust to the odd slow repetition (a clock dip)
    stage_ms = {s: statistics.median(se[r][i].elapsed_time(se[r][i + 1]) for r in range(n_rep))
                for i, s in enumerate(stages)}
    work = work_per_step(cfg, counts.cpu().numpy())

    # ---- end to end through moe_forward_host (pinned host buffers) ----------
    hws = torch.empty(moe.moe_forward_host_workspace_size(shape), dtype=torch.uint8, device=dev)
    h_host = inp["hidden"].pin_memory()
    l_host = inp["logits"].pin_memory()
    o_host = torch.empty(cfg.T, cfg.H, dtype=torch.bfloat16).pin_memory()

    def e2e_step():
        moe.moe_forward_host(h_host, l_host, d["w_gu"], scales[0], d["w_d"], scales[1], shape, o_host, hws, stream)

    for _ in range(W):
        e2e_step()
    barrier()
    torch.cuda.synchronize()
    ea, eb = ev(), ev()
    ea.record(stream)
    for _ in range(K):
        e2e_step()
    eb.record(stream)
    torch.cuda.synchronize()
    e_ms = max_over_ranks(ea.elapsed_time(eb))
    e2e = {"value": world * cfg.T * K / (e_ms / 1e3), "unit": UNIT,
           "h2d_bytes_per_step": h_host.numel() * h_host.element_size() + l_host.numel() * l_host.element_size(),
           "d2h_bytes_per_step": o_host.numel() * o_host.element_size()}

    err = moe.moe_get_device_error()
    if err:
        raise SystemExit(f"device error flag {err} raised during the benchmark of {cfg.name}")

    # ---- roofline of the dominant kernel -------------------------------------
    # each stage is timed on its own (a sub-millisecond launch between events),
    # so a tensor-bound kernel is held against the burst bf16 peak
    peaks, peak_src = read_peaks()
    dom = "fused" if fused else max(("gemm_swiglu", "gemm_down"), key=lambda s: stage_ms[s])
    wk = work[dom]
    # an MXFP8 contraction's peak: the measured bf16 peak times the nominal
    # fp8 / bf16 ratio of 2 (4.5 / 2.25 PFLOP/s dense)
    fp8 = cfg.fmt in ("mxfp8", "mxfp4")     # FP8 (or FP4 x FP8) operands on the block-scaled MMA
    tensor_peak = peaks["bf16_tflops"] * (2.0 if fp8 else 1.0)
    ridge = tensor_peak * 1e12 / (peaks["hbm_gbs"] * 1e9)
    launch_ms = stage_ms[dom]
    if fused:
        # the step is this one kernel after a one-warp counter reset: its
        # average duration over the timed region is the step time (the stage
        # pass times it alone, without the overlap of consecutive calls)
        launch_ms = ms_max / K
    sec = launch_ms / 1e3
    if wk["flops"] / wk["bytes"] < ridge:
        roof = {"bound": "hbm", "achieved": wk["bytes"] / sec / 1e9, "peak": peaks["hbm_gbs"], "unit": "GB/s"}
        which = "hbm_gbs"
    else:
        roof = {"bound": "tensor", "achieved": wk["flops"] / sec / 1e12, "peak": tensor_peak, "unit": "TFLOP/s"}
        which = ("bf16_tflops x 2 (fp8 / bf16 nominal ratio)" if fp8 else "bf16_tflops") + \
            " (burst: the kernel is timed alone)"
    roof["frac"] = roof["achieved"] / roof["peak"]
    roof["traffic"] = profiled_traffic(dom, cfg.name)
    roof["kernel"] = dom
    roof["algorithmic_per_launch"] = wk["bytes"] if roof["bound"] == "hbm" else wk["flops"]
    roof["peak_source"] = f"{peak_src} {which}"
    roof["launch_ms"] = launch_ms
    if fused:
        roof["launch_source"] = "timed region (K steps, each the counter reset and this kernel)"

    layer_s = ms_max / 1e3 / K
    res = {"value": value, "ms_per_step": ms_max / K, "steps": K, "step_ms": step_ms, "roofline": roof,
           "layer": dict(layer_fractions(cfg, work, layer_s, peaks), stage_ms=stage_ms), "e2e": e2e,
           "gpu_launches": launches_per_step(cfg) * K, "clocks": clocks}
    if graph:
        res["cuda_graph"] = graph
    cpu = None
    if headline and rank == 0 and world == 1 and not args.no_cpu_baseline:
        cpu = cpu_baseline(cfg, inp, args.cpu_budget_s)
    del d, ws, out, ids, wts, counts, offsets, perm, inv, hp, act, y, pws, hws
    torch.cuda.empty_cache()
    return res, cpu


def run_ours(args, rank, world, local):
    import torch
    import torch.distributed as dist

    import mixture_experts_expert_top_b200 as moe

    if not torch.cuda.is_available():
        raise SystemExit("bench.py needs a CUDA device (B200)")
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    if world > 1:
        import datetime
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120), device_id=dev)
    moe.lib()
    props = torch.cuda.get_device_properties(dev)
    uuid = f"GPU-{props.uuid}" if getattr(props, "uuid", None) else str(local)
    sampler = ClockSampler(uuid, local)
    sampler.start()
    try:
        cfg = get_workload(args.workload, args.set)
        head, cpu = measure(cfg, args, dev, world, rank, sampler, headline=True)
        others = {}
        for name in extra_workloads(args):
            c = get_workload(name)
            r, _ = measure(c, args, dev, world, rank, sampler, headline=False)
            others[name] = dict(r, config=c.describe())
    finally:
        sampler.stop()
    result = {
        "metric": METRIC, "value": head["value"], "unit": UNIT, "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": head["ms_per_step"], "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "bf16" if cfg.fmt == "bf16" else "bf16 (int4 weights)",
        "data": "synthetic (seeded N(0,1) tokens and logits, N(0,0.02) random-init expert weights)",
        "config": config_of(cfg, world),
        "roofline": head["roofline"], "layer": head["layer"], "step_ms": head["step_ms"], "e2e": head["e2e"],
        "gpu_launches": head["gpu_launches"], "clocks": head["clocks"],
        "workloads": others,
    }
    if "cuda_graph" in head:
        result["cuda_graph"] = head["cuda_graph"]
    if cpu:
        result["cpu_baseline"] = cpu
    if world > 1:
        dist.destroy_process_group()
    return result


# ------------------------------------------------------------ the oracle arm --

def _oracle_tokens_per_s(cfg, inp, tokens, reps_budget_s, min_reps=1):
    import oracle
    t0 = time.perf_counter()
    reps = 0
    while True:
        oracle.forward_tokens(inp, cfg.k, tokens, fmt=cfg.fmt)
        reps += 1
        el = time.perf_counter() - t0
        if reps >= min_reps and el >= reps_budget_s:
            break
    return reps * len(tokens) / el, reps, el


def cpu_baseline(cfg, inp, budget_s):
    import oracle
    n = cfg.T
    tokens = list(range(n))
    # one calibration pass on a few tokens to size the sample to the budget
    t0 = time.perf_counter()
    oracle.forward_tokens(inp, cfg.k, tokens[: min(4, n)], fmt=cfg.fmt)
    per_tok = (time.perf_counter() - t0) / min(4, n)
    ntok = max(1, min(n, int(budget_s / max(per_tok, 1e-9))))
    v, reps, el = _oracle_tokens_per_s(cfg, inp, tokens[:ntok], budget_s)
    return {"value": v, "unit": UNIT, "cores": oracle.num_threads(), "cpu_model": host_cpu_model(),
            "kind": "oracle",
            "sample": f"{reps} x {ntok} tokens of {cfg.name} (all k={cfg.k} experts per token, full H/I), "
                      f"{el:.1f} s of CPU time on {oracle.num_threads()} threads"}


def run_reference(args, rank, world):
    if rank != 0:
        return None
    import moe_synth
    import oracle
    cfg = get_workload(args.workload, args.set)
    inp = moe_synth.gen_inputs(cfg, seed=args.seed)
    # size each step so that warmup + steps fit the budget
    t0 = time.perf_counter()
    oracle.forward_tokens(inp, cfg.k, [0], fmt=cfg.fmt)
    per_tok = time.perf_counter() - t0
    per_step = args.ref_budget_s / (args.steps + args.warmup)
    ntok = max(1, min(cfg.T, int(per_step / max(per_tok, 1e-9))))
    tokens = list(range(ntok))
    for _ in range(args.warmup):
        oracle.forward_tokens(inp, cfg.k, tokens, fmt=cfg.fmt)
    t0 = time.perf_counter()
    for _ in range(args.steps):
        oracle.forward_tokens(inp, cfg.k, tokens, fmt=cfg.fmt)
    el = time.perf_counter() - t0
    value = args.steps * ntok / el
    sample = f"{ntok} of {cfg.T} tokens per step (all k={cfg.k} experts per token, full H/I)"
    return {
        "impl": "reference", "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": el * 1e3 / args.steps,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64 accumulate",
        "data": "synthetic (seeded N(0,1) tokens and logits, N(0,0.02) random-init expert weights)",
        "config": config_of(cfg, world),
        "cpu_baseline": {"value": value, "unit": UNIT, "cores": oracle.num_threads(), "cpu_model": host_cpu_model(),
                         "kind": "oracle", "sample": sample},
        "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }


def relaunch_under_torchrun(args, argv) -> int:
    """--gpus N > 1 started as a plain process: run the same command as N
    ranks under torchrun (one process per GPU) and return its exit status."""
    cmd = [sys.executable, "-m", "torch.distributed.run", "--nnodes=1", f"--nproc-per-node={args.gpus}",
           "--master-addr", "127.0.0.1", "--master-port", str(free_port()), os.path.abspath(__file__), *argv]
    return subprocess.call(cmd)


def main(argv=None):
    argv = list(sys.argv[1:] if argv is None else argv)
    args = parse_args(argv)
    if args.gpus > 1 and "WORLD_SIZE" not in os.environ:
        raise SystemExit(relaunch_under_torchrun(args, argv))
    rank, world, local = dist_env()
    if world != args.gpus:
        raise SystemExit(f"--gpus {args.gpus} but WORLD_SIZE={world}")
    if args.impl == "reference":
        res = run_reference(args, rank, world)
    else:
        res = run_ours(args, rank, world, local)
    if rank == 0 and res is not None:
        print(json.dumps(res), flush=True)


if __name__ == "__main__":
    main()
