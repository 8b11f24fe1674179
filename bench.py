#!/usr/bin/env python
"""Benchmark of the MoE expert-FFN layer (libmoe_b200) on B200.

One step = one whole layer call (route, permute + gather, grouped GEMM
gate/up + SwiGLU, grouped GEMM down, finalize) over one batch of synthetic
tokens, through the C ABI. The default workload is the Qwen3-30B-A3B-shaped
decode layer: T=64, H=2048, I=768, E=128, top_k=8, bf16 weights (1.2 GB of
expert weights, larger than the 126 MB L2, so no flush is needed between
steps).

  python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME] [--impl ours|reference]

With --gpus N > 1 (one process per GPU under torchrun) every rank runs its
own replica on its own token batch (token-sharded data parallel: the layer
needs no exchange between ranks), and value = all ranks' tokens / the
slowest rank's time.

--impl reference times the CPU oracle (the plain C reference in oracle/) on
the host cores, on the same workload, metric and unit.
"""

from __future__ import annotations

import argparse
import hashlib
import json
import os
import re
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
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}
NORTH_STAR_HBM_GBS = 8000.0       # the roofline literals the layer's target is stated against
NORTH_STAR_BF16_TFLOPS = 2250.0
PROFILE_DIR = os.path.join(ROOT, "profiles")
# the grouped-GEMM kernels' sources: a change to any of them invalidates stored counters
KERNEL_SOURCES = ["mixture_experts_expert_top_b200/csrc/gemm_sm100.cu",
                  "mixture_experts_expert_top_b200/csrc/gemm_prefill_sm100.cu",
                  "mixture_experts_expert_top_b200/csrc/gemm_common.cuh",
                  "mixture_experts_expert_top_b200/csrc/common.cuh",
                  "mixture_experts_expert_top_b200/csrc/launch_util.cuh"]


# ----------------------------------------------------------------- helpers --

def parse_args(argv=None):
    ap = argparse.ArgumentParser(description=__doc__.split("\n")[0])
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=2000)
    ap.add_argument("--warmup", type=int, default=20)
    ap.add_argument("--workload", default="qwen3_decode")
    ap.add_argument("--set", action="append", default=[], metavar="KEY=VALUE",
                    help="override a workload field (T, H, I, E, k), e.g. for a smaller profiling case")
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
    return a


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


def kernel_source_hash() -> str:
    h = hashlib.sha256()
    for rel in KERNEL_SOURCES:
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
    if not m_hash or not m_tr or m_hash.group(1) != kernel_source_hash():
        return None
    return float(m_tr.group(1))


class ClockSampler:
    """nvidia-smi samples of SM clock and throttle reasons during a region."""

    FIELDS = ["index", "clocks.sm", "clocks.max.sm", "power.draw", "clocks_event_reasons.active",
              "clocks_event_reasons.hw_slowdown", "clocks_event_reasons.hw_thermal_slowdown",
              "clocks_event_reasons.sw_thermal_slowdown", "clocks_event_reasons.sw_power_cap"]

    def __init__(self, gpu_id: str, period_ms: int = 50):
        self.gpu_id = gpu_id
        self.period_ms = period_ms
        self.proc = None
        self.lines = []
        self.t0 = self.t1 = None

    def start(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", self.gpu_id, f"--query-gpu={','.join(self.FIELDS)}",
                 "--format=csv,noheader,nounits", f"-lms", str(self.period_ms)],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except OSError:
            self.proc = None
            return
        self._reader = threading.Thread(target=self._read, daemon=True)
        self._reader.start()

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append((time.time(), line.strip()))

    def mark_begin(self):
        self.t0 = time.time()

    def mark_end(self):
        self.t1 = time.time()

    def stop(self):
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": [], "samples": 0}
        time.sleep(2 * self.period_ms / 1000.0)
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        rows = []
        for ts, line in self.lines:
            parts = [p.strip() for p in line.split(",")]
            if len(parts) != len(self.FIELDS):
                continue
            rows.append((ts, parts))
        inside = [r for ts, r in rows if self.t0 is not None and self.t0 <= ts <= (self.t1 or ts)]
        use = inside or [r for _, r in rows]
        sm = [float(r[1]) for r in use if _isnum(r[1])]
        smax = [float(r[2]) for r in use if _isnum(r[2])]
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({n for r in use for n, v in zip(names, r[5:9]) if v.lower().startswith("active")})
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": max(smax) if smax else None,
                "reasons": reasons, "samples": len(use), "samples_inside_timed_region": len(inside),
                "power_w_max": max((float(r[3]) for r in use if _isnum(r[3])), default=None)}


def _isnum(s):
    try:
        float(s)
        return True
    except ValueError:
        return False


# -------------------------------------------------------- workload accounting --

def work_per_step(cfg, counts):
    """Algorithmic bytes and FLOPs of each kernel for one step, from the real
    per-expert counts (experts with no rows read no weights)."""
    T, H, I, E, k = cfg.T, cfg.H, cfg.I, cfg.E, cfg.k
    P = T * k
    active = int(sum(1 for c in counts if c > 0))
    if cfg.fmt == "bf16":
        w_gu = active * 2 * I * H * 2
        w_d = active * H * I * 2
    else:
        w_gu = active * 2 * I * (H // 2 + (H // 128) * 2)
        w_d = active * H * (I // 2 + (I // 128) * 2)
    return {
        "active_experts": active,
        "weight_bytes": w_gu + w_d,
        "gemm_swiglu": {"bytes": w_gu + P * H * 2 + P * I * 2 + (E + 1) * 4, "flops": 2 * P * 2 * I * H},
        "gemm_down": {"bytes": w_d + P * I * 2 + P * H * 2 + (E + 1) * 4, "flops": 2 * P * H * I},
        "route": {"bytes": T * E * 4 + P * 8, "flops": 0},
        "permute": {"bytes": P * 4 * 3 + (2 * E + 1) * 4 + T * H * 2 + P * H * 2, "flops": 0},
        "finalize": {"bytes": P * H * 2 + T * H * 2 + P * 8, "flops": 0},
        "layer_flops": 2 * P * 3 * H * I,
    }


def launches_per_step(cfg) -> int:
    """Kernels one moe_forward call enqueues for this workload (the library's own count)."""
    import mixture_experts_expert_top_b200 as moe
    return moe.moe_forward_kernel_count(moe.Shape.of(cfg.T, cfg.H, cfg.I, cfg.E, cfg.k, cfg.fmt))


# ------------------------------------------------------------------ our arm --

def workload(args):
    import moe_synth
    cfg = moe_synth.get_config(args.workload)
    over = {}
    for kv in args.set:
        k, v = kv.split("=", 1)
        if k not in ("T", "H", "I", "E", "k"):
            raise SystemExit(f"--set: unknown field {k}")
        over[k] = int(v)
    if over:
        cfg = cfg.with_(**over, name=cfg.name + "+" + ",".join(f"{k}={v}" for k, v in sorted(over.items())))
    return cfg


def run_ours(args, rank, world, local):
    import numpy as np
    import torch
    import torch.distributed as dist

    import moe_synth
    import mixture_experts_expert_top_b200 as moe

    if not torch.cuda.is_available():
        raise SystemExit("bench.py needs a CUDA device (B200)")
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    if world > 1:
        import datetime
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120), device_id=dev)
    moe.lib()
    cfg = workload(args)
    # weights are the same on every rank (replicas); each rank draws its own tokens
    inp = moe_synth.gen_inputs(cfg, seed=args.seed)
    if rank:
        inp["hidden"] = moe_synth.gen_hidden(cfg, seed=args.seed + rank)
        inp["logits"] = moe_synth.gen_logits(cfg, seed=args.seed + rank)
    d = {n: t.to(dev) for n, t in inp.items()}
    shape = moe.Shape.of(cfg.T, cfg.H, cfg.I, cfg.E, cfg.k, cfg.fmt)
    ws = torch.empty(moe.moe_workspace_size(shape), dtype=torch.uint8, device=dev)
    out = torch.empty(cfg.T, cfg.H, dtype=torch.bfloat16, device=dev)
    stream = torch.cuda.current_stream(dev)
    scales = (d.get("w_gu_scales"), d.get("w_d_scales"))

    def step():
        moe.moe_forward(d["hidden"], d["logits"], d["w_gu"], scales[0], d["w_d"], scales[1], shape, out, ws, stream)

    # ---- device-timed value: K whole-layer steps ---------------------------
    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()
    props = torch.cuda.get_device_properties(dev)
    gpu_id = f"GPU-{props.uuid}" if getattr(props, "uuid", None) else str(local)
    sampler = ClockSampler(gpu_id)
    sampler.start()
    time.sleep(0.2)
    barrier()
    torch.cuda.synchronize()
    t_start, t_end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    sampler.mark_begin()
    t_start.record(stream)
    for _ in range(args.steps):
        step()
    t_end.record(stream)
    torch.cuda.synchronize()
    sampler.mark_end()
    barrier()
    ms = t_start.elapsed_time(t_end)
    clocks = sampler.stop()
    ms_max = max_over_ranks(ms)
    value = world * cfg.T * args.steps / (ms_max / 1e3)

    # ---- per-kernel durations (same kernels, one C-ABI call per stage) -----
    P = cfg.P
    i32 = dict(dtype=torch.int32, device=dev)
    ids = torch.empty(cfg.T, cfg.k, **i32)
    wts = torch.empty(cfg.T, cfg.k, dtype=torch.float32, device=dev)
    counts = torch.empty(cfg.E, **i32)
    offsets = torch.empty(cfg.E + 1, **i32)
    perm = torch.empty(P, **i32)
    inv = torch.empty(P, **i32)
    # the same gate/up kernel as moe_forward: rows read through perm, or a gathered copy
    in_gemm = moe.moe_forward_gathers_in_gemm(shape)
    hp = None if in_gemm else torch.empty(P, cfg.H, dtype=torch.bfloat16, device=dev)
    act = torch.empty(P, cfg.I, dtype=torch.bfloat16, device=dev)
    y = torch.empty(P, cfg.H, dtype=torch.bfloat16, device=dev)
    pws = torch.empty(max(1, moe.moe_permute_workspace_size(shape)), dtype=torch.uint8, device=dev)
    stages = ["route", "permute", "gemm_swiglu", "gemm_down", "finalize"]
    calls = [
        lambda: moe.moe_route(d["logits"], shape, ids, wts, stream),
        (lambda: moe.moe_permute(ids, shape, counts, offsets, perm, inv, None, None, pws, stream)) if in_gemm else
        (lambda: moe.moe_permute(ids, shape, counts, offsets, perm, inv, d["hidden"], hp, pws, stream)),
        (lambda: moe.moe_grouped_gemm_swiglu(d["hidden"], perm, offsets, d["w_gu"], scales[0], shape, act, stream))
        if in_gemm else
        (lambda: moe.moe_grouped_gemm_swiglu(hp, None, offsets, d["w_gu"], scales[0], shape, act, stream)),
        lambda: moe.moe_grouped_gemm_down(act, offsets, d["w_d"], scales[1], shape, y, stream),
        lambda: moe.moe_finalize(y, wts, inv, shape, out, stream),
    ]
    for _ in range(args.warmup):
        for c in calls:
            c()
    torch.cuda.synchronize()
    n_rep = args.steps
    ev = [[torch.cuda.Event(enable_timing=True) for _ in range(len(calls) + 1)] for _ in range(n_rep)]
    for r in range(n_rep):
        ev[r][0].record(stream)
        for i, c in enumerate(calls):
            c()
            ev[r][i + 1].record(stream)
    torch.cuda.synchronize()
    # median over repetitions: robust to the odd slow repetition (a clock dip)
    stage_ms = {s: statistics.median(ev[r][i].elapsed_time(ev[r][i + 1]) for r in range(n_rep))
                for i, s in enumerate(stages)}
    counts_h = counts.cpu().numpy()
    work = work_per_step(cfg, counts_h)

    # ---- end to end through moe_forward_host (pinned host buffers) ----------
    hws = torch.empty(moe.moe_forward_host_workspace_size(shape), dtype=torch.uint8, device=dev)
    h_host = inp["hidden"].pin_memory()
    l_host = inp["logits"].pin_memory()
    o_host = torch.empty(cfg.T, cfg.H, dtype=torch.bfloat16).pin_memory()

    def e2e_step():
        moe.moe_forward_host(h_host, l_host, d["w_gu"], scales[0], d["w_d"], scales[1], shape, o_host, hws, stream)

    for _ in range(args.warmup):
        e2e_step()
    barrier()
    torch.cuda.synchronize()
    e_start, e_end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e_start.record(stream)
    for _ in range(args.steps):
        e2e_step()
    e_end.record(stream)
    torch.cuda.synchronize()
    e_ms = max_over_ranks(e_start.elapsed_time(e_end))
    e2e_value = world * cfg.T * args.steps / (e_ms / 1e3)
    h2d = h_host.numel() * h_host.element_size() + l_host.numel() * l_host.element_size()
    d2h = o_host.numel() * o_host.element_size()

    err = moe.moe_get_device_error()
    if err:
        raise SystemExit(f"device error flag {err} raised during the benchmark")

    # ---- roofline of the dominant kernel -------------------------------------
    peaks, peak_src = read_peaks()
    dom = max(("gemm_swiglu", "gemm_down"), key=lambda s: stage_ms[s])
    wk = work[dom]
    ai = wk["flops"] / wk["bytes"]
    ridge = peaks["bf16_tflops_sustained"] * 1e12 / (peaks["hbm_gbs"] * 1e9)
    sec = stage_ms[dom] / 1e3
    if ai < ridge:
        roof = {"bound": "hbm", "achieved": wk["bytes"] / sec / 1e9, "peak": peaks["hbm_gbs"], "unit": "GB/s"}
    else:
        roof = {"bound": "tensor", "achieved": wk["flops"] / sec / 1e12, "peak": peaks["bf16_tflops_sustained"],
                "unit": "TFLOP/s"}
    roof["frac"] = roof["achieved"] / roof["peak"]
    roof["traffic"] = profiled_traffic(dom, cfg.name)
    roof["kernel"] = dom
    roof["algorithmic_per_launch"] = wk["bytes"] if roof["bound"] == "hbm" else wk["flops"]
    roof["peak_source"] = f"{peak_src} ({'hbm_gbs' if roof['bound'] == 'hbm' else 'bf16_tflops_sustained'})"
    roof["launch_ms"] = stage_ms[dom]

    layer_s = ms_max / 1e3 / args.steps
    result = {
        "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": ms_max / args.steps, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "bf16" if cfg.fmt == "bf16" else "bf16 (int4 weights)",
        "data": "synthetic (seeded N(0,1) tokens and logits, N(0,0.02) random-init expert weights)",
        "config": {"workload": cfg.describe(), "T": cfg.T, "H": cfg.H, "I": cfg.I, "E": cfg.E, "top_k": cfg.k,
                   "weights": cfg.fmt, "global_batch": world * cfg.T,
                   "parallelism": "replicas (token-sharded, no collective)" if world > 1 else "single GPU",
                   "l2": f"inputs larger than L2: {work['weight_bytes'] / 1e9:.3f} GB of expert weights read per step"},
        "roofline": roof,
        "layer": {"active_experts": work["active_experts"], "weight_bytes": work["weight_bytes"],
                  "flops": work["layer_flops"],
                  "hbm_frac_of_measured": work["weight_bytes"] / layer_s / (peaks["hbm_gbs"] * 1e9),
                  "hbm_frac_of_8TBps": work["weight_bytes"] / layer_s / (NORTH_STAR_HBM_GBS * 1e9),
                  "tensor_frac_of_2250TF": work["layer_flops"] / layer_s / (NORTH_STAR_BF16_TFLOPS * 1e12),
                  "stage_ms": stage_ms},
        "e2e": {"value": e2e_value, "unit": UNIT, "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h},
        "gpu_launches": launches_per_step(cfg) * args.steps,
        "clocks": clocks,
    }
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        result["cpu_baseline"] = cpu_baseline(cfg, inp, args.cpu_budget_s)
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
    return {"value": v, "unit": UNIT, "cores": oracle.num_threads(), "kind": "oracle",
            "sample": f"{reps} x {ntok} tokens of {cfg.name} (all k={cfg.k} experts per token, full H/I), "
                      f"{el:.1f} s of CPU time on {oracle.num_threads()} threads"}


def run_reference(args, rank, world):
    if rank != 0:
        return None
    import moe_synth
    import oracle
    cfg = workload(args)
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
        "data": "synthetic", "config": {"workload": cfg.describe(), "global_batch": cfg.T},
        "cpu_baseline": {"value": value, "unit": UNIT, "cores": oracle.num_threads(), "kind": "oracle",
                         "sample": sample},
        "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }


def main(argv=None):
    args = parse_args(argv)
    rank, world, local = dist_env()
    if world != args.gpus and "WORLD_SIZE" in os.environ:
        raise SystemExit(f"--gpus {args.gpus} but WORLD_SIZE={world}")
    world = max(world, 1)
    if args.impl == "reference":
        res = run_reference(args, rank, world)
    else:
        res = run_ours(args, rank, world, local)
    if rank == 0 and res is not None:
        print(json.dumps(res), flush=True)


if __name__ == "__main__":
    main()
