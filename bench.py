#!/usr/bin/env python
"""Benchmark of the action-expert denoise loop (one JSON line on rank 0).

    python bench.py [--gpus N] [--steps K] [--warmup W] [--config NAME]
                    [--impl ours|reference] [--no-secondary] [--no-cpu-baseline]

A "step" is one pae_denoise call: the whole hot path (input projection, 18
expert layers, output projection and Euler update, for all Euler steps) over
one batch of synthetic action chunks whose prefix K/V is already cached.
Throughput follows the pages' definition: batch size over synchronised batch
time (PhyAI report, Sec. 5.2 / Eq. 9), here chunks/s.  Timing: W untimed
warm-up calls, then K calls between CUDA events on the launching stream,
bracketed by a barrier and a device synchronise; the max over ranks is taken.
Each rank runs an independent replica (pi0.5 requests are data-parallel with no
exchange in the loop), so scaling is weak and there is no collective on the
data path.  The weights (623 MB of projections) are larger than L2, so every
Euler step streams them from HBM; no L2 flush is needed.

--impl reference times the float64 CPU oracle instead (the only reference this
build has), on a bounded sample of the same workload.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import os
import statistics
import sys
import threading
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import workloads as wl  # noqa: E402

METRIC = "denoise-loop action chunks/s at bs1 and bs32; achieved HBM GB/s / TC util vs peak"
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}


# --------------------------------------------------------------------- helpers
def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return d, "measured"
    return dict(FALLBACK_PEAKS), "fallback"


def dist_env():
    ws = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return ws, rank, local


class ClockSampler:
    """Samples SM clock and throttle reasons through NVML while running."""

    REASONS = {0x8: "hw_slowdown", 0x40: "hw_thermal_slowdown", 0x20: "sw_thermal_slowdown",
               0x4: "sw_power_cap", 0x80: "hw_power_brake_slowdown", 0x1: "gpu_idle"}

    def __init__(self, index: int, period_s: float = 0.005):
        self.index = index
        self.period = period_s
        self.samples = []
        self.reasons = set()
        self.max_mhz = None
        self._stop = threading.Event()
        self._t = None
        self.ok = False

    def start(self):
        try:
            import pynvml
            pynvml.nvmlInit()
            h = pynvml.nvmlDeviceGetHandleByIndex(self.index)
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(h, pynvml.NVML_CLOCK_SM)
            self.ok = True
        except Exception:
            return self

        def run():
            while not self._stop.is_set():
                try:
                    self.samples.append(pynvml.nvmlDeviceGetClockInfo(h, pynvml.NVML_CLOCK_SM))
                    r = pynvml.nvmlDeviceGetCurrentClocksEventReasons(h)
                    for bit, name in self.REASONS.items():
                        if r & bit and name != "gpu_idle":
                            self.reasons.add(name)
                except Exception:
                    pass
                time.sleep(self.period)

        self._t = threading.Thread(target=run, daemon=True)
        self._t.start()
        return self

    def stop(self):
        self._stop.set()
        if self._t:
            self._t.join()
        if not self.ok or not self.samples:
            return None
        return {"sm_mhz": float(statistics.median(self.samples)), "sm_max_mhz": float(self.max_mhz),
                "reasons": sorted(self.reasons), "samples": len(self.samples), "source": "nvml"}


FUSED_NORM = [0]  # PAE_OPT_FUSED_NORM for every context the benchmark creates
DATAFLOW = [-1]   # PAE_OPT_DATAFLOW for every context (-1: the library default)
FACTORED = [-1]   # PAE_OPT_FACTORED_NORM for every context (-1: the library default)


def algorithmic(cfg: wl.ExpertConfig, batch: int, lens=None):
    """Algorithmic bytes and FLOPs per launch of each kernel class and per
    Euler step (weights and prefix/action K/V once, activations once; table
    build excluded)."""
    D, F, A, H, L = cfg.width, cfg.mlp_dim, cfg.action_dim, cfg.chunk, cfg.layers
    qkv, att = cfg.qkv_dim, cfg.attn_dim
    M = batch * H
    if lens is None:
        lens = [cfg.prefix] * batch
    if cfg.dtype == wl.W4A16:
        wb = lambda n, k: n * k / 2 + n * (k // cfg.group_size) * 2  # noqa: E731
    else:
        es = 4 if cfg.dtype == wl.FP32 else 2
        wb = lambda n, k: n * k * es  # noqa: E731
    ae = 4 if cfg.dtype == wl.FP32 else 2
    kv_tokens = sum(p + H for p in lens)
    out = {
        "qkv": {"bytes": wb(qkv, D) + M * D * ae + M * qkv * ae, "flops": 2 * M * qkv * D},
        "attention": {"bytes": 2 * kv_tokens * cfg.n_kv_heads * cfg.head_dim * ae + 2 * M * att * ae,
                      "flops": 4 * cfg.n_q_heads * H * cfg.head_dim * sum(p + H for p in lens)},
        "o_proj": {"bytes": wb(D, att) + M * att * ae + 2 * M * D * 4, "flops": 2 * M * D * att},
        "gate_up": {"bytes": wb(2 * F, D) + M * D * ae + M * F * ae, "flops": 2 * M * 2 * F * D},
        "down": {"bytes": wb(D, F) + M * F * ae + 2 * M * D * 4, "flops": 2 * M * D * F},
    }
    # in/out projections stay in the activation dtype (bf16 in int4 mode)
    step_w = L * (wb(qkv, D) + wb(D, att) + wb(2 * F, D) + wb(D, F)) + 2 * D * A * (4 if cfg.dtype == wl.FP32 else 2)
    step_kv = L * 2 * sum(lens) * cfg.n_kv_heads * cfg.head_dim * ae
    step_flops = L * (out["qkv"]["flops"] + out["o_proj"]["flops"] + out["gate_up"]["flops"] +
                      out["down"]["flops"] + out["attention"]["flops"]) + 2 * 2 * M * A * D
    # the persistent kernel and the dataflow loop run a whole call (all Euler steps) in one launch
    out["persistent"] = {"bytes": cfg.steps * (step_w + step_kv), "flops": cfg.steps * step_flops}
    out["dataflow"] = dict(out["persistent"])
    return out, {"bytes": step_w + step_kv, "flops": step_flops}


# The files each kernel class is compiled from (its own file and the headers
# it includes); a traffic figure stays valid while these are unchanged.
_GEMM_SOURCES = ["k_tc_gemm.cu", "epilogue.cuh", "internal.h", "common.cuh", "launch.cuh"]
KERNEL_SOURCES = {
    "attention": ["k_attn_tc.cu", "internal.h", "common.cuh", "launch.cuh"],
    "gemm": _GEMM_SOURCES,
    "qkv": _GEMM_SOURCES,
    "o_proj": _GEMM_SOURCES,
    "gate_up": _GEMM_SOURCES,
    "down": _GEMM_SOURCES,
    "transition": ["k_token.cu", "internal.h", "common.cuh", "launch.cuh"],
    "norm": ["k_token.cu", "internal.h", "common.cuh", "launch.cuh"],
    "dataflow": ["k_flow.cu", "epilogue.cuh", "internal.h", "common.cuh", "launch.cuh"],
}


def src_hash(kernel=None):
    """Hash of the kernel sources: all of csrc, or the files of one kernel class."""
    h = hashlib.sha256()
    csrc = os.path.join(ROOT, "flow_matching_action_pi0_b200", "csrc")
    names = KERNEL_SOURCES.get(kernel) or [n for n in os.listdir(csrc) if n.endswith((".cu", ".cuh", ".h"))]
    for name in sorted(names):
        with open(os.path.join(csrc, name), "rb") as f:
            h.update(name.encode() + f.read())
    return h.hexdigest()[:16]


def ncu_traffic(workload: str, kernel: str):
    """DRAM bytes per launch from the committed ncu summary, if it was taken
    on the current kernel sources (else None)."""
    p = os.path.join(ROOT, "profiles", "ncu_traffic.json")
    if not os.path.exists(p):
        return None
    with open(p) as f:
        d = json.load(f)
    e = d.get(f"{workload}:{kernel}")
    if not e or e.get("src_sha") != src_hash(kernel if kernel in KERNEL_SOURCES else None):
        return None
    return e.get("dram_bytes_per_launch")


def blas_threads():
    try:
        from threadpoolctl import threadpool_info
        n = [i["num_threads"] for i in threadpool_info() if i.get("user_api") == "blas"]
        return int(max(n)) if n else 1
    except Exception:
        return os.cpu_count() or 1


# --------------------------------------------------------------- oracle timing
def oracle_sample_time(cfg, W, ks, vs, noise, euler_steps: int):
    """Seconds the float64 oracle takes for one request over `euler_steps`
    Euler steps of the workload's grid (tables excluded, as on the GPU)."""
    return oracle_sample_times(cfg, W, ks, vs, noise, euler_steps)[0]


def oracle_sample_times(cfg, W, ks, vs, noise, euler_steps: int, min_seconds: float = 0.0, max_reps: int = 1):
    """Times of repeated oracle runs of one request (`euler_steps` Euler steps,
    tables excluded), repeated until `min_seconds` of work or `max_reps` runs;
    the weights are converted once, outside the timed runs."""
    import oracle
    p = oracle.params_from_weights(cfg, W)
    grid = wl.uniform_grid(cfg.steps)
    tabs = oracle.modulation_tables(grid, p)[:euler_steps]
    kp = [np.asarray(a, np.float64) for a in ks[0]]
    vp = [np.asarray(a, np.float64) for a in vs[0]]
    x0 = noise[0].astype(np.float64)
    times = []
    while not times or (sum(times) < min_seconds and len(times) < max_reps):
        t0 = time.perf_counter()
        oracle.denoise_row(x0.copy(), tabs, p, kp, vp)
        times.append(time.perf_counter() - t0)
    return times


def run_reference(args, cfg):
    ws, rank, _ = dist_env()
    if rank != 0:
        return 0
    W = wl.make_weights(cfg)
    lens = wl.prefix_lengths(cfg)[:1]
    ks, vs = wl.make_prefix(cfg, lengths=lens)
    noise = wl.make_noise(cfg, batch=1)
    # one Euler step of one request per step, the weights converted once
    ts = oracle_sample_times(cfg, W, ks, vs, noise, 1, min_seconds=float("inf"),
                             max_reps=args.warmup + args.steps)
    per = ts[args.warmup:]
    t_euler = float(np.mean(per))
    chunk_s = t_euler * cfg.steps            # one request, all Euler steps
    value = 1.0 / chunk_s                    # rows are independent: chunks/s
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": "chunks/s", "n_gpus": ws,
        "steps": args.steps, "warmup": args.warmup,
        # what one timed step is: one Euler step of one request
        "ms_per_step": t_euler * 1e3,
        "step": "one Euler step of one request (the oracle's unit of work)",
        "chunk_ms_extrapolated": chunk_s * 1e3,
        "batch_ms_extrapolated": chunk_s * 1e3 * cfg.batch,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic", "config": workload_config(cfg),
        "cpu_baseline": {"value": value, "unit": "chunks/s", "cores": blas_threads(), "kind": "oracle",
                         "sample": f"one request, one Euler step per timed step (x{cfg.steps} for a chunk)"},
        "e2e": {"value": value, "unit": "chunks/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)
    return 0


def workload_config(cfg, batch=None):
    return {"workload": cfg.name, "batch": cfg.batch if batch is None else batch, "chunk": cfg.chunk,
            "action_dim": cfg.action_dim, "prefix": cfg.prefix, "euler_steps": cfg.steps,
            "layers": cfg.layers, "width": cfg.width, "heads": f"{cfg.n_q_heads}q/{cfg.n_kv_heads}kv",
            "head_dim": cfg.head_dim, "mlp_dim": cfg.mlp_dim, "weights": cfg.dtype,
            "l2": "no flush: inputs larger than L2 (projection weights stream from HBM every Euler step)",
            "parallelism": "replicas (one independent context per GPU)"}


# ------------------------------------------------------------------ GPU timing
def setup_context(cfg, W, batch: int, lens=None):
    import flow_matching_action_pi0_b200 as fm
    from workloads import device as wd
    dev_w = wd.upload_weights(cfg, W)
    ex = fm.ActionExpert(fm.make_config(**wd.abi_config(cfg, max_batch=batch)), dev_w)
    del dev_w
    ex.set_option(fm.PAE_OPT_FUSED_NORM, FUSED_NORM[0])
    if DATAFLOW[0] >= 0:
        ex.set_option(fm.PAE_OPT_DATAFLOW, DATAFLOW[0])
    if FACTORED[0] >= 0:
        ex.set_option(fm.PAE_OPT_FACTORED_NORM, FACTORED[0])
    if lens is None:
        lens = [cfg.prefix] * batch
    ks, vs = wl.make_prefix(cfg, lengths=lens)
    kd, vd = wd.upload_prefix(cfg, ks, vs)
    for b in range(batch):
        ex.set_prefix(b, kd[b], vd[b], lens[b])
    t0 = time.perf_counter()
    ex.precompute_tables(wl.uniform_grid(cfg.steps))
    ex.sync()
    table_ms = (time.perf_counter() - t0) * 1e3
    return ex, ks, vs, kd, vd, lens, table_ms


def timed(fn, steps, warmup, stream, barrier):
    import torch
    for _ in range(warmup):
        fn()
    torch.cuda.synchronize()
    barrier()
    torch.cuda.synchronize()
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for _ in range(steps):
        fn()
    e1.record(stream)
    torch.cuda.synchronize()
    barrier()
    return e0.elapsed_time(e1) / steps


def profile_classes(ex, nd, od, stream, args):
    """Live per-kernel timing: the same loop with CUDA events around every
    launch (PAE_OPT_PROFILE), a few calls, per class the mean device time per
    launch, the launches per call and the time per call."""
    import flow_matching_action_pi0_b200 as fm
    ex.set_option(fm.PAE_OPT_PROFILE, (1 << len(fm.KERNEL_CLASSES)) - 1)
    n_prof = max(3, min(args.steps, 10))
    for _ in range(2):
        ex.denoise(nd, od, stream)
    stream.synchronize()
    tot = {c: 0.0 for c in fm.KERNEL_CLASSES}
    cnt = {c: 0 for c in fm.KERNEL_CLASSES}
    for _ in range(n_prof):
        ex.denoise(nd, od, stream)
        stream.synchronize()
        for i, c in enumerate(fm.KERNEL_CLASSES):
            t, n = ex.profile_read(i)
            tot[c] += t
            cnt[c] += n
    ex.set_option(fm.PAE_OPT_PROFILE, 0)
    return {c: {"ms_per_launch": (tot[c] / cnt[c]) if cnt[c] else 0.0, "launches_per_step": cnt[c] // n_prof,
                "ms_per_step": tot[c] / n_prof} for c in fm.KERNEL_CLASSES}


def measure(cfg, W, batch, args, stream, barrier, maxr, lens=None, with_e2e=True, gpu_index=0):
    import torch
    import flow_matching_action_pi0_b200 as fm
    ex, ks, vs, kd, vd, lens, table_ms = setup_context(cfg, W, batch, lens)
    noise = wl.make_noise(cfg, batch=batch)
    nd = torch.from_numpy(noise).cuda()
    od = torch.empty_like(nd)
    res = {"lens": lens}
    with torch.cuda.stream(stream):
        clk = ClockSampler(gpu_index).start()
        ms = timed(lambda: ex.denoise(nd, od, stream), args.steps, args.warmup, stream, barrier)
        res["clocks"] = clk.stop()
        res["ms_per_step"] = maxr(ms)
        res["persistent"] = ex.query(fm.PAE_Q_PERSISTENT, batch)
        res["dataflow"] = ex.query(fm.PAE_Q_DATAFLOW, batch)
        # kernels per pae_denoise call: one persistent or dataflow launch, or the captured graph's kernel nodes
        res["graph_kernels"] = 1 if (res["persistent"] or res["dataflow"]) else \
            ex.query(fm.PAE_Q_GRAPH_KERNELS, batch)
        res["splits"] = ex.query(fm.PAE_Q_SPLITS, batch)
        res["token_tile"] = ex.query(fm.PAE_Q_TOKEN_TILE, batch)
        res["table_ms"] = table_ms
        if with_e2e:
            nh = torch.from_numpy(noise).pin_memory()
            oh = torch.empty_like(nh).pin_memory()
            for _ in range(args.warmup):
                ex.denoise_host(nh, oh, stream)
            torch.cuda.synchronize()
            barrier()
            t0 = time.perf_counter()
            for _ in range(args.steps):
                ex.denoise_host(nh, oh, stream)
                stream.synchronize()      # result read back on the host every step
            wall = (time.perf_counter() - t0) / args.steps
            res["e2e_ms"] = maxr(wall * 1e3)
            res["io_bytes"] = int(nh.numel() * 4)
        res["kernels"] = profile_classes(ex, nd, od, stream, args)
    res["ex"] = ex
    res["ks"], res["vs"] = ks, vs
    res["noise"] = noise
    return res


def class_fractions(per_c, dur_ms, peaks):
    """Both roofline fractions of one kernel class from its algorithmic bytes and
    FLOPs per launch and its measured duration per launch."""
    if dur_ms <= 0:
        return None
    dur = dur_ms * 1e-3
    gbs = per_c["bytes"] / dur / 1e9
    tfs = per_c["flops"] / dur / 1e12
    ridge = (peaks["bf16_tflops_sustained"] * 1e12) / (peaks["hbm_gbs"] * 1e9)
    return {"bound": "hbm" if per_c["flops"] / max(per_c["bytes"], 1) < ridge else "tensor",
            "ms_per_launch": dur_ms, "algorithmic_bytes_per_launch": per_c["bytes"],
            "algorithmic_flops_per_launch": per_c["flops"], "achieved_gbs": gbs, "frac_hbm": gbs / peaks["hbm_gbs"],
            "achieved_tflops": tfs, "frac_tensor": tfs / peaks["bf16_tflops_sustained"]}


def roofline_for(cfg, batch, res, peaks, peak_kind, lens):
    """Roofline block for the kernel class that sets the bound of the loop.

    The loop is HBM-bound when its algorithmic bytes take longer at the HBM
    peak than its FLOPs at the tensor peak (batch 1); the class reported is
    then the one that moves the most bytes per Euler step (the gate/up
    projection).  Otherwise (batch 32, ragged 16) it is the class with the
    largest share of the measured step time.  Per-class durations come from
    CUDA events around every launch of the same loop; those events serialise
    the launches (no programmatic overlap), so each duration is an upper bound
    and each achieved figure a lower bound."""
    per, step = algorithmic(cfg, batch, lens)
    ks = res["kernels"]
    total = sum(v["ms_per_step"] for v in ks.values()) or 1.0
    hbm_t = step["bytes"] / (peaks["hbm_gbs"] * 1e9)
    tc_t = step["flops"] / (peaks["bf16_tflops_sustained"] * 1e12)
    timed_classes = [c for c in per if ks.get(c, {}).get("launches_per_step", 0) > 0]
    if not timed_classes:  # one persistent launch: the whole call is the kernel
        timed_classes = ["persistent"]
    if hbm_t >= tc_t:
        dom = max(timed_classes, key=lambda c: per[c]["bytes"] * ks[c]["launches_per_step"])
    else:
        dom = max(timed_classes, key=lambda c: ks[c]["ms_per_step"])
    fr = class_fractions(per[dom], ks[dom]["ms_per_launch"], peaks)
    hbm_bound = fr["bound"] == "hbm"
    if hbm_bound:
        rl = {"bound": "hbm", "unit": "GB/s", "achieved": fr["achieved_gbs"], "peak": peaks["hbm_gbs"],
              "frac": fr["frac_hbm"]}
    else:
        rl = {"bound": "tensor", "unit": "TFLOP/s", "achieved": fr["achieved_tflops"],
              "peak": peaks["bf16_tflops_sustained"], "frac": fr["frac_tensor"]}
    rl.update({"kernel": dom, "algorithmic_bytes_per_launch": per[dom]["bytes"],
               "algorithmic_flops_per_launch": per[dom]["flops"],
               "peak_source": f"{peak_kind} ({'hbm_gbs' if hbm_bound else 'bf16_tflops_sustained'})",
               "ms_per_launch": ks[dom]["ms_per_launch"], "share_of_step": ks[dom]["ms_per_step"] / total,
               "timing": "CUDA events around each launch (serialised; duration is an upper bound)",
               "traffic": ncu_traffic(cfg.name if batch == cfg.batch else f"{cfg.name}@{batch}", dom)})
    rl["per_class"] = {c: class_fractions(per[c], ks[c]["ms_per_launch"], peaks) for c in timed_classes}
    wname = cfg.name if batch == cfg.batch else f"{cfg.name}@{batch}"
    for c in timed_classes:
        rl["per_class"][c]["traffic"] = ncu_traffic(wname, c)
    # whole loop against the HBM and tensor rooflines
    t_step = res["ms_per_step"] * 1e-3 / cfg.steps
    loop = {"euler_step_us": t_step * 1e6, "bytes_per_euler_step": step["bytes"],
            "flops_per_euler_step": step["flops"], "hbm_roofline_us": hbm_t * 1e6,
            "tensor_roofline_us": tc_t * 1e6, "frac_of_roofline": max(hbm_t, tc_t) / t_step,
            "frac_hbm": hbm_t / t_step, "frac_tensor": tc_t / t_step,
            "achieved_gbs": step["bytes"] / t_step / 1e9, "achieved_tflops": step["flops"] / t_step / 1e12}
    shares = {c: ks[c]["ms_per_step"] / total for c in ks}
    return rl, loop, shares


def run_minimal(args, cfg):
    """Warm-up and timed pae_denoise calls only (for ncu launch ranges): the
    launches before the timed region are 1 (weight transpose) + batch
    (prefix lengths) + 6 (tables: time MLP, modulation rows, two projected
    shift tables) + warmup x graph kernels."""
    import torch
    import flow_matching_action_pi0_b200 as fm
    torch.cuda.set_device(0)
    W = wl.make_weights(cfg)
    ex, *_ = setup_context(cfg, W, cfg.batch, wl.prefix_lengths(cfg))
    ex.set_option(fm.PAE_OPT_PDL, args.pdl)
    ex.set_option(fm.PAE_OPT_PERSISTENT, args.persistent)
    if args.max_splitk:
        ex.set_option(fm.PAE_OPT_MAX_SPLITK, args.max_splitk)
    nd = torch.from_numpy(wl.make_noise(cfg)).cuda()
    od = torch.empty_like(nd)
    stream = torch.cuda.Stream()
    with torch.cuda.stream(stream):
        ms = timed(lambda: ex.denoise(nd, od, stream), args.steps, args.warmup, stream, lambda: None)
    persist = ex.query(fm.PAE_Q_PERSISTENT, cfg.batch)
    flow = ex.query(fm.PAE_Q_DATAFLOW, cfg.batch)
    k = 1 if (persist or flow) else ex.query(fm.PAE_Q_GRAPH_KERNELS, cfg.batch)
    print(json.dumps({"workload": cfg.name, "pdl": args.pdl, "persistent": persist, "dataflow": flow,
                      "max_splitk": args.max_splitk, "ms_per_step": ms,
                      "splits": ex.query(fm.PAE_Q_SPLITS, cfg.batch), "graph_kernels": k,
                      "launches_before_timed": 1 + cfg.batch + 6 + args.warmup * k}), flush=True)
    ex.close()
    return 0


def rank_helpers(world_size: int, device: str = "cuda"):
    """Barrier and max-over-ranks for the timing protocol (the process group
    must already exist when world_size > 1).  Replicas share nothing else."""
    if world_size <= 1:
        return (lambda: None), (lambda v: float(v))
    import torch
    import torch.distributed as dist

    def barrier():
        dist.barrier()

    def maxr(v):
        t = torch.tensor([float(v)], device=device)
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
        return float(t.item())

    return barrier, maxr


def measure_ragged(args, stream, barrier, maxr, ws, gpu_index):
    """Ragged batch 16: per-request prefix lengths drawn on [512, 1024]; every
    timed step re-sets 8 rows with fresh prefixes (a new observation each) and
    keeps 8 (cache hits), then runs the denoise loop."""
    import torch
    import flow_matching_action_pi0_b200 as fm
    from workloads import device as wd
    cfg = wl.RAGGED_BF16_BS16
    W = wl.make_weights(cfg)
    lens = wl.prefix_lengths(cfg)
    ex, ks, vs, kd, vd, lens, _ = setup_context(cfg, W, cfg.batch, lens)
    # a second set of prefixes for the fresh rows, swapped in alternately
    ks2, vs2 = wl.make_prefix(cfg, lengths=lens[:8], seed=1000 + cfg.index)
    kd2, vd2 = wd.upload_prefix(cfg, ks2, vs2)
    noise = wl.make_noise(cfg)
    nd = torch.from_numpy(noise).cuda()
    od = torch.empty_like(nd)
    flip = [0]

    def step():
        src_k, src_v = (kd2, vd2) if flip[0] % 2 == 0 else (kd[:8], vd[:8])
        for r in range(8):
            ex.set_prefix(r, src_k[r], src_v[r], lens[r], stream)
        flip[0] += 1
        ex.denoise(nd, od, stream)

    peaks, peak_kind = load_peaks()
    with torch.cuda.stream(stream):
        clk = ClockSampler(gpu_index).start()
        ms = maxr(timed(step, args.steps, args.warmup, stream, barrier))
        ms_loop = maxr(timed(lambda: ex.denoise(nd, od, stream), args.steps, args.warmup, stream, barrier))
        clocks = clk.stop()
        kernels = profile_classes(ex, nd, od, stream, args)
    ex.close()
    # rooflines of the denoise loop itself (cached rows only: the set_prefix
    # copies are not loop work)
    rl, loop, shares = roofline_for(cfg, cfg.batch, {"kernels": kernels, "ms_per_step": ms_loop}, peaks, peak_kind,
                                    lens)
    return {"value": ws * cfg.batch / (ms * 1e-3), "unit": "chunks/s", "ms_per_step": ms,
            "ms_per_step_cached_only": ms_loop, "prefix_lengths": lens, "roofline": rl, "loop_roofline": loop,
            "kernel_shares": shares, "clocks": clocks,
            "kernels_ms_per_launch": {c: v["ms_per_launch"] for c, v in kernels.items()},
            "note": "each step: 8 fresh set_prefix calls (new observations) + 8 cached rows + pae_denoise; "
                    "rooflines are for the loop alone (ms_per_step_cached_only)"}


def measure_prefix_production(args, stream, barrier, maxr, peaks, gpu_index):
    """pae_set_prefix_hidden at the pi0.5 shape: 18 layers, a 968-token prefix
    whose hidden states are 2048 wide (a Gemma-2B-like prefix model), keys
    rotated (RoPE): per layer an RMSNorm and a [968 x 2048] x [2048 x 512]
    projection written straight into the K/V slot.  One step = one new
    observation of one request."""
    import torch
    import flow_matching_action_pi0_b200 as fm
    from workloads import device as wd
    Dp = 2048
    cfg = wl.PI05_BF16_BS1.replace(name="pi05_prefix_production", prefix_width=Dp, rope_base=10000.0)
    W = dict(wl.make_weights(cfg))
    g = np.random.default_rng(77)
    L, P = cfg.layers, cfg.prefix
    kvr = 2 * cfg.n_kv_heads * cfg.head_dim
    W["w_prefix_kv"] = [wl.round_bf16(g.standard_normal((kvr, Dp)) * 0.02) for _ in range(L)]
    dev_w = wd.upload_weights(cfg, W)
    ex = fm.ActionExpert(fm.make_config(**wd.abi_config(cfg, max_batch=1)), dev_w)
    del dev_w
    hs = [torch.randn(P, Dp, device="cuda").to(torch.bfloat16) for _ in range(L)]
    with torch.cuda.stream(stream):
        clk = ClockSampler(gpu_index).start()
        ms = maxr(timed(lambda: ex.set_prefix_hidden(0, hs, P, stream), args.steps, args.warmup, stream, barrier))
        clocks = clk.stop()
    ex.close()
    flops = 2.0 * L * P * Dp * kvr
    bytes_ = L * (kvr * Dp * 2 + P * Dp * 2 * 2 + P * kvr * 2)  # weights, hidden in + normalised out/in, K/V out
    return {"ms_per_observation": ms, "observations_per_s": 1e3 / ms, "prefix_tokens": P, "hidden_width": Dp,
            "layers": L, "algorithmic_flops": flops, "algorithmic_bytes": bytes_,
            "achieved_tflops": flops / (ms * 1e-3) / 1e12,
            "frac_tensor": flops / (ms * 1e-3) / 1e12 / peaks["bf16_tflops_sustained"],
            "achieved_gbs": bytes_ / (ms * 1e-3) / 1e9, "frac_hbm": bytes_ / (ms * 1e-3) / 1e9 / peaks["hbm_gbs"],
            "clocks": clocks,
            "note": "pae_set_prefix_hidden: per layer RMSNorm + K/V projection (keys rotated) into the slot"}


def measure_persistent(cfg, W, args, stream, barrier, maxr, ws):
    """The same batch-1 workload through the persistent kernel (one launch per
    call, grid barriers between phases) instead of the captured graph."""
    import torch
    import flow_matching_action_pi0_b200 as fm
    lens = wl.prefix_lengths(cfg)
    ex, *_ = setup_context(cfg, W, cfg.batch, lens)
    ex.set_option(fm.PAE_OPT_PERSISTENT, 1)
    nd = torch.from_numpy(wl.make_noise(cfg)).cuda()
    od = torch.empty_like(nd)
    with torch.cuda.stream(stream):
        ms = maxr(timed(lambda: ex.denoise(nd, od, stream), args.steps, args.warmup, stream, barrier))
    used = ex.query(fm.PAE_Q_PERSISTENT, cfg.batch)
    ex.close()
    return {"value": ws * cfg.batch / (ms * 1e-3), "unit": "chunks/s", "ms_per_step": ms, "persistent": used,
            "note": "one cooperative launch per call; slower than the captured graph on this workload"}


def run_ours(args, cfg):
    import torch
    ws, rank, local = dist_env()
    torch.cuda.set_device(local)
    if ws > 1:
        import datetime
        import torch.distributed as dist
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=180),
                                device_id=torch.device("cuda", local))
    barrier, maxr = rank_helpers(ws)
    import flow_matching_action_pi0_b200 as fm
    fm.lib()
    peaks, peak_kind = load_peaks()
    stream = torch.cuda.Stream()
    W = wl.make_weights(cfg)
    lens = wl.prefix_lengths(cfg)
    gpu_index = local
    res = measure(cfg, W, cfg.batch, args, stream, barrier, maxr, lens=lens, gpu_index=gpu_index)
    ms = res["ms_per_step"]
    value = ws * cfg.batch / (ms * 1e-3)
    rl, loop, shares = roofline_for(cfg, cfg.batch, res, peaks, peak_kind, lens)
    line = {
        "metric": METRIC, "value": value, "unit": "chunks/s", "n_gpus": ws, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": ms, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "bf16" if cfg.dtype == wl.BF16 else cfg.dtype,
        "data": "synthetic: seeded N(0,0.02) weights, N(0,1) prefix K/V and noise",
        "config": workload_config(cfg), "per_euler_step_us": ms * 1e3 / cfg.steps,
        "roofline": rl, "loop_roofline": loop, "kernel_shares": shares,
        "kernels_ms_per_launch": {c: v["ms_per_launch"] for c, v in res["kernels"].items()},
        "gpu_launches": int(res["graph_kernels"]) * args.steps,
        "kernels_per_call": int(res["graph_kernels"]),
        "loop": ("persistent kernel" if res["persistent"] else
                 f"dataflow loop (one launch, clusters of {res['dataflow']})" if res["dataflow"] else
                 "captured graph"),
        "splitk": {"qkv": res["splits"] & 255, "o": (res["splits"] >> 8) & 255,
                   "gate_up": (res["splits"] >> 16) & 255, "down": (res["splits"] >> 24) & 255},
        "token_tile": res["token_tile"], "table_build_ms": res["table_ms"],
        "clocks": res["clocks"],
        "e2e": {"value": ws * cfg.batch / (res["e2e_ms"] * 1e-3), "unit": "chunks/s",
                "h2d_bytes_per_step": res["io_bytes"], "d2h_bytes_per_step": res["io_bytes"],
                "ms_per_step": res["e2e_ms"], "api": "pae_denoise_host (pinned host buffers)"},
    }
    ex = res.pop("ex")
    ex.close()
    del res
    torch.cuda.empty_cache()
    if args.secondary and cfg.name == wl.PI05_BF16_BS1.name:
        c32 = wl.PI05_BF16_BS32
        r32 = measure(c32, W, c32.batch, args, stream, barrier, maxr, with_e2e=False, gpu_index=gpu_index)
        rl32, loop32, sh32 = roofline_for(c32, c32.batch, r32, peaks, peak_kind, r32["lens"])
        line["secondary"] = {c32.name: {
            "value": ws * c32.batch / (r32["ms_per_step"] * 1e-3), "unit": "chunks/s",
            "ms_per_step": r32["ms_per_step"], "roofline": rl32, "loop_roofline": loop32,
            "kernel_shares": sh32, "clocks": r32["clocks"],
            "kernels_ms_per_launch": {c: v["ms_per_launch"] for c, v in r32["kernels"].items()},
            "splitk": r32["splits"], "token_tile": r32["token_tile"],
            "note": "same weights as the batch-1 line; 32 independent 968-token prefixes"}}
        r32.pop("ex").close()
        del r32
    if args.secondary and cfg.name == wl.PI05_BF16_BS1.name:
        line.setdefault("secondary", {})[wl.RAGGED_BF16_BS16.name] = measure_ragged(args, stream, barrier, maxr,
                                                                                   ws, gpu_index)
    if args.secondary and cfg.name == wl.PI05_BF16_BS1.name:
        line.setdefault("secondary", {})["pi05_bf16_bs1_persistent_kernel"] = measure_persistent(
            cfg, W, args, stream, barrier, maxr, ws)
    if args.secondary and cfg.name == wl.PI05_BF16_BS1.name:
        line.setdefault("secondary", {})["pi05_prefix_production"] = measure_prefix_production(
            args, stream, barrier, maxr, peaks, gpu_index)
    if args.secondary and cfg.name == wl.PI05_BF16_BS1.name:
        c4 = wl.PI05_W4A16_BS1
        W4 = wl.make_weights(c4)
        r4 = measure(c4, W4, c4.batch, args, stream, barrier, maxr, with_e2e=False, gpu_index=gpu_index)
        rl4, loop4, sh4 = roofline_for(c4, c4.batch, r4, peaks, peak_kind, r4["lens"])
        line.setdefault("secondary", {})[c4.name] = {
            "value": ws * c4.batch / (r4["ms_per_step"] * 1e-3), "unit": "chunks/s",
            "ms_per_step": r4["ms_per_step"], "roofline": rl4, "loop_roofline": loop4, "kernel_shares": sh4,
            "clocks": r4["clocks"],
            "kernels_ms_per_launch": {c: v["ms_per_launch"] for c, v in r4["kernels"].items()},
            "note": "int4 weights (group 128, bf16 scales), bf16 activations"}
        r4.pop("ex").close()
        del r4, W4
    if args.cpu_baseline and ws == 1 and rank == 0:
        # a bounded sample: one request, all Euler steps, repeated to >= 10 s (at most 8 runs)
        ts = oracle_sample_times(cfg, W, *wl.make_prefix(cfg, lengths=lens[:1]), wl.make_noise(cfg, batch=1),
                                 cfg.steps, min_seconds=10.0, max_reps=8)
        t = sum(ts) / len(ts)
        line["cpu_baseline"] = {"value": 1.0 / t, "unit": "chunks/s", "cores": blas_threads(), "kind": "oracle",
                                "sample": f"one request of the workload, all {cfg.steps} Euler steps, "
                                          f"{len(ts)} runs ({sum(ts):.1f} s); requests are independent"}
    if rank == 0:
        print(json.dumps(line), flush=True)
    if ws > 1:
        import torch.distributed as dist
        dist.barrier()
        dist.destroy_process_group()
    return 0


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=50)
    ap.add_argument("--warmup", type=int, default=10)
    ap.add_argument("--config", default=wl.PI05_BF16_BS1.name, choices=sorted(wl.CONFIGS))
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--no-secondary", dest="secondary", action="store_false")
    ap.add_argument("--no-cpu-baseline", dest="cpu_baseline", action="store_false")
    ap.add_argument("--minimal", action="store_true", help="only warm-up and timed calls (for profilers)")
    ap.add_argument("--pdl", type=int, default=1, help="programmatic dependent launch inside the loop (1/0)")
    ap.add_argument("--max-splitk", type=int, default=0, help="cap on the projection split-K (0: library default)")
    ap.add_argument("--fused-norm", type=int, default=0,
                    help="adaRMSNorm inside the projections for batches of <= 64 tokens (1/0; 0 keeps norm kernels)")
    ap.add_argument("--dataflow", type=int, default=-1,
                    help="dataflow loop for batches of <= 64 tokens (1/0; -1 keeps the library default)")
    ap.add_argument("--factored-norm", dest="factored_norm", type=int, default=-1,
                    help="adaRMSNorm factored into the projections' epilogues (1/0; -1 keeps the library default)")
    ap.add_argument("--persistent", type=int, default=0,
                    help="persistent kernel for batches of <= 64 tokens (1/0; 0 runs the captured graph)")
    args = ap.parse_args()
    if args.warmup < 3:
        args.warmup = 3
    cfg = wl.CONFIGS[args.config]
    FUSED_NORM[0] = args.fused_norm
    DATAFLOW[0] = args.dataflow
    FACTORED[0] = args.factored_norm
    if args.impl == "reference":
        return run_reference(args, cfg)
    if args.minimal:
        return run_minimal(args, cfg)
    return run_ours(args, cfg)


if __name__ == "__main__":
    sys.exit(main())
