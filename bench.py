"""Benchmark of the routed MoE FFN layer on B200 (one JSON line on rank 0).

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME] [--impl ours|reference]

A step is one whole layer forward (router, top-k, dispatch, grouped SwiGLU GEMMs,
weighted combine with the gated shared expert) over one batch of T tokens, inputs
resident in HBM. By default the line's headline is the 2.4T-shaped prefill layer (T=8192,
hidden 8192, 512 experts top-10, inter 2048, shared 2048) in tokens/s; the Flash-Next-shaped
decode layer (T=64, reported in µs/layer), the Flash-Next-shaped prefill layer and the skewed
2.4T-shaped layer (T=16384) are measured in the same run and reported under "workloads",
each with its own clocks, roofline and error statistics. --workload NAME measures one
workload only. Under torchrun each rank runs its own replica on its own token batch (weak
scaling, no data-path collective); the time is the max over ranks of CUDA-event time.

Reported for each workload beside the device-timed value:
* e2e         -- the same metric through moe_layer_forward_host: pinned host x copied in,
                 layer, out copied back, every step inside the timed region;
* roofline    -- the dominant kernel's algorithmic bytes (or FLOPs) per launch / its mean
                 launch time (CUDA events on the launch stream), against the measured peak
                 in MEASURED_PEAKS.json;
* layer       -- the whole layer's TC % (FLOPs / (peak x time)), HBM % (bytes / (bandwidth
                 x time)) and roofline %, dense-equivalent and executed FLOPs separately;
* errors      -- max |gpu - oracle| / RMS and mean relative error of the timed output on
                 sampled tokens against the fp64 oracle, and the near-tie count;
* cpu_baseline-- the fp64 oracle on the host cores on a bounded token sample (headline,
                 rank 0, N=1);
* clocks      -- nvidia-smi SM clocks and throttle reasons sampled during the timed regions.

--impl reference times the oracle (the only other implementation of this layer) on the
headline workload on the host cores; under torchrun only rank 0 runs it.
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
sys.path.insert(0, ROOT)

METRIC = "MoE-layer tokens/s (prefill), µs/layer (decode); % of TC or HBM roofline"
PEAKS_FILE = os.path.join(ROOT, "MEASURED_PEAKS.json")
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}
KERNEL_SOURCES = {  # kernel id -> source file whose hash a stored ncu traffic figure carries
    "gate_up": ("stream_swiglu.cu", "tc_gemm.cu", "tc2_gemm.cu", "tc_common.cuh", "sm100_ptx.cuh"),
    "down": ("stream_swiglu.cu", "tc_gemm.cu", "tc2_gemm.cu", "tc_common.cuh", "sm100_ptx.cuh"),
    "gate_up_f16": ("tc_gemm.cu", "tc2_gemm.cu", "tc_common.cuh", "sm100_ptx.cuh"),
    "down_f16": ("tc2_gemm.cu", "tc_common.cuh", "sm100_ptx.cuh"),
    "router_logits": ("router.cu", "tc_gemm.cu", "tc_common.cuh", "sm100_ptx.cuh"),
    "router_topk": ("router.cu",),
    "permute": ("permute.cu",),
    "combine": ("combine.cu",),
    "gate_up_fp8": ("tc8_gemm.cu", "tc_common.cuh", "sm100_ptx.cuh"),
    "down_fp8": ("tc8_gemm.cu", "tc_common.cuh", "sm100_ptx.cuh"),
}
# oracle token sample per workload for the CPU baseline (about 10-30 s on a host)
CPU_SAMPLE = {"tiny": 64, "flash_decode": 16, "flash_prefill": 32, "flash_prefill_e64": 32,
              "t24_prefill_e16": 2, "t24_prefill": 2, "t24_skewed": 2}


def log(*a):
    print(*a, file=sys.stderr, flush=True)


def load_peaks():
    try:
        with open(PEAKS_FILE) as f:
            p = json.load(f)
        return p, "measured"
    except (OSError, ValueError):
        return dict(FALLBACK_PEAKS), "fallback"


# --------------------------------------------------------------------------- clocks

class ClockSampler:
    """nvidia-smi SM clock / throttle-reason sampler for one GPU (by UUID)."""

    FIELDS = ("timestamp,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, uuid: str, period_ms: int = 100):
        self.rows = []
        self.proc = None
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", uuid, f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                 "-lms", str(period_ms)], stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            self.thread = threading.Thread(target=self._read, daemon=True)
            self.thread.start()
        except OSError:
            self.proc = None

    def _read(self):
        for line in self.proc.stdout:
            parts = [p.strip() for p in line.split(",")]
            if len(parts) != 9:
                continue
            try:
                ts = time.mktime(time.strptime(parts[0].split(".")[0], "%Y/%m/%d %H:%M:%S"))
                ts += float("0." + parts[0].split(".")[1]) if "." in parts[0] else 0.0
                self.rows.append((ts, float(parts[1]), float(parts[2]), parts[5], parts[6], parts[7], parts[8]))
            except (ValueError, IndexError):
                continue

    def stop(self):
        if self.proc:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()

    def summary(self, windows):
        if not self.proc:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": [], "samples": 0,
                    "note": "nvidia-smi unavailable"}
        inside = [r for r in self.rows if any(a - 0.15 <= r[0] <= b + 0.15 for a, b in windows)]
        note = "samples inside the timed regions"
        if not inside:
            inside = self.rows[-5:]
            note = "timed regions shorter than the sampling period: last samples before stop"
        if not inside:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": [], "samples": 0, "note": "no samples"}
        names = ("hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap")
        reasons = sorted({names[i] for r in inside for i in range(4) if r[3 + i].lower() == "active"})
        return {"sm_mhz": statistics.median(r[1] for r in inside), "sm_max_mhz": max(r[2] for r in inside),
                "reasons": reasons, "samples": len(inside), "note": note}


# --------------------------------------------------------------------------- roofline

def algorithmic_bytes(kernel: str, cfg, n_active: int, fp8: bool = False, h_bytes: int = 4) -> float:
    """Bytes a launch of `kernel` must move at least (each operand once). fp8: the routed
    experts as E4M3 codes (1 byte per weight) plus one fp32 scale per weight row. h_bytes:
    bytes per element of the intermediate h (4: the bf16 pair hi + lo; 2: one fp16 value,
    with the fp16 down operands)."""
    T, H, I, Is, R = cfg.T, cfg.H, cfg.I, cfg.Is, cfg.R
    if fp8 and kernel == "gate_up":
        return n_active * 2 * I * (H + 4) + (2 * Is * H + T * H) * 2 + (R * I + T * Is) * h_bytes
    if fp8 and kernel == "down":
        return n_active * H * (I + 4) + H * Is * 2 + (R * I + T * Is) * h_bytes + T * H * 4
    if kernel == "gate_up":  # activated experts' gate|up + shared gate|up + x + h out
        return (n_active * 2 * I * H + 2 * Is * H + T * H) * 2 + (R * I + T * Is) * h_bytes
    if kernel == "down":  # activated experts' down + shared down + h in + out (fp32)
        return (n_active * H * I + H * Is) * 2 + (R * I + T * Is) * h_bytes + T * H * 4
    if kernel == "router_logits":
        return cfg.E * H * 4 + T * H * 2 + T * cfg.E * 4
    if kernel == "router_topk":
        return T * cfg.E * 4 + T * H * 2 + T * H * 4
    if kernel == "permute":
        return R * 4 * 4
    if kernel == "combine":
        return (R + T) * H * 4 + T * H * 4
    return 0.0


def kernel_flops(kernel: str, cfg) -> float:
    T, H, I, Is, R, E = cfg.T, cfg.H, cfg.I, cfg.Is, cfg.R, cfg.E
    if kernel == "gate_up":
        return 4.0 * (R * H * I + T * H * Is)
    if kernel == "down":
        return 2.0 * (R * H * I + T * H * Is)
    if kernel == "router_logits":
        return 2.0 * T * H * E
    return 0.0


def stored_traffic(kernel: str, workload: str):
    """Per-launch DRAM bytes from a committed ncu summary, if taken on the current source."""
    path = os.path.join(ROOT, "profiles", f"{kernel}_{workload}.md")
    if not os.path.exists(path):
        return None
    text = open(path).read()
    m = re.search(r"traffic_per_launch_bytes\s*=\s*([0-9.eE+]+)", text)
    h = re.search(r"source_sha256\s*=\s*([0-9a-f]{64})", text)
    if not m or not h or h.group(1) != source_hash(kernel):
        return None
    return float(m.group(1))


def source_hash(kernel: str) -> str:
    """Hash of the code (comments and whitespace removed) of the files a kernel is built from:
    a stored ncu traffic figure stays valid across comment edits, not across code changes."""
    hsh = hashlib.sha256()
    for f in KERNEL_SOURCES.get(kernel, ()):
        p = os.path.join(ROOT, "sparse_moe_expert_fp32_b200", "csrc", f)
        if os.path.exists(p):
            src = open(p, encoding="utf-8").read()
            src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
            src = re.sub(r"//[^\n]*", "", src)
            hsh.update(re.sub(r"\s+", "", src).encode())
    return hsh.hexdigest()


# --------------------------------------------------------------------------- CPU oracle

def oracle_sample(cfg, seed: int, ntok: int, fp8: bool = False):
    """Inputs for timing the oracle on `ntok` sampled tokens (weights made beforehand; with
    fp8, the routed experts quantised and dequantised as the FP8 layer uses them)."""
    import numpy as np

    import oracle
    import synth

    host = synth.host_inputs(cfg, seed=seed)
    rng = np.random.default_rng(99)
    rows = sorted(rng.choice(cfg.T, min(ntok, cfg.T), replace=False).tolist())
    x = host.x[rows]
    logits = oracle.router_logits(x, host.w_router, host.router_bias)
    ids, _ = oracle.topk_select(logits, cfg.k)
    src = oracle.Fp8Experts(host.gate_up, host.down) if fp8 else host
    gu = {int(e): src.gate_up(int(e)) for e in np.unique(ids)}
    dn = {int(e): src.down(int(e)) for e in np.unique(ids)}
    return host, x, gu, dn, rows


def time_oracle(cfg, host, x, gu, dn, with_result: bool = False):
    """Seconds the oracle takes for the layer on the token rows x (and its result)."""
    import oracle

    t0 = time.perf_counter()
    ref = oracle.moe_forward(x, host.w_router, host.router_bias, gu.__getitem__, dn.__getitem__,
                             host.ws_gate_up, host.ws_down, host.w_shared_gate, cfg.k)
    dt = time.perf_counter() - t0
    return (dt, ref) if with_result else dt


def blas_threads() -> int:
    try:
        from threadpoolctl import threadpool_info

        n = [i.get("num_threads", 1) for i in threadpool_info() if i.get("user_api") == "blas"]
        return max(n) if n else 1
    except Exception:  # noqa: BLE001
        return os.cpu_count() or 1


# --------------------------------------------------------------------------- arms

def dist_setup():
    import torch

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        import datetime

        import torch.distributed as dist

        torch.cuda.set_device(local)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=torch.device("cuda", local))
    elif torch.cuda.is_available():
        torch.cuda.set_device(0)
    return world, rank, local


def dist_barrier(world: int) -> None:
    """Barrier over the ranks of the job (no-op on one process)."""
    if world > 1:
        import torch.distributed as dist

        dist.barrier()


def dist_max(v: float, world: int, device) -> float:
    """The largest of every rank's `v` (each rank's device time: the job takes the slowest)."""
    if world == 1:
        return v
    import torch
    import torch.distributed as dist

    t = torch.tensor([v], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def job_value(tokens_per_rank_step: int, steps: int, world: int, ms: float) -> float:
    """Whole-job throughput in tokens/s: every rank's tokens over the slowest rank's time."""
    return tokens_per_rank_step * steps * world / (ms / 1e3)


def run_reference(args, cfg, world, rank):
    if rank != 0:
        return None
    ntok = CPU_SAMPLE.get(cfg.name, 8)
    fp8 = bool(getattr(args, "fp8", False))
    host, x, gu, dn, rows = oracle_sample(cfg, 0, ntok, fp8)
    for _ in range(args.warmup):
        time_oracle(cfg, host, x, gu, dn)
    total = 0.0
    for _ in range(args.steps):
        total += time_oracle(cfg, host, x, gu, dn)
    value = len(rows) * args.steps / total
    cores = blas_threads()
    sample = f"{len(rows)} of {cfg.T} tokens of the {cfg.name} layer per step, fp64 oracle on host cores"
    return {"metric": METRIC, "value": value, "unit": "tokens/s", "impl": "reference",
            "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": 1e3 * total / args.steps, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": config_block(cfg, "fp8" if fp8 else None, "fp64 oracle on the host cores"),
            "cpu_baseline": {"value": value, "unit": "tokens/s", "cores": cores, "kind": "oracle",
                             "sample": sample},
            "e2e": {"value": value, "unit": "tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}


def config_block(cfg, variant, timed_as="CUDA graph replay of one layer forward per step"):
    return {"workload": cfg.name, "description": cfg.description, "T": cfg.T, "H": cfg.H, "E": cfg.E,
            "k": cfg.k, "I": cfg.I, "Is": cfg.Is, "zipf_s": cfg.zipf_s, "zero_rows_pct": cfg.zero_rows_pct,
            "variant": variant, "accumulate": "fp32", "output": "fp32",
            "timed_as": timed_as,
            "l2": "inputs larger than L2 (expert weight bank exceeds the 126 MB L2)"
            if cfg.E * 3 * cfg.H * cfg.I * 2 > 126e6 else "L2-resident (tiny layer)",
            "parallelism": "replicas: one token batch per GPU, no collective"}


def layer_totals(cfg, n_active: int, I_exec=None) -> dict:
    """Algorithmic work of one layer forward: FLOPs of the expert GEMMs and the router
    (dense-equivalent: every routed row at width I; executed: at the width the GEMMs ran,
    I_exec after zero-channel compaction) and the bytes it must move at least (activated
    routed experts, shared expert, router matrix, x in, out as fp32)."""
    T, H, E, I, Is, R = cfg.T, cfg.H, cfg.E, cfg.I, cfg.Is, cfg.R
    Ix = I if I_exec is None else I_exec
    router = 2.0 * T * H * E
    dense = 6.0 * (R * H * I + T * H * Is) + router
    executed = 6.0 * (R * H * Ix + T * H * Is) + router
    nbytes = (n_active * 3 * H * Ix + 3 * H * Is) * 2 + E * H * 4 + T * H * 2 + T * H * 4
    return {"flops_dense_equivalent": dense, "flops_executed": executed, "bytes": float(nbytes)}


def layer_fractions(tot: dict, seconds: float, peaks: dict) -> dict:
    """TC % = F / (P t), HBM % = B / (BW t), roofline % = max(F / P, B / BW) / t."""
    P = peaks["bf16_tflops"] * 1e12
    Ps = peaks.get("bf16_tflops_sustained", peaks["bf16_tflops"]) * 1e12
    BW = peaks["hbm_gbs"] * 1e9
    F, B = tot["flops_executed"], tot["bytes"]
    return {"tc_pct": 100.0 * F / (P * seconds), "tc_pct_of_sustained": 100.0 * F / (Ps * seconds),
            "tc_pct_dense_equivalent": 100.0 * tot["flops_dense_equivalent"] / (P * seconds),
            "hbm_pct": 100.0 * B / (BW * seconds),
            "roofline_pct": 100.0 * max(F / P, B / BW) / seconds,
            "bound": "tensor" if F / P > B / BW else "hbm",
            "roofline_us": 1e6 * max(F / P, B / BW), **tot}


def error_stats(gpu_out, gpu_ids, ref: dict, k: int) -> dict:
    """Layer output against the fp64 oracle on the sampled tokens: max |d| / RMS(ref) and
    sum |d| / sum |ref|; tokens whose id sets differ (near-ties) are counted and left out."""
    import numpy as np

    keep, ties = [], 0
    for i in range(len(gpu_ids)):
        if set(int(v) for v in gpu_ids[i]) == set(int(v) for v in ref["ids"][i]):
            keep.append(i)
        else:
            ties += 1
    g = np.asarray(gpu_out, dtype=np.float64)[keep]
    r = np.asarray(ref["out"], dtype=np.float64)[keep]
    d = np.abs(g - r)
    rms = float(np.sqrt(np.mean(r * r))) if r.size else 0.0
    return {"tokens": len(gpu_ids), "max_abs_over_rms": float(d.max() / rms) if d.size else None,
            "mean_rel": float(d.sum() / np.abs(r).sum()) if d.size else None,
            "sample_id_sets_differ": ties,
            "sample_near_ties_fp64": int(sum(1 for g_ in ref["gap"] if g_ < 1e-5)),
            "tolerance": {"max_abs_over_rms": 1e-2, "mean_rel": 2e-3}}


def kernel_roofline(kernels: dict, cfg, n_active: int, peaks: dict, peak_kind: str, fp8: bool,
                    traffic_workload: str, h_bytes: int = 4) -> dict:
    """Roofline of the dominant kernel (largest total device time): algorithmic bytes (or
    FLOPs) per launch over its mean launch time, against the measured peak."""
    dom = max(kernels, key=lambda k: kernels[k]["ms_per_launch"] * kernels[k]["launches"])
    dom_bytes = algorithmic_bytes(dom, cfg, n_active, fp8, h_bytes)
    bound = "tensor" if kernel_flops(dom, cfg) / max(dom_bytes, 1) > 290 else "hbm"
    per_launch_s = kernels[dom]["ms_per_launch"] / 1e3
    if bound == "hbm":
        achieved = dom_bytes / per_launch_s / 1e9
        peak, unit = peaks["hbm_gbs"], "GB/s"
    else:
        achieved = kernel_flops(dom, cfg) / per_launch_s / 1e12
        peak, unit = peaks["bf16_tflops"], "TFLOP/s"
    return {"bound": bound, "kernel": dom, "achieved": achieved, "peak": peak, "unit": unit,
            "frac": achieved / peak,
            "peak_source": f"{peak_kind} ({'hbm_gbs' if bound == 'hbm' else 'bf16_tflops'})",
            "algorithmic_bytes_per_launch": dom_bytes,
            "algorithmic_flops_per_launch": kernel_flops(dom, cfg),
            "activated_experts": n_active,
            "timed_from": "mean of the kernel's launch durations (CUDA events on its stream) over "
                          "host-launched steps right after the graph-timed region",
            "traffic": stored_traffic(dom + ("_fp8" if fp8 else ("_f16" if h_bytes == 2 else "")),
                                      traffic_workload)}


def measure_workload(args, cfg, world, rank, local, sampler, want_cpu_baseline: bool) -> dict:
    """Everything the line reports for one workload: device-resident value, per-kernel
    times, roofline, layer fractions, end-to-end value, clocks, errors against the oracle."""
    import numpy as np
    import torch

    import sparse_moe_expert_fp32_b200 as moe
    import synth

    variant = {"auto": moe.MOE_VARIANT_AUTO, "stream": moe.MOE_VARIANT_STREAM,
               "tc": moe.MOE_VARIANT_TC, "tc2": moe.MOE_VARIANT_TC2}[args.variant]
    full_cfg = cfg
    dev = synth.device_inputs(cfg, seed=0, x_seed=rank, device=f"cuda:{local}")
    compact = None
    if args.compact:
        # weight pre-pass (once, at load time): drop zero gate/up channels and their down
        # columns; the layer then runs with I = I_c
        t0 = time.time()
        dev, I_c = moe.compact_zero_channels(moe.shape_of(cfg), dev)
        torch.cuda.synchronize()
        compact = {"I": cfg.I, "I_c": I_c, "prepass_s": round(time.time() - t0, 3)}
        cfg = cfg.replace(I=I_c)
        torch.cuda.empty_cache()
    s = moe.shape_of(cfg)
    fp8 = None
    if args.fp8:
        # weight pre-pass (once, at load time): routed experts to E4M3 codes + fp32 row
        # scales; the bf16 routed banks are then freed (the FP8 layer does not read them)
        t0 = time.time()
        q = moe.quantize_fp8_experts(s, dev)
        torch.cuda.synchronize()
        fp8 = {"expert_weights": "E4M3 codes, one fp32 scale per weight row (amax/448)",
               "shared_expert_and_router": "bf16 / fp32", "prepass_s": round(time.time() - t0, 3)}
        dev["w_gate_up"] = None
        dev["w_down"] = None
        torch.cuda.empty_cache()
        qs = moe.make_fp8_experts(q)
    down_f16 = None
    if fp8 is None and not args.down_bf16_pair and args.variant != "stream":
        # weight pre-pass (once, at load time): the down matrices re-encoded as fp16(W * 2^8)
        # so that the down GEMM takes h as one fp16 value (one MMA per K step). Not with the
        # FP8 experts: their down GEMM takes h as four E4M3 pieces (16 bits)
        t0 = time.time()
        dev = moe.prepare_down_f16(s, dev)
        torch.cuda.synchronize()
        down_f16 = {"prepass_s": round(time.time() - t0, 3),
                    "weights": "W_down re-encoded once as fp16(W * 2^8): exact for 2^-25 <= |w| < 256",
                    "h": "fp16(h * 2^-8): 11 significant bits for |h| >= 2^-6 (the bf16 pair hi + lo "
                         "carries 16); fp32 accumulation"}
    ws = moe.alloc_workspace(s, host_staging=True, variant=variant)
    out = torch.empty((cfg.T, cfg.H), dtype=torch.float32, device="cuda")
    ids = torch.empty((cfg.T, cfg.k), dtype=torch.int32, device="cuda")
    gap = torch.empty((cfg.T,), dtype=torch.float32, device="cuda")
    stream = torch.cuda.current_stream()
    w = moe.make_weights(dev)

    if args.staged:
        # the four stage entry points, y materialised in fp32 and combined by its own kernel
        R = cfg.T * cfg.k
        st_ids = torch.empty((cfg.T, cfg.k), dtype=torch.int32, device="cuda")
        st_w = torch.empty((cfg.T, cfg.k), dtype=torch.float32, device="cuda")
        st_sg = torch.empty((cfg.T,), dtype=torch.float32, device="cuda")
        st_gap = torch.empty((cfg.T,), dtype=torch.float32, device="cuda")
        st_off = torch.empty((cfg.E + 1,), dtype=torch.int32, device="cuda")
        st_tok = torch.empty((R,), dtype=torch.int32, device="cuda")
        st_ar = torch.empty((R,), dtype=torch.int32, device="cuda")
        st_y = torch.empty((R, cfg.H), dtype=torch.float32, device="cuda")
        st_ys = torch.empty((cfg.T, cfg.H), dtype=torch.float32, device="cuda")

    def layer(x_dev, out_dev, topk_ids=None, gap_out=None):
        if fp8 is not None:
            moe.moe_layer_forward_fp8(s, x_dev, w, qs, out_dev, ws, topk_ids=topk_ids, gap=gap_out)
        elif args.staged:
            moe.moe_router_topk(s, x_dev, w, st_ids, st_w, st_sg, st_gap, ws)
            moe.moe_permute(s, st_ids, st_off, st_tok, st_ar, ws)
            moe.moe_grouped_swiglu(s, x_dev, st_tok, st_off, w, st_y, st_ys, ws)
            moe.moe_unpermute_combine(s, st_y, st_ys, st_ar, st_w, st_sg, out_dev)
            if topk_ids is not None:
                topk_ids.copy_(st_ids)
            if gap_out is not None:
                gap_out.copy_(st_gap)
        else:
            moe.moe_layer_forward(s, x_dev, w, out_dev, ws, topk_ids=topk_ids, gap=gap_out)

    x_in = torch.empty_like(dev["x"])
    out_in = torch.empty_like(out)

    def layer_host(x_host, out_host):
        if fp8 is not None or args.staged:  # the copies the host-buffer entry point makes
            x_in.copy_(x_host, non_blocking=True)
            layer(x_in, out_in)
            out_host.copy_(out_in, non_blocking=True)
        else:
            moe.moe_layer_forward_host(s, x_host, w, out_host, ws)

    layer(dev["x"], out, topk_ids=ids, gap_out=gap)
    st, flags = moe.moe_device_status(ws)
    if st != moe.MOE_OK:
        raise RuntimeError(f"{cfg.name}: device status {st} ({flags})")
    ids_np = ids.cpu().numpy()
    n_active = int(np.unique(ids_np).size)
    counts = np.bincount(ids_np.ravel(), minlength=cfg.E)
    near_ties_gpu = int((gap.cpu().numpy() < 1e-5).sum())
    for _ in range(args.warmup):
        layer(dev["x"], out)
    torch.cuda.synchronize()

    # ---- device-resident timed region: one layer forward per step, replayed from a CUDA
    # graph (as a served layer would run; --no-graph launches every kernel from the host)
    graph = None
    moe.moe_profile_enable(True)  # fill the library's event pool before any capture
    layer(dev["x"], out)
    torch.cuda.synchronize()
    moe.moe_profile_collect()
    per_step = None
    if not args.no_graph:
        graph = torch.cuda.CUDAGraph()
        n_cap = moe.moe_launch_count()
        with torch.cuda.graph(graph, capture_error_mode="thread_local"):
            layer(dev["x"], out)
        per_step = moe.moe_launch_count() - n_cap
        stream = torch.cuda.current_stream()
        for _ in range(2):
            graph.replay()
        torch.cuda.synchronize()
    dist_barrier(world)
    torch.cuda.synchronize()
    n0 = moe.moe_launch_count()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    windows = []
    w0 = time.time()
    e0.record(stream)
    for _ in range(args.steps):
        if graph is not None:
            graph.replay()
        else:
            layer(dev["x"], out)
    e1.record(stream)
    torch.cuda.synchronize()
    windows.append((w0, time.time()))
    launches = per_step * args.steps if graph is not None else moe.moe_launch_count() - n0
    if graph is not None:
        # per-kernel device times: host-launched steps right after the graph-timed ones
        # (the same kernels on the same data; events inside a graph cannot be timed)
        moe.moe_profile_collect()
        for _ in range(min(args.steps, 50)):
            layer(dev["x"], out)
        torch.cuda.synchronize()
    moe.moe_profile_enable(False)
    prof = moe.moe_profile_collect()
    dist_barrier(world)
    ms = dist_max(e0.elapsed_time(e1), world, "cuda")
    st, flags = moe.moe_device_status(ws)
    if st != moe.MOE_OK:
        raise RuntimeError(f"{cfg.name}: device status after the timed region {st} ({flags})")
    out_np = out.cpu().numpy()  # the last timed step's output (same inputs every step)

    # ---- end to end through the host-buffer entry point
    x_host = dev["x"].cpu().pin_memory()
    out_host = torch.empty((cfg.T, cfg.H), dtype=torch.float32).pin_memory()
    for _ in range(max(1, min(args.warmup, 3))):
        layer_host(x_host, out_host)
    torch.cuda.synchronize()
    dist_barrier(world)
    w0 = time.time()
    e0.record(stream)
    for _ in range(args.steps):
        layer_host(x_host, out_host)
    e1.record(stream)
    torch.cuda.synchronize()
    windows.append((w0, time.time()))
    dist_barrier(world)
    ms_e2e = dist_max(e0.elapsed_time(e1), world, "cuda")
    st, flags = moe.moe_device_status(ws)
    if st != moe.MOE_OK:
        raise RuntimeError(f"{cfg.name}: device status after timing {st} ({flags})")
    del graph, ws, dev, w, out, out_in, x_in
    if args.staged:
        del st_y, st_ys
    torch.cuda.empty_cache()
    if rank != 0:
        return None

    peaks, peak_kind = load_peaks()
    kernels = {k: {"ms_per_launch": v[0] / v[1], "launches": v[1], "share": None}
               for k, v in prof.items() if v[1] > 0}
    tot = sum(v[0] for v in prof.values()) or 1.0
    for k, v in prof.items():
        if v[1] > 0:
            kernels[k]["share"] = v[0] / tot
    is8 = fp8 is not None
    seconds = ms / args.steps / 1e3
    totals = layer_totals(full_cfg, n_active, I_exec=cfg.I)
    if is8:  # routed experts at one byte per weight plus a 4-byte scale per row
        totals["bytes"] = (n_active * (3 * cfg.H * cfg.I + 4 * (2 * cfg.I + cfg.H)) + 3 * cfg.H * cfg.Is * 2
                           + cfg.E * cfg.H * 4 + cfg.T * cfg.H * 6)
    res = {"workload": cfg.name, "value": job_value(cfg.T, args.steps, world, ms), "unit": "tokens/s",
           "ms_per_step": ms / args.steps, "us_per_layer": 1e3 * ms / args.steps,
           "steps": args.steps,
           "config": config_block(full_cfg, "fp8" if args.fp8 else
                                  (args.variant + "+staged" if args.staged else args.variant),
                                  "host launches of one layer forward per step" if args.no_graph
                                  else "CUDA graph replay of one layer forward per step"),
           "zero_channel_compaction": compact, "fp8_experts": fp8, "down_operands_fp16": down_f16,
           "roofline": kernel_roofline(kernels, cfg, n_active, peaks, peak_kind, is8, cfg.name,
                                       h_bytes=2 if down_f16 else 4),
           "layer": {**layer_fractions(totals, seconds, peaks), "peaks": f"{peak_kind} (MEASURED_PEAKS.json)"
                     if peak_kind == "measured" else "fallback"},
           "graph": not args.no_graph,
           "e2e": {"value": job_value(cfg.T, args.steps, world, ms_e2e), "unit": "tokens/s",
                   "h2d_bytes_per_step": cfg.T * cfg.H * 2, "d2h_bytes_per_step": cfg.T * cfg.H * 4},
           "gpu_launches": launches, "kernels": kernels,
           "expert_load": {"active": n_active, "max_rows": int(counts.max()),
                           "mean_rows_active": float(counts[counts > 0].mean()),
                           "min_rows_active": int(counts[counts > 0].min())},
           "near_ties": {"tokens_gap_below_1e-5": near_ties_gpu,
                         "note": "10th/11th logit gap of the kernel's own routing, all tokens"},
           "clocks": sampler.summary(windows) if sampler else None}
    # errors against the fp64 oracle on sampled tokens of the timed inputs (rank 0's batch);
    # the oracle's time on the same sample is the CPU baseline
    if not args.no_oracle and rank == 0:
        ntok = ERROR_SAMPLE.get(full_cfg.name, 8)
        host, x, gu, dn, rows = oracle_sample(full_cfg, 0, ntok, is8)
        dt, ref = time_oracle(full_cfg, host, x, gu, dn, with_result=True)
        res["errors"] = error_stats(out_np[rows], ids_np[rows], ref, cfg.k)
        if want_cpu_baseline:
            res["cpu_baseline"] = {
                "value": len(rows) / dt, "unit": "tokens/s", "cores": blas_threads(), "kind": "oracle",
                "sample": f"{len(rows)} of {full_cfg.T} tokens of the {full_cfg.name} layer (seed 0), full "
                          f"layer per token in fp64; expert weights made{' (FP8, dequantised)' if is8 else ''}"
                          " before timing", "seconds": dt}
    return res


HEADLINE = "t24_prefill"
# "+fp8": the same workload with the routed experts in FP8 (as --fp8)
SUITE = ("t24_prefill", "flash_decode", "flash_prefill", "t24_skewed", "flash_decode+fp8")
# tokens the oracle evaluates per workload for the error statistics (and the CPU baseline)
ERROR_SAMPLE = {"tiny": 64, "flash_decode": 16, "flash_prefill": 16, "flash_prefill_e64": 16,
                "flash_decode_e64": 16, "t24_prefill_e16": 4, "t24_prefill": 4, "t24_skewed": 4}


def main():
    import synth

    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--workload", default=None, choices=sorted(synth.CONFIGS),
                    help="one workload only (default: the 2.4T-shaped prefill layer as the "
                         "headline, with the decode, Flash-Next prefill and skewed layers beside it)")
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--variant", default="auto", choices=["auto", "stream", "tc", "tc2"])
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-oracle", action="store_true",
                    help="skip the oracle error statistics and the CPU baseline")
    ap.add_argument("--no-graph", action="store_true", help="launch every kernel from the host")
    ap.add_argument("--staged", action="store_true",
                    help="time the four stage entry points (y in fp32, separate combine) "
                         "instead of the fused layer forward")
    ap.add_argument("--fp8", action="store_true",
                    help="routed experts in FP8 (E4M3 + fp32 row scales, quantised before timing)")
    ap.add_argument("--compact", action="store_true",
                    help="zero-channel compaction of the routed experts before timing (weight pre-pass)")
    ap.add_argument("--down-bf16-pair", action="store_true",
                    help="keep the down GEMM on the bf16 weights with h as the bf16 pair hi + lo "
                         "(default: the fp16 down-operand pre-pass runs before timing)")
    args = ap.parse_args()
    args.warmup = max(args.warmup, 3)
    if args.staged and (args.fp8 or args.compact):
        ap.error("--staged times the bf16 stage entry points on the full bank: "
                 "it does not combine with --fp8 or --compact")
    if args.no_oracle:
        args.no_cpu_baseline = True
    names = [args.workload] if args.workload else list(SUITE)
    if args.workload is None and (args.fp8 or args.compact or args.staged):
        names = [n for n in names if "+" not in n]

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    if args.impl == "reference":
        line = run_reference(args, synth.CONFIGS[names[0].split("+")[0]], world, rank)
        if line is not None:
            print(json.dumps(line), flush=True)
        return

    import torch

    world, rank, local = dist_setup()
    sampler = None
    if rank == 0:
        props = torch.cuda.get_device_properties(local)
        uuid = str(getattr(props, "uuid", ""))
        sampler = ClockSampler(uuid if uuid.startswith("GPU-") else f"GPU-{uuid}")
        time.sleep(1.5)  # nvidia-smi start-up
    results = []
    try:
        for i, name in enumerate(names):
            base, _, extra = name.partition("+")
            wargs = argparse.Namespace(**vars(args))
            if extra == "fp8":
                wargs.fp8 = True
            r = measure_workload(wargs, synth.CONFIGS[base], world, rank, local, sampler,
                                 want_cpu_baseline=(i == 0 and world == 1
                                                    and not args.no_cpu_baseline))
            if extra:
                r["workload"] = name
            results.append(r)
    finally:
        if sampler:
            sampler.stop()
        if world > 1:
            import torch.distributed as dist

            dist.destroy_process_group()
    if rank != 0:
        return
    head = results[0]
    line = {"metric": METRIC, "value": head["value"], "unit": "tokens/s", "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": head["ms_per_step"],
            "us_per_layer": head["us_per_layer"], "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None,
            "dtype": ("e4m3 (routed gate|up and down MMAs: x as 2, h as 4 E4M3 pieces), bf16 (shared "
                      "expert), fp32 accumulation and output" if args.fp8 else
                      "bf16 (router split, gate|up MMAs)" + (", bf16 (down MMAs)" if head.get(
                          "down_operands_fp16") is None else ", fp16 (down MMAs)")
                      + ", fp32 accumulation and output"),
            "data": "synthetic (seeded counter-based generator: x~N(0,1), weights~N(0,0.02), random "
                    "router; the skewed layer adds a Zipf(1.1) router bias and 71% zero gate/up channels)"}
    for key in ("config", "roofline", "layer", "e2e", "gpu_launches", "kernels", "clocks", "errors",
                "near_ties", "expert_load", "cpu_baseline", "zero_channel_compaction", "fp8_experts",
                "down_operands_fp16", "graph"):
        if key in head:
            line[key] = head[key]
    if len(results) > 1:
        line["gpu_launches"] = sum(r["gpu_launches"] for r in results)
        line["gpu_launches_note"] = "all workloads' timed regions (the headline's alone: " \
                                    f"{head['gpu_launches']})"
        line["workloads"] = {r["workload"]: {k: v for k, v in r.items() if k not in ("workload",)}
                             for r in results[1:]}
    print(json.dumps(line), flush=True)


if __name__ == "__main__":
    main()
