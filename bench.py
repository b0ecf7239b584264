#!/usr/bin/env python3
"""Benchmark of the hybrid W4A4 + outlier linear layer on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
                    [--workload NAME] [--no-cpu-baseline]

One step = one layer call (quik_linear), one pass of the hot path over one
batch: quantise + reorder the activations, then the INT4 x INT4 GEMM with the
outlier sub-product and the dequantising epilogue; the weights are packed
once before timing (offline).  The default workload is the
Llama-7B attention projection (M=2048 tokens, N=K=4096, 128 FP16 outliers).

Timing: W untimed warm-up steps, then exactly K steps; before every step a
256 MiB buffer is written (flushing the 126 MB L2, outside the step's
events); each step is bracketed by CUDA events on the launching stream
(quantise and GEMM separately); the K steps are bracketed by a barrier and
torch.cuda.synchronize() on both sides; the reported time is the max over
ranks.  With N > 1 every rank runs an independent replica on its own GPU
(weak scaling; the layer has no exchange step), and `value` is the ops of all
ranks divided by the slowest rank's time.

Prints ONE JSON line (rank 0).
"""
from __future__ import annotations

import argparse
import datetime
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

METRIC = "W4A4+outlier linear TOPS & µs/call at Llama shapes; % of dense INT8 peak"
UNIT = "TOPS"
FLUSH_BYTES = 256 << 20
PROFILE_DIR = os.path.join(ROOT, "profiles")
GEMM_SOURCES = [os.path.join(ROOT, "mixed_precision_quantized_quantize_b200", "csrc", f)
                for f in ("gemm.cu", "gemm_persistent.cu", "sm100.cuh")]
# nominal dense-rate ratio INT8 : BF16 on B200 (4.5 : 2.25 PFLOP/s)
INT8_PER_BF16 = 2.0
FALLBACK_BF16_TFLOPS = 1590.0
FALLBACK_HBM_GBS = 6650.0


def parse():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=200)
    ap.add_argument("--warmup", type=int, default=10)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", default=None)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    return ap.parse_args()


def dist_env():
    return (int(os.environ.get("RANK", "0")), int(os.environ.get("LOCAL_RANK", "0")),
            int(os.environ.get("WORLD_SIZE", "1")))


# ----------------------------------------------------------------- peaks and profiles
def measured_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            d = json.load(f)
        return d, "measured"
    except (OSError, ValueError):
        return {"bf16_tflops": FALLBACK_BF16_TFLOPS, "hbm_gbs": FALLBACK_HBM_GBS}, "fallback"


def gemm_source_hash() -> str:
    h = hashlib.sha256()
    for p in GEMM_SOURCES:
        with open(p, "rb") as f:
            h.update(f.read())
    return h.hexdigest()[:16]


def gemm_kernel(cfg):
    """The GEMM kernel the library dispatches for this layer, and its profile file."""
    fits = cfg.k_o <= (256 if cfg.outlier_int8 else 128)
    if cfg.sparse24 and cfg.M <= 32:
        return ("w4a4_gemv24 (2:4-sparse INT4 weights as the sparse MMA operand, tcgen05.mma.sp "
                "kind::i8; 128 W rows x 32 tokens per CTA)", f"w4a4_gemv24_{cfg.name}.md")
    persistent = ("w4a4_gemm_persistent (persistent warp-specialised CTA pairs, 256 weight rows "
                  "x 256 tokens per tile, double-buffered TMEM accumulators; INT4 codes widened "
                  "to INT8, tcgen05 kind::i8; FP16 outliers as kind::f16 MMAs onto the "
                  "dequantised tile)")
    persistent2 = ("w4a4_gemm_persistent2 (the persistent kernel with 256 weight rows x 512 tokens per "
                   "tile: each widened weight k-block feeds two 256-token halves, two TMEM "
                   "accumulators, all-warps epilogue per tile; tcgen05 kind::i8, FP16 outliers as "
                   "kind::f16 MMAs onto the dequantised tile)")

    def tiles512(packed):
        # the library's rule for 512-token tiles: one wave of them where
        # 256-token tiles need two or more, with at most as many FP16
        # outlier units as operand stages (three with packed activations,
        # four with the layer call's widened ones)
        n_wt = -(-cfg.N // 256)
        tiles1, tiles2 = -(-cfg.M // 256) * n_wt, -(-cfg.M // 512) * n_wt
        return -(-cfg.k_o // 64) <= (3 if packed else 4) and tiles2 <= 74 and tiles1 > 74

    if cfg.sparse24:
        # the timed GEMM is quik_gemm on packed codes and the expanded weights
        two = tiles512(True)
        return ((persistent2 if two else persistent) + " on the 2:4 weights expanded to dense codes "
                "(more than 32 tokens; the expansion is timed separately)",
                f"w4a4_gemm_persistent{'2' if two else ''}_{cfg.name}.md")
    if cfg.act_bits == 8:
        return (("w4a4_gemm_pair with INT8 activations and weights (W8A8)" if cfg.weight_bits == 8 else
                 "w4a4_gemm_pair with INT8 activations (W4A8; weights widened from INT4)")
                + ", tcgen05 kind::i8 on CTA pairs", f"w4a4_gemm_{cfg.name}.md")
    if cfg.group == 0 and cfg.M <= 32 and fits:
        return ("w4a4_gemv (decode shapes: W rows as the MMA's M, tokens as N; INT4 codes "
                "widened to INT8, tcgen05 kind::i8)", f"w4a4_gemv_{cfg.name}.md")
    if cfg.group == 0 and (cfg.k_o == 0 or not cfg.outlier_int8):
        # the norm-fused workload's GEMM is timed through quik_gemm on packed
        # codes; the others' inside the layer call, on widened codes
        if tiles512(cfg.rmsnorm):
            return persistent2, f"w4a4_gemm_persistent2_{cfg.name}.md"
        return persistent, f"w4a4_gemm_persistent_{cfg.name}.md"
    if cfg.group == 0:
        return ("w4a4_gemm_pair (INT4 codes widened to INT8, tcgen05 kind::i8 on CTA pairs)",
                f"w4a4_gemm_{cfg.name}.md")
    return ("w4a4_gemm (grouped scales; INT4 codes widened to INT8, tcgen05 kind::i8)",
            f"w4a4_gemm_grouped_{cfg.name}.md")


def profiled_traffic(profile_file):
    """dram bytes per launch from the committed ncu summary, if it matches this kernel."""
    try:
        with open(os.path.join(PROFILE_DIR, profile_file)) as f:
            text = f.read()
    except OSError:
        return None
    vals = {}
    for line in text.splitlines():
        if line.startswith("traffic_bytes_per_launch:"):
            vals["t"] = line.split(":", 1)[1].strip()
        if line.startswith("gemm_source_sha256_16:"):
            vals["h"] = line.split(":", 1)[1].strip()
    if vals.get("h") != gemm_source_hash() or "t" not in vals:
        return None
    try:
        return float(vals["t"])
    except ValueError:
        return None


def library_context(cfg, X, W, flush, steps: int = 20):
    """Same-shape library GEMMs for context (never this library's arithmetic): the fp16
    product the method replaces (torch.matmul -> cuBLAS) and cuBLASLt INT8
    (torch._int_mm, where its shape rules allow), each with the L2 flushed."""
    import torch

    def timed(fn):
        for _ in range(3):
            flush.zero_()
            fn()
        ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
              for _ in range(steps)]
        for a, b in ev:
            flush.zero_()
            a.record()
            fn()
            b.record()
        torch.cuda.synchronize()
        return float(np.median([a.elapsed_time(b) for a, b in ev])) * 1e3

    Wt = W.t()
    out = {"fp16_matmul_us": round(timed(lambda: torch.matmul(X, Wt)), 2)}
    try:
        g = torch.Generator(device=X.device).manual_seed(5)
        Xi = torch.randint(-7, 8, (cfg.M, cfg.K), dtype=torch.int8, device=X.device, generator=g)
        Wi = torch.randint(-7, 8, (cfg.K, cfg.N), dtype=torch.int8, device=X.device, generator=g)
        out["int8_int_mm_us"] = round(timed(lambda: torch._int_mm(Xi, Wi)), 2)
    except (RuntimeError, TypeError):
        out["int8_int_mm_us"] = None
    return out


# ----------------------------------------------------------------- clocks (NVML, read only)
class ClockSampler:
    """Samples SM clock, power and throttle reasons every ~5 ms in a thread."""

    REASONS = {
        "gpu_idle": 0x1, "applications_clocks_setting": 0x2, "sw_power_cap": 0x4,
        "hw_slowdown": 0x8, "sync_boost": 0x10, "sw_thermal_slowdown": 0x20,
        "hw_thermal_slowdown": 0x40, "hw_power_brake_slowdown": 0x80,
        "display_clock_setting": 0x100,
    }

    def __init__(self, index: int):
        self.samples, self.reasons = [], 0
        self.max_mhz = None
        self._stop = threading.Event()
        self._ok = False
        try:
            import pynvml
            pynvml.nvmlInit()
            self.nv = pynvml
            self.h = pynvml.nvmlDeviceGetHandleByIndex(index)
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self.h, pynvml.NVML_CLOCK_SM)
            self._ok = True
        except Exception:  # noqa: BLE001 - clocks are reported as unavailable
            self._ok = False

    def _run(self):
        while not self._stop.is_set():
            try:
                self.samples.append(self.nv.nvmlDeviceGetClockInfo(self.h, self.nv.NVML_CLOCK_SM))
                self.reasons |= self.nv.nvmlDeviceGetCurrentClocksEventReasons(self.h)
            except Exception:  # noqa: BLE001
                pass
            time.sleep(0.005)

    def __enter__(self):
        if self._ok:
            self.t = threading.Thread(target=self._run, daemon=True)
            self.t.start()
        return self

    def __exit__(self, *exc):
        if self._ok:
            self._stop.set()
            self.t.join()

    def summary(self):
        if not self._ok:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvml unavailable"]}
        names = [n for n, b in self.REASONS.items() if self.reasons & b]
        return {"sm_mhz": statistics.median(self.samples) if self.samples else None,
                "sm_max_mhz": self.max_mhz, "reasons": names, "samples": len(self.samples)}


# ----------------------------------------------------------------- CPU oracle legs
def cpu_oracle_step(cfg, d, rows: int):
    """One bounded CPU pass of the layer: quantise `rows` token rows (with the
    RMS norm folded in, for a norm-fused workload), then their full output rows
    (every column) from the pre-packed weights."""
    import oracle
    X = d["X"][:rows].numpy()
    if cfg.rmsnorm:
        xq = oracle.rmsnorm_quantize_rows(X, d["gamma"].numpy(), d["eps"], d["perm_np"], cfg.k_o,
                                          cfg.group, cfg.outlier_int8, cfg.act_bits)
    else:
        xq = oracle.quantize_rows(X, d["perm_np"], cfg.k_o, cfg.group, cfg.outlier_int8,
                                  cfg.act_bits)
    wq = d["w_oracle"]
    oracle.linear(xq[0], xq[1], xq[2] if cfg.k_o else None, xq[3], wq[0], wq[1],
                  wq[2] if cfg.k_o else None, wq[3], d["bias_np"], cfg.K, cfg.k_o, cfg.group)


def prepare_cpu_inputs(cfg, d):
    import oracle
    d["perm_np"] = d["perm"].numpy()
    d["bias_np"] = None if d["bias"] is None else d["bias"].numpy()
    if cfg.sparse24:  # the 2:4 weights, expanded to dense codes for the oracle's product
        Qs, meta, sw, Wo, swo = oracle.prune24_quantize_rows(d["W"].numpy(), d["perm_np"], cfg.k_o,
                                                             cfg.outlier_int8)
        d["w_oracle"] = (oracle.unpack24(Qs, meta), sw, Wo, swo)
    else:
        d["w_oracle"] = oracle.quantize_rows(d["W"].numpy(), d["perm_np"], cfg.k_o, cfg.group,
                                             cfg.outlier_int8, cfg.weight_bits)


def cpu_baseline(cfg, d, budget_s: float = 10.0):
    """Time the oracle, as it stands, on a bounded sample of the workload."""
    import oracle
    prepare_cpu_inputs(cfg, d)
    threads = oracle.num_threads()
    rows = max(1, min(cfg.M, threads))
    while True:
        t0 = time.perf_counter()
        cpu_oracle_step(cfg, d, rows)
        dt = time.perf_counter() - t0
        if dt >= budget_s or rows >= cfg.M:
            break
        rows = min(cfg.M, max(rows + 1, int(rows * min(8.0, 1.2 * budget_s / max(dt, 1e-3)))))
    ops = 2.0 * rows * cfg.N * cfg.K
    return {"value": ops / dt / 1e12, "unit": UNIT, "cores": threads, "kind": "oracle",
            "sample": f"{rows} of {cfg.M} token rows x all {cfg.N} columns "
                      f"(quantise + fp64 layer output), {dt:.1f} s"}


# ----------------------------------------------------------------- path roofline
def path_roofline(cfg, peaks: dict, t_step_s: float) -> dict:
    """The layer call's floor, serial: the quantiser's bytes at HBM speed,
    then the GEMM's slower of its tensor work and its bytes.  The INT4 part
    runs at the INT8 rate (twice that on the 2:4 sparse kernel), an FP16
    outlier block at the FP16 rate (the bf16 figure), an INT8 one at the INT8
    rate."""
    bw = float(peaks["hbm_gbs"]) * 1e9
    p_f16 = float(peaks["bf16_tflops"]) * 1e12
    p_i8 = p_f16 * INT8_PER_BF16
    p_int4 = p_i8 * (2.0 if cfg.sparse24 and cfg.M <= 32 else 1.0)
    p_out = p_i8 if cfg.outlier_int8 else p_f16
    t_tensor = 2.0 * cfg.M * cfg.N * cfg.K_i / p_int4 + 2.0 * cfg.M * cfg.N * cfg.k_o / p_out
    t_gemm = max(t_tensor, cfg.gemm_bytes / bw)
    t_quant = cfg.quant_bytes / bw
    t_roof = t_gemm + t_quant
    return {"t_roof_us": round(t_roof * 1e6, 4), "t_us": round(t_step_s * 1e6, 2),
            "frac": round(t_roof / t_step_s, 4) if t_step_s > 0 else None,
            "gemm_roof_us": round(t_gemm * 1e6, 4), "quantise_roof_us": round(t_quant * 1e6, 4),
            "gemm_bound": "tensor" if t_tensor >= cfg.gemm_bytes / bw else "hbm"}


# ----------------------------------------------------------------- aggregation
def aggregate(step_times_s, ops_per_rank: float, world: int, reduce_max):
    """Whole-job throughput from this rank's per-step times (weak scaling:
    every rank does ops_per_rank per step)."""
    local = float(sum(step_times_s))
    total = reduce_max(local)
    steps = len(step_times_s)
    value = world * ops_per_rank * steps / total / 1e12
    return value, total / steps


# ----------------------------------------------------------------- our arm
def run_ours(args, rank, local_rank, world):
    import torch
    import torch.distributed as dist

    import mixed_precision_quantized_quantize_b200 as q
    from mixed_precision_quantized_quantize_b200 import workloads as wl

    torch.cuda.set_device(local_rank)
    dev = torch.device("cuda", local_rank)
    if world > 1:
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=dev)

    def reduce_max(x):
        if world == 1:
            return x
        t = torch.tensor([x], dtype=torch.float64, device=dev)
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
        return float(t.item())

    def barrier():
        if world > 1:
            dist.barrier(device_ids=[local_rank])

    name = args.workload or wl.BENCH_CONFIG
    cfg = wl.CONFIGS[name]
    d = wl.make_layer(cfg)
    X = d["X"].to(dev)
    perm = d["perm"].to(dev)
    bias = d["bias"].to(dev) if d["bias"] is not None else None
    gamma = d["gamma"].to(dev) if cfg.rmsnorm else None
    eps = d.get("eps", 0.0)
    if cfg.sparse24:
        layer = q.QuikLinear24(d["W"].to(dev), perm, cfg.k_o, cfg.outlier_int8, bias)
    else:
        layer = q.QuikLinear(d["W"].to(dev), perm, cfg.k_o, cfg.group, cfg.outlier_int8, bias,
                             act_bits=cfg.act_bits, weight_bits=cfg.weight_bits, norm_weight=gamma,
                             norm_eps=eps)
    shape = layer.shape(cfg.M)
    Xq, sx, Xo, sxo = q._binding._quant_outputs(cfg.M, cfg.K, cfg.k_o, cfg.group,
                                                cfg.outlier_int8, dev, cfg.act_bits)
    Y = torch.empty((cfg.M, cfg.N), dtype=torch.float16, device=dev)
    flush = torch.empty(FLUSH_BYTES, dtype=torch.uint8, device=dev)
    stream = torch.cuda.current_stream(dev)

    ws_bytes = q.quik_workspace_size_24(shape) if cfg.sparse24 else q.quik_workspace_size(shape)
    ws = torch.empty((ws_bytes,), dtype=torch.uint8, device=dev)
    # the 2:4 prefill path: the dense copy of the weights its layer call makes
    prefill24 = cfg.sparse24 and cfg.M > 32
    Wd = (torch.empty((cfg.N, cfg.K_i // 2), dtype=torch.uint8, device=dev)
          if prefill24 else None)

    def step():
        # one layer call: quantise + reorder (behind the RMS norm, for a
        # norm-fused workload), then the GEMM (which may start while the
        # quantiser finishes: programmatic dependent launch)
        if cfg.sparse24:
            q.quik_linear_24(shape, X, perm, layer.Wq24, layer.Wmeta, layer.w_scale, layer.Wo,
                             layer.wo_scale, bias, Y, ws, stream=stream)
        elif cfg.rmsnorm:
            q.quik_rmsnorm_linear(shape, X, gamma, eps, perm, layer.Wq, layer.w_scale, layer.Wo,
                                  layer.wo_scale, bias, Y, ws, stream=stream)
        else:
            q.quik_linear(shape, X, perm, layer.Wq, layer.w_scale, layer.Wo, layer.wo_scale, bias,
                          Y, ws, stream=stream)

    def split_step(ev):
        # the same two kernels through the two public calls, with an event
        # between them: the per-kernel breakdown
        ev[0].record(stream)
        if cfg.rmsnorm:
            q.quik_rmsnorm_quantize_reorder(shape, X, gamma, eps, perm, Xq, sx, Xo, sxo,
                                            stream=stream)
        else:
            q.quik_quantize_reorder(shape, X, perm, Xq, sx, Xo, sxo, stream=stream)
        ev[1].record(stream)
        if prefill24:
            q.quik_expand_weights_24(shape, layer.Wq24, layer.Wmeta, Wd, stream=stream)
            ev[3].record(stream)
            q.quik_gemm(shape, Xq, sx, Xo, sxo, Wd, layer.w_scale, layer.Wo, layer.wo_scale, bias,
                        Y, stream=stream)
        elif cfg.sparse24:
            q.quik_gemm_24(shape, Xq, sx, Xo, sxo, layer.Wq24, layer.Wmeta, layer.w_scale, layer.Wo,
                           layer.wo_scale, bias, Y, stream=stream)
        else:
            q.quik_gemm(shape, Xq, sx, Xo, sxo, layer.Wq, layer.w_scale, layer.Wo, layer.wo_scale,
                        bias, Y, stream=stream)
        ev[2].record(stream)

    # the layer call with an event between its two kernels (quik_linear_timed:
    # the GEMM then waits for the quantiser instead of overlapping its tail)
    timed_layer = not cfg.sparse24 and not cfg.rmsnorm

    def marked_step(ev):
        ev[0].record(stream)
        q.quik_linear_timed(shape, X, perm, layer.Wq, layer.w_scale, layer.Wo, layer.wo_scale,
                            bias, Y, ws, ev[1], stream=stream)
        ev[2].record(stream)

    for _ in range(max(3, args.warmup)):
        flush.zero_()
        step()
    torch.cuda.synchronize()
    assert q.quik_sync_check(stream) == q.QUIK_OK

    events = [[torch.cuda.Event(enable_timing=True) for _ in range(2)] for _ in range(args.steps)]
    sampler = ClockSampler(local_rank)
    barrier()
    torch.cuda.synchronize()
    with sampler:
        for i in range(args.steps):
            flush.zero_()
            events[i][0].record(stream)
            step()
            events[i][1].record(stream)
        torch.cuda.synchronize()
    barrier()
    status = q.quik_sync_check(stream)
    if status != q.QUIK_OK:
        raise RuntimeError(f"device error after timed region: {q.status_string(status)}")
    step_s = [e[0].elapsed_time(e[1]) / 1e3 for e in events]
    value, t_step = aggregate(step_s, cfg.ops, world, reduce_max)
    t_step_median = reduce_max(float(np.median(step_s)))
    # per-kernel breakdown (separate, untimed-for-value pass)
    n_split = max(10, args.steps // 4)
    sev = [[torch.cuda.Event(enable_timing=True) for _ in range(4)] for _ in range(n_split)]
    for _ in range(3):  # warm-up: the first launches of the split path's kernels
        split_step([torch.cuda.Event(enable_timing=True) for _ in range(4)])
    torch.cuda.synchronize()
    for i in range(n_split):
        flush.zero_()
        split_step(sev[i])
    torch.cuda.synchronize()
    g0 = 3 if prefill24 else 1  # the GEMM starts after the expansion on the 2:4 prefill path
    # per-kernel breakdown: medians over the split steps
    gemm_avg = reduce_max(float(np.median([e[g0].elapsed_time(e[2]) / 1e3 for e in sev])))
    expand_avg = (reduce_max(float(np.median([e[1].elapsed_time(e[3]) / 1e3 for e in sev])))
                  if prefill24 else None)
    quant_avg = reduce_max(float(np.median([e[0].elapsed_time(e[1]) / 1e3 for e in sev])))
    split_avg = reduce_max(float(np.median([e[0].elapsed_time(e[2]) / 1e3 for e in sev])))
    layer_quant = layer_gemm = None
    if timed_layer:
        mev = [[torch.cuda.Event(enable_timing=True) for _ in range(3)] for _ in range(n_split)]
        for _ in range(3):
            marked_step([torch.cuda.Event(enable_timing=True) for _ in range(3)])
        torch.cuda.synchronize()
        for i in range(n_split):
            flush.zero_()
            marked_step(mev[i])
        torch.cuda.synchronize()
        layer_quant = reduce_max(float(np.median([e[0].elapsed_time(e[1]) / 1e3 for e in mev])))
        layer_gemm = reduce_max(float(np.median([e[1].elapsed_time(e[2]) / 1e3 for e in mev])))
    # the dominant kernel: the layer call's own GEMM where it can be timed
    # apart, else quik_gemm's
    dom_avg = layer_gemm if layer_gemm is not None else gemm_avg

    # ---- end to end through the public call with host buffers (pinned)
    Xh = d["X"].pin_memory()
    Yh = torch.empty((cfg.M, cfg.N), dtype=torch.float16).pin_memory()
    Xd = torch.empty_like(X)
    e2e_steps = max(10, args.steps // 4)

    def e2e_step():
        Xd.copy_(Xh, non_blocking=True)
        layer(Xd, out=Y, stream=stream)
        Yh.copy_(Y, non_blocking=True)

    for _ in range(3):
        e2e_step()
    torch.cuda.synchronize()
    ev = [[torch.cuda.Event(enable_timing=True) for _ in range(2)] for _ in range(e2e_steps)]
    barrier()
    torch.cuda.synchronize()
    for i in range(e2e_steps):
        flush.zero_()
        ev[i][0].record(stream)
        e2e_step()
        ev[i][1].record(stream)
    torch.cuda.synchronize()
    barrier()
    e2e_value, _ = aggregate([a.elapsed_time(b) / 1e3 for a, b in ev], cfg.ops, world, reduce_max)

    # ---- the same step with a warm L2 (no flush between steps)
    wev = [[torch.cuda.Event(enable_timing=True) for _ in range(2)] for _ in range(20)]
    torch.cuda.synchronize()
    for i in range(20):
        wev[i][0].record(stream)
        step()
        wev[i][1].record(stream)
    torch.cuda.synchronize()
    warm_us = float(np.median([a.elapsed_time(b) for a, b in wev])) * 1e3
    context = library_context(cfg, X, d["W"].to(dev), flush)
    context["warm_l2_us_per_call"] = round(warm_us, 2)
    if cfg.rmsnorm:
        # the unfused pipeline: torch's RMS norm writes the normalised fp16
        # rows, then the plain layer call quantises them
        def unfused():
            Xn = torch.nn.functional.rms_norm(X, (cfg.K,), gamma, eps)
            q.quik_linear(shape, Xn, perm, layer.Wq, layer.w_scale, layer.Wo, layer.wo_scale,
                          bias, Y, ws, stream=stream)

        uev = [[torch.cuda.Event(enable_timing=True) for _ in range(2)] for _ in range(20)]
        for _ in range(3):
            flush.zero_()
            unfused()
        for i in range(20):
            flush.zero_()
            uev[i][0].record(stream)
            unfused()
            uev[i][1].record(stream)
        torch.cuda.synchronize()
        context["unfused_torch_rms_norm_then_layer_us"] = round(
            float(np.median([a.elapsed_time(b) for a, b in uev])) * 1e3, 2)
    context["layer_speedup_vs_fp16_matmul"] = round(context["fp16_matmul_us"] / (t_step * 1e6), 3)

    peaks, peak_kind = measured_peaks()
    int8_peak = float(peaks["bf16_tflops"]) * INT8_PER_BF16
    # the 2:4-sparse MMA does half the multiply-adds of the INT4 part: its
    # dense-equivalent peak is twice the dense one (ops stay 2 M N K)
    sparse_x = 2.0 if cfg.sparse24 and not prefill24 else 1.0
    tensor_peak = int8_peak * sparse_x
    gemm_tops = cfg.ops / dom_avg / 1e12
    kernel_name, profile_file = gemm_kernel(cfg)
    hbm_peak = float(peaks["hbm_gbs"])
    timed_as = ("the layer call's GEMM launch: quik_linear_timed, CUDA events around it on the "
                "launching stream, L2 flushed before each call" if timed_layer else
                "quik_gemm, CUDA events around it on the launching stream, L2 flushed before each "
                "call")
    # the path's bound: the slower of the tensor work and the bytes it must move
    if cfg.gemm_bytes / (hbm_peak * 1e9) > cfg.ops / (tensor_peak * 1e12):
        roofline = {
            "bound": "hbm", "kernel": kernel_name, "timed_as": timed_as,
            "achieved": round(cfg.gemm_bytes / dom_avg / 1e9, 1), "peak": hbm_peak,
            "unit": "GB/s", "frac": round(cfg.gemm_bytes / dom_avg / 1e9 / hbm_peak, 4),
            "traffic": profiled_traffic(profile_file),
            "algorithmic_bytes_per_launch": cfg.gemm_bytes,
            "peak_source": f"{peak_kind} HBM copy bandwidth",
        }
    else:
        roofline = {
            "bound": "tensor", "kernel": kernel_name, "timed_as": timed_as,
            "achieved": round(gemm_tops, 2), "peak": round(tensor_peak, 1), "unit": "TFLOP/s",
            "frac": round(gemm_tops / tensor_peak, 4),
            "traffic": profiled_traffic(profile_file),
            "algorithmic_bytes_per_launch": cfg.gemm_bytes,
            "peak_source": (f"{peak_kind} bf16 burst {peaks['bf16_tflops']} TFLOP/s x "
                            f"{INT8_PER_BF16} (nominal INT8:BF16 dense ratio)"
                            + (" x 2 (2:4-sparse MMA, dense-equivalent)" if sparse_x > 1 else "")
                            + "; integer ops counted 2 per multiply-add"),
        }
    line = {
        "metric": METRIC,
        "value": round(value, 2),
        "unit": UNIT,
        "n_gpus": world,
        "steps": args.steps,
        "warmup": max(3, args.warmup),
        "ms_per_step": round(t_step * 1e3, 5),
        "ms_per_step_median": round(t_step_median * 1e3, 5),
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": ("int4" if cfg.act_bits == 4 else
                  "int8" if cfg.weight_bits == 8 else "int4 weights x int8 activations"),
        "data": "synthetic",
        "config": {
            "workload": name, "M": cfg.M, "N": cfg.N, "K": cfg.K, "k_o": cfg.k_o,
            "group_size": cfg.group, "outliers": "int8" if cfg.outlier_int8 else "fp16",
            "bias": cfg.bias, "parallelism": f"replicas x{world}" if world > 1 else "single GPU",
            "l2": "flushed before every step (256 MiB write, outside the step's events)",
            "step": ("quik_linear_24: quantise + reorder, then the 2:4-sparse GEMM" if cfg.sparse24
                     else "quik_rmsnorm_linear: RMS norm folded into quantise + reorder, then the GEMM"
                     if cfg.rmsnorm else "quik_linear: quantise + reorder, then the GEMM")
                    + " (weights packed once, offline)",
        },
        "us_per_call": round(t_step * 1e6, 2),
        "pct_int8_peak": round(100.0 * value / world / int8_peak, 2),
        "breakdown_us": {**({"layer_quantize_reorder": round(layer_quant * 1e6, 2),
                            "layer_gemm": round(layer_gemm * 1e6, 2)} if timed_layer else {}),
                         "quik_quantize_reorder": round(quant_avg * 1e6, 2),
                         "quik_gemm": round(gemm_avg * 1e6, 2),
                         "two_calls_with_event_between": round(split_avg * 1e6, 2),
                         **({"expand_weights_24": round(expand_avg * 1e6, 2)} if prefill24 else {})},
        "roofline": roofline,
        "path_roofline": path_roofline(cfg, peaks, t_step),
        "e2e": {"value": round(e2e_value, 2), "unit": UNIT,
                "h2d_bytes_per_step": X.numel() * 2, "d2h_bytes_per_step": Y.numel() * 2,
                "call": ("quik_linear_24" if cfg.sparse24 else "quik_rmsnorm_linear" if cfg.rmsnorm
                         else "quik_linear")
                        + " via QuikLinear, pinned host X in, host Y out"},
        "gpu_launches": (3 if prefill24 else 2) * args.steps,
        "clocks": sampler.summary(),
        "context": context,
    }
    if world > 1:
        dist.barrier(device_ids=[local_rank])
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        line["cpu_baseline"] = cpu_baseline(cfg, d)
    if world > 1:
        dist.destroy_process_group()
    if rank == 0:
        print(json.dumps(line), flush=True)


# ----------------------------------------------------------------- reference arm (the oracle)
def run_reference(args, rank, world):
    if rank != 0:
        return
    import oracle
    from mixed_precision_quantized_quantize_b200 import workloads as wl
    name = args.workload or wl.BENCH_CONFIG
    cfg = wl.CONFIGS[name]
    d = wl.make_layer(cfg)
    prepare_cpu_inputs(cfg, d)
    threads = oracle.num_threads()
    rows = max(1, min(cfg.M, threads))  # one token row per OpenMP thread per step
    for _ in range(max(3, args.warmup)):
        cpu_oracle_step(cfg, d, rows)
    times = []
    for _ in range(args.steps):
        t0 = time.perf_counter()
        cpu_oracle_step(cfg, d, rows)
        times.append(time.perf_counter() - t0)
    ops = 2.0 * rows * cfg.N * cfg.K
    t = float(np.mean(times))
    value = ops / t / 1e12
    sample = (f"each step: {rows} of {cfg.M} token rows x all {cfg.N} columns "
              f"(quantise + fp64 layer output)")
    print(json.dumps({
        "impl": "reference", "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world,
        "steps": args.steps, "warmup": max(3, args.warmup), "ms_per_step": t * 1e3,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "int4",
        "data": "synthetic",
        "config": {"workload": name, "M": cfg.M, "N": cfg.N, "K": cfg.K, "k_o": cfg.k_o,
                   "group_size": cfg.group, "outliers": "int8" if cfg.outlier_int8 else "fp16",
                   "parallelism": "host cores (OpenMP over rows)"},
        "cpu_baseline": {"value": value, "unit": UNIT, "cores": threads, "kind": "oracle",
                         "sample": sample},
        "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }), flush=True)


def main():
    args = parse()
    rank, local_rank, world = dist_env()
    if args.impl == "reference":
        run_reference(args, rank, world)
    else:
        run_ours(args, rank, local_rank, world)


if __name__ == "__main__":
    main()
