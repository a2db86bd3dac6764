#!/usr/bin/env python
"""Benchmark of the fine-grained MoE layer forward on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME] [--impl ours|reference]

One step = one pass of the whole hot path over one batch held in HBM:
gate GEMM + sigmoid + bias-shifted top-k + weights + load histogram
(moe_route), expert-contiguous permutation (moe_permute), the routed and
shared grouped SwiGLU GEMMs (moe_ffn_up / moe_ffn_down: one launch each for
both expert sets), the weighted
combine (moe_combine) and the bias update at the end of the step
(moe_load_and_bias_update; with N > 1 the counts are first summed over the
ranks with an NCCL all-reduce -- the one exchange the method has).  Each rank
processes its own T tokens (weak scaling, token-sharded data parallel with
replicated weights).

Timing: W warm-up steps, then K steps bracketed by a barrier and a device
synchronize, measured with CUDA events on the launching stream; the slowest
rank's time is reported.  CUDA events between the stages give each kernel's
duration inside the timed region (roofline of the dominant kernel).  The
layer weights (22.6 GB for the DeepSeek-V3 shape) are far larger than the
126 MB L2, so no flush is needed between steps.

The e2e leg runs the same steps through moe_layer_forward (or
moe_layer_forward_fp8) with each step's tokens copied from pinned host memory
and its output copied back, double-buffered on two copy streams so that the
copies of one step overlap the compute of the next.

Rank 0 prints one JSON line.  With the default workload (v3_prefill) the
line also carries, under "workloads", the decode-shaped workload (T=64 per
call, 1000 calls with fresh tokens each) and the skewed-routing workload
(T=32768, Zipf(1.2) popularity, 200 steps with the bias updated every step,
reporting the most-loaded expert's rows over the mean per step), each timed
the same way with its own roofline (HBM for decode, tensor for skew).

--backward times moe_layer_backward instead (one GPU, its own JSON line): the
gradients of x, the gate and every expert weight plus the sequence-wise
balance loss for a routing computed once before timing.
"""
from __future__ import annotations

import argparse
import datetime
import hashlib
import json
import os
import statistics
import subprocess
import sys
import tempfile
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

METRIC = "MoE layer fwd tokens/s (V3-shaped, bf16) and % of BF16 tensor / HBM roofline"
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}
STAGES = ["route", "permute", "ffn_up", "ffn_down", "combine", "bias_update"]
# E4M3 expert workloads: the token rows are quantized (1x32 tiles) in the step, h in the gate/up epilogue
STAGES_FP8 = ["route", "quant_x", "permute", "ffn_up", "ffn_down", "combine", "bias_update"]
DOMINANT = "ffn_up"
WORKLOADS = ["v3_prefill", "v3_decode", "small_bf16", "skew_stress", "tiny_fp32", "v3_prefill_fp8",
             "v3_decode_fp8", "small_fp8"]


def parse_args():
    ap = argparse.ArgumentParser(description=__doc__.split("\n\n")[0])
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=200)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--workload", default="v3_prefill", choices=WORKLOADS)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--cpu-tokens", type=int, default=0, help="oracle sample size (0: per-workload default)")
    ap.add_argument("--T", type=int, default=0, help="override tokens per GPU (profiling slices)")
    ap.add_argument("--E", type=int, default=0, help="override routed experts (profiling slices)")
    ap.add_argument("--I", type=int, default=0,
                    help="override the expert width I = Is (profiling slices: the router at full size in little memory)")
    ap.add_argument("--no-extra", action="store_true",
                    help="v3_prefill only: skip the decode and skew workloads of the default line")
    ap.add_argument("--decode-calls", type=int, default=1000, help="decode workload: timed calls (fresh x each)")
    ap.add_argument("--skew-steps", type=int, default=200, help="skew workload: timed steps")
    ap.add_argument("--backward", action="store_true",
                    help="time moe_layer_backward (one GPU) instead of the forward step; prints its own line")
    return ap.parse_args()


def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            d = json.load(f)
        return d, "measured"
    except (OSError, ValueError):
        return dict(FALLBACK_PEAKS), "fallback"


# --------------------------------------------------------------- clocks

class ClockSampler:
    """SM clock, power and throttle reasons sampled while the timed region
    runs: NVML polled from a thread every 5 ms (nvidia-smi at 50 ms if NVML
    is unavailable)."""
    REASONS = ("hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap")
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_id: str, period_s: float = 0.005):
        self.gpu_id = gpu_id
        self.period = period_s
        self.samples = []
        self.proc = None
        self.thread = None
        self.nvml = None

    def start(self):
        import threading
        try:
            import pynvml
            pynvml.nvmlInit()
            uuid_or_idx = self.gpu_id
            h = (pynvml.nvmlDeviceGetHandleByUUID(uuid_or_idx) if not uuid_or_idx.isdigit()
                 else pynvml.nvmlDeviceGetHandleByIndex(int(uuid_or_idx)))
            self.nvml = (pynvml, h)
        except Exception:
            self.nvml = None
        if self.nvml is not None:
            self.stop_evt = threading.Event()
            self.thread = threading.Thread(target=self._poll, daemon=True)
            self.thread.start()
            return
        fd, self.path = tempfile.mkstemp(prefix="clocks_", suffix=".csv")
        os.close(fd)
        try:
            self.out = open(self.path, "w")
            self.proc = subprocess.Popen(["nvidia-smi", "-i", self.gpu_id, f"--query-gpu={self.FIELDS}",
                                          "--format=csv,noheader,nounits", "-lms", "50"], stdout=self.out,
                                         stderr=subprocess.DEVNULL)
        except OSError:
            self.proc = None

    def _poll(self):
        pynvml, h = self.nvml
        bits = {"hw_slowdown": pynvml.nvmlClocksEventReasonHwSlowdown,
                "hw_thermal_slowdown": pynvml.nvmlClocksEventReasonHwThermalSlowdown,
                "sw_thermal_slowdown": pynvml.nvmlClocksEventReasonSwThermalSlowdown,
                "sw_power_cap": pynvml.nvmlClocksEventReasonSwPowerCap}
        smax = pynvml.nvmlDeviceGetMaxClockInfo(h, pynvml.NVML_CLOCK_SM)
        while not self.stop_evt.is_set():
            try:
                sm = pynvml.nvmlDeviceGetClockInfo(h, pynvml.NVML_CLOCK_SM)
                pw = pynvml.nvmlDeviceGetPowerUsage(h) / 1000.0
                rs = pynvml.nvmlDeviceGetCurrentClocksEventReasons(h)
                self.samples.append((float(sm), float(smax), pw, [n for n, b in bits.items() if rs & b]))
            except Exception:
                pass
            self.stop_evt.wait(self.period)

    def stop(self):
        if self.thread is not None:
            self.stop_evt.set()
            self.thread.join(timeout=5)
            rows = self.samples
            src = "nvml 5 ms"
        elif self.proc is not None:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()
            self.out.close()
            rows = []
            with open(self.path) as f:
                for line in f:
                    parts = [p.strip() for p in line.split(",")]
                    if len(parts) < 9:
                        continue
                    try:
                        rows.append((float(parts[1]), float(parts[2]), float(parts[3]),
                                     [n for n, v in zip(self.REASONS, parts[5:9]) if v.lower() == "active"]))
                    except ValueError:
                        continue
            os.unlink(self.path)
            src = "nvidia-smi 50 ms"
        else:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["no clock source"], "samples": 0}
        sm = [r[0] for r in rows]
        reasons = sorted({n for r in rows for n in r[3]})
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": max(r[1] for r in rows) if rows else None,
                "reasons": reasons, "samples": len(rows), "source": src,
                "power_w_median": statistics.median(r[2] for r in rows) if rows else None}


# ------------------------------------------------------------ oracle leg

DEFAULT_CPU_TOKENS = {"v3_prefill": 12, "v3_decode": 12, "skew_stress": 12, "small_bf16": 48, "tiny_fp32": 128,
                      "v3_prefill_fp8": 12, "v3_decode_fp8": 12, "small_fp8": 48}


def oracle_sample(cfg, p, x, n_tok):
    """Times the CPU oracle on the first n_tok tokens of x: routing
    (affinities + top-k + weights), then every routed expert those tokens
    use and the shared experts.  Expert weights are copied to the host
    before the clock starts; only oracle arithmetic is timed.
    Returns (seconds, tokens, threads)."""
    import numpy as np
    import oracle
    from fine_grained_moe_gate_b200.inputs import to_numpy

    oracle.build()
    xs = to_numpy(x[:n_tok])
    wg = to_numpy(p["w_gate"])
    bias = p["bias"].detach().cpu().numpy()
    t0 = time.perf_counter()
    s = oracle.affinity(xs, wg)
    idx, w = oracle.select(s, bias, cfg.k)
    secs = time.perf_counter() - t0
    yacc = np.zeros((n_tok, cfg.d), np.float64)
    for sidx in range(cfg.S):
        a, b, c = to_numpy(p["ws1"][sidx]), to_numpy(p["ws3"][sidx]), to_numpy(p["ws2"][sidx])
        t0 = time.perf_counter()
        oracle.expert_accumulate(xs, np.arange(n_tok, dtype=np.int32), np.ones(n_tok), a, b, c, yacc)
        secs += time.perf_counter() - t0
    for e in np.unique(idx):
        ii, jj = np.nonzero(idx == e)
        a, b, c = to_numpy(p["w1"][e]), to_numpy(p["w3"][e]), to_numpy(p["w2"][e])
        t0 = time.perf_counter()
        oracle.expert_accumulate(xs[ii], ii.astype(np.int32), w[ii, jj].astype(np.float64), a, b, c, yacc)
        secs += time.perf_counter() - t0
    t0 = time.perf_counter()
    oracle.finalize(yacc, xs.dtype)
    secs += time.perf_counter() - t0
    threads = int(os.environ.get("OMP_NUM_THREADS", "0")) or len(os.sched_getaffinity(0))
    return secs, n_tok, threads


def oracle_sample_fp8(cfg, p, x, n_tok):
    """oracle_sample for the E4M3 expert workloads: routing, per-tile
    quantization of x, and for every expert the tokens use (and the shared
    experts) the FP8 gate/up, per-tile quantization of h and the FP8 down.
    The expert weights are quantized by the oracle itself, expert by expert,
    before the clock starts; only the forward's oracle arithmetic is timed."""
    import numpy as np
    import oracle
    from fine_grained_moe_gate_b200.inputs import to_numpy

    oracle.build()
    xs = to_numpy(x[:n_tok])
    wg = to_numpy(p["w_gate"])
    bias = p["bias"].detach().cpu().numpy()
    d, I, S, Is = cfg.d, cfg.I, cfg.S, cfg.Is
    t0 = time.perf_counter()
    s = oracle.affinity(xs, wg)
    idx, w = oracle.select(s, bias, cfg.k)
    xq, xe = oracle.quantize_mx(xs)
    secs = time.perf_counter() - t0
    yacc = np.zeros((n_tok, d), np.float64)
    if S > 0:
        q1, e1 = oracle.quantize_mx(to_numpy(p["ws1"]).reshape(S * Is, d))
        q3, e3 = oracle.quantize_mx(to_numpy(p["ws3"]).reshape(S * Is, d))
        q2, e2 = oracle.quantize_mx(to_numpy(p["ws2"]), nseg=S)
        t0 = time.perf_counter()
        hq, he = oracle.quantize_mx(oracle.expert_up_mx(xq, xe, q1, e1, q3, e3))
        yacc += oracle.expert_down_mx(hq, he, q2, e2)
        secs += time.perf_counter() - t0
    for e in np.unique(idx):
        ii, jj = np.nonzero(idx == e)
        q1, e1 = oracle.quantize_mx(to_numpy(p["w1"][e]))
        q3, e3 = oracle.quantize_mx(to_numpy(p["w3"][e]))
        q2, e2 = oracle.quantize_mx(to_numpy(p["w2"][e]))
        t0 = time.perf_counter()
        hq, he = oracle.quantize_mx(oracle.expert_up_mx(xq[ii], xe[ii], q1, e1, q3, e3))
        yacc[ii] += w[ii, jj].astype(np.float64)[:, None] * oracle.expert_down_mx(hq, he, q2, e2)
        secs += time.perf_counter() - t0
    t0 = time.perf_counter()
    oracle.finalize(yacc, xs.dtype)
    secs += time.perf_counter() - t0
    threads = int(os.environ.get("OMP_NUM_THREADS", "0")) or len(os.sched_getaffinity(0))
    return secs, n_tok, threads


def run_oracle_sample(cfg, p, x, n_tok):
    return (oracle_sample_fp8 if cfg.dtype == "fp8" else oracle_sample)(cfg, p, x, n_tok)


def cpu_baseline_record(cfg, secs, n_tok, threads, label):
    return {"value": n_tok / secs, "unit": "tokens/s", "cores": threads, "kind": "oracle",
            "sample": (f"{label}: {n_tok} of {cfg.T} tokens of the {cfg.name} batch through the whole layer "
                       f"(routing over all {cfg.E} experts, every routed expert those tokens use, "
                       f"{cfg.S} shared); {secs:.2f} s of oracle arithmetic, scaled to tokens/s; "
                       f"OpenMP over tokens/rows, up to {threads} threads")}


# ------------------------------------------------------------ our leg

def traffic_record(kernel_file: str, workload_name: str):
    """Per-launch DRAM bytes of the dominant kernel on this workload from the
    committed ncu summary, if the kernel source is unchanged since it was
    captured."""
    path = os.path.join(ROOT, "profiles", "traffic.json")
    try:
        with open(path) as f:
            rec = json.load(f)
        with open(kernel_file, "rb") as f:
            digest = hashlib.sha256(f.read()).hexdigest()[:16]
        ent = rec.get(workload_name, {}).get(DOMINANT)
        if ent and ent.get("source_sha256_16") == digest:
            return ent.get("dram_bytes_per_launch")
    except (OSError, ValueError):
        pass
    return None


def workload(args):
    from fine_grained_moe_gate_b200.inputs import CONFIGS
    cfg = CONFIGS[args.workload]
    over = {}
    if args.T:
        over["T"] = args.T
    if args.E:
        over["E"] = args.E
    if args.I:
        over["I"] = over["Is"] = args.I
    if over:
        tag = ",".join(f"{k}={v}" for k, v in over.items())
        cfg = cfg.scaled(name=f"{cfg.name}[{tag}]", **over)
    return cfg


class LayerStep:
    """Device buffers and the step of one workload on one rank: route,
    (quantize x,) permute, gate/up, (quantize h,) down, combine, counts
    all-reduce when N > 1, bias update.  ``xs`` are the step inputs, cycled."""

    def __init__(self, cfg, dev, world, p, xs, stream):
        import torch
        import fine_grained_moe_gate_b200 as moe
        from fine_grained_moe_gate_b200 import dist as mdist
        self.moe, self.mdist, self.torch = moe, mdist, torch
        self.cfg, self.p, self.xs, self.stream = cfg, p, xs, stream
        self.sh = moe.shape_of(cfg)
        self.sh_global = moe.shape_of(cfg, T=mdist.global_token_count(cfg.T, world))  # the step's batch
        self.fp8 = cfg.dtype == "fp8"
        self.stages = STAGES_FP8 if self.fp8 else STAGES
        T, k, d, E = cfg.T, cfg.k, cfg.d, cfg.E
        dt = cfg.torch_dtype
        e = lambda *s, dtype=torch.int32: torch.empty(s, dtype=dtype, device=dev)
        self.idx, self.w, self.counts = e(T, k), e(T, k, dtype=torch.float32), e(E)
        self.offsets, self.perm, self.inv = e(E + 1), e(T * k), e(T * k)
        self.pws = e(max(moe.moe_permute_workspace_size(self.sh), 256), dtype=torch.uint8)
        self.x_perm = e(T * k, d, dtype=dt)   # x_perm, then y_perm
        if not self.fp8:  # (E4M3: h leaves the gate/up launch already quantized)
            self.h = e(T * k, cfg.I, dtype=dt)
            self.hs = e(T, max(1, cfg.S * cfg.Is), dtype=dt)
        self.shared_out = e(T, d, dtype=dt) if cfg.S > 0 else None
        self.y = e(T, d, dtype=dt)
        if self.fp8:  # E4M3 expert weights with tile scales, quantized once before timing
            self.q8 = moe.quantize_experts_fp8(p)
            self.w8 = moe.fp8_experts(self.q8)
            SIs = max(128, cfg.S * cfg.Is)
            tok = moe.MOE_SF_TOKENS
            self.xq, self.xsc = e(T, d, dtype=torch.uint8), moe.fp8_scales(T, d, tok, dev)
            self.xq_perm = e(T * k, d, dtype=torch.uint8)
            # token scales as the GEMMs' tile images: x's routed and shared tiles, h's and hs's
            self.x_img, self.xsh_img = moe.fp8_tile_images(T * k, E, d, dev), moe.fp8_tile_images(T, 1, d, dev)
            self.hq, self.h_img = e(T * k, cfg.I, dtype=torch.uint8), moe.fp8_tile_images(T * k, E, cfg.I, dev)
            self.hsq, self.hs_img = e(T, SIs, dtype=torch.uint8), moe.fp8_tile_images(T, 1, SIs, dev)
            torch.cuda.synchronize()

    def __call__(self, i, ev=None):
        moe, cfg, p, st, sh = self.moe, self.cfg, self.p, self.stream, self.sh
        x = self.xs[i % len(self.xs)]
        rec = (lambda j: ev[j].record(st)) if ev is not None else (lambda j: None)
        sh_ = cfg.S > 0
        T, k = cfg.T, cfg.k
        rec(0)
        moe.moe_route(x, p["w_gate"], p["bias"], sh, self.idx, self.w, self.counts, None, st)
        rec(1)
        if self.fp8:
            moe.moe_quantize_fp8(x, T, cfg.d, 1, moe.MOE_SF_TOKENS, self.xq, self.xsc, st)
            rec(2)
            moe.moe_permute(self.xq, self.idx, self.counts, sh, self.xq_perm, self.offsets, self.perm, self.inv,
                            self.pws, st)
            rec(3)
            moe.moe_fp8_tile_scales(self.xsc, T, cfg.d, self.perm, k, self.offsets, cfg.E, T * k, self.x_img, st)
            if sh_:
                moe.moe_fp8_tile_scales(self.xsc, T, cfg.d, None, 1, None, 1, T, self.xsh_img, st)
            moe.moe_ffn_up_fp8_quant(self.xq_perm, self.x_img, self.offsets, self.xq if sh_ else None, self.xsh_img,
                                     self.w8, sh, self.hq, self.h_img, self.hsq if sh_ else None,
                                     self.hs_img if sh_ else None, st)
            rec(4)
            moe.moe_ffn_down_fp8(self.hq, self.h_img, self.offsets, self.hsq if sh_ else None, self.hs_img, self.w8,
                                 sh, self.x_perm, self.shared_out, st)
            j = 5
        else:
            moe.moe_permute(x, self.idx, self.counts, sh, self.x_perm, self.offsets, self.perm, self.inv, self.pws, st)
            rec(2)
            moe.moe_ffn_up(self.x_perm, self.offsets, p["w1"], p["w3"], x if sh_ else None, p["ws1"], p["ws3"], sh,
                           self.h, self.hs, st)
            rec(3)
            moe.moe_ffn_down(self.h, self.offsets, p["w2"], self.hs if sh_ else None, p["ws2"], sh, self.x_perm,
                             self.shared_out, st)
            j = 4
        rec(j)
        moe.moe_combine(self.x_perm, self.w, self.inv, self.shared_out, sh, self.y, st)
        rec(j + 1)
        self.mdist.allreduce_counts(self.counts)
        moe.moe_load_and_bias_update(self.counts, self.sh_global, cfg.step_size, None, p["bias"], None, st)
        rec(j + 2)


def _gpu_id(local):
    gpu_id = str(local)
    vis = os.environ.get("CUDA_VISIBLE_DEVICES")
    if vis:
        gpu_id = vis.split(",")[local].strip()
    return gpu_id


def timed_steps(step, steps, warmup, world, local, dev, on_step=None):
    """W untimed steps, then K steps between a barrier + synchronize on both
    sides, CUDA events on the launching stream (and between the stages);
    max over ranks.  Returns (ms_total, stage_ms, launches, clocks)."""
    import torch
    import torch.distributed as dist
    import fine_grained_moe_gate_b200 as moe
    stream = step.stream

    def barrier():
        if world > 1:
            dist.barrier()
        torch.cuda.synchronize()

    for i in range(warmup):
        step(i)
    st = moe.moe_get_last_error(stream)
    if st != 0:
        raise moe.MoEError(st, f"{step.cfg.name}: warm-up steps")
    clocks = ClockSampler(_gpu_id(local))
    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(len(step.stages) + 1)] for _ in range(steps)]
    start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    barrier()
    clocks.start()
    launches0 = moe.moe_kernel_launch_count()
    start.record(stream)
    for i in range(steps):
        step(warmup + i, evs[i])
        if on_step is not None:
            on_step(i)
    end.record(stream)
    launches = moe.moe_kernel_launch_count() - launches0
    barrier()
    clk = clocks.stop()
    st = moe.moe_get_last_error(stream)
    if st != 0:
        raise moe.MoEError(st, f"{step.cfg.name}: timed steps")
    stage_ms = {name: statistics.mean(e[j].elapsed_time(e[j + 1]) for e in evs)
                for j, name in enumerate(step.stages)}
    t = torch.tensor([start.elapsed_time(end)], dtype=torch.float64, device=dev)
    if world > 1:
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item()), stage_ms, launches, clk


def roofline_records(step, stage_ms, peaks, peak_src, dominant_ms=None):
    """Roofline of the dominant kernel (the gate/up launch, routed + shared
    sets): tensor FLOP/s against the measured burst bf16 peak (the kernel is
    timed in a sub-second region; the sustained figure is the seconds-long
    power-capped one) and the HBM bytes it must move against the measured
    copy bandwidth.  Returns (primary, alternate, touched experts)."""
    moe, cfg, p, sh = step.moe, step.cfg, step.p, step.sh
    T, k, d = cfg.T, cfg.k, cfg.d
    SIs = cfg.S * cfg.Is
    flops_per_launch = T * k * 4 * d * cfg.I + T * 4 * d * SIs   # gate + up, real rows only
    dom_ms = stage_ms[DOMINANT] if dominant_ms is None else dominant_ms
    achieved = flops_per_launch / (dom_ms / 1e3) / 1e12
    # algorithmic bytes of that launch: W1 + W3 of the routed experts that got
    # rows (counted by routing each input once more, outside the timed region)
    # and of the shared experts, the token rows read and h written
    touched = []
    for xx in step.xs[:8]:
        moe.moe_route(xx, p["w_gate"], p["bias"], sh, step.idx, step.w, step.counts, None, step.stream)
        touched.append(int((step.counts > 0).sum().item()))
    n_touched = statistics.mean(touched)
    esz = {"bf16": 2, "fp8": 1}.get(cfg.dtype, 4)
    if step.fp8:  # E4M3 codes (weights and token rows in, h out), each with one scale byte per 32
        bytes_per_launch = (n_touched * 2 * cfg.I * d + 2 * SIs * d + T * k * d + T * d + T * k * cfg.I +
                            T * SIs) * 33 // 32
    else:
        bytes_per_launch = (n_touched * 2 * cfg.I * d + T * k * (d + cfg.I) + 2 * SIs * d + T * (d + SIs)) * esz
    hbm_gbs = bytes_per_launch / (dom_ms / 1e3) / 1e9
    hbm_peak = float(peaks.get("hbm_gbs", FALLBACK_PEAKS["hbm_gbs"]))
    traffic = traffic_record(os.path.join(ROOT, "fine_grained_moe_gate_b200", "csrc", "gemm_tc.cu"), cfg.name)
    roof_hbm = {"bound": "hbm", "kernel": "gate/up projection (routed + shared)", "achieved": round(hbm_gbs, 1),
                "peak": hbm_peak, "unit": "GB/s", "frac": round(hbm_gbs / hbm_peak, 4),
                "frac_of_nominal_8000": round(hbm_gbs / 8000.0, 4),
                "traffic": traffic, "bytes_per_launch": int(bytes_per_launch), "experts_touched": n_touched,
                "ms_per_launch": round(dom_ms, 4), "peak_kind": f"hbm_gbs ({peak_src}, copy bandwidth)"}
    burst = float(peaks.get("bf16_tflops", FALLBACK_PEAKS["bf16_tflops"]))
    sus = float(peaks.get("bf16_tflops_sustained", FALLBACK_PEAKS["bf16_tflops_sustained"]))
    if cfg.dtype in ("bf16", "fp8"):
        mult = 2.0 if step.fp8 else 1.0  # nominal dense E4M3 / bf16 ratio 4.5 / 2.25
        peak = mult * burst
        roof = {"bound": "tensor",
                "kernel": "tc_grouped_gemm_kernel<up%s> (routed + shared experts, SwiGLU epilogue)"
                          % (", E4M3" if step.fp8 else ""),
                "achieved": round(achieved, 2), "peak": peak, "unit": "TFLOP/s", "frac": round(achieved / peak, 4),
                "frac_of_sustained": round(achieved / (mult * sus), 4), "traffic": traffic,
                "peak_kind": ("%sbf16_tflops (%s, burst): the kernel is timed in a sub-second region"
                              % ("2 x " if step.fp8 else "", peak_src)),
                "flops_per_launch": flops_per_launch, "ms_per_launch": round(dom_ms, 4)}
    else:
        roof = {"bound": "alu", "kernel": "simt_grouped_gemm_kernel (fp32 FFMA; routed and shared launches)",
                "achieved": round(achieved, 3), "peak": None, "unit": "TFLOP/s", "frac": None, "traffic": None,
                "flops_per_launch": flops_per_launch, "ms_per_launch": round(dom_ms, 4)}
    if cfg.name.startswith("v3_decode"):
        # a few tokens per expert: the launch streams the touched experts' weights
        roof, roof_hbm = roof_hbm, roof
    return roof, roof_hbm, n_touched


def layer_weight_bytes(cfg, n_touched):
    """HBM bytes of the weights one layer step must read: W1, W3, W2 of the
    touched experts, the shared experts and W_gate (the decode workload's
    bound)."""
    esz = {"bf16": 2, "fp8": 1}.get(cfg.dtype, 4)
    gate = cfg.E * cfg.d * (2 if cfg.dtype == "fp8" else esz)
    return int((n_touched * 3 * cfg.I * cfg.d + 3 * cfg.S * cfg.Is * cfg.d) * esz + gate)


def measure_extra(name, args, world, rank, local, dev, peaks, peak_src, n_steps, n_x):
    """One more workload of the default line (decode, skew): its own layer
    and inputs, timed like the main line; returns its record."""
    import torch
    from fine_grained_moe_gate_b200 import dist as mdist
    from fine_grained_moe_gate_b200.inputs import CONFIGS, make_layer, make_tokens
    cfg = CONFIGS[name]
    stream = torch.cuda.current_stream()
    p = make_layer(cfg, dev)
    xs = [make_tokens(cfg, dev, step=mdist.shard_step(i, rank, world)) for i in range(n_x)]
    step = LayerStep(cfg, dev, world, p, xs, stream)
    loads = None
    if cfg.zipf_s > 0:
        loads = torch.empty((n_steps, cfg.E), dtype=torch.int32, device=dev)
        on_step = lambda i: loads[i].copy_(step.counts, non_blocking=True)  # 1 KB device copy per step
    else:
        on_step = None
    ms_total, stage_ms, launches, clk = timed_steps(step, n_steps, max(3, args.warmup), world, local, dev, on_step)
    roof, roof_alt, n_touched = roofline_records(step, stage_ms, peaks, peak_src)
    ms = ms_total / n_steps
    rec = {"value": round(world * cfg.T * n_steps / (ms_total / 1e3), 1), "unit": "tokens/s",
           "ms_per_step": round(ms, 4), "steps": n_steps, "warmup": max(3, args.warmup),
           "config": {"workload": cfg.name, "T_per_gpu": cfg.T, "d": cfg.d, "E": cfg.E, "k": cfg.k, "I": cfg.I,
                      "S": cfg.S, "Is": cfg.Is, "inputs": f"{n_x} pre-drawn batches, cycled"
                      + (" (fresh x every call)" if n_x >= n_steps else "")},
           "roofline": roof, "roofline_alt": roof_alt,
           "stages_ms": {k_: round(v, 4) for k_, v in stage_ms.items()},
           "gpu_launches": int(launches), "clocks": clk}
    if cfg.name.startswith("v3_decode"):
        wb = layer_weight_bytes(cfg, n_touched)
        hbm = float(peaks.get("hbm_gbs", FALLBACK_PEAKS["hbm_gbs"]))
        gbs = wb / (ms / 1e3) / 1e9
        rec["layer_hbm"] = {"bytes_per_step": wb, "achieved_gbs": round(gbs, 1), "frac": round(gbs / hbm, 4),
                            "frac_of_nominal_8000": round(gbs / 8000.0, 4),
                            "what": "weights of the touched experts (W1, W3, W2), the shared expert and W_gate "
                                    "per step / step time, against the measured copy bandwidth"}
    else:
        rec["layer_tflops"] = round(cfg.flops() / (ms / 1e3) / 1e12, 2)
    if loads is not None:
        c = loads.double()
        ratio = (c.max(1).values / c.mean(1)).cpu().tolist()
        rec["load_max_over_mean"] = {"first": round(ratio[0], 3), "last": round(ratio[-1], 3),
                                     "min": round(min(ratio), 3), "median": round(statistics.median(ratio), 3),
                                     "max": round(max(ratio), 3),
                                     "what": "per timed step: the most-loaded expert's rows / mean rows per expert "
                                             "(counts summed over ranks), bias updated every step"}
    del step, p, xs
    torch.cuda.empty_cache()
    return rec


def run_ours(args, world, rank, local):
    import torch
    import torch.distributed as dist

    import fine_grained_moe_gate_b200 as moe
    from fine_grained_moe_gate_b200 import dist as mdist
    from fine_grained_moe_gate_b200.inputs import make_layer, make_tokens

    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    if world > 1:
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120), device_id=dev)
    cfg = workload(args)
    sh = moe.shape_of(cfg)
    stream = torch.cuda.current_stream()

    p = make_layer(cfg, dev)
    fp8 = cfg.dtype == "fp8"
    n_x = max(1, min(4, args.steps + args.warmup))
    xs = [make_tokens(cfg, dev, step=mdist.shard_step(i, rank, world)) for i in range(n_x)]
    step = LayerStep(cfg, dev, world, p, xs, stream)
    T, k, d, E = cfg.T, cfg.k, cfg.d, cfg.E
    dt = cfg.torch_dtype
    ms_total, stage_ms, launches, clk = timed_steps(step, args.steps, args.warmup, world, local, dev)
    ms_per_step = ms_total / args.steps
    tokens_per_s = world * T * args.steps / (ms_total / 1e3)

    def barrier():
        if world > 1:
            dist.barrier()
        torch.cuda.synchronize()

    # ---- e2e: public call, host buffers, copies inside the timed region
    e2e = None
    if not args.no_e2e:
        # Double-buffered: the tokens of step i+1 go up (copy stream) and the
        # output of step i comes down (another copy stream) while step i+1
        # computes; every step still copies its own x in and its y out, all
        # inside the timed region.
        ws = torch.empty(moe.moe_workspace_size(sh), dtype=torch.uint8, device=dev)
        nb = 2
        x_dev = [torch.empty((T, d), dtype=dt, device=dev) for _ in range(nb)]
        y_dev = [torch.empty((T, d), dtype=dt, device=dev) for _ in range(nb)]
        x_host = [xx.cpu().pin_memory() for xx in xs]
        y_host = [torch.empty((T, d), dtype=dt).pin_memory() for _ in range(nb)]
        s_in, s_out = torch.cuda.Stream(device=dev), torch.cuda.Stream(device=dev)
        ev_in = [torch.cuda.Event() for _ in range(nb)]     # x_dev[b] holds the step's tokens
        ev_done = [torch.cuda.Event() for _ in range(nb)]   # the step using buffer b has computed
        ev_out = [torch.cuda.Event() for _ in range(nb)]    # y_dev[b] has reached the host
        idx, w, counts = step.idx, step.w, step.counts

        def issue_h2d(i):
            bb = i % nb
            s_in.wait_event(ev_done[bb])                    # the step that last read x_dev[bb] is done
            with torch.cuda.stream(s_in):
                x_dev[bb].copy_(x_host[i % n_x], non_blocking=True)
            ev_in[bb].record(s_in)

        def e2e_step(i, last):
            bb = i % nb
            stream.wait_event(ev_in[bb])
            stream.wait_event(ev_out[bb])                   # y_dev[bb] is no longer being copied out
            if fp8:
                moe.moe_layer_forward_fp8(x_dev[bb], p["w_gate"], p["bias"], step.w8, sh, y_dev[bb], idx, w, counts,
                                          ws, stream)
            else:
                moe.moe_layer_forward(x_dev[bb], p["w_gate"], p["bias"], p["w1"], p["w3"], p["w2"], p["ws1"],
                                      p["ws3"], p["ws2"], sh, y_dev[bb], idx, w, counts, ws, stream)
            mdist.allreduce_counts(counts)
            moe.moe_load_and_bias_update(counts, step.sh_global, cfg.step_size, None, p["bias"], None, stream)
            ev_done[bb].record(stream)
            if not last:
                issue_h2d(i + 1)
            s_out.wait_event(ev_done[bb])
            with torch.cuda.stream(s_out):
                y_host[bb].copy_(y_dev[bb], non_blocking=True)
            ev_out[bb].record(s_out)

        def e2e_run(n):
            s_in.wait_event(start_ev)
            issue_h2d(0)
            for i in range(n):
                e2e_step(i, i == n - 1)
            stream.wait_event(ev_out[(n - 1) % nb])

        start_ev = torch.cuda.Event()
        start_ev.record(stream)
        e2e_run(args.warmup)
        barrier()
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record(stream)
        start_ev = a
        e2e_run(args.steps)
        b.record(stream)
        barrier()
        te = torch.tensor([a.elapsed_time(b)], dtype=torch.float64, device=dev)
        if world > 1:
            dist.all_reduce(te, op=dist.ReduceOp.MAX)
        e2e = {"value": world * T * args.steps / (float(te.item()) / 1e3), "unit": "tokens/s",
               "h2d_bytes_per_step": x_dev[0].numel() * x_dev[0].element_size(),
               "d2h_bytes_per_step": y_host[0].numel() * y_host[0].element_size(),
               "ms_per_step": float(te.item()) / args.steps,
               "pipelining": "copy-in of step i+1 and copy-out of step i overlap step i+1's compute (2 buffers)"}
        st = moe.moe_get_last_error(stream)
        if st != 0:
            raise moe.MoEError(st, "e2e steps")
        del ws, x_dev, y_dev, x_host, y_host

    peaks, peak_src = load_peaks()
    roof, roof_hbm, n_touched = roofline_records(step, stage_ms, peaks, peak_src)
    esz = {"bf16": 2, "fp8": 1}.get(cfg.dtype, 4)
    layer_flops = cfg.flops()
    step_tflops = layer_flops / (ms_per_step / 1e3) / 1e12
    burst = float(peaks.get("bf16_tflops", FALLBACK_PEAKS["bf16_tflops"]))
    weights_gb = (p["w1"].numel() * 3 + p["ws1"].numel() * 3) * esz / 1e9

    cpu = None
    if world == 1 and rank == 0 and not args.no_cpu_baseline:
        n_tok = args.cpu_tokens or DEFAULT_CPU_TOKENS[args.workload]
        secs, n, threads = run_oracle_sample(cfg, p, xs[0], min(n_tok, T))
        cpu = cpu_baseline_record(cfg, secs, n, threads, "oracle sample")

    # ---- the other workloads of the default line (decode-shaped, skewed routing)
    extras = {}
    if not args.no_extra and args.workload == "v3_prefill" and not (args.T or args.E or args.I):
        del step, xs
        p.clear()
        torch.cuda.empty_cache()
        extras["v3_decode"] = measure_extra("v3_decode", args, world, rank, local, dev, peaks, peak_src,
                                            args.decode_calls, args.decode_calls)
        extras["skew_stress"] = measure_extra("skew_stress", args, world, rank, local, dev, peaks, peak_src,
                                              args.skew_steps, 8)

    if rank == 0:
        line = {
            "metric": METRIC, "value": round(tokens_per_s, 1), "unit": "tokens/s", "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(ms_per_step, 4),
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": cfg.dtype,
            "data": "synthetic (seeded N(0,1) tokens, N(0,std) weights of the stated shape"
                    + ("; expert weights quantized to E4M3 with 1x32 power-of-two tile scales before timing)"
                       if fp8 else ")"),
            "config": {"workload": cfg.name, "T_per_gpu": T, "global_batch": T * world, "d": d, "E": E, "k": k,
                       "I": cfg.I, "S": cfg.S, "Is": cfg.Is, "parallelism": f"dp{world}",
                       "l2": f"inputs larger than L2: layer weights read every step ({weights_gb:.1f} GB)",
                       "bias_update": "every step"},
            "roofline": roof,
            "roofline_alt": roof_hbm,
            "layer_tflops": round(step_tflops, 2),
            "layer_frac_of_peak": round(step_tflops / (burst * (2.0 if fp8 else 1.0)), 4)
            if cfg.dtype in ("bf16", "fp8") else None,
            "layer_peak_kind": "bf16_tflops burst (x2 for E4M3)",
            "stages_ms": {k_: round(v, 4) for k_, v in stage_ms.items()},
            "cpu_baseline": cpu,
            "e2e": e2e,
            "gpu_launches": int(launches),
            "clocks": clk,
            "impl": "ours",
        }
        if extras:
            line["workloads"] = extras
        print(json.dumps(line), flush=True)
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()


def run_reference(args, world, rank, local):
    """The oracle as the reference arm: rank 0 times it on the host cores on
    a bounded token sample per step; other ranks exit without work."""
    if rank != 0:
        return
    import torch
    from fine_grained_moe_gate_b200.inputs import make_layer, make_tokens

    cfg = workload(args)
    dev = torch.device("cuda", local) if torch.cuda.is_available() else torch.device("cpu")
    if dev.type == "cuda":
        torch.cuda.set_device(local)
    p = make_layer(cfg, dev)
    x = make_tokens(cfg, dev, 0)
    n_tok = args.cpu_tokens or max(2, DEFAULT_CPU_TOKENS[args.workload] // 3)
    n_tok = min(n_tok, cfg.T)
    for _ in range(args.warmup):
        run_oracle_sample(cfg, p, x, n_tok)
    total, threads = 0.0, 1
    for _ in range(args.steps):
        secs, n, threads = run_oracle_sample(cfg, p, x, n_tok)
        total += secs
    value = n_tok * args.steps / total
    rec = cpu_baseline_record(cfg, total, n_tok * args.steps, threads, "reference arm (oracle)")
    rec["value"] = value
    line = {
        "metric": METRIC, "value": round(value, 4), "unit": "tokens/s", "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": round(1e3 * total / args.steps, 3), "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": cfg.dtype,
        "data": "synthetic (seeded N(0,1) tokens, N(0,std) weights of the stated shape)",
        "config": {"workload": cfg.name, "T_per_gpu": cfg.T, "global_batch": cfg.T * world, "d": cfg.d, "E": cfg.E,
                   "k": cfg.k, "I": cfg.I, "S": cfg.S, "Is": cfg.Is, "parallelism": f"dp{world}",
                   "sample_tokens_per_step": n_tok},
        "impl": "reference",
        "cpu_baseline": rec,
        "e2e": {"value": round(value, 4), "unit": "tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


# fp32 FFMA peak for the SIMT backward: 148 SMs x 128 fp32 lanes x 2 FLOP per
# cycle at the 1965 MHz maximum SM clock
FP32_SIMT_PEAK_TFLOPS = 148 * 128 * 2 * 1.965e9 / 1e12


def run_backward(args, world, rank, local):
    """One step = moe_layer_backward over the workload's batch: gradients of
    x, the gate and all expert weights plus the sequence-wise balance loss
    (alpha 1e-4, one sequence per 4096 tokens or the whole batch), for a
    routing computed once before timing."""
    import torch

    import fine_grained_moe_gate_b200 as moe
    from fine_grained_moe_gate_b200.inputs import make_layer, make_tokens

    if world > 1:
        if rank == 0:
            print(json.dumps({"metric": "MoE layer backward", "unavailable": "--backward runs on one GPU"}))
        return
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    cfg = workload(args)
    if cfg.dtype == "fp8":
        raise SystemExit("--backward: E4M3 layers have no backward")
    sh = moe.shape_of(cfg)
    p = make_layer(cfg, dev)
    x = make_tokens(cfg, dev)
    T, d, E, k, I, S, Is = cfg.T, cfg.d, cfg.E, cfg.k, cfg.I, cfg.S, cfg.Is
    idx = torch.empty((T, k), dtype=torch.int32, device=dev)
    w = torch.empty((T, k), dtype=torch.float32, device=dev)
    counts = torch.empty(E, dtype=torch.int32, device=dev)
    aff = torch.empty((T, E), dtype=torch.float32, device=dev)
    moe.moe_route(x, p["w_gate"], p["bias"], sh, idx, w, counts, aff)
    g = torch.Generator(device=dev).manual_seed(cfg.seed + 101)
    dy = torch.randn((T, d), generator=g, device=dev)
    f32 = lambda *shp: torch.empty(shp, dtype=torch.float32, device=dev)
    out = [f32(T, d), f32(E, d), f32(E, I, d), f32(E, I, d), f32(E, d, I)]
    sh_out = [f32(S, Is, d), f32(S, Is, d), f32(S, d, Is)] if S else [None, None, None]
    loss = f32(1)
    L = 4096 if T % 4096 == 0 else T
    ws = torch.empty(moe.moe_backward_workspace_size(sh, L), dtype=torch.uint8, device=dev)
    shw = [p["ws1"], p["ws3"], p["ws2"]] if S else [None, None, None]

    def step():
        moe.moe_layer_backward(x, p["w_gate"], p["w1"], p["w3"], p["w2"], *shw, sh, idx, w, counts, aff, dy, 1e-4, L,
                               *out, *sh_out, loss, ws)

    for _ in range(max(args.warmup, 1)):
        step()
    torch.cuda.synchronize()
    steps = max(1, args.steps)
    clocks = ClockSampler(os.environ.get("CUDA_VISIBLE_DEVICES", str(local)).split(",")[0])
    clocks.start()
    n0 = moe.moe_kernel_launch_count()
    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    torch.cuda.synchronize()
    a.record()
    for _ in range(steps):
        step()
    b.record()
    torch.cuda.synchronize()
    ck = clocks.stop()
    launches = moe.moe_kernel_launch_count() - n0
    st = moe.moe_get_last_error()
    if st != 0:
        raise SystemExit(f"device status {moe.STATUS.get(st, st)}")
    ms = a.elapsed_time(b) / steps
    # bf16 layers whose widths are multiples of 128 run the expert contractions on the tensor cores
    tc = cfg.dtype == "bf16" and d % 128 == 0 and I % 128 == 0 and (S == 0 or Is % 128 == 0)
    # FLOPs (2 per multiply-add): per routed row the recomputed a and g (4 d I), dh (2 d I), dx_perm
    # (4 d I) and dW1, dW3, dW2 (6 d I) = 16 d I, plus the recomputed o (2 d I) on the SIMT path (the
    # tensor-core path takes the combine weights' gradient from dh instead); per token the shared
    # experts 16 d S Is and the router's dx and dW_g 4 d E
    flop = T * k * (16 if tc else 18) * d * I + T * 16 * d * S * Is + T * 4 * d * E
    tflops = flop / (ms * 1e-3) / 1e12
    if tc:
        peaks, peak_src = load_peaks()
        burst = float(peaks.get("bf16_tflops", FALLBACK_PEAKS["bf16_tflops"]))
        roof = {"bound": "tensor", "achieved": round(tflops, 2), "peak": burst, "unit": "TFLOP/s",
                "frac": round(tflops / burst, 4), "traffic": None,
                "peak_kind": f"bf16_tflops ({peak_src}, burst): the backward is timed in a sub-second region; "
                             "FLOPs of the router (2 d E per token, fp32 SIMT) included"}
    else:
        roof = {"bound": "alu", "achieved": round(tflops, 3), "peak": round(FP32_SIMT_PEAK_TFLOPS, 1),
                "unit": "TFLOP/s", "frac": round(tflops / FP32_SIMT_PEAK_TFLOPS, 4), "traffic": None,
                "peak_kind": "derived: 148 SMs x 128 fp32 FMA lanes x 2 FLOP x 1965 MHz"}
    line = {
        "metric": "MoE layer backward tokens/s (%s)" % ("tcgen05 bf16 contractions" if tc else "fp32 SIMT contractions"),
        "value": round(T / (ms * 1e-3), 2),
        "unit": "tokens/s", "n_gpus": 1, "steps": steps, "warmup": args.warmup, "ms_per_step": round(ms, 3),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16" if tc else "f32",
        "data": "synthetic (seeded N(0,1) tokens and dy, N(0,std) weights of the stated shape)",
        "config": {"workload": cfg.name + " backward", "T": T, "d": d, "E": E, "k": k, "I": I, "S": S, "Is": Is,
                   "balance_alpha": 1e-4, "seq_len": L,
                   "l2": "weights and activations far larger than L2 at these shapes; no flush"},
        "roofline": roof, "tflops": round(tflops, 2),
        "gpu_launches": int(launches), "clocks": ck,
    }
    print(json.dumps(line), flush=True)


def main():
    args = parse_args()
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world != args.gpus:
        print(f"warning: --gpus {args.gpus} but WORLD_SIZE={world}; using WORLD_SIZE", file=sys.stderr)
    if args.backward:
        run_backward(args, world, rank, local)
    elif args.impl == "reference":
        run_reference(args, world, rank, local)
    else:
        run_ours(args, world, rank, local)


if __name__ == "__main__":
    main()
