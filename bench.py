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

Rank 0 prints one JSON line.

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
# E4M3 expert workloads: token rows and h are quantized per row in the step
STAGES_FP8 = ["route", "quant_x", "permute", "ffn_up", "quant_h", "ffn_down", "combine", "bias_update"]
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
    """nvidia-smi samples of the SM clock and throttle reasons while the
    timed region runs."""
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_id: str):
        self.gpu_id = gpu_id
        self.proc = None
        self.path = None

    def start(self):
        fd, self.path = tempfile.mkstemp(prefix="clocks_", suffix=".csv")
        os.close(fd)
        try:
            self.out = open(self.path, "w")
            self.proc = subprocess.Popen(["nvidia-smi", "-i", self.gpu_id, f"--query-gpu={self.FIELDS}",
                                          "--format=csv,noheader,nounits", "-lms", "50"], stdout=self.out,
                                         stderr=subprocess.DEVNULL)
        except OSError:
            self.proc = None

    def stop(self):
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"], "samples": 0}
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
                if len(parts) >= 9:
                    rows.append(parts)
        os.unlink(self.path)
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = set()
        sm, smax, pw = [], [], []
        for r in rows:
            try:
                sm.append(float(r[1]))
                smax.append(float(r[2]))
                pw.append(float(r[3]))
            except ValueError:
                continue
            for n, v in zip(names, r[5:9]):
                if v.lower() == "active":
                    reasons.add(n)
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": max(smax) if smax else None,
                "reasons": sorted(reasons), "samples": len(sm),
                "power_w_median": statistics.median(pw) if pw else None}


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
    """oracle_sample for the E4M3 expert workloads: routing, per-token
    quantization of x, and for every expert the tokens use (and the shared
    experts) the FP8 gate/up, per-row quantization of h and the FP8 down.
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
    xq, xsc = oracle.quantize_rows_fp8(xs)
    secs = time.perf_counter() - t0
    yacc = np.zeros((n_tok, d), np.float64)
    if S > 0:
        q1, s1 = oracle.quantize_rows_fp8(to_numpy(p["ws1"]).reshape(S * Is, d))
        q3, s3 = oracle.quantize_rows_fp8(to_numpy(p["ws3"]).reshape(S * Is, d))
        q2, s2 = oracle.quantize_rows_fp8(to_numpy(p["ws2"]), nseg=S)
        t0 = time.perf_counter()
        hq, hsc = oracle.quantize_rows_fp8(oracle.expert_up_fp8(xq, xsc, q1, s1, q3, s3))
        yacc += oracle.expert_down_fp8(hq, hsc, q2, s2)
        secs += time.perf_counter() - t0
    for e in np.unique(idx):
        ii, jj = np.nonzero(idx == e)
        q1, s1 = oracle.quantize_rows_fp8(to_numpy(p["w1"][e]))
        q3, s3 = oracle.quantize_rows_fp8(to_numpy(p["w3"][e]))
        q2, s2 = oracle.quantize_rows_fp8(to_numpy(p["w2"][e]))
        t0 = time.perf_counter()
        hq, hsc = oracle.quantize_rows_fp8(oracle.expert_up_fp8(xq[ii], xsc[ii], q1, s1, q3, s3))
        yacc[ii] += w[ii, jj].astype(np.float64)[:, None] * oracle.expert_down_fp8(hq, hsc, q2, s2)
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
    if over:
        tag = ",".join(f"{k}={v}" for k, v in over.items())
        cfg = cfg.scaled(name=f"{cfg.name}[{tag}]", **over)
    return cfg


def run_ours(args, world, rank, local):
    import numpy as np
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
    sh_global = moe.shape_of(cfg, T=mdist.global_token_count(cfg.T, world))  # the step's batch, all ranks
    stream = torch.cuda.current_stream()

    p = make_layer(cfg, dev)
    fp8 = cfg.dtype == "fp8"
    stages = STAGES_FP8 if fp8 else STAGES
    if fp8:  # E4M3 expert weights, quantized once per output row before timing
        q8 = moe.quantize_experts_fp8(p)
        w8 = moe.fp8_experts(q8)
        torch.cuda.synchronize()
    n_x = max(1, min(4, args.steps + args.warmup))
    xs = [make_tokens(cfg, dev, step=mdist.shard_step(i, rank, world)) for i in range(n_x)]

    T, k, d, E = cfg.T, cfg.k, cfg.d, cfg.E
    dt = cfg.torch_dtype
    idx = torch.empty((T, k), dtype=torch.int32, device=dev)
    w = torch.empty((T, k), dtype=torch.float32, device=dev)
    counts = torch.empty(E, dtype=torch.int32, device=dev)
    offsets = torch.empty(E + 1, dtype=torch.int32, device=dev)
    perm = torch.empty(T * k, dtype=torch.int32, device=dev)
    inv = torch.empty(T * k, dtype=torch.int32, device=dev)
    pws = torch.empty(max(moe.moe_permute_workspace_size(sh), 256), dtype=torch.uint8, device=dev)
    x_perm = torch.empty((T * k, d), dtype=dt, device=dev)   # x_perm, then y_perm
    h = torch.empty((T * k, cfg.I), dtype=dt, device=dev)
    hs = torch.empty((T, max(1, cfg.S * cfg.Is)), dtype=dt, device=dev)
    shared_out = torch.empty((T, d), dtype=dt, device=dev) if cfg.S > 0 else None
    y = torch.empty((T, d), dtype=dt, device=dev)
    if fp8:
        SIs = max(1, cfg.S * cfg.Is)
        xq = torch.empty((T, d), dtype=torch.uint8, device=dev)
        xsc = torch.empty(T, dtype=torch.float32, device=dev)
        xq_perm = torch.empty((T * k, d), dtype=torch.uint8, device=dev)
        hq = torch.empty((T * k, cfg.I), dtype=torch.uint8, device=dev)
        h_sc = torch.empty(T * k, dtype=torch.float32, device=dev)
        hsq = torch.empty((T, SIs), dtype=torch.uint8, device=dev)
        hs_sc = torch.empty(T, dtype=torch.float32, device=dev)

    def step_fp8(i, ev=None):
        x = xs[i % n_x]
        rec = (lambda j: ev[j].record(stream)) if ev is not None else (lambda j: None)
        sh_ = cfg.S > 0
        rec(0)
        moe.moe_route(x, p["w_gate"], p["bias"], sh, idx, w, counts, None, stream)
        rec(1)
        moe.moe_quantize_fp8(x, T, d, 1, xq, xsc, stream)
        rec(2)
        moe.moe_permute(xq, idx, counts, sh, xq_perm, offsets, perm, inv, pws, stream)
        rec(3)
        moe.moe_ffn_up_fp8(xq_perm, perm, xsc, offsets, xq if sh_ else None, w8, sh, h, hs if sh_ else None, stream)
        rec(4)
        moe.moe_quantize_fp8(h, T * k, cfg.I, 1, hq, h_sc, stream)
        if sh_:
            moe.moe_quantize_fp8(hs, T, cfg.S * cfg.Is, 1, hsq, hs_sc, stream)
        rec(5)
        moe.moe_ffn_down_fp8(hq, h_sc, offsets, hsq if sh_ else None, hs_sc, w8, sh, x_perm, shared_out, stream)
        rec(6)
        moe.moe_combine(x_perm, w, inv, shared_out, sh, y, stream)
        rec(7)
        mdist.allreduce_counts(counts)
        moe.moe_load_and_bias_update(counts, sh_global, cfg.step_size, None, p["bias"], None, stream)
        rec(8)

    def step(i, ev=None):
        x = xs[i % n_x]
        rec = (lambda j: ev[j].record(stream)) if ev is not None else (lambda j: None)
        rec(0)
        moe.moe_route(x, p["w_gate"], p["bias"], sh, idx, w, counts, None, stream)
        rec(1)
        moe.moe_permute(x, idx, counts, sh, x_perm, offsets, perm, inv, pws, stream)
        rec(2)
        xs_ = x if cfg.S > 0 else None
        moe.moe_ffn_up(x_perm, offsets, p["w1"], p["w3"], xs_, p["ws1"], p["ws3"], sh, h, hs, stream)
        rec(3)
        moe.moe_ffn_down(h, offsets, p["w2"], hs if cfg.S > 0 else None, p["ws2"], sh, x_perm, shared_out, stream)
        rec(4)
        moe.moe_combine(x_perm, w, inv, shared_out, sh, y, stream)
        rec(5)
        mdist.allreduce_counts(counts)
        moe.moe_load_and_bias_update(counts, sh_global, cfg.step_size, None, p["bias"], None, stream)
        rec(6)

    if fp8:
        step = step_fp8

    def barrier():
        if world > 1:
            dist.barrier()
        torch.cuda.synchronize()

    for i in range(args.warmup):
        step(i)
    st = moe.moe_get_last_error(stream)
    if st != 0:
        raise moe.MoEError(st, "warm-up steps")

    gpu_id = str(local)
    vis = os.environ.get("CUDA_VISIBLE_DEVICES")
    if vis:
        gpu_id = vis.split(",")[local].strip()
    clocks = ClockSampler(gpu_id)
    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(len(stages) + 1)] for _ in range(args.steps)]
    start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    barrier()
    clocks.start()
    launches0 = moe.moe_kernel_launch_count()
    start.record(stream)
    for i in range(args.steps):
        step(args.warmup + i, evs[i])
    end.record(stream)
    launches = moe.moe_kernel_launch_count() - launches0
    barrier()
    clk = clocks.stop()
    st = moe.moe_get_last_error(stream)
    if st != 0:
        raise moe.MoEError(st, "timed steps")
    ms_local = start.elapsed_time(end)
    stage_ms = {}
    for j, name in enumerate(stages):
        stage_ms[name] = statistics.mean(e[j].elapsed_time(e[j + 1]) for e in evs)
    t = torch.tensor([ms_local], dtype=torch.float64, device=dev)
    if world > 1:
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
    ms_total = float(t.item())
    ms_per_step = ms_total / args.steps
    tokens_per_s = world * T * args.steps / (ms_total / 1e3)

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
                moe.moe_layer_forward_fp8(x_dev[bb], p["w_gate"], p["bias"], w8, sh, y_dev[bb], idx, w, counts, ws,
                                          stream)
            else:
                moe.moe_layer_forward(x_dev[bb], p["w_gate"], p["bias"], p["w1"], p["w3"], p["w2"], p["ws1"],
                                      p["ws3"], p["ws2"], sh, y_dev[bb], idx, w, counts, ws, stream)
            mdist.allreduce_counts(counts)
            moe.moe_load_and_bias_update(counts, sh_global, cfg.step_size, None, p["bias"], None, stream)
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

    # ---- roofline of the dominant kernel (gate/up grouped GEMM, routed + shared sets)
    peaks, peak_src = load_peaks()
    SIs = cfg.S * cfg.Is
    flops_per_launch = T * k * 4 * d * cfg.I + T * 4 * d * SIs   # gate + up, real rows only
    dom_ms = stage_ms[DOMINANT]
    achieved = flops_per_launch / (dom_ms / 1e3) / 1e12
    # algorithmic bytes of that launch: W1 + W3 of the routed experts that got
    # rows (counted by routing each input once more, outside the timed region)
    # and of the shared experts, the token rows read and h written
    touched = []
    for xx in xs:
        moe.moe_route(xx, p["w_gate"], p["bias"], sh, idx, w, counts, None, stream)
        touched.append(int((counts > 0).sum().item()))
    n_touched = statistics.mean(touched)
    esz = {"bf16": 2, "fp8": 1}.get(cfg.dtype, 4)
    if fp8:  # E4M3 weights and token rows in, bf16 h out
        bytes_per_launch = (n_touched * 2 * cfg.I * d + 2 * SIs * d + T * k * d + T * d) + \
            (T * k * cfg.I + T * SIs) * 2
    else:
        bytes_per_launch = (n_touched * 2 * cfg.I * d + T * k * (d + cfg.I) + 2 * SIs * d + T * (d + SIs)) * esz
    hbm_gbs = bytes_per_launch / (dom_ms / 1e3) / 1e9
    hbm_peak = float(peaks.get("hbm_gbs", FALLBACK_PEAKS["hbm_gbs"]))
    traffic = traffic_record(os.path.join(ROOT, "fine_grained_moe_gate_b200", "csrc", "gemm_tc.cu"), cfg.name)
    roof_hbm = {"bound": "hbm", "kernel": "gate/up projection (routed + shared)", "achieved": round(hbm_gbs, 1), "peak": hbm_peak,
                "unit": "GB/s", "frac": round(hbm_gbs / hbm_peak, 4),
                "frac_of_nominal_8000": round(hbm_gbs / 8000.0, 4),
                "traffic": traffic, "bytes_per_launch": int(bytes_per_launch), "experts_touched": n_touched,
                "peak_kind": f"hbm_gbs ({peak_src}, copy bandwidth)"}
    bf16_sus = float(peaks.get("bf16_tflops_sustained", FALLBACK_PEAKS["bf16_tflops_sustained"]))
    if cfg.dtype == "bf16":
        peak = bf16_sus
        roof = {"bound": "tensor", "kernel": "tc_grouped_gemm_kernel<up> (routed + shared experts, SwiGLU epilogue)",
                "achieved": round(achieved, 2), "peak": peak, "unit": "TFLOP/s", "frac": round(achieved / peak, 4),
                "traffic": traffic,
                "peak_kind": f"bf16_tflops_sustained ({peak_src}): the kernel is timed inside a long step",
                "flops_per_launch": flops_per_launch, "ms_per_launch": round(dom_ms, 4)}
    elif fp8:
        peak = 2.0 * bf16_sus  # nominal dense E4M3 / bf16 ratio 4.5 / 2.25 times the measured bf16 figure
        roof = {"bound": "tensor", "kernel": "tc_grouped_gemm_kernel<up, E4M3> (routed + shared experts)",
                "achieved": round(achieved, 2), "peak": peak, "unit": "TFLOP/s", "frac": round(achieved / peak, 4),
                "traffic": traffic,
                "peak_kind": f"2 x bf16_tflops_sustained ({peak_src}; nominal fp8/bf16 dense ratio 4.5/2.25)",
                "flops_per_launch": flops_per_launch, "ms_per_launch": round(dom_ms, 4)}
    else:
        roof = {"bound": "alu", "kernel": "simt_grouped_gemm_kernel (fp32 FFMA; routed and shared launches)", "achieved": round(achieved, 3),
                "peak": None, "unit": "TFLOP/s", "frac": None, "traffic": None,
                "flops_per_launch": flops_per_launch, "ms_per_launch": round(dom_ms, 4)}
    if cfg.name.startswith("v3_decode"):
        # a few tokens per expert: the launch streams the touched experts' weights
        roof, roof_hbm = roof_hbm, roof
    layer_flops = cfg.flops()
    step_tflops = layer_flops / (ms_per_step / 1e3) / 1e12

    cpu = None
    if world == 1 and rank == 0 and not args.no_cpu_baseline:
        n_tok = args.cpu_tokens or DEFAULT_CPU_TOKENS[args.workload]
        secs, n, threads = run_oracle_sample(cfg, p, xs[0], min(n_tok, T))
        cpu = cpu_baseline_record(cfg, secs, n, threads, "oracle sample")

    if rank == 0:
        line = {
            "metric": METRIC, "value": round(tokens_per_s, 1), "unit": "tokens/s", "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(ms_per_step, 4),
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": cfg.dtype,
            "data": "synthetic (seeded N(0,1) tokens, N(0,std) weights of the stated shape"
                    + ("; expert weights quantized to E4M3 per output row before timing)" if fp8 else ")"),
            "config": {"workload": cfg.name, "T_per_gpu": T, "global_batch": T * world, "d": d, "E": E, "k": k,
                       "I": cfg.I, "S": cfg.S, "Is": cfg.Is, "parallelism": f"dp{world}",
                       "l2": "inputs larger than L2: layer weights read every step "
                             f"({(p['w1'].numel() * 3 + p['ws1'].numel() * 3) * esz / 1e9:.1f} GB)",
                       "bias_update": "every step"},
            "roofline": roof,
            "roofline_alt": roof_hbm,
            "layer_tflops": round(step_tflops, 2),
            "layer_frac_of_peak": round(step_tflops / (bf16_sus * (2.0 if fp8 else 1.0)), 4)
            if cfg.dtype in ("bf16", "fp8") else None,
            "stages_ms": {k_: round(v, 4) for k_, v in stage_ms.items()},
            "cpu_baseline": cpu,
            "e2e": e2e,
            "gpu_launches": int(launches),
            "clocks": clk,
            "impl": "ours",
        }
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
    # FLOPs (2 per multiply-add): per routed row the recomputed a, g and o (6 d I), dh (2 d I), dx_perm
    # (4 d I) and dW1, dW3, dW2 (6 d I) = 18 d I; per token the shared experts 16 d S Is (no o) and the
    # router's dx and dW_g 4 d E
    flop = T * k * 18 * d * I + T * 16 * d * S * Is + T * 4 * d * E
    tflops = flop / (ms * 1e-3) / 1e12
    line = {
        "metric": "MoE layer backward tokens/s (fp32 SIMT contractions)", "value": round(T / (ms * 1e-3), 2),
        "unit": "tokens/s", "n_gpus": 1, "steps": steps, "warmup": args.warmup, "ms_per_step": round(ms, 3),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f32",
        "data": "synthetic (seeded N(0,1) tokens and dy, N(0,std) weights of the stated shape)",
        "config": {"workload": cfg.name + " backward", "T": T, "d": d, "E": E, "k": k, "I": I, "S": S, "Is": Is,
                   "balance_alpha": 1e-4, "seq_len": L,
                   "l2": "weights and activations far larger than L2 at these shapes; no flush"},
        "roofline": {"bound": "alu", "achieved": round(tflops, 3), "peak": round(FP32_SIMT_PEAK_TFLOPS, 1),
                     "unit": "TFLOP/s", "frac": round(tflops / FP32_SIMT_PEAK_TFLOPS, 4), "traffic": None,
                     "peak_kind": "derived: 148 SMs x 128 fp32 FMA lanes x 2 FLOP x 1965 MHz"},
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
