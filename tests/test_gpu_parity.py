"""GPU parity: every C-ABI call against the CPU oracle on the same seeded
inputs, at sizes the oracle finishes in seconds that still span several
tiles and ragged tails.

Bars: routing indices, counts, offsets, permutation and bias updates are
bit-exact (both sides select on the kernel's fp32 affinities); the kernel's
own affinities are within the fp32-accumulation bound derived in
gpu_harness.affinity_tolerance; layer outputs within relative Frobenius 1e-5
(fp32) and 5e-3 (bf16).
"""
import numpy as np
import pytest
import torch

import fine_grained_moe_gate_b200 as moe
import oracle
from fine_grained_moe_gate_b200.inputs import CONFIGS, make_layer, make_tokens, to_numpy

from gpu_harness import (DEV, as_f64, check_layer_elementwise, check_route_parity, check_status, grouped_swiglu,
                         layer_forward, oracle_rows, oracle_terms, oracle_terms_from_h, permute, rel_fro, route,
                         to_f64_rows)

pytestmark = pytest.mark.gpu

TINY = CONFIGS["tiny_fp32"]
SMALL = CONFIGS["small_bf16"]
V3 = CONFIGS["v3_prefill"]


@pytest.fixture(autouse=True)
def _clean_status():
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    moe.moe_get_last_error()
    yield


# ------------------------------------------------------------------ router

def test_route_tiny_fp32_full():
    sh = moe.shape_of(TINY)
    p = make_layer(TINY, DEV)
    x = make_tokens(TINY, DEV)
    idx, w, counts, aff = route(sh, x, p["w_gate"], p["bias"])
    check_status()
    check_route_parity(x, p["w_gate"], p["bias"], sh.k, idx, w, counts, aff, "auto")


ROUTER_BF16 = [
    dict(T=300, d=512, E=64, k=6),        # small_bf16 routing shape, ragged token tile
    dict(T=1000, d=1024, E=256, k=8),     # V3 routing, 8 token tiles
    dict(T=77, d=128, E=40, k=3),         # E not a multiple of 16
    dict(T=130, d=64, E=8, k=8),          # k = E
    dict(T=64, d=256, E=32, k=12),        # k > 8 (16-wide top-k registers)
    dict(T=1, d=64, E=16, k=2),
    # CTA-pair tiles of 256 tokens (large batches)
    dict(T=4964, d=256, E=72, k=6),       # last pair's second CTA entirely past T; N/2 = 40 rows per CTA
    dict(T=8192, d=1024, E=256, k=8),     # V3 routing width, K split over 2 pairs
    dict(T=6000, d=192, E=24, k=4),       # uneven K slices (3 blocks over 2 pairs), N = 32
    dict(T=20000, d=128, E=256, k=12),    # k > 8, no K split, more pairs than one wave
    dict(T=5000, d=128, E=8, k=2),        # the smallest pair MMA: N = 16, 8 W_gate rows per CTA
]


@pytest.mark.parametrize("c", ROUTER_BF16, ids=lambda c: "T{T}_d{d}_E{E}_k{k}".format(**c))
def test_route_bf16_tensor_cores(c):
    cfg = V3.scaled(T=c["T"], d=c["d"], E=c["E"], k=c["k"], w_std=0.02, bias_range=0.05)
    sh = moe.shape_of(cfg)
    p = make_layer(cfg.scaled(I=128, Is=128, S=0), DEV)
    x = make_tokens(cfg, DEV)
    idx, w, counts, aff = route(sh, x, p["w_gate"], p["bias"])
    check_status()
    # the first tile and the ragged last ones
    rows = np.unique(np.concatenate([np.arange(min(c["T"], 256)), np.arange(max(c["T"] - 300, 0), c["T"])]))
    check_route_parity(x, p["w_gate"], p["bias"], sh.k, idx, w, counts, aff, "auto", self_rows=rows)


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
def test_route_exact_ties_go_to_lower_index(dtype):
    """Duplicate gate rows and equal biases give exactly equal scores; the
    lower expert index must win every tie ("In code", route: topk; ties by
    lower index)."""
    cfg = V3.scaled(T=256, d=128, E=32, k=5, dtype=dtype)
    sh = moe.shape_of(cfg)
    g = torch.Generator(device=DEV).manual_seed(3)
    wg = torch.randn((8, cfg.d), generator=g, device=DEV) * 0.1
    wg = wg.repeat(4, 1).to(cfg.torch_dtype).contiguous()   # expert e == expert e % 8
    bias = torch.zeros(cfg.E, device=DEV)
    x = make_tokens(cfg, DEV)
    idx, w, counts, aff = route(sh, x, wg, bias)
    check_status()
    o_idx, _ = check_route_parity(x, wg, bias, sh.k, idx, w, counts, aff, "auto", self_rows=np.arange(32))
    # each chosen expert must be the lowest index among its equal-score copies
    idx_np = o_idx
    for t in range(cfg.T):
        for e in idx_np[t]:
            assert e < 8 or (e - 8) in idx_np[t]


def test_route_tiny_experts_brute_force():
    """fp32 path on tiny E: GPU selection equals the brute-force best
    k-subset of the biased affinities."""
    import itertools
    cfg = TINY.scaled(T=40, d=32, E=6, k=2)
    sh = moe.shape_of(cfg)
    p = make_layer(cfg.scaled(I=8, Is=8, S=0), DEV)
    x = make_tokens(cfg, DEV)
    idx, w, counts, aff = route(sh, x, p["w_gate"], p["bias"])
    check_status()
    v = aff.cpu().numpy() + p["bias"].cpu().numpy()
    for t in range(cfg.T):
        best = max(itertools.combinations(range(cfg.E), cfg.k), key=lambda s: (sum(float(v[t, i]) for i in s),
                                                                                [-i for i in s]))
        assert set(idx[t].tolist()) == set(best)


def test_route_empty_batch():
    sh = moe.shape_of(TINY, T=0)
    p = make_layer(TINY.scaled(I=8, Is=8), DEV)
    counts = torch.full((TINY.E,), 7, dtype=torch.int32, device=DEV)
    moe.moe_route(None, p["w_gate"], p["bias"], sh, None, None, counts)
    torch.cuda.synchronize()
    check_status()
    assert int(counts.abs().sum()) == 0


# ------------------------------------------------------------- bias update

@pytest.mark.parametrize("with_target", [False, True])
def test_bias_update_bit_exact(with_target):
    cfg = TINY
    sh = moe.shape_of(cfg)
    p = make_layer(cfg, DEV)
    x = make_tokens(cfg, DEV)
    idx, w, counts, aff = route(sh, x, p["w_gate"], p["bias"])
    target = None
    if with_target:
        target = torch.linspace(0.0, 0.1, cfg.E, device=DEV, dtype=torch.float32)
    bias = p["bias"].clone()
    load = torch.empty(cfg.E, device=DEV)
    moe.moe_load_and_bias_update(counts, sh, 1e-3, target, bias, load)
    torch.cuda.synchronize()
    check_status()
    ob, ol = oracle.bias_update(counts.cpu().numpy(), p["bias"].cpu().numpy(), cfg.T, cfg.k, 1e-3,
                                None if target is None else target.cpu().numpy())
    assert (bias.cpu().numpy().view(np.uint32) == ob.view(np.uint32)).all()
    assert (load.cpu().numpy().view(np.uint32) == ol.view(np.uint32)).all()
    # step 0: the bias does not move
    b0 = p["bias"].clone()
    moe.moe_load_and_bias_update(counts, sh, 0.0, None, b0, None)
    torch.cuda.synchronize()
    assert torch.equal(b0, p["bias"])


def test_bias_trajectory_small_bf16_ten_steps():
    """small_bf16 balancing loop, 10 steps with fresh tokens per step: the
    bias after every step equals the oracle's bit for bit (injected mode)."""
    cfg = SMALL.scaled(T=1024)  # routing only: full d and E, fewer tokens
    sh = moe.shape_of(cfg)
    p = make_layer(cfg.scaled(I=128, Is=128), DEV)
    bias_gpu = p["bias"].clone()
    bias_orc = p["bias"].cpu().numpy().copy()
    for step in range(SMALL.steps):
        x = make_tokens(cfg, DEV, step)
        idx, w, counts, aff = route(sh, x, p["w_gate"], bias_gpu)
        o_idx, _ = oracle.select(aff.cpu().numpy(), bias_orc, cfg.k)
        assert (idx.cpu().numpy() == o_idx).all()
        o_counts = oracle.histogram(o_idx, cfg.E)
        moe.moe_load_and_bias_update(counts, sh, cfg.step_size, None, bias_gpu)
        torch.cuda.synchronize()
        bias_orc, _ = oracle.bias_update(o_counts, bias_orc, cfg.T, cfg.k, cfg.step_size)
        assert (bias_gpu.cpu().numpy().view(np.uint32) == bias_orc.view(np.uint32)).all(), f"step {step}"
    check_status()


# ----------------------------------------------------------------- permute

@pytest.mark.parametrize("dtype,T,E,k", [("f32", 128, 256, 8), ("bf16", 1000, 64, 6), ("bf16", 1, 16, 4),
                                         ("f32", 300, 7, 7)])
def test_permute_bit_exact(dtype, T, E, k):
    cfg = V3.scaled(T=T, d=128, E=E, k=k, dtype=dtype, I=128, Is=128, S=0)
    sh = moe.shape_of(cfg)
    p = make_layer(cfg, DEV)
    x = make_tokens(cfg, DEV)
    idx, w, counts, _ = route(sh, x, p["w_gate"], p["bias"], with_aff=False)
    x_perm, offsets, perm, inv = permute(sh, x, idx, counts)
    check_status()
    o_off, o_perm, o_inv = oracle.permute(idx.cpu().numpy(), E)
    assert (offsets.cpu().numpy() == o_off).all()
    assert (perm.cpu().numpy() == o_perm).all()
    assert (inv.cpu().numpy() == o_inv).all()
    src = torch.as_tensor(o_perm // k, device=DEV, dtype=torch.long)
    assert torch.equal(x_perm.view(torch.int16 if dtype == "bf16" else torch.int32),
                       x[src].view(torch.int16 if dtype == "bf16" else torch.int32))


def test_permute_reports_inconsistent_counts():
    cfg = TINY.scaled(T=256, E=32, k=4, I=8, Is=8)
    sh = moe.shape_of(cfg)
    p = make_layer(cfg, DEV)
    x = make_tokens(cfg, DEV)
    idx, w, counts, _ = route(sh, x, p["w_gate"], p["bias"], with_aff=False)
    bad = counts.clone()
    bad[3] += 1
    permute(sh, x, idx, bad)
    assert moe.moe_get_last_error() == 6
    assert moe.moe_get_last_error() == 0   # read-and-clear


def test_permute_reports_out_of_range_expert():
    cfg = TINY.scaled(T=128, E=16, k=2, I=8, Is=8)
    sh = moe.shape_of(cfg)
    x = make_tokens(cfg, DEV)
    idx = torch.randint(0, 16, (cfg.T, cfg.k), device=DEV, dtype=torch.int32)
    idx[:, 1] = (idx[:, 0] + 1) % 16
    idx[5, 1] = 99
    counts = torch.bincount(idx.clamp(max=15).flatten().long(), minlength=16).int()
    x_perm, offsets, perm, inv = permute(sh, x, idx, counts)
    assert moe.moe_get_last_error() == 6


# ------------------------------------------------- grouped SwiGLU (experts)

def _group_case(dtype, d, I, S, Is, sizes, seed=0):
    E = len(sizes)
    cfg = V3.scaled(T=sum(sizes), d=d, E=E, k=1, I=I, S=S, Is=Is, dtype=dtype, w_std=0.05)
    p = make_layer(cfg, DEV)
    g = torch.Generator(device=DEV).manual_seed(seed)
    x_perm = torch.randn((sum(sizes), d), generator=g, device=DEV).to(cfg.torch_dtype)
    offsets = torch.tensor(np.concatenate([[0], np.cumsum(sizes)]), dtype=torch.int32, device=DEV)
    return cfg, p, x_perm, offsets


@pytest.mark.parametrize("dtype,d,I,sizes", [
    ("bf16", 256, 128, [300, 0, 1, 128, 129, 7, 0, 255]),   # ragged M tiles, empty groups
    ("bf16", 512, 384, [64, 200, 3]),                       # 3 N tiles of the up projection, 2 of the down
    ("f32", 96, 40, [70, 0, 5, 33]),
])
def test_grouped_swiglu_against_oracle(dtype, d, I, sizes):
    cfg, p, x_perm, offsets = _group_case(dtype, d, I, 0, 128, sizes)
    sh = moe.shape_of(cfg)
    y_perm, _ = grouped_swiglu(sh, x_perm, offsets, p)
    check_status()
    xs = to_numpy(x_perm)
    yacc = np.zeros((xs.shape[0], d), np.float64)
    off = offsets.cpu().numpy()
    for e in range(len(sizes)):
        rows = np.arange(off[e], off[e + 1], dtype=np.int32)
        if len(rows):
            oracle.expert_accumulate(xs[rows], rows, np.ones(len(rows)), to_numpy(p["w1"][e]), to_numpy(p["w3"][e]),
                                     to_numpy(p["w2"][e]), yacc)
    ref = to_f64_rows(oracle.finalize(yacc, xs.dtype))
    err = rel_fro(as_f64(y_perm), ref)
    assert err <= (1e-5 if dtype == "f32" else 5e-3), err


@pytest.mark.parametrize("dtype,S,Is", [("bf16", 2, 256), ("bf16", 1, 128), ("f32", 2, 24)])
def test_shared_experts_against_oracle(dtype, S, Is):
    d = 256 if dtype == "bf16" else 64
    T = 333
    cfg, p, x_perm, offsets = _group_case(dtype, d, 128 if dtype == "bf16" else 16, S, Is, [T])
    sh = moe.shape_of(cfg)
    x = x_perm  # shared experts see the token rows themselves
    _, shared_out = grouped_swiglu(sh, x_perm, offsets, p, x=x)
    check_status()
    xs = to_numpy(x)
    yacc = np.zeros((T, d), np.float64)
    for s in range(S):
        oracle.expert_accumulate(xs, np.arange(T, dtype=np.int32), np.ones(T), to_numpy(p["ws1"][s]),
                                 to_numpy(p["ws3"][s]), to_numpy(p["ws2"][s]), yacc)
    ref = to_f64_rows(oracle.finalize(yacc, xs.dtype))
    err = rel_fro(as_f64(shared_out), ref)
    assert err <= (1e-5 if dtype == "f32" else 5e-3), err


# ----------------------------------------------------------------- combine

@pytest.mark.parametrize("dtype", ["f32", "bf16"])
def test_combine_against_float64(dtype):
    T, k, d = 257, 6, 128
    tdt = torch.float32 if dtype == "f32" else torch.bfloat16
    g = torch.Generator(device=DEV).manual_seed(1)
    y_perm = torch.randn((T * k, d), generator=g, device=DEV).to(tdt)
    shared = torch.randn((T, d), generator=g, device=DEV).to(tdt)
    inv = torch.randperm(T * k, generator=g, device=DEV).to(torch.int32)
    w = torch.rand((T, k), generator=g, device=DEV)
    y = torch.empty((T, d), dtype=tdt, device=DEV)
    sh = moe.MoEShape(T, d, 8, k, 128, 1, 128, moe.MOE_F32 if dtype == "f32" else moe.MOE_BF16)
    moe.moe_combine(y_perm, w, inv, shared, sh, y)
    torch.cuda.synchronize()
    check_status()
    yp = as_f64(y_perm)[inv.cpu().numpy().astype(np.int64)].reshape(T, k, d)
    ref = as_f64(shared) + (w.cpu().numpy().astype(np.float64)[:, :, None] * yp).sum(axis=1)
    err = rel_fro(as_f64(y), ref)
    assert err <= (1e-6 if dtype == "f32" else 4e-3), err


# ------------------------------------------------------------ whole layer

def test_layer_tiny_fp32_full():
    """tiny_fp32 end to end: the oracle recomputes everything from the
    kernel's routing and must agree within 1e-5."""
    cfg = TINY
    sh = moe.shape_of(cfg)
    p = make_layer(cfg, DEV)
    x = make_tokens(cfg, DEV)
    y, idx, w, counts = layer_forward(sh, p, x)
    check_status()
    # routing parity against an independent route call with affinities
    ridx, rw, rcounts, aff = route(sh, x, p["w_gate"], p["bias"])
    assert torch.equal(ridx, idx) and torch.equal(rw, w) and torch.equal(rcounts, counts)
    check_route_parity(x, p["w_gate"], p["bias"], sh.k, idx, w, counts, aff, "auto")
    n = {k_: to_numpy(v) for k_, v in p.items()}
    ref = oracle.layer_output(to_numpy(x), idx.cpu().numpy(), w.cpu().numpy(), n["w1"], n["w3"], n["w2"], n["ws1"],
                              n["ws3"], n["ws2"])
    err = rel_fro(as_f64(y), ref)
    assert err <= 1e-5, err
    # one bias-update step (the workload's single balancing step)
    bias = p["bias"].clone()
    moe.moe_load_and_bias_update(counts, sh, cfg.step_size, None, bias)
    torch.cuda.synchronize()
    ob, _ = oracle.bias_update(counts.cpu().numpy(), p["bias"].cpu().numpy(), cfg.T, cfg.k, cfg.step_size)
    assert (bias.cpu().numpy().view(np.uint32) == ob.view(np.uint32)).all()


@pytest.mark.parametrize("shape", [
    dict(T=512, d=512, E=64, k=6, I=256, S=2, Is=256),     # small_bf16 family, scaled
    dict(T=300, d=256, E=256, k=8, I=128, S=1, Is=128),    # V3 routing fan-out, many near-empty experts
    dict(T=96, d=128, E=8, k=8, I=128, S=0, Is=128),       # k = E, no shared expert
])
def test_layer_bf16_against_oracle(shape):
    cfg = SMALL.scaled(**shape, w_std=0.05, bias_kind="uniform", bias_range=0.02)
    sh = moe.shape_of(cfg)
    p = make_layer(cfg, DEV)
    if cfg.S == 0:
        p["ws1"] = p["ws3"] = p["ws2"] = None
    x = make_tokens(cfg, DEV)
    y, idx, w, counts = layer_forward(sh, p, x)
    check_status()
    ridx, rw, rcounts, aff = route(sh, x, p["w_gate"], p["bias"])
    assert torch.equal(ridx, idx) and torch.equal(rw, w)
    check_route_parity(x, p["w_gate"], p["bias"], sh.k, idx, w, counts, aff, "auto", self_rows=np.arange(64))
    n = {k_: (to_numpy(v) if v is not None else None) for k_, v in p.items()}
    if cfg.S == 0:
        z = np.zeros((0, cfg.Is, cfg.d), np.uint16)
        n["ws1"] = n["ws3"] = z
        n["ws2"] = np.zeros((0, cfg.d, cfg.Is), np.uint16)
    ref = oracle.layer_output(to_numpy(x), idx.cpu().numpy(), w.cpu().numpy(), n["w1"], n["w3"], n["w2"], n["ws1"],
                              n["ws3"], n["ws2"])
    err = rel_fro(as_f64(y), to_f64_rows(ref))
    assert err <= 5e-3, err
    # element by element, every token, against the oracle's down projections and combine of the
    # GPU's own h (the staged calls, bit-identical to the layer)
    x_perm, offsets, perm, inv = permute(sh, x, idx, counts)
    T, k, I, S, Is = cfg.T, cfg.k, cfg.I, cfg.S, cfg.Is
    h = torch.empty((T * k, I), dtype=torch.bfloat16, device=DEV)
    hs = torch.empty((T, max(1, S * Is)), dtype=torch.bfloat16, device=DEV)
    moe.moe_ffn_up(x_perm, offsets, p["w1"], p["w3"], x if S else None, p["ws1"], p["ws3"], sh, h, hs)
    torch.cuda.synchronize()
    y_ref, mag = oracle_terms_from_h(p, h, hs, idx, w, inv, np.arange(T), S)
    check_layer_elementwise(y, y_ref, mag)


def test_layer_is_deterministic():
    cfg = SMALL.scaled(T=700, d=256, E=64, k=6, I=128, S=2, Is=128)
    sh = moe.shape_of(cfg)
    p = make_layer(cfg, DEV)
    x = make_tokens(cfg, DEV)
    a = layer_forward(sh, p, x)
    b = layer_forward(sh, p, x)
    for u, v in zip(a, b):
        assert torch.equal(u.view(torch.uint8) if u.dtype != torch.int32 else u,
                           v.view(torch.uint8) if v.dtype != torch.int32 else v)
    check_status()


@pytest.mark.parametrize("dtype", ["bf16", "f32"])
def test_expert_up_gather_equals_permuted_rows(dtype):
    """moe_expert_up reading token rows through perm_tok (no x_perm copy)
    gives the same h, bit for bit, as reading the permuted copy."""
    cfg = V3.scaled(T=700, d=256 if dtype == "bf16" else 96, E=16, k=4, I=256 if dtype == "bf16" else 40, S=0,
                    dtype=dtype, w_std=0.05)
    sh = moe.shape_of(cfg)
    p = make_layer(cfg, DEV)
    x = make_tokens(cfg, DEV)
    idx, w, counts, _ = route(sh, x, p["w_gate"], p["bias"], with_aff=False)
    x_perm, offsets, perm, inv = permute(sh, x, idx, counts)
    h1 = torch.empty((cfg.T * cfg.k, cfg.I), dtype=x.dtype, device=DEV)
    h2 = torch.empty_like(h1)
    moe.moe_expert_up(x_perm, None, offsets, p["w1"], p["w3"], sh, moe.MOE_ROUTED, h1)
    moe.moe_expert_up(x, perm, offsets, p["w1"], p["w3"], sh, moe.MOE_ROUTED, h2)
    torch.cuda.synchronize()
    check_status()
    bits = torch.int16 if dtype == "bf16" else torch.int32
    assert torch.equal(h1.view(bits), h2.view(bits))


@pytest.mark.parametrize("dtype,S", [("bf16", 2), ("bf16", 0), ("f32", 2)])
def test_ffn_one_launch_per_projection_equals_separate_sets(dtype, S):
    """moe_ffn_up / moe_ffn_down run the routed and the shared set in one
    launch each; every output equals, bit for bit, the per-set calls.  The
    shared set is wider than a routed expert (S*Is = 4 I) and contracts over
    a longer K on the way down, so per-set tile counts and K blocks differ."""
    bf = dtype == "bf16"
    cfg = V3.scaled(T=700, d=256 if bf else 96, E=16, k=4, I=128 if bf else 16, S=S, Is=256 if bf else 24,
                    dtype=dtype, w_std=0.05)
    sh = moe.shape_of(cfg)
    p = make_layer(cfg, DEV)
    x = make_tokens(cfg, DEV)
    idx, w, counts, _ = route(sh, x, p["w_gate"], p["bias"], with_aff=False)
    x_perm, offsets, perm, inv = permute(sh, x, idx, counts)
    rows, SIs = cfg.T * cfg.k, max(1, cfg.S * cfg.Is)
    new = lambda *shape: torch.full(shape, float("nan"), dtype=x.dtype, device=DEV)
    h1, h2 = new(rows, cfg.I), new(rows, cfg.I)
    hs1, hs2 = new(cfg.T, SIs), new(cfg.T, SIs)
    y1, y2 = new(rows, cfg.d), new(rows, cfg.d)
    so1, so2 = new(cfg.T, cfg.d), new(cfg.T, cfg.d)
    xs_ = x if S > 0 else None
    moe.moe_ffn_up(x_perm, offsets, p["w1"], p["w3"], xs_, p["ws1"], p["ws3"], sh, h1, hs1)
    moe.moe_ffn_down(h1, offsets, p["w2"], hs1 if S > 0 else None, p["ws2"], sh, y1, so1)
    moe.moe_expert_up(x_perm, None, offsets, p["w1"], p["w3"], sh, moe.MOE_ROUTED, h2)
    moe.moe_expert_down(h2, offsets, p["w2"], sh, moe.MOE_ROUTED, y2)
    if S > 0:
        moe.moe_expert_up(x, None, None, p["ws1"], p["ws3"], sh, moe.MOE_SHARED, hs2)
        moe.moe_expert_down(hs2, None, p["ws2"], sh, moe.MOE_SHARED, so2)
    torch.cuda.synchronize()
    check_status()
    bits = torch.int16 if bf else torch.int32
    pairs = [(h1, h2), (y1, y2)] + ([(hs1, hs2), (so1, so2)] if S > 0 else [])
    for a, b in pairs:
        assert torch.isfinite(a.float()).all()
        assert torch.equal(a.view(bits), b.view(bits))
    if S == 0:  # the shared buffers are left alone
        assert torch.isnan(hs1.float()).all() and torch.isnan(so1.float()).all()


def test_bounded_wait_times_out_and_context_survives():
    """Failure detection without a fault: a device wait that nothing ends
    gives up after its limit, reports MOE_ERR_TIMEOUT through the status
    word, and the next layer call runs normally."""
    import time
    t0 = time.perf_counter()
    moe.moe_selftest_bounded_wait(50_000)          # 50 ms limit
    assert moe.moe_get_last_error() == 7           # MOE_ERR_TIMEOUT (read and cleared)
    assert time.perf_counter() - t0 < 5.0
    assert moe.moe_get_last_error() == 0
    cfg = SMALL.scaled(T=128, d=256, E=16, k=2, I=128, S=1, Is=128)
    sh = moe.shape_of(cfg)
    p = make_layer(cfg, DEV)
    x = make_tokens(cfg, DEV)
    y, idx, w, counts = layer_forward(sh, p, x)
    check_status()
    assert int(counts.sum()) == cfg.T * cfg.k
    assert torch.isfinite(y.float()).all()


@pytest.mark.parametrize("shape", [
    dict(T=512, d=512, E=64, k=6, I=256, S=2, Is=256),
    dict(T=300, d=256, E=256, k=8, I=128, S=1, Is=128),
    dict(T=96, d=384, E=8, k=8, I=128, S=0, Is=128),       # no shared set; d % 256 == 128
])
def test_down_with_fused_combine_against_oracle(shape):
    """moe_ffn_down_combine + moe_combine_finish (the weighted combine in the
    down projection's epilogue, fp32 additions) against the oracle's layer,
    element by element, and the accumulator left cleared."""
    cfg = SMALL.scaled(**shape, w_std=0.05, bias_kind="uniform", bias_range=0.02)
    sh = moe.shape_of(cfg)
    p = make_layer(cfg, DEV)
    x = make_tokens(cfg, DEV)
    T, k, d, I, S, Is = cfg.T, cfg.k, cfg.d, cfg.I, cfg.S, cfg.Is
    idx, w, counts, _ = route(sh, x, p["w_gate"], p["bias"], with_aff=False)
    x_perm, offsets, perm, inv = permute(sh, x, idx, counts)
    h = torch.empty((T * k, I), dtype=torch.bfloat16, device=DEV)
    hs = torch.empty((T, max(1, S * Is)), dtype=torch.bfloat16, device=DEV)
    moe.moe_ffn_up(x_perm, offsets, p["w1"], p["w3"], x if S else None, p["ws1"], p["ws3"], sh, h, hs)
    acc = torch.zeros((T, d), dtype=torch.float32, device=DEV)
    y = torch.empty((T, d), dtype=torch.bfloat16, device=DEV)
    moe.moe_ffn_down_combine(h, offsets, p["w2"], hs if S else None, p["ws2"], perm, w, sh, acc)
    moe.moe_combine_finish(acc, sh, y)
    torch.cuda.synchronize()
    check_status()
    assert bool((acc == 0).all()), "accumulator not cleared"
    y_ref, mag = oracle_terms_from_h(p, h, hs, idx, w, inv, np.arange(T), S)
    err = check_layer_elementwise(y, y_ref, mag)
    assert err <= 5e-3, err
