"""Expert parallelism on one GPU: W ranks emulated in one process, their
buffers plain allocations on the same device, the ranks advanced in lock step
through the same staged forward (dist.ep_forward_steps) that the multi-GPU
driver runs.  Page: crackai.dev "DeepSeek-V3", "How It Works" (all-to-all
dispatch/combine kernels).

Bars: every rank's layer output against the CPU oracle's layer over the
ranks' concatenated batch with the ranks' own routing (relative Frobenius
5e-3 bf16 / 1e-5 fp32); and, bit for bit, the single-GPU layer over the same
batch -- the receive buffers hold each expert's rows in the single-GPU
permutation's order, so the same tiles compute the same sums (the
single-GPU kernels are checked element by element in the parity tests).
"""
import numpy as np
import pytest
import torch

import fine_grained_moe_gate_b200 as moe
from fine_grained_moe_gate_b200 import dist as mdist
from fine_grained_moe_gate_b200.inputs import CONFIGS, make_layer, make_tokens

import oracle
from fine_grained_moe_gate_b200.inputs import to_numpy
from gpu_harness import DEV, as_f64, check_status, rel_fro, to_f64_rows

pytestmark = pytest.mark.gpu


@pytest.fixture(autouse=True)
def _clean_status():
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    moe.moe_get_last_error()
    yield


def _run_emulated(cfg, world, p, xs, capacity=None):
    bufs = [mdist.EPBuffers(cfg, world, DEV, capacity=capacity) for _ in range(world)]
    recv_ptrs = [b.recv.data_ptr() for b in bufs]
    back_ptrs = [b.back.data_ptr() for b in bufs]
    gens = []
    for r in range(world):
        pr = dict(p)
        pr.update(mdist.local_experts(p, r, world))
        gens.append(mdist.ep_forward_steps(moe, cfg, r, world, xs[r], pr, bufs[r], recv_ptrs, back_ptrs))
    msgs = [next(g) for g in gens]
    assert all(m[0] == "counts" for m in msgs)
    counts_all = torch.stack([m[1] for m in msgs]).contiguous()        # the all-gather
    msgs = [g.send(counts_all) for g in gens]
    outs = [None] * world
    while any(o is None for o in outs):
        assert all(m is None or m[0] == "barrier" for m in msgs)         # one stream: the barrier is stream order
        nxt = []
        for r, g in enumerate(gens):
            try:
                nxt.append(g.send(None))
            except StopIteration as stop:
                outs[r] = stop.value
                nxt.append(None)
        msgs = nxt
    torch.cuda.synchronize()
    return outs, bufs, counts_all


def _oracle_check(cfg, world, p, xs, bufs, outs):
    """The ranks' outputs against the oracle's layer over the concatenated
    batch, routed by the ranks' own decisions (injected routing)."""
    x = torch.cat(xs)
    idx = torch.cat([b.idx for b in bufs])
    w = torch.cat([b.w for b in bufs])
    got = torch.cat(outs)
    n = {k_: to_numpy(v) for k_, v in p.items()}
    if cfg.S == 0:
        n["ws1"] = n["ws3"] = np.zeros((0, cfg.Is, cfg.d), n["w1"].dtype)
        n["ws2"] = np.zeros((0, cfg.d, cfg.Is), n["w1"].dtype)
    ref = oracle.layer_output(to_numpy(x), idx.cpu().numpy(), w.cpu().numpy(), n["w1"], n["w3"], n["w2"], n["ws1"],
                              n["ws3"], n["ws2"])
    err = rel_fro(as_f64(got), to_f64_rows(ref))
    assert err <= (5e-3 if cfg.dtype == "bf16" else 1e-5), err


def _single_gpu(cfg, world, p, xs, bufs):
    """The single-GPU staged layer over the concatenated batch, routed by the ranks' own decisions."""
    T = cfg.T * world
    big = cfg.scaled(T=T)
    sh = moe.shape_of(big)
    x = torch.cat(xs)
    idx = torch.cat([b.idx for b in bufs])
    w = torch.cat([b.w for b in bufs])
    counts = torch.stack([b.counts for b in bufs]).sum(0).to(torch.int32)
    k, d, E = cfg.k, cfg.d, cfg.E
    x_perm = torch.empty((T * k, d), dtype=x.dtype, device=DEV)
    offsets = torch.empty(E + 1, dtype=torch.int32, device=DEV)
    perm = torch.empty(T * k, dtype=torch.int32, device=DEV)
    inv = torch.empty(T * k, dtype=torch.int32, device=DEV)
    pws = torch.empty(max(moe.moe_permute_workspace_size(sh), 256), dtype=torch.uint8, device=DEV)
    moe.moe_permute(x, idx, counts, sh, x_perm, offsets, perm, inv, pws)
    h = torch.empty((T * k, cfg.I), dtype=x.dtype, device=DEV)
    y_perm = torch.empty((T * k, d), dtype=x.dtype, device=DEV)
    moe.moe_expert_up(x_perm, None, offsets, p["w1"], p["w3"], sh, moe.MOE_ROUTED, h)
    moe.moe_expert_down(h, offsets, p["w2"], sh, moe.MOE_ROUTED, y_perm)
    shared_out = None
    if cfg.S > 0:
        hs = torch.empty((T, cfg.S * cfg.Is), dtype=x.dtype, device=DEV)
        shared_out = torch.empty((T, d), dtype=x.dtype, device=DEV)
        moe.moe_expert_up(x, None, None, p["ws1"], p["ws3"], sh, moe.MOE_SHARED, hs)
        moe.moe_expert_down(hs, None, p["ws2"], sh, moe.MOE_SHARED, shared_out)
    y = torch.empty((T, d), dtype=x.dtype, device=DEV)
    moe.moe_combine(y_perm, w, inv, shared_out, sh, y)
    torch.cuda.synchronize()
    check_status()
    return y


@pytest.mark.parametrize("dtype,world,T,E,k", [("bf16", 4, 96, 16, 4), ("bf16", 2, 333, 8, 2), ("f32", 2, 50, 8, 3),
                                               ("bf16", 8, 40, 8, 4)])
def test_ep_emulated_ranks_equal_single_gpu(dtype, world, T, E, k):
    bf = dtype == "bf16"
    cfg = CONFIGS["small_bf16"].scaled(name="ep_case", T=T, d=256 if bf else 96, E=E, k=k, I=128 if bf else 40, S=1,
                                       Is=128 if bf else 24, dtype=dtype, w_std=0.05, bias_kind="uniform",
                                       bias_range=0.02)
    p = make_layer(cfg, DEV)
    xs = [make_tokens(cfg, DEV, step=r) for r in range(world)]
    outs, bufs, counts_all = _run_emulated(cfg, world, p, xs)
    check_status()
    _oracle_check(cfg, world, p, xs, bufs, outs)
    # every rank received exactly the rows routed to its experts, from everyone
    Epr = E // world
    ca = counts_all.cpu().numpy()
    for o in range(world):
        ro = bufs[o].recv_offsets.cpu().numpy()
        assert ro[-1] == ca[:, o * Epr:(o + 1) * Epr].sum()
    y_single = _single_gpu(cfg, world, p, xs, bufs)
    bits = torch.int16 if bf else torch.int32
    got = torch.cat(outs)
    assert torch.equal(got.view(bits), y_single.view(bits))


def test_ep_skewed_routing_one_rank_gets_most_rows():
    """Most rows go to one rank's experts (a strong bias): the receive
    layout and the return addresses still hold."""
    world = 4
    cfg = CONFIGS["small_bf16"].scaled(name="ep_skew", T=128, d=256, E=16, k=2, I=128, S=0, Is=128, w_std=0.05,
                                       bias_kind="zero")
    p = make_layer(cfg, DEV)
    p["bias"][0:4] = 10.0                      # experts 0-3 (rank 0) win almost every slot
    xs = [make_tokens(cfg, DEV, step=r) for r in range(world)]
    outs, bufs, counts_all = _run_emulated(cfg, world, p, xs)
    check_status()
    assert bufs[0].recv_offsets[-1].item() >= world * cfg.T * cfg.k * 0.9
    _oracle_check(cfg, world, p, xs, bufs, outs)
    y_single = _single_gpu(cfg, world, p, xs, bufs)
    assert torch.equal(torch.cat(outs).view(torch.int16), y_single.view(torch.int16))


def test_ep_receive_capacity_from_balanced_load():
    """Receive buffers of 2*T*k rows instead of W*T*k (mdist.ep_capacity with
    factor 2): enough for a balanced routing; outputs as the oracle's and
    the single-GPU layer's."""
    world = 4
    cfg = CONFIGS["small_bf16"].scaled(name="ep_cap", T=256, d=256, E=16, k=4, I=128, S=1, Is=128, w_std=0.05,
                                       bias_kind="zero")
    p = make_layer(cfg, DEV)
    xs = [make_tokens(cfg, DEV, step=r) for r in range(world)]
    cap = mdist.ep_capacity(cfg, world, 2.0)
    assert cap == 2 * cfg.T * cfg.k < world * cfg.T * cfg.k
    outs, bufs, counts_all = _run_emulated(cfg, world, p, xs, capacity=cap)
    check_status()
    assert all(b.recv.shape[0] == cap and b.h_recv.shape[0] == cap for b in bufs)
    _oracle_check(cfg, world, p, xs, bufs, outs)
    y_single = _single_gpu(cfg, world, p, xs, bufs)
    assert torch.equal(torch.cat(outs).view(torch.int16), y_single.view(torch.int16))


def test_ep_receive_overflow_is_refused_not_dropped():
    """A step whose routing sends more rows to one owner than its receive
    capacity: the plan reports MOE_ERR_DEVICE_CHECK and neither the dispatch
    nor the return stores a row (the return buffers keep their fill)."""
    world = 4
    cfg = CONFIGS["small_bf16"].scaled(name="ep_ovf", T=128, d=256, E=16, k=2, I=128, S=0, Is=128, w_std=0.05,
                                       bias_kind="zero")
    p = make_layer(cfg, DEV)
    p["bias"][0:4] = 10.0                      # rank 0's experts get almost every row: ~W*T*k > 2*T*k
    xs = [make_tokens(cfg, DEV, step=r) for r in range(world)]
    cap = mdist.ep_capacity(cfg, world, 2.0)
    bufs = [mdist.EPBuffers(cfg, world, DEV, capacity=cap) for _ in range(world)]
    for b in bufs:
        b.recv.fill_(-3.0)
        b.back.fill_(-5.0)
    recv_ptrs = [b.recv.data_ptr() for b in bufs]
    back_ptrs = [b.back.data_ptr() for b in bufs]
    gens = []
    for r in range(world):
        pr = dict(p)
        pr.update(mdist.local_experts(p, r, world))
        gens.append(mdist.ep_forward_steps(moe, cfg, r, world, xs[r], pr, bufs[r], recv_ptrs, back_ptrs))
    msgs = [next(g) for g in gens]
    counts_all = torch.stack([m[1] for m in msgs]).contiguous()
    assert counts_all[:, 0:4].sum().item() > cap
    for g in gens:
        assert g.send(counts_all) == ("barrier",)       # dispatch issued (it must store nothing)
    torch.cuda.synchronize()
    assert moe.moe_get_last_error() == 6                 # MOE_ERR_DEVICE_CHECK from the plan
    for b in bufs:
        assert bool((b.recv == -3.0).all()), "a row was stored past the refused plan"
    for g in gens:
        assert g.send(None) == ("barrier",)             # the GEMMs and the return
    torch.cuda.synchronize()
    moe.moe_get_last_error()
    for b in bufs:
        assert bool((b.back == -5.0).all()), "a row was returned under the refused plan"
