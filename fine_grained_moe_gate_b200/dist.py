"""Multi-GPU plumbing of the layer: token-sharded data parallelism.

Every rank holds the full layer (weights replicated) and routes its own share
of the step's tokens; everything on the path is per token except the load
over the whole batch of the step, which the bias update needs (kbwen.com
DeepSeek tag page, "A bias term for each expert": the load is monitored over
the whole batch of the step).  That is the one exchange: the per-expert
counts are summed over the ranks (an all-reduce of E int32 over NCCL) and
every rank then applies the identical update with the global token count, so
the biases stay bit-identical without ever being sent.
"""
from __future__ import annotations

import math

import torch


def shard_step(step: int, rank: int, world: int) -> int:
    """Token-draw index of this rank's shard of step ``step`` (feeds
    ``inputs.make_tokens``); shards of one step never repeat a draw."""
    return step * world + rank


def global_token_count(tokens_per_rank: int, world: int) -> int:
    return tokens_per_rank * world


def allreduce_counts(counts: torch.Tensor, group=None) -> torch.Tensor:
    """Sum the per-expert counts of all ranks in place (no-op on one rank)."""
    import torch.distributed as dist
    if dist.is_available() and dist.is_initialized() and dist.get_world_size(group) > 1:
        dist.all_reduce(counts, op=dist.ReduceOp.SUM, group=group)
    return counts


# ---- backward under token-sharded data parallelism ---------------------------------
#
# Each rank runs moe_layer_backward on its own tokens.  x's gradient stays
# per rank; the weight gradients of the replicated layer are sums over the
# tokens of all ranks, so they are summed over the ranks (the backward's one
# exchange).  The balance loss is a mean over the batch's sequences: with
# every rank holding whole sequences, a rank runs its backward with its share
# of the weight, alpha * (its sequences / all sequences), and the summed
# gradients and losses are then exactly those of the whole batch.

WEIGHT_GRADS = ("dw_gate", "dw1", "dw3", "dw2", "dws1", "dws3", "dws2")


def local_balance_alpha(alpha: float, tokens_per_rank: int, world: int) -> float:
    """The balance-loss weight one rank's backward uses so that the sum over
    the ranks is the batch's loss (equal, whole-sequence shards)."""
    return alpha * tokens_per_rank / global_token_count(tokens_per_rank, world)


def allreduce_grads(grads: dict, group=None) -> dict:
    """Sum the weight gradients (and the balance loss, key 'balance_loss',
    a 1-element tensor) over the ranks in place; other entries (dx) are left
    per rank.  No-op on one rank."""
    import torch.distributed as dist
    if not (dist.is_available() and dist.is_initialized() and dist.get_world_size(group) > 1):
        return grads
    for name in WEIGHT_GRADS + ("balance_loss",):
        t = grads.get(name)
        if t is not None:
            dist.all_reduce(t, op=dist.ReduceOp.SUM, group=group)
    return grads


# ---- expert parallelism ---------------------------------------------------------
#
# Experts sharded over the ranks (rank o owns experts [o*E/W, (o+1)*E/W)),
# tokens kept where they are: each rank routes its own tokens, the step's
# counts are gathered (a few KB), and the token rows travel to the experts'
# owners and the expert outputs back through the library's peer-store
# kernels (moe_ep_dispatch / moe_ep_return) -- no NCCL data all-to-all.

def exchange_counts(counts: torch.Tensor, world: int, group=None) -> torch.Tensor:
    """All ranks' per-expert counts [W][E] (int32), gathered in rank order."""
    import torch.distributed as dist
    out = torch.empty((world, counts.numel()), dtype=counts.dtype, device=counts.device)
    if world == 1:
        out[0].copy_(counts)
        return out
    dist.all_gather_into_tensor(out, counts.reshape(1, -1).contiguous(), group=group)
    return out


def local_experts(p: dict, rank: int, world: int) -> dict:
    """Views of the expert weights rank `rank` owns (contiguous slices)."""
    E = p["w1"].shape[0]
    e0, e1 = rank * E // world, (rank + 1) * E // world
    return {"w1": p["w1"][e0:e1], "w3": p["w3"][e0:e1], "w2": p["w2"][e0:e1]}


def ep_capacity(cfg, world: int, factor: float | None = None) -> int:
    """Rows of every rank's receive buffer.  None: W*T*k, the most that can
    ever arrive (every rank sending all its rows to one owner).  A factor f
    gives ceil(f*T*k) (at most W*T*k): with the bias keeping the load near
    k/E per expert an owner receives about T*k rows per step, so f = 2 leaves
    room for a 2x imbalance; a step that would need more is refused on the
    device (moe_ep_plan) instead of dropping rows."""
    full = world * cfg.T * cfg.k
    if factor is None:
        return full
    return max(1, min(full, int(math.ceil(factor * cfg.T * cfg.k))))


class EPBuffers:
    """One rank's per-step device buffers for ep_forward_steps.  `recv` and
    `back` are the buffers peers store into: allocate them where peers can
    reach them (symmetric memory across GPUs; any allocation on one GPU).
    `capacity` rows (ep_capacity) size the receive buffer and the
    intermediate h of the received rows; the expert outputs overwrite the
    received rows in place (they are read by the up projection only, which
    runs first, and the next step's stores come after this step's return)."""

    def __init__(self, cfg, world: int, device, recv=None, back=None, capacity: int | None = None):
        T, k, d, E, I = cfg.T, cfg.k, cfg.d, cfg.E, cfg.I
        dt = cfg.torch_dtype
        cap = ep_capacity(cfg, world) if capacity is None else int(capacity)
        self.capacity = cap
        i32 = torch.int32
        self.recv = recv if recv is not None else torch.empty((cap, d), dtype=dt, device=device)
        if self.recv.shape[0] < cap:
            raise ValueError(f"receive buffer holds {self.recv.shape[0]} rows, capacity {cap}")
        self.back = back if back is not None else torch.empty((T * k, d), dtype=dt, device=device)
        self.h_recv = torch.empty((cap, I), dtype=dt, device=device)
        self.y_recv = self.recv
        self.idx = torch.empty((T, k), dtype=i32, device=device)
        self.w = torch.empty((T, k), dtype=torch.float32, device=device)
        self.counts = torch.empty(E, dtype=i32, device=device)
        self.offsets = torch.empty(E + 1, dtype=i32, device=device)
        self.perm = torch.empty(T * k, dtype=i32, device=device)
        self.inv = torch.empty(T * k, dtype=i32, device=device)
        self.recv_offsets = torch.empty(E // world + 1, dtype=i32, device=device)
        self.hs = torch.empty((T, max(1, cfg.S * cfg.Is)), dtype=dt, device=device)
        self.shared_out = torch.empty((T, d), dtype=dt, device=device) if cfg.S > 0 else None
        self.y = torch.empty((T, d), dtype=dt, device=device)
        self.flag = torch.zeros(1, dtype=torch.float32, device=device)
        self._pws = None
        self._plan = None

    def scratch(self, moe, sh, world):
        if self._pws is None:
            self._pws = torch.empty(max(moe.moe_permute_workspace_size(sh), 256), dtype=torch.uint8,
                                    device=self.y.device)
            self._plan = torch.empty(max(moe.moe_ep_plan_size(world, sh), 256) // 4, dtype=torch.int32,
                                     device=self.y.device)
        return self._pws, self._plan


def ep_forward_steps(moe, cfg, rank: int, world: int, x, p: dict, bufs: EPBuffers, recv_ptrs, back_ptrs,
                     stream=None):
    """One rank's expert-parallel layer forward, as a generator.

    Yields ("counts", counts) and expects the step's counts of all ranks
    [W][E] to be sent back; yields ("barrier",) where every rank's peer
    stores must be complete before it is resumed.  Returns y [T][d] (the
    generator's value).  p holds the replicated router weights and shared
    experts plus this rank's experts (``local_experts``); recv_ptrs[o] is
    rank o's receive buffer, back_ptrs[s] rank s's return buffer."""
    from . import MoEShape, MOE_SHARED, shape_of
    sh = shape_of(cfg)
    Epr = cfg.E // world
    # the GEMMs on the receive buffer: this rank's experts, rows by offsets,
    # bufs.capacity rows (k = 1 so that the local expert count may be < k)
    sh_local = MoEShape(bufs.capacity, cfg.d, Epr, 1, cfg.I, 0, cfg.Is, sh.dtype)
    pws, plan = bufs.scratch(moe, sh, world)
    moe.moe_route(x, p["w_gate"], p["bias"], sh, bufs.idx, bufs.w, bufs.counts, None, stream)
    counts_all = yield ("counts", bufs.counts)
    moe.moe_permute(x, bufs.idx, bufs.counts, sh, None, bufs.offsets, bufs.perm, bufs.inv, pws, stream)
    moe.moe_ep_plan(counts_all, world, rank, sh, bufs.capacity, plan, bufs.recv_offsets, stream)
    moe.moe_ep_dispatch(x, bufs.perm, plan, world, rank, sh, recv_ptrs, stream)
    yield ("barrier",)
    moe.moe_ffn_up(bufs.recv, bufs.recv_offsets, p["w1"], p["w3"], None, None, None, sh_local, bufs.h_recv, None,
                   stream)
    moe.moe_ffn_down(bufs.h_recv, bufs.recv_offsets, p["w2"], None, None, sh_local, bufs.y_recv, None, stream)
    if cfg.S > 0:
        moe.moe_expert_up(x, None, None, p["ws1"], p["ws3"], sh, MOE_SHARED, bufs.hs, stream)
        moe.moe_expert_down(bufs.hs, None, p["ws2"], sh, MOE_SHARED, bufs.shared_out, stream)
    moe.moe_ep_return(bufs.y_recv, plan, world, rank, sh, back_ptrs, stream)
    yield ("barrier",)
    moe.moe_combine(bufs.back, bufs.w, bufs.inv, bufs.shared_out, sh, bufs.y, stream)
    return bufs.y


def ep_forward(moe, cfg, rank: int, world: int, x, p: dict, bufs: EPBuffers, recv_ptrs, back_ptrs, group=None):
    """ep_forward_steps driven across processes: counts gathered with
    all_gather, barriers as a stream-ordered all-reduce of one float (it
    completes on every rank only after every rank's earlier kernels, so the
    peer stores have landed).  Not run on more than one GPU in this build."""
    import torch.distributed as dist
    gen = ep_forward_steps(moe, cfg, rank, world, x, p, bufs, recv_ptrs, back_ptrs)
    msg = next(gen)
    while True:
        try:
            if msg[0] == "counts":
                msg = gen.send(exchange_counts(msg[1], world, group))
            else:
                dist.all_reduce(bufs.flag, group=group)
                msg = gen.send(None)
        except StopIteration as stop:
            return stop.value


def ep_symmetric_buffers(cfg, world: int, device, group_name: str, capacity: int | None = None):
    """Receive and return buffers in symmetric memory, with every rank's
    device pointers (torch.distributed._symmetric_memory; NVLink peers).
    capacity: receive rows (ep_capacity; default W*T*k).  Returns (recv,
    back, recv_ptrs, back_ptrs).  Not run on more than one GPU in this
    build."""
    import torch.distributed._symmetric_memory as symm_mem
    T, k, d = cfg.T, cfg.k, cfg.d
    cap = ep_capacity(cfg, world) if capacity is None else int(capacity)
    recv = symm_mem.empty((cap, d), dtype=cfg.torch_dtype, device=device)
    back = symm_mem.empty((T * k, d), dtype=cfg.torch_dtype, device=device)
    hr = symm_mem.rendezvous(recv, group_name)
    hb = symm_mem.rendezvous(back, group_name)
    return recv, back, list(hr.buffer_ptrs), list(hb.buffer_ptrs)
