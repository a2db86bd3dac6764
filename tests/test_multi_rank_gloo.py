"""The multi-GPU path's host logic on CPU with world size 2 (gloo): token
shards per rank, the one exchange (per-expert counts summed over ranks) and
the bias update with the global token count ("A bias term for each expert":
the load is taken over the whole batch of the step).  The oracle stands in
for the per-rank kernels, which need a GPU."""
import datetime
import json
import os
import socket
import tempfile

import numpy as np
import pytest
import torch
import torch.multiprocessing as mp

WORLD = 2
STEPS = 3


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _cfg():
    from fine_grained_moe_gate_b200.inputs import CONFIGS
    return CONFIGS["tiny_fp32"].scaled(T=48, d=64, E=32, k=4, I=8, Is=8)


def _worker(rank, port, out_dir, fail_rank):
    import torch.distributed as dist

    import oracle
    from fine_grained_moe_gate_b200 import dist as mdist
    from fine_grained_moe_gate_b200.inputs import make_layer, make_tokens, to_numpy

    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=WORLD, timeout=datetime.timedelta(seconds=10))
    cfg = _cfg()
    p = make_layer(cfg, "cpu")                      # same seed on every rank: replicated weights
    wg = to_numpy(p["w_gate"])
    bias = p["bias"].numpy().copy()
    result = {"rank": rank, "biases": [], "error": None}
    try:
        for step in range(STEPS):
            x = make_tokens(cfg, "cpu", step=mdist.shard_step(step, rank, WORLD))
            s = oracle.affinity(to_numpy(x), wg)
            idx, _ = oracle.select(s, bias, cfg.k)
            counts = torch.from_numpy(oracle.histogram(idx, cfg.E))
            if rank == fail_rank:
                raise RuntimeError("injected host-side failure before the exchange")
            mdist.allreduce_counts(counts)
            bias, _ = oracle.bias_update(counts.numpy(), bias, mdist.global_token_count(cfg.T, WORLD), cfg.k,
                                         cfg.step_size)
            result["biases"].append(bias.view(np.uint32).tolist())
    except Exception as e:  # reported to the parent, never hangs the test
        result["error"] = f"{type(e).__name__}: {e}"
    with open(os.path.join(out_dir, f"rank{rank}.json"), "w") as f:
        json.dump(result, f)
    try:
        dist.destroy_process_group()
    except Exception:
        pass


def _run(fail_rank):
    out_dir = tempfile.mkdtemp(prefix="gloo_")
    mp.start_processes(_worker, args=(_free_port(), out_dir, fail_rank), nprocs=WORLD, join=True,
                       start_method="spawn")
    return [json.load(open(os.path.join(out_dir, f"rank{r}.json"))) for r in range(WORLD)]


def test_two_ranks_keep_identical_bias_equal_to_single_process():
    import oracle
    from fine_grained_moe_gate_b200 import dist as mdist
    from fine_grained_moe_gate_b200.inputs import make_layer, make_tokens, to_numpy

    res = _run(fail_rank=-1)
    for r in res:
        assert r["error"] is None, r["error"]
    assert res[0]["biases"] == res[1]["biases"]     # bit-identical on every rank, every step
    # single process over the concatenated batch of each step
    cfg = _cfg()
    p = make_layer(cfg, "cpu")
    wg = to_numpy(p["w_gate"])
    bias = p["bias"].numpy().copy()
    for step in range(STEPS):
        x = torch.cat([make_tokens(cfg, "cpu", step=mdist.shard_step(step, r, WORLD)) for r in range(WORLD)])
        idx, _ = oracle.select(oracle.affinity(to_numpy(x), wg), bias, cfg.k)
        bias, _ = oracle.bias_update(oracle.histogram(idx, cfg.E), bias, x.shape[0], cfg.k, cfg.step_size)
        assert bias.view(np.uint32).tolist() == res[0]["biases"][step], f"step {step}"


def test_a_failed_rank_ends_the_exchange_with_an_error_not_a_hang():
    res = _run(fail_rank=1)
    assert "injected" in res[1]["error"]
    assert res[0]["error"] is not None             # the survivor's all-reduce errored out within the timeout
    assert len(res[0]["biases"]) == 0


def _ep_worker(rank, port, out_dir):
    import torch.distributed as dist

    import oracle
    from fine_grained_moe_gate_b200 import dist as mdist
    from fine_grained_moe_gate_b200.inputs import make_layer, make_tokens, to_numpy

    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=WORLD, timeout=datetime.timedelta(seconds=10))
    cfg = _cfg()
    p = make_layer(cfg, "cpu")
    x = make_tokens(cfg, "cpu", step=mdist.shard_step(0, rank, WORLD))
    idx, _ = oracle.select(oracle.affinity(to_numpy(x), to_numpy(p["w_gate"])), p["bias"].numpy(), cfg.k)
    counts = torch.from_numpy(oracle.histogram(idx, cfg.E))
    allc = mdist.exchange_counts(counts, WORLD)
    with open(os.path.join(out_dir, f"ep{rank}.json"), "w") as f:
        json.dump({"counts_all": allc.tolist(), "own": counts.tolist()}, f)
    dist.destroy_process_group()


def test_expert_parallel_counts_exchange():
    """Expert parallelism's one host-side exchange: every rank ends with the
    same [W][E] counts in rank order, from which each owner's receive size
    (its experts' columns summed over the sources) follows."""
    out_dir = tempfile.mkdtemp(prefix="gloo_ep_")
    mp.start_processes(_ep_worker, args=(_free_port(), out_dir), nprocs=WORLD, join=True, start_method="spawn")
    res = [json.load(open(os.path.join(out_dir, f"ep{r}.json"))) for r in range(WORLD)]
    assert res[0]["counts_all"] == res[1]["counts_all"]
    assert res[0]["counts_all"] == [res[r]["own"] for r in range(WORLD)]
    cfg = _cfg()
    allc = np.array(res[0]["counts_all"])
    Epr = cfg.E // WORLD
    recv = [allc[:, o * Epr:(o + 1) * Epr].sum() for o in range(WORLD)]
    assert sum(recv) == WORLD * cfg.T * cfg.k


# ---- backward under token-sharded data parallelism

def _bwd_cfg():
    from fine_grained_moe_gate_b200.inputs import CONFIGS
    return CONFIGS["tiny_fp32"].scaled(T=12, d=16, E=8, k=2, I=8, S=1, Is=8)


BWD_ALPHA, BWD_SEQ = 0.05, 4


def _bwd_grads(cfg, x, p, alpha):
    """Oracle backward (stands in for moe_layer_backward) of one rank's tokens."""
    import oracle
    from oracle import backward as ob
    from fine_grained_moe_gate_b200.inputs import to_numpy

    xn = to_numpy(x)
    s = oracle.affinity(xn, to_numpy(p["w_gate"]))
    idx, w = oracle.select(s, p["bias"].numpy(), cfg.k)
    g = torch.Generator().manual_seed(int(x.sum().abs().item() * 1000) % (1 << 31))
    dy = torch.randn((x.shape[0], cfg.d), generator=g, dtype=torch.float64).numpy()
    out = ob.layer_backward(xn, to_numpy(p["w_gate"]), idx, w, s, *[to_numpy(p[n]) for n in
                            ("w1", "w3", "w2", "ws1", "ws3", "ws2")], dy, alpha=alpha, seq_len=BWD_SEQ)
    return out, dy


def _bwd_worker(rank, port, out_dir):
    import torch.distributed as dist

    from fine_grained_moe_gate_b200 import dist as mdist
    from fine_grained_moe_gate_b200.inputs import make_layer, make_tokens

    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=WORLD, timeout=datetime.timedelta(seconds=10))
    cfg = _bwd_cfg()
    p = make_layer(cfg, "cpu")
    x = make_tokens(cfg, "cpu", step=mdist.shard_step(0, rank, WORLD))
    out, _ = _bwd_grads(cfg, x, p, mdist.local_balance_alpha(BWD_ALPHA, cfg.T, WORLD))
    grads = {n: torch.from_numpy(np.ascontiguousarray(out[n])) for n in mdist.WEIGHT_GRADS}
    grads["balance_loss"] = torch.tensor([out["balance_loss"]], dtype=torch.float64)
    mdist.allreduce_grads(grads)
    np.savez(os.path.join(out_dir, f"bwd{rank}.npz"), dx=out["dx"], **{n: t.numpy() for n, t in grads.items()})
    dist.destroy_process_group()


def test_backward_data_parallel_equals_whole_batch():
    """Two ranks, each with its own tokens: after the weight-gradient
    all-reduce every rank holds the whole batch's weight gradients and
    balance loss, and each rank's dx is the whole batch's dx for its rows."""
    from fine_grained_moe_gate_b200 import dist as mdist
    from fine_grained_moe_gate_b200.inputs import make_layer, make_tokens

    out_dir = tempfile.mkdtemp(prefix="gloo_bwd_")
    mp.start_processes(_bwd_worker, args=(_free_port(), out_dir), nprocs=WORLD, join=True, start_method="spawn")
    res = [dict(np.load(os.path.join(out_dir, f"bwd{r}.npz"))) for r in range(WORLD)]
    cfg = _bwd_cfg()
    p = make_layer(cfg, "cpu")
    xs = [make_tokens(cfg, "cpu", step=mdist.shard_step(0, r, WORLD)) for r in range(WORLD)]
    # the whole batch in one process: same tokens, same per-rank dy, the batch's alpha
    import oracle
    from oracle import backward as ob
    from fine_grained_moe_gate_b200.inputs import to_numpy
    dys = [_bwd_grads(cfg, x, p, 0.0)[1] for x in xs]
    x = torch.cat(xs)
    s = oracle.affinity(to_numpy(x), to_numpy(p["w_gate"]))
    idx, w = oracle.select(s, p["bias"].numpy(), cfg.k)
    ref = ob.layer_backward(to_numpy(x), to_numpy(p["w_gate"]), idx, w, s, *[to_numpy(p[n]) for n in
                            ("w1", "w3", "w2", "ws1", "ws3", "ws2")], np.concatenate(dys), alpha=BWD_ALPHA,
                            seq_len=BWD_SEQ)
    for r in range(WORLD):
        for n in mdist.WEIGHT_GRADS:
            assert np.allclose(res[r][n], ref[n], rtol=1e-12, atol=1e-14), (r, n)
        assert abs(float(res[r]["balance_loss"][0]) - ref["balance_loss"]) < 1e-14
        assert np.allclose(res[r]["dx"], ref["dx"][r * cfg.T:(r + 1) * cfg.T], rtol=1e-12, atol=1e-14)
