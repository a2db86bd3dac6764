"""GPU parity at the workloads' full sizes, through moe_layer_forward (the
call the bench times): routing, counts and the bias step are checked for
every token (injected mode), the kernel's affinities and the layer output on
sampled tokens the oracle computes one by one."""
import numpy as np
import pytest
import torch

import fine_grained_moe_gate_b200 as moe
import oracle
from fine_grained_moe_gate_b200.inputs import CONFIGS, make_layer, make_tokens

from gpu_harness import (DEV, as_f64, check_route_parity, check_status, layer_forward, oracle_rows, rel_fro, route,
                         to_f64_rows)

pytestmark = pytest.mark.gpu


def _full_check(cfg, p, x, n_sample, seed, s_tol="auto"):
    sh = moe.shape_of(cfg)
    y, idx, w, counts = layer_forward(sh, p, x)
    check_status()
    ridx, rw, rcounts, aff = route(sh, x, p["w_gate"], p["bias"])
    assert torch.equal(ridx, idx) and torch.equal(rw, w) and torch.equal(rcounts, counts)
    rng = np.random.default_rng(seed)
    rows = np.sort(rng.choice(cfg.T, size=min(64, cfg.T), replace=False))
    check_route_parity(x, p["w_gate"], p["bias"], cfg.k, idx, w, counts, aff, s_tol, self_rows=rows)
    assert int(counts.sum()) == cfg.T * cfg.k       # no dropped tokens
    tokens = np.sort(rng.choice(cfg.T, size=n_sample, replace=False))
    ref = to_f64_rows(oracle_rows(p, x, idx, w, tokens, cfg.S))
    got = as_f64(y[torch.as_tensor(tokens, device=DEV)])
    err = rel_fro(got, ref)
    assert err <= 5e-3, err
    return y, idx, w, counts


@pytest.fixture(scope="module")
def v3_layer():
    cfg = CONFIGS["v3_prefill"]
    p = make_layer(cfg, DEV)
    yield cfg, p
    del p
    torch.cuda.empty_cache()


def test_v3_prefill_full(v3_layer):
    cfg, p = v3_layer
    x = make_tokens(cfg, DEV)
    _full_check(cfg, p, x, n_sample=6, seed=2)


def test_v3_decode_calls(v3_layer):
    """T=64 per call with fresh tokens each call (calls 0, 1 and 999)."""
    cfg_p, p = v3_layer
    cfg = CONFIGS["v3_decode"]
    for call in (0, 1, 999):
        x = make_tokens(cfg, DEV, call)
        _full_check(cfg, p, x, n_sample=4, seed=call)


def test_small_bf16_full_and_ten_steps():
    cfg = CONFIGS["small_bf16"]
    sh = moe.shape_of(cfg)
    p = make_layer(cfg, DEV)
    bias0 = p["bias"].clone()
    bias_orc = p["bias"].cpu().numpy().copy()
    for step in range(cfg.steps):
        x = make_tokens(cfg, DEV, step)
        if step in (0, cfg.steps - 1):
            y, idx, w, counts = _full_check(cfg, p, x, n_sample=24, seed=step)
        else:
            y, idx, w, counts = layer_forward(sh, p, x)
        ridx, rw, rc, aff = route(sh, x, p["w_gate"], p["bias"])
        o_idx, _ = oracle.select(aff.cpu().numpy(), bias_orc, cfg.k)
        assert (o_idx == idx.cpu().numpy()).all()
        moe.moe_load_and_bias_update(counts, sh, cfg.step_size, None, p["bias"])
        torch.cuda.synchronize()
        bias_orc, _ = oracle.bias_update(oracle.histogram(o_idx, cfg.E), bias_orc, cfg.T, cfg.k, cfg.step_size)
        assert (p["bias"].cpu().numpy().view(np.uint32) == bias_orc.view(np.uint32)).all(), f"step {step}"
    assert not torch.equal(bias0, p["bias"])
    check_status()


def test_skew_stress_routing_and_sampled_output():
    """Zipf-skewed popularity: head experts get thousands of rows (many M
    tiles); five bias steps bit-exact, output on sampled tokens."""
    cfg = CONFIGS["skew_stress"]
    sh = moe.shape_of(cfg)
    p = make_layer(cfg, DEV)
    bias_orc = p["bias"].cpu().numpy().copy()
    for step in range(5):
        x = make_tokens(cfg, DEV, step)
        if step == 0:
            y, idx, w, counts = _full_check(cfg, p, x, n_sample=3, seed=4)
            c = counts.cpu().numpy()
            assert c.max() > 8 * c.mean()    # the workload really is skewed
        else:
            y, idx, w, counts = layer_forward(sh, p, x)
        _, _, _, aff = route(sh, x, p["w_gate"], p["bias"])
        o_idx, _ = oracle.select(aff.cpu().numpy(), bias_orc, cfg.k)
        assert (o_idx == idx.cpu().numpy()).all()
        moe.moe_load_and_bias_update(counts, sh, cfg.step_size, None, p["bias"])
        torch.cuda.synchronize()
        bias_orc, _ = oracle.bias_update(oracle.histogram(o_idx, cfg.E), bias_orc, cfg.T, cfg.k, cfg.step_size)
        assert (p["bias"].cpu().numpy().view(np.uint32) == bias_orc.view(np.uint32)).all()
    check_status()
