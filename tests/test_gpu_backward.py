"""GPU parity of the layer backward (moe_layer_backward) against the backward
oracle (oracle/backward.py, float64), on the same tensors and the same
selection: the kernel's own routing (idx, w, s) is injected into the oracle.

Pages cited (title, section):
  "DeepSeek V3 From Scratch": "In code" (route, renormalised unbiased weights).
  "Scaling Efficiency: A Deep Dive into the DeepSeek-V3 Architecture":
      DeepSeekMoE sketch (shared + weighted routed SwiGLU experts).
  kbwen.com DeepSeek tag page: "A bias term for each expert" (the bias carries
      no gradient; the complementary sequence-wise balance loss).

Bar: every gradient within a relative Frobenius error of 2e-5 (fp32 layer) or
2e-4 (bf16 layer on the fp32 SIMT path) of the oracle's, and elementwise
within 1e-3 of the gradient's largest magnitude.  Inputs are exact in both;
the kernel accumulates in fp32 (relative error ~ K * 2^-24 on the longest
sums, K <= a few hundred here) against the oracle's float64; in bf16 layers
both round the recomputed h to bf16, and an h within fp32 error of a
rounding boundary may land on the other neighbour (2^-8 of one element).
bf16 layers whose widths are multiples of 128 run their contractions on the
tensor cores with bf16 operands: do = w dy, da, dg (and dy for the shared
experts) are rounded to bf16 (relative error up to 2^-9 each, about 1e-3
RMS, carried into every gradient built from them, twice for dx), so there
the bar is the forward's bf16 one: 5e-3 relative Frobenius, elementwise 5e-3
of the largest magnitude.  Gradients of experts no token chose are exactly
zero on both paths.
"""
import numpy as np
import pytest
import torch

import fine_grained_moe_gate_b200 as moe
from fine_grained_moe_gate_b200.inputs import CONFIGS, make_layer, make_tokens, to_numpy
from oracle import backward as ob

from gpu_harness import DEV, check_status, rel_fro, route

pytestmark = pytest.mark.gpu

NAMES = ("dx", "dw_gate", "dw1", "dw3", "dw2", "dws1", "dws3", "dws2")


@pytest.fixture(autouse=True)
def _clean_status():
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    moe.moe_get_last_error()
    yield


def _run(cfg, alpha=0.0, seq_len=0, bias=None):
    sh = moe.shape_of(cfg)
    p = make_layer(cfg, DEV)
    if bias is not None:
        p["bias"] = bias.to(DEV)
    x = make_tokens(cfg, DEV)
    idx, w, counts, aff = route(sh, x, p["w_gate"], p["bias"])
    g = torch.Generator(device=DEV).manual_seed(cfg.seed + 101)
    dy = torch.randn((cfg.T, cfg.d), generator=g, device=DEV)
    T, d, E, I, S, Is = cfg.T, cfg.d, cfg.E, cfg.I, cfg.S, cfg.Is
    f = lambda *s: torch.full(s, float("nan"), device=DEV)  # poisoned: every element must be written
    out = dict(dx=f(T, d), dw_gate=f(E, d), dw1=f(E, I, d), dw3=f(E, I, d), dw2=f(E, d, I),
               dws1=f(S, Is, d) if S else None, dws3=f(S, Is, d) if S else None, dws2=f(S, d, Is) if S else None)
    loss = torch.full((1,), float("nan"), device=DEV)
    ws = torch.empty(max(moe.moe_backward_workspace_size(sh, seq_len if alpha > 0 else 0), 256), dtype=torch.uint8,
                     device=DEV)
    moe.moe_layer_backward(x, p["w_gate"], p["w1"], p["w3"], p["w2"], p["ws1"] if S else None,
                           p["ws3"] if S else None, p["ws2"] if S else None, sh, idx, w, counts, aff, dy, alpha,
                           seq_len, out["dx"], out["dw_gate"], out["dw1"], out["dw3"], out["dw2"], out["dws1"],
                           out["dws3"], out["dws2"], loss, ws)
    torch.cuda.synchronize()
    check_status()
    npx = lambda t: to_numpy(t)
    ref = ob.layer_backward(npx(x), npx(p["w_gate"]), idx.cpu().numpy(), w.cpu().numpy(), aff.cpu().numpy(),
                            npx(p["w1"]), npx(p["w3"]), npx(p["w2"]), npx(p["ws1"]) if S else None,
                            npx(p["ws3"]) if S else None, npx(p["ws2"]) if S else None, dy.cpu().numpy(),
                            alpha=alpha, seq_len=seq_len, round_h="bf16" if cfg.dtype == "bf16" else "f32")
    got = {n: (t.cpu().numpy().astype(np.float64) if t is not None else None) for n, t in out.items()}
    return got, ref, float(loss.item()), idx.cpu().numpy()


def _tensor_cores(c):
    """The tensor-core path: bf16 and every width a multiple of 128."""
    return c["dtype"] == "bf16" and c["d"] % 128 == 0 and c["I"] % 128 == 0 and (c["S"] == 0 or c["Is"] % 128 == 0)


def _tols(c):
    if c["dtype"] == "f32":
        return 2e-5, 1e-3
    return (5e-3, 5e-3) if _tensor_cores(c) else (2e-4, 1e-3)


def _check(got, ref, tol, elem=1e-3):
    for n in NAMES:
        if got[n] is None:
            continue
        g, r = got[n], ref[n]
        assert np.all(np.isfinite(g)), n
        assert rel_fro(g, r) < tol, (n, rel_fro(g, r))
        assert np.max(np.abs(g - r)) <= elem * max(np.max(np.abs(r)), 1e-30), (n, np.max(np.abs(g - r)))


CASES = {
    "bf16_base": dict(dtype="bf16", T=96, d=128, E=8, k=2, I=128, S=1, Is=128),
    "bf16_ragged_two_shared": dict(dtype="bf16", T=200, d=192, E=16, k=4, I=256, S=2, Is=128),
    "bf16_no_shared": dict(dtype="bf16", T=130, d=64, E=12, k=3, I=128, S=0, Is=128),
    "f32": dict(dtype="f32", T=50, d=40, E=6, k=3, I=24, S=1, Is=16),
    # tensor-core path: ragged experts, two shared experts, partial 256-wide tiles
    # (d, I = 384), experts of several 256-row token tiles and 64-row stages
    "tc_ragged_two_shared": dict(dtype="bf16", T=200, d=256, E=16, k=4, I=256, S=2, Is=128),
    "tc_wide": dict(dtype="bf16", T=300, d=384, E=8, k=2, I=384, S=1, Is=256),
    "tc_big_experts": dict(dtype="bf16", T=600, d=256, E=4, k=2, I=256, S=1, Is=128),
    "tc_no_shared": dict(dtype="bf16", T=130, d=128, E=12, k=3, I=128, S=0, Is=128),
}


@pytest.mark.parametrize("name", list(CASES))
@pytest.mark.parametrize("alpha", [0.0, 0.05])
def test_backward_matches_oracle(name, alpha):
    c = CASES[name]
    cfg = CONFIGS["small_bf16"].scaled(name="bwd_" + name, w_std=0.05, bias_kind="uniform", bias_range=0.02, seed=3,
                                       **c)
    L = 10 if c["T"] % 10 == 0 else c["T"]
    got, ref, loss, _ = _run(cfg, alpha=alpha, seq_len=L if alpha > 0 else 0)
    _check(got, ref, *_tols(c))
    if alpha > 0:
        assert abs(loss - ref["balance_loss"]) <= 1e-5 * abs(ref["balance_loss"])
    else:
        assert loss == 0.0


def test_backward_unchosen_experts_get_zero_gradient():
    """A strong bias steers every token to experts 0..3 of 16: the other
    experts' weight gradients are exactly zero, the rest match the oracle."""
    cfg = CONFIGS["small_bf16"].scaled(name="bwd_skew", T=64, d=128, E=16, k=2, I=128, S=1, Is=128, w_std=0.05,
                                       bias_kind="zero", seed=4)
    bias = torch.zeros(16)
    bias[:4] = 10.0
    got, ref, _, idx = _run(cfg, bias=bias)
    assert set(np.unique(idx)) <= {0, 1, 2, 3}
    for n in ("dw1", "dw3", "dw2"):
        assert np.all(got[n][4:] == 0.0), n
    _check(got, ref, *_tols(dict(dtype="bf16", d=128, I=128, S=1, Is=128)))


def test_backward_pages_balance_weight_and_long_sequence():
    """The pages' loss weight 0.0001 over one sequence spanning the batch."""
    cfg = CONFIGS["small_bf16"].scaled(name="bwd_seq", T=256, d=128, E=32, k=4, I=128, S=1, Is=128, w_std=0.05,
                                       bias_kind="uniform", bias_range=0.02, seed=5)
    got, ref, loss, _ = _run(cfg, alpha=1e-4, seq_len=256)
    _check(got, ref, *_tols(dict(dtype="bf16", d=128, I=128, S=1, Is=128)))
    assert abs(loss - ref["balance_loss"]) <= 1e-5 * abs(ref["balance_loss"])


def test_backward_rejects_bad_arguments():
    cfg = CONFIGS["small_bf16"].scaled(name="bwd_args", T=32, d=64, E=8, k=2, I=128, S=0, Is=128, seed=6)
    sh = moe.shape_of(cfg)
    z = torch.zeros(1 << 16, device=DEV)
    ws = torch.empty(moe.moe_backward_workspace_size(sh, 5), dtype=torch.uint8, device=DEV)
    args = [z] * 5 + [None] * 3
    with pytest.raises(moe.MoEError) as ei:   # alpha > 0 with a sequence length that does not divide T
        moe.moe_layer_backward(*args, sh, z, z, z, z, z, 0.1, 5, z, z, z, z, z, None, None, None, z, ws)
    assert ei.value.status == 1
    with pytest.raises(moe.MoEError) as ei:   # workspace too small
        moe.moe_layer_backward(*args, sh, z, z, z, z, z, 0.0, 0, z, z, z, z, z, None, None, None, z, ws[:256])
    assert ei.value.status == 4
