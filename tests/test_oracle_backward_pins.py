"""Pins for the backward oracle (oracle/backward.py), CPU only.

Each check compares the oracle's gradients with something other than its own
formulas: central finite differences of a forward (itself checked against
the C oracle's forward), torch autograd of the same function in float64, a
closed form of the balance loss, and invariants of the renormalised gate.

Pages cited (title, section):
  "DeepSeek V3 From Scratch": "In code" (route, unbiased renormalised weights).
  "Scaling Efficiency: A Deep Dive into the DeepSeek-V3 Architecture":
      DeepSeekMoE sketch (shared + routed experts, weighted combine).
  kbwen.com DeepSeek tag page: "A bias term for each expert" (the
      complementary sequence-wise balance loss, weight 0.0001; its formula
      is not on the pages -- parity unpinned by them).
"""
import numpy as np
import pytest
import torch

import oracle
from oracle import backward as ob


def _problem(T=6, d=8, E=4, k=2, I=6, S=1, Is=4, seed=0, scale=0.4):
    rng = np.random.default_rng(seed)
    p = dict(
        x=rng.normal(size=(T, d)),
        w_gate=rng.normal(size=(E, d)) * scale,
        w1=rng.normal(size=(E, I, d)) * scale,
        w3=rng.normal(size=(E, I, d)) * scale,
        w2=rng.normal(size=(E, d, I)) * scale,
        ws1=rng.normal(size=(S, Is, d)) * scale,
        ws3=rng.normal(size=(S, Is, d)) * scale,
        ws2=rng.normal(size=(S, d, Is)) * scale,
    )
    s = 1.0 / (1.0 + np.exp(-(p["x"] @ p["w_gate"].T)))
    bias = rng.uniform(-0.05, 0.05, size=E)
    idx = np.argsort(-(s + bias), axis=1, kind="stable")[:, :k].astype(np.int32)
    dy = rng.normal(size=(T, d))
    return p, idx, dy


def _objective(p, idx, dy, alpha, L):
    y, s, _ = ob.layer_forward_f64(p["x"], p["w_gate"], idx, p["w1"], p["w3"], p["w2"], p["ws1"], p["ws3"],
                                   p["ws2"])
    val = float((dy * y).sum())
    if alpha > 0:
        val += ob.balance_loss(s, idx, alpha, L)[0]
    return val


def _analytic(p, idx, dy, alpha, L):
    _, s, w = ob.layer_forward_f64(p["x"], p["w_gate"], idx, p["w1"], p["w3"], p["w2"], p["ws1"], p["ws3"],
                                   p["ws2"])
    return ob.layer_backward(p["x"], p["w_gate"], idx, w, s, p["w1"], p["w3"], p["w2"], p["ws1"], p["ws3"],
                             p["ws2"], dy, alpha=alpha, seq_len=L)


def test_forward_restatement_matches_c_oracle():
    """The float64 forward used for the finite differences agrees with the C
    oracle's layer output (fp32 inputs, h rounded to fp32 on both sides)."""
    p, idx, _ = _problem(T=20, d=16, E=6, k=3, I=12, S=2, Is=8, seed=3)
    f32 = {n: v.astype(np.float32) for n, v in p.items()}
    y, s, w = ob.layer_forward_f64(f32["x"], f32["w_gate"], idx, f32["w1"], f32["w3"], f32["w2"], f32["ws1"],
                                   f32["ws3"], f32["ws2"], round_h="f32")
    yc = oracle.layer_output(f32["x"], idx, w.astype(np.float32), f32["w1"], f32["w3"], f32["w2"], f32["ws1"],
                             f32["ws3"], f32["ws2"])
    assert np.max(np.abs(y - yc)) <= 2e-6 * max(1.0, np.max(np.abs(y)))
    sc = oracle.affinity(f32["x"], f32["w_gate"])
    assert np.max(np.abs(s - sc)) < 1e-6


@pytest.mark.parametrize("alpha,L", [(0.0, 0), (0.3, 3), (0.3, 6)])
def test_backward_matches_central_differences(alpha, L):
    p, idx, dy = _problem(seed=1)
    g = _analytic(p, idx, dy, alpha, L)
    rng = np.random.default_rng(7)
    eps = 1e-6
    names = {"x": "dx", "w_gate": "dw_gate", "w1": "dw1", "w3": "dw3", "w2": "dw2", "ws1": "dws1", "ws3": "dws3",
             "ws2": "dws2"}
    for n, gn in names.items():
        for _ in range(6):
            i = tuple(int(rng.integers(0, m)) for m in p[n].shape)
            q = {kk: v.copy() for kk, v in p.items()}
            q[n][i] += eps
            fp = _objective(q, idx, dy, alpha, L)
            q[n][i] -= 2 * eps
            fm = _objective(q, idx, dy, alpha, L)
            fd = (fp - fm) / (2 * eps)
            assert abs(fd - g[gn][i]) <= 1e-6 * max(1.0, abs(fd)), (n, i, fd, g[gn][i])


def test_backward_matches_torch_autograd():
    """Same function written with torch float64 ops, differentiated by autograd."""
    p, idx, dy = _problem(T=9, d=10, E=5, k=3, I=7, S=2, Is=5, seed=2)
    alpha, L = 0.25, 3
    tp = {n: torch.tensor(v, dtype=torch.float64, requires_grad=True) for n, v in p.items()}
    ti = torch.tensor(idx, dtype=torch.long)
    x = tp["x"]
    s = torch.sigmoid(x @ tp["w_gate"].T)
    sel = torch.gather(s, 1, ti)
    w = sel / sel.sum(1, keepdim=True)
    y = torch.zeros_like(x)
    for j in range(tp["ws1"].shape[0]):
        y = y + (torch.nn.functional.silu(x @ tp["ws1"][j].T) * (x @ tp["ws3"][j].T)) @ tp["ws2"][j].T
    for t in range(x.shape[0]):
        for j in range(idx.shape[1]):
            e = int(idx[t, j])
            hh = torch.nn.functional.silu(tp["w1"][e] @ x[t]) * (tp["w3"][e] @ x[t])
            y = y.index_add(0, torch.tensor([t]), (w[t, j] * (tp["w2"][e] @ hh))[None])
    T, E = s.shape
    k = idx.shape[1]
    bal = 0.0
    for b in range(T // L):
        sb = s[b * L:(b + 1) * L]
        cnt = torch.zeros(E, dtype=torch.float64).index_add(0, ti[b * L:(b + 1) * L].reshape(-1),
                                                             torch.ones(L * k, dtype=torch.float64))
        f = cnt * E / (k * L)
        P = (sb / sb.sum(1, keepdim=True)).mean(0)
        bal = bal + alpha * (f * P).sum()
    obj = (torch.tensor(dy) * y).sum() + bal / (T // L)
    obj.backward()
    g = _analytic(p, idx, dy, alpha, L)
    for n, gn in (("x", "dx"), ("w_gate", "dw_gate"), ("w1", "dw1"), ("w3", "dw3"), ("w2", "dw2"),
                  ("ws1", "dws1"), ("ws3", "dws3"), ("ws2", "dws2")):
        ref = tp[n].grad.numpy()
        assert np.allclose(g[gn], ref, rtol=1e-10, atol=1e-12), n
    assert abs(g["balance_loss"] - float(bal.detach()) / (T // L)) < 1e-12


def test_balance_loss_uniform_affinities_closed_form():
    """All affinities equal: P_i = 1/E, sum_i f_i = E, so the loss is alpha
    and ds_ti = alpha / (nb L) * (f_i - 1) / (E c)."""
    T, E, k, L, c, alpha = 12, 8, 2, 4, 0.3, 0.01
    rng = np.random.default_rng(4)
    idx = np.stack([rng.choice(E, size=k, replace=False) for _ in range(T)]).astype(np.int32)
    s = np.full((T, E), c)
    loss, ds = ob.balance_loss(s, idx, alpha, L)
    assert abs(loss - alpha) < 1e-15
    nb = T // L
    for b in range(nb):
        cnt = np.bincount(idx[b * L:(b + 1) * L].ravel(), minlength=E)
        f = cnt * E / (k * L)
        expect = alpha / (nb * L) * (f - 1.0) / (E * c)
        assert np.allclose(ds[b * L:(b + 1) * L], expect[None, :], rtol=1e-12, atol=1e-15)


def test_renormalised_gate_is_scale_invariant():
    """w depends on the chosen scores only up to a common factor, so the
    gradient through the renormalisation is orthogonal to them:
    sum_j ds_{t,idx_j} s_{t,idx_j} = 0 for every token (no balance loss)."""
    p, idx, dy = _problem(T=10, E=6, k=3, seed=5)
    g = _analytic(p, idx, dy, 0.0, 0)
    _, s, _ = ob.layer_forward_f64(p["x"], p["w_gate"], idx, p["w1"], p["w3"], p["w2"], p["ws1"], p["ws3"], p["ws2"])
    dot = (np.take_along_axis(g["ds"], idx, 1) * np.take_along_axis(s, idx, 1)).sum(1)
    assert np.max(np.abs(dot)) < 1e-12
    # and unchosen experts get no gradient from the combine
    mask = np.ones_like(s, bool)
    np.put_along_axis(mask, idx, False, 1)
    assert np.all(g["ds"][mask] == 0.0)


def test_single_expert_gate_gets_no_gradient():
    """E = k = 1: the weight is identically 1, so the gate weights get exactly
    zero gradient and dx is the plain SwiGLU-MLP input gradient."""
    p, idx, dy = _problem(T=5, d=6, E=1, k=1, I=4, S=1, Is=3, seed=6)
    g = _analytic(p, idx, dy, 0.0, 0)
    assert np.all(g["dw_gate"] == 0.0)
    x = torch.tensor(p["x"], requires_grad=True)

    def mlp(w1, w3, w2):
        return (torch.nn.functional.silu(x @ torch.tensor(w1).T) * (x @ torch.tensor(w3).T)) @ torch.tensor(w2).T

    y = mlp(p["w1"][0], p["w3"][0], p["w2"][0]) + mlp(p["ws1"][0], p["ws3"][0], p["ws2"][0])
    (torch.tensor(dy) * y).sum().backward()
    assert np.allclose(g["dx"], x.grad.numpy(), rtol=1e-11, atol=1e-13)


def test_backward_is_linear_in_dy():
    p, idx, dy = _problem(seed=8)
    dy2 = np.random.default_rng(9).normal(size=dy.shape)
    g1, g2, g12 = (_analytic(p, idx, v, 0.0, 0) for v in (dy, dy2, dy + dy2))
    for n in ("dx", "dw_gate", "dw1", "dw3", "dw2", "dws1", "dws3", "dws2"):
        assert np.allclose(g12[n], g1[n] + g2[n], rtol=1e-10, atol=1e-12), n
