"""Pins for the CPU oracle: each check compares it with something other than
itself -- brute force, library routines on special cases, closed forms, the
pages' worked example, or invariants the pages state.  CPU only.

Pages cited (title, section):
  "DeepSeek V3 From Scratch": "The idea", "Worked example", "In code".
  "Scaling Efficiency: A Deep Dive into the DeepSeek-V3 Architecture":
      DeepSeekMoE sketch (shared + routed, weighted combine).
  kbwen.com DeepSeek tag page: "A bias term for each expert".
"""
import itertools
import json
import os

import numpy as np
import pytest
import torch

import oracle

HERE = os.path.dirname(os.path.abspath(__file__))
F32_EPS = 2.0 ** -24


# ---------------------------------------------------------------- selection

def _brute_force_topk(v, k):
    """Best k-subset by total score; equal totals broken by the
    lexicographically smallest sorted index list."""
    best, best_key = None, None
    for sub in itertools.combinations(range(len(v)), k):
        total = sum(float(v[i]) for i in sub)   # dyadic values: exact
        key = (-total, sub)
        if best_key is None or key < best_key:
            best, best_key = sub, key
    return set(best)


@pytest.mark.parametrize("E", [1, 2, 3, 5, 8, 12])
def test_select_brute_force_with_ties(oracle_lib, E):
    """Selection = the best-scoring k-subset (brute force over all C(E,k)),
    ties to lower expert index; slots in descending score, equal scores by
    ascending index ("In code", route: topk on affinity + bias)."""
    rng = np.random.default_rng(100 + E)
    for k in range(1, min(4, E) + 1):
        for _ in range(40):
            T = 3
            # dyadic affinities in (0,1) and dyadic biases: fp32 sums exact,
            # and few distinct values so ties are frequent
            s = (rng.integers(1, 8, size=(T, E)) / 8.0).astype(np.float32)
            b = (rng.integers(-2, 3, size=E) / 16.0).astype(np.float32)
            idx, w = oracle.select(s, b, k)
            v = s + b
            for t in range(T):
                assert set(idx[t].tolist()) == _brute_force_topk(v[t], k)
                for j in range(k - 1):
                    a, c = idx[t, j], idx[t, j + 1]
                    assert v[t, a] > v[t, c] or (v[t, a] == v[t, c] and a < c)


def test_select_matches_torch_topk_tie_free(oracle_lib):
    """Tie-free scores: the oracle's slots equal torch.topk(s + b) (sorted)."""
    g = torch.Generator().manual_seed(5)
    T, E, k = 64, 256, 8
    s = torch.rand((T, E), generator=g, dtype=torch.float32) * 0.9 + 0.05
    b = (torch.rand(E, generator=g, dtype=torch.float32) - 0.5) * 0.1
    idx, _ = oracle.select(s.numpy(), b.numpy(), k)
    ref = torch.topk(s + b, k, dim=-1).indices.numpy()
    assert (idx == ref).all()


def test_select_no_bias_equals_topk_of_logits(oracle_lib):
    """b = 0: sigmoid is monotone, so the route equals topk of x @ W_g^T."""
    rng = np.random.default_rng(7)
    x = rng.standard_normal((32, 48)).astype(np.float32)
    wg = (rng.standard_normal((40, 48)) * 0.3).astype(np.float32)
    w, idx, s = oracle.route(x, wg, np.zeros(40, np.float32), 5)
    logits = torch.from_numpy(x.astype(np.float64)) @ torch.from_numpy(wg.astype(np.float64)).T
    ref = torch.topk(logits, 5, dim=-1).indices.numpy()
    assert (idx == ref).all()


# ------------------------------------------------------------------ weights

def test_weights_definition_and_sum(oracle_lib):
    """Weights are the unbiased affinities of the chosen k renormalised to
    sum to 1 ("The idea"; "In code": weights / weights.sum())."""
    rng = np.random.default_rng(11)
    T, E, k = 200, 64, 6
    s = rng.uniform(0.01, 0.99, size=(T, E)).astype(np.float32)
    b = rng.uniform(-0.05, 0.05, size=E).astype(np.float32)
    idx, w = oracle.select(s, b, k)
    assert (w > 0).all()
    sel = np.take_along_axis(s, idx, axis=1).astype(np.float64)
    exact = sel / sel.sum(axis=1, keepdims=True)
    assert np.all(np.abs(w - exact) <= 3 * F32_EPS * exact)
    assert np.all(np.abs(w.astype(np.float64).sum(axis=1) - 1.0) <= k * F32_EPS * 2)
    for t in range(T):
        assert len(set(idx[t].tolist())) == k


def test_bias_affects_selection_only(oracle_lib):
    """Changing the bias of experts that stay unselected leaves every
    weight bit-identical ("The idea": the bias acts only on which experts
    are selected; "A bias term for each expert")."""
    rng = np.random.default_rng(12)
    T, E, k = 6, 64, 4
    s = rng.uniform(0.05, 0.95, size=(T, E)).astype(np.float32)
    b1 = np.zeros(E, np.float32)
    idx1, w1 = oracle.select(s, b1, k)
    never = np.setdiff1d(np.arange(E), np.unique(idx1))
    assert len(never) > 0
    b2 = b1.copy()
    b2[never] = -0.5          # pushes unselected experts further down
    idx2, w2 = oracle.select(s, b2, k)
    assert (idx1 == idx2).all()
    assert (w1.view(np.uint32) == w2.view(np.uint32)).all()
    # a bias that does reorder the selected set changes the slots, but the
    # weight of each selected expert is still its own s over the same sum
    b3 = b1.copy()
    b3[idx1[:, 0]] = 0.0
    b3[idx1[:, -1]] = 0.6     # the slot-(k-1) expert of each row jumps up
    idx3, w3 = oracle.select(s, b3, k)
    for t in range(T):
        if set(idx3[t]) == set(idx1[t]):
            m1 = dict(zip(idx1[t].tolist(), w1[t].tolist()))
            m3 = dict(zip(idx3[t].tolist(), w3[t].tolist()))
            for e in m1:
                assert abs(m1[e] - m3[e]) <= 2 * F32_EPS * m1[e]


# ----------------------------------------------------------- worked example

def test_worked_example(oracle_lib):
    """Rank-9 expert with bias +0.05 joins the top 8; one update pushes its
    bias down and it drops out again ("Worked example"; "In code",
    update_bias with step 1e-3)."""
    with open(os.path.join(HERE, "golden", "worked_example.json")) as f:
        ex = json.load(f)
    E, k, e12, step = ex["E"], ex["k"], ex["expert"], ex["step"]
    rng = np.random.default_rng(27)
    T = 16
    # one token pattern repeated over the batch: eight experts above expert
    # 12, expert 12 ninth, 0.0495 below the eighth, the rest far below
    base = rng.uniform(0.05, 0.30, size=E).astype(np.float32)
    top = [3, 40, 77, 100, 150, 180, 200, 250]
    vals = [0.90, 0.86, 0.82, 0.78, 0.74, 0.70, 0.66, 0.62]
    for e, v in zip(top, vals):
        base[e] = v
    base[e12] = np.float32(0.62 - 0.0495)
    s = np.tile(base, (T, 1))
    order = np.argsort(-base, kind="stable")
    assert int(np.where(order == e12)[0][0]) + 1 == ex["unbiased_rank_1based"]

    bias0 = np.zeros(E, np.float32)
    idx0, _ = oracle.select(s, bias0, k)
    assert (e12 in idx0[0]) == ex["expect"]["selected_without_bias"]

    bias = bias0.copy()
    bias[e12] = np.float32(ex["bias"])
    idx1, w1 = oracle.select(s, bias, k)
    assert (e12 in idx1[0]) == ex["expect"]["selected_with_bias"]
    assert top[-1] not in idx1[0]                # the former eighth drops out
    assert list(idx1[0]).index(e12) == k - 1     # it enters at the last slot
    assert abs(float(w1[0].astype(np.float64).sum()) - 1.0) <= k * F32_EPS * 2
    j = list(idx1[0]).index(e12)
    exact = float(s[0, e12]) / s[0, idx1[0]].astype(np.float64).sum()   # unbiased s
    assert abs(float(w1[0, j]) - exact) <= 3 * F32_EPS * exact

    counts = oracle.histogram(idx1, E)
    new_bias, load = oracle.bias_update(counts, bias, T, k, step)
    direction = np.sign(float(new_bias[e12]) - float(bias[e12]))
    assert direction == ex["expect"]["bias_direction_after_update"]
    assert new_bias[e12] == np.float32(np.float32(ex["bias"]) - np.float32(step))
    idx2, _ = oracle.select(s, new_bias, k)
    assert e12 not in idx2[0]


# -------------------------------------------------------------- bias update

@pytest.mark.parametrize("T,E,k", [(128, 256, 8), (4096, 64, 6), (64, 16, 2)])
def test_bias_update_closed_form(oracle_lib, T, E, k):
    """b_new = b + step * sign(k/E - c/T), a fixed +-step, 0 at equality
    ("In code", update_bias; "A bias term for each expert").  T, E are
    powers of two here, so the fp32 comparison is the exact integer one
    sign(k*T - E*c)."""
    rng = np.random.default_rng(T + E)
    counts = rng.multinomial(T * k, np.ones(E) / E).astype(np.int32)
    counts[0] = T * k // E                      # exactly at target
    counts[1] = 0                               # idle
    counts[2] = min(T, counts[2] + T // 2)      # overloaded
    b = rng.uniform(-0.05, 0.05, size=E).astype(np.float32)
    step = np.float32(1e-3)
    new_b, load = oracle.bias_update(counts, b, T, k, 1e-3)
    sign = np.sign(k * T - E * counts.astype(np.int64))
    for i in range(E):
        expect = np.float32(b[i] + np.float32(sign[i]) * step)
        assert new_b[i] == expect
        delta = float(new_b[i]) - float(b[i])
        if sign[i] == 0:
            assert delta == 0.0
        else:
            assert abs(abs(delta) - float(step)) <= np.spacing(np.float32(abs(new_b[i]) + 1e-3))
            assert np.sign(delta) == sign[i]
    assert (load == (counts / np.float32(T)).astype(np.float32)).all()
    zero_b, _ = oracle.bias_update(counts, b, T, k, 0.0)
    assert (zero_b == b).all()


# ------------------------------------------------------ histogram, permute

def test_histogram_and_permutation(oracle_lib):
    rng = np.random.default_rng(3)
    T, E, k = 300, 20, 3
    s = rng.uniform(0, 1, size=(T, E)).astype(np.float32)
    idx, _ = oracle.select(s, np.zeros(E, np.float32), k)
    counts = oracle.histogram(idx, E)
    assert (counts == np.bincount(idx.ravel(), minlength=E)).all()
    assert counts.sum() == T * k                 # no dropped tokens
    offsets, perm, inv = oracle.permute(idx, E)
    assert offsets[0] == 0 and offsets[-1] == T * k
    assert (np.diff(offsets) == counts).all()
    assert (perm == np.argsort(idx.ravel(), kind="stable")).all()
    assert (inv[perm] == np.arange(T * k)).all()
    assert (perm[inv] == np.arange(T * k)).all()


# ----------------------------------------------------------------- affinity

def test_affinity_matches_float64_library(oracle_lib):
    rng = np.random.default_rng(9)
    x = rng.standard_normal((20, 96)).astype(np.float32)
    wg = (rng.standard_normal((30, 96)) * 0.1).astype(np.float32)
    s = oracle.affinity(x, wg)
    z = torch.from_numpy(x.astype(np.float64)) @ torch.from_numpy(wg.astype(np.float64)).T
    ref = torch.sigmoid(z).to(torch.float32).numpy()
    diff = np.abs(s.view(np.int32).astype(np.int64) - ref.view(np.int32).astype(np.int64))
    assert diff.max() <= 1


def test_affinity_bf16_widening(oracle_lib):
    g = torch.Generator().manual_seed(4)
    x = torch.randn((8, 64), generator=g).to(torch.bfloat16)
    wg = (torch.randn((16, 64), generator=g) * 0.1).to(torch.bfloat16)
    from fine_grained_moe_gate_b200.inputs import to_numpy
    s = oracle.affinity(to_numpy(x), to_numpy(wg))
    ref = torch.sigmoid(x.double() @ wg.double().T).float().numpy()
    diff = np.abs(s.view(np.int32).astype(np.int64) - ref.view(np.int32).astype(np.int64))
    assert diff.max() <= 1


# ------------------------------------------------------- experts, combine

def _swiglu64(x, w1, w3, w2, round_h=None):
    a = x @ w1.T
    g = x @ w3.T
    h = torch.nn.functional.silu(a) * g
    if round_h is not None:
        h = h.to(round_h).double()
    return h @ w2.T


def _layer_inputs(T, d, E, I, S, Is, seed, dtype=torch.float32):
    g = torch.Generator().manual_seed(seed)
    p = dict(
        x=torch.randn((T, d), generator=g),
        w1=torch.randn((E, I, d), generator=g) * 0.1,
        w3=torch.randn((E, I, d), generator=g) * 0.1,
        w2=torch.randn((E, d, I), generator=g) * 0.1,
        ws1=torch.randn((S, Is, d), generator=g) * 0.1,
        ws3=torch.randn((S, Is, d), generator=g) * 0.1,
        ws2=torch.randn((S, d, Is), generator=g) * 0.1,
    )
    return {n: v.to(dtype) for n, v in p.items()}


def _np(p):
    from fine_grained_moe_gate_b200.inputs import to_numpy
    return {n: to_numpy(v) for n, v in p.items()}


def _rel_fro(a, b):
    a, b = np.asarray(a, np.float64), np.asarray(b, np.float64)
    return np.linalg.norm(a - b) / np.linalg.norm(b)


def test_layer_single_expert_is_dense(oracle_lib):
    """E = k = 1: every token goes to expert 0 with weight 1, so
    y = shared(x) + expert(x) (DeepSeekMoE sketch: shared_out + routed_out)."""
    T, d, I, S, Is = 10, 24, 16, 1, 12
    p = _layer_inputs(T, d, 1, I, S, Is, 1)
    idx = np.zeros((T, 1), np.int32)
    w = np.ones((T, 1), np.float32)
    n = _np(p)
    y = oracle.layer_output(n["x"], idx, w, n["w1"], n["w3"], n["w2"], n["ws1"], n["ws3"], n["ws2"])
    P = {k_: v.double() for k_, v in p.items()}
    ref = _swiglu64(P["x"], P["ws1"][0], P["ws3"][0], P["ws2"][0]) + _swiglu64(P["x"], P["w1"][0], P["w3"][0], P["w2"][0])
    assert _rel_fro(y, ref.numpy()) < 2e-7


def test_layer_single_expert_bf16(oracle_lib):
    """bf16: h is rounded to bf16 once before the down projection and y once
    at the end; the same recipe through torch's own bf16 cast."""
    T, d, I, S, Is = 6, 32, 16, 2, 8
    p = _layer_inputs(T, d, 1, I, S, Is, 2, torch.bfloat16)
    idx = np.zeros((T, 1), np.int32)
    w = np.ones((T, 1), np.float32)
    n = _np(p)
    y = oracle.layer_output(n["x"], idx, w, n["w1"], n["w3"], n["w2"], n["ws1"], n["ws3"], n["ws2"])
    P = {k_: v.double() for k_, v in p.items()}
    ref = sum(_swiglu64(P["x"], P["ws1"][s], P["ws3"][s], P["ws2"][s], torch.bfloat16) for s in range(S))
    ref = ref + _swiglu64(P["x"], P["w1"][0], P["w3"][0], P["w2"][0], torch.bfloat16)
    yt = torch.from_numpy(y.view(np.int16)).view(torch.bfloat16).double()
    # one final bf16 rounding on each side (<= 1 bf16 ulp apart) and rare
    # 1-ulp h disagreements from fp64 summation order
    assert _rel_fro(yt.numpy(), ref.numpy()) < 4e-3
    assert np.allclose(yt.numpy(), ref.numpy(), rtol=2 ** -7, atol=1e-3)


def test_layer_zero_down_is_shared_only(oracle_lib):
    """W2 = 0 for every routed expert: only the shared expert remains."""
    T, d, E, I, S, Is = 12, 16, 6, 8, 1, 8
    p = _layer_inputs(T, d, E, I, S, Is, 3)
    p["w2"] = torch.zeros_like(p["w2"])
    n = _np(p)
    s = oracle.affinity(n["x"], (np.random.default_rng(0).standard_normal((E, d)) * 0.2).astype(np.float32))
    idx, w = oracle.select(s, np.zeros(E, np.float32), 2)
    y = oracle.layer_output(n["x"], idx, w, n["w1"], n["w3"], n["w2"], n["ws1"], n["ws3"], n["ws2"])
    P = {k_: v.double() for k_, v in p.items()}
    ref = _swiglu64(P["x"], P["ws1"][0], P["ws3"][0], P["ws2"][0]).float().numpy()
    assert _rel_fro(y, ref) < 2e-7


def test_layer_all_experts_is_dense_mixture(oracle_lib):
    """k = E with zero bias: y = shared(x) + sum_i (s_i / sum s) expert_i(x),
    a dense mixture computed here with float64 library matmuls."""
    T, d, E, I, S, Is = 9, 20, 5, 12, 1, 10
    p = _layer_inputs(T, d, E, I, S, Is, 4)
    wg = torch.randn((E, d), generator=torch.Generator().manual_seed(8)) * 0.3
    n = _np(p)
    w, idx, s = oracle.route(n["x"], wg.numpy(), np.zeros(E, np.float32), E)
    y = oracle.layer_output(n["x"], idx, w, n["w1"], n["w3"], n["w2"], n["ws1"], n["ws3"], n["ws2"])
    P = {k_: v.double() for k_, v in p.items()}
    aff = torch.sigmoid(P["x"] @ wg.double().T)
    gates = aff / aff.sum(dim=1, keepdim=True)
    ref = _swiglu64(P["x"], P["ws1"][0], P["ws3"][0], P["ws2"][0])
    for e in range(E):
        ref = ref + gates[:, e:e + 1] * _swiglu64(P["x"], P["w1"][e], P["w3"][e], P["w2"][e])
    assert _rel_fro(y, ref.numpy()) < 1e-6


def test_layer_routed_mixture_masked_loop(oracle_lib):
    """General routing, checked against the pages' own formulation: a
    per-expert masked loop with float64 library matmuls (DeepSeekMoE
    sketch: routed_out[mask] += w * expert(x[mask])), weights from the
    oracle's unbiased routing."""
    T, d, E, I, S, Is, k = 40, 32, 8, 16, 2, 8, 3
    p = _layer_inputs(T, d, E, I, S, Is, 5)
    wg = torch.randn((E, d), generator=torch.Generator().manual_seed(9)) * 0.3
    bias = np.random.default_rng(1).uniform(-0.05, 0.05, E).astype(np.float32)
    n = _np(p)
    w, idx, s = oracle.route(n["x"], wg.numpy(), bias, k)
    y = oracle.layer_output(n["x"], idx, w, n["w1"], n["w3"], n["w2"], n["ws1"], n["ws3"], n["ws2"])
    P = {k_: v.double() for k_, v in p.items()}
    ref = sum(_swiglu64(P["x"], P["ws1"][q], P["ws3"][q], P["ws2"][q]) for q in range(S))
    it, wt = torch.from_numpy(idx.astype(np.int64)), torch.from_numpy(w).double()
    for e in range(E):
        mask = (it == e).any(dim=-1)
        if mask.any():
            slot = (it[mask] == e).nonzero(as_tuple=True)[1]
            ref[mask] += wt[mask, slot].unsqueeze(-1) * _swiglu64(P["x"][mask], P["w1"][e], P["w3"][e], P["w2"][e])
    assert _rel_fro(y, ref.numpy()) < 2e-7


def test_expert_up_down_against_float64_library(oracle_lib):
    """The two projections of one expert (DeepSeekMoE sketch: one SwiGLU MLP
    per expert): expert_up against torch float64 silu(x W1^T) * (x W3^T)
    rounded once to bf16; expert_down against a float64 matmul of the same
    h.  A transposed weight or a swapped W1/W3 fails these (W1 != W3)."""
    n, d, I = 7, 40, 24
    p = _layer_inputs(n, d, 1, I, 1, 8, 6, torch.bfloat16)
    nb = _np(p)
    h = oracle.expert_up(nb["x"], nb["w1"][0], nb["w3"][0])
    P = {k_: v.double() for k_, v in p.items()}
    ref = (torch.nn.functional.silu(P["x"] @ P["w1"][0].T) * (P["x"] @ P["w3"][0].T)).to(torch.bfloat16)
    got = torch.from_numpy(h.view(np.int16)).view(torch.bfloat16)
    diff = (got.double() - ref.double()).abs()
    # float64 sums in another order may land on the other side of a bf16
    # rounding boundary: at most one ulp, and rarely
    assert (diff <= 2.0 ** -7 * ref.double().abs() + 1e-30).all()
    assert (diff > 0).float().mean() < 0.01
    swapped = oracle.expert_up(nb["x"], nb["w3"][0], nb["w1"][0])
    assert not np.array_equal(swapped, h)
    o = oracle.expert_down(h, nb["w2"][0])
    ref_o = got.double() @ P["w2"][0].T
    assert np.allclose(o, ref_o.numpy(), rtol=1e-12, atol=1e-12)
    # fp32 layer: the split equals the fused accumulation exactly
    pf = _np(_layer_inputs(n, d, 1, I, 1, 8, 7))
    yacc = np.zeros((n, d), np.float64)
    oracle.expert_accumulate(pf["x"], np.arange(n, dtype=np.int32), np.ones(n), pf["w1"][0], pf["w3"][0],
                             pf["w2"][0], yacc)
    o32 = oracle.expert_down(oracle.expert_up(pf["x"], pf["w1"][0], pf["w3"][0]), pf["w2"][0])
    assert np.array_equal(o32, yacc)
