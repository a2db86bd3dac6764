"""GPU parity at the workloads' full sizes, in the launch configuration the
bench times: routing, counts and the bias step are checked for every token
(injected mode), the kernel's affinities on sampled tokens, the grouped
GEMMs' outputs element by element over whole experts (the most-loaded one,
a median one, the last one and the shared set), and the layer output element
by element on sampled tokens the oracle computes one by one."""
import numpy as np
import pytest
import torch

import fine_grained_moe_gate_b200 as moe
import oracle
from fine_grained_moe_gate_b200.inputs import CONFIGS, make_layer, make_tokens, to_numpy

from gpu_harness import (DEV, as_f64, check_bf16_close, check_layer_elementwise, check_route_parity, check_status,
                         layer_forward, oracle_terms, oracle_terms_from_h, permute, rel_fro, route, to_f64_rows)

pytestmark = pytest.mark.gpu


def _rows_to_check(r0, r1, dense_limit):
    """Every row of [r0, r1) when there are at most dense_limit of them; else
    every 7th row and the last 16, which still reaches every 256-row token tile."""
    if r1 - r0 <= dense_limit:
        return np.arange(r0, r1)
    return np.unique(np.concatenate([np.arange(r0, r1, 7), np.arange(max(r0, r1 - 16), r1)]))


def _feature_subset(total, tile, offs):
    """A few output features of every `tile`-wide feature tile, at the given
    offsets inside the tile (chosen to reach both CTAs of a pair and every
    TMEM lane quarter of each)."""
    f = np.concatenate([t + np.asarray(offs) for t in range(0, total, tile)])
    return f[f < total]


UP_OFFS = (0, 17, 40, 63, 64, 81, 104, 127)        # 128-feature up tiles: 64 per CTA, 32 per lane quarter
DOWN_OFFS = (0, 45, 100, 127, 128, 160, 201, 255)   # 256-feature down tiles: 128 per CTA


def _projection_checks(cfg, p, x, idx, counts, y_layer, w):
    """moe_permute, moe_ffn_up, moe_ffn_down and moe_combine as the bench
    calls them.  For the most-loaded expert, a median-loaded one, the last
    expert with rows and the shared set: h (gate/up + SwiGLU epilogue)
    against the oracle's up projection of the same token rows, and y_perm /
    shared_out (down) against the oracle's down projection of the GPU's own h
    (so that each launch is checked alone), element by element.  Small
    experts are checked in full; large ones on every 7th row and a feature
    subset that reaches every tile."""
    sh = moe.shape_of(cfg)
    T, k, d, I, S, Is = cfg.T, cfg.k, cfg.d, cfg.I, cfg.S, cfg.Is
    x_perm, offsets, perm, inv = permute(sh, x, idx, counts)
    h = torch.empty((T * k, I), dtype=x.dtype, device=DEV)
    hs = torch.empty((T, S * Is), dtype=x.dtype, device=DEV)
    moe.moe_ffn_up(x_perm, offsets, p["w1"], p["w3"], x, p["ws1"], p["ws3"], sh, h, hs)
    y_perm = torch.empty((T * k, d), dtype=x.dtype, device=DEV)
    shared_out = torch.empty((T, d), dtype=x.dtype, device=DEV)
    moe.moe_ffn_down(h, offsets, p["w2"], hs, p["ws2"], sh, y_perm, shared_out)
    y = torch.empty((T, d), dtype=x.dtype, device=DEV)
    moe.moe_combine(y_perm, w, inv, shared_out, sh, y)
    torch.cuda.synchronize()
    check_status()
    assert torch.equal(y.view(torch.int16), y_layer.view(torch.int16))   # the staged calls are the layer
    c = counts.cpu().numpy()
    off = offsets.cpu().numpy()
    nz = np.nonzero(c)[0]
    by_load = nz[np.argsort(c[nz], kind="stable")]
    picks = sorted({int(by_load[-1]), int(by_load[len(by_load) // 2]), int(nz[-1])})
    fu_all, fd_all = np.arange(I), np.arange(d)
    for e in picks:
        r0, r1 = int(off[e]), int(off[e + 1])
        rows = _rows_to_check(r0, r1, 2048)
        fu = fu_all if r1 - r0 <= 512 else _feature_subset(I, 128, UP_OFFS)
        fd = fd_all if r1 - r0 <= 320 else _feature_subset(d, 256, DOWN_OFFS)
        rt = torch.as_tensor(rows, device=DEV)
        xr = to_numpy(x_perm[rt])
        h_ref = oracle.expert_up(xr, to_numpy(p["w1"][e][torch.as_tensor(fu, device=DEV)]),
                                 to_numpy(p["w3"][e][torch.as_tensor(fu, device=DEV)]))
        check_bf16_close(as_f64(h[rt][:, torch.as_tensor(fu, device=DEV)]), to_f64_rows(h_ref),
                         f"{cfg.name} h of expert {e} ({r1 - r0} rows)")
        o_ref = oracle.expert_down(to_numpy(h[rt]), to_numpy(p["w2"][e][torch.as_tensor(fd, device=DEV)]))
        check_bf16_close(as_f64(y_perm[rt][:, torch.as_tensor(fd, device=DEV)]), o_ref,
                         f"{cfg.name} y_perm of expert {e} ({r1 - r0} rows)")
    if S > 0:
        rows = _rows_to_check(0, T, 640) if T > 640 else np.arange(T)
        rt = torch.as_tensor(rows, device=DEV)
        fu = _feature_subset(Is, 128, UP_OFFS)
        fd = _feature_subset(d, 256, DOWN_OFFS)
        xr = to_numpy(x[rt])
        hs_rows = hs[rt]
        o_ref = np.zeros((len(rows), len(fd)), np.float64)
        for s in range(S):
            h_ref = oracle.expert_up(xr, to_numpy(p["ws1"][s][torch.as_tensor(fu, device=DEV)]),
                                     to_numpy(p["ws3"][s][torch.as_tensor(fu, device=DEV)]))
            check_bf16_close(as_f64(hs_rows[:, torch.as_tensor(s * Is + fu, device=DEV)]), to_f64_rows(h_ref),
                             f"{cfg.name} hs of shared expert {s}")
            o_ref += oracle.expert_down(to_numpy(hs_rows[:, s * Is:(s + 1) * Is]),
                                        to_numpy(p["ws2"][s][torch.as_tensor(fd, device=DEV)]))
        check_bf16_close(as_f64(shared_out[rt][:, torch.as_tensor(fd, device=DEV)]), o_ref,
                         f"{cfg.name} shared_out")
    return h, hs, inv


def _full_check(cfg, p, x, n_sample, seed, s_tol="auto", projections=False):
    sh = moe.shape_of(cfg)
    y, idx, w, counts = layer_forward(sh, p, x)
    check_status()
    ridx, rw, rcounts, aff = route(sh, x, p["w_gate"], p["bias"])
    assert torch.equal(ridx, idx) and torch.equal(rw, w) and torch.equal(rcounts, counts)
    rng = np.random.default_rng(seed)
    rows = np.sort(rng.choice(cfg.T, size=min(64, cfg.T), replace=False))
    check_route_parity(x, p["w_gate"], p["bias"], cfg.k, idx, w, counts, aff, s_tol, self_rows=rows)
    assert int(counts.sum()) == cfg.T * cfg.k       # no dropped tokens
    tokens = np.sort(rng.choice(cfg.T, size=min(n_sample, cfg.T), replace=False))
    yt = y[torch.as_tensor(tokens, device=DEV)]
    # the layer bar (5e-3 relative Frobenius for bf16) against the oracle computed from scratch
    y_ref, _ = oracle_terms(p, x, idx, w, tokens, cfg.S)
    err = rel_fro(as_f64(yt), to_f64_rows(oracle.finalize(y_ref, np.uint16)))
    assert err <= 5e-3, err
    if projections:
        # every kernel's output element by element: the projections, then the down projections and
        # the combine of the sampled tokens from the GPU's own h
        h, hs, inv = _projection_checks(cfg, p, x, idx, counts, y, w)
        y_ref_h, mag = oracle_terms_from_h(p, h, hs, idx, w, inv, tokens, cfg.S)
        check_layer_elementwise(yt, y_ref_h, mag)
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
    _full_check(cfg, p, x, n_sample=64, seed=2, projections=True)


def test_v3_decode_calls(v3_layer):
    """T=64 per call with fresh tokens each call (calls 0, 1 and 999)."""
    cfg_p, p = v3_layer
    cfg = CONFIGS["v3_decode"]
    for call in (0, 1, 999):
        x = make_tokens(cfg, DEV, call)
        _full_check(cfg, p, x, n_sample=64 if call == 0 else 16, seed=call, projections=call == 0)


def test_small_bf16_full_and_ten_steps():
    cfg = CONFIGS["small_bf16"]
    sh = moe.shape_of(cfg)
    p = make_layer(cfg, DEV)
    bias0 = p["bias"].clone()
    bias_orc = p["bias"].cpu().numpy().copy()
    for step in range(cfg.steps):
        x = make_tokens(cfg, DEV, step)
        if step in (0, cfg.steps - 1):
            y, idx, w, counts = _full_check(cfg, p, x, n_sample=64, seed=step, projections=step == 0)
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
            # logits carry the per-expert offsets: the derived affinity bound, uncapped
            y, idx, w, counts = _full_check(cfg, p, x, n_sample=64, seed=4, s_tol="derived", projections=True)
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


def test_skew_stress_bias_trajectory_200_steps():
    """The skew workload's load trajectory ("A bias term for each expert":
    the bias moves by the fixed step at the end of every step): 200 steps of
    routing and bias update, a fresh batch per step; every step's choices
    and bias bit-exact against the oracle taking the kernel's affinities."""
    cfg = CONFIGS["skew_stress"]
    sh = moe.shape_of(cfg)
    p = make_layer(cfg, DEV)
    bias_orc = p["bias"].cpu().numpy().copy()
    for step in range(200):
        x = make_tokens(cfg, DEV, step)
        idx, _, counts, aff = route(sh, x, p["w_gate"], p["bias"])
        o_idx, _ = oracle.select(aff.cpu().numpy(), bias_orc, cfg.k)
        assert (o_idx == idx.cpu().numpy()).all(), f"step {step}"
        assert (oracle.histogram(o_idx, cfg.E) == counts.cpu().numpy()).all(), f"step {step}"
        moe.moe_load_and_bias_update(counts, sh, cfg.step_size, None, p["bias"])
        torch.cuda.synchronize()
        bias_orc, _ = oracle.bias_update(oracle.histogram(o_idx, cfg.E), bias_orc, cfg.T, cfg.k, cfg.step_size)
        assert (p["bias"].cpu().numpy().view(np.uint32) == bias_orc.view(np.uint32)).all(), f"step {step}"
    check_status()


# ------------------------------------------------------------------ FP8 experts

def _oracle_rows_fp8(p, x, idx, w, tokens, cfg):
    """The oracle's per-tile FP8 layer output for the sampled tokens ("DeepSeek
    V3 From Scratch", "The idea": fine-grained quantization tiles): tokens
    quantized by tiles, every expert they use quantized by the oracle from
    its bf16 weights (one expert at a time) and run from its E4M3 codes, h
    quantized by tiles per assignment row, outputs summed in double."""
    from fine_grained_moe_gate_b200.inputs import to_numpy
    d, I, S, Is = cfg.d, cfg.I, cfg.S, cfg.Is
    tokens = np.asarray(tokens)
    xq, xe = oracle.quantize_mx(to_numpy(x[torch.as_tensor(tokens, device=DEV)]))
    yacc = np.zeros((len(tokens), d), np.float64)
    if S > 0:
        q1, e1 = oracle.quantize_mx(to_numpy(p["ws1"]).reshape(S * Is, d))
        q3, e3 = oracle.quantize_mx(to_numpy(p["ws3"]).reshape(S * Is, d))
        q2, e2 = oracle.quantize_mx(to_numpy(p["ws2"]), nseg=S)
        hq, he = oracle.quantize_mx(oracle.expert_up_mx(xq, xe, q1, e1, q3, e3))
        yacc += oracle.expert_down_mx(hq, he, q2, e2)
    idx_np, w_np = idx.cpu().numpy()[tokens], w.cpu().numpy()[tokens]
    for e in np.unique(idx_np):
        ii, jj = np.nonzero(idx_np == e)
        q1, e1 = oracle.quantize_mx(to_numpy(p["w1"][e]))
        q3, e3 = oracle.quantize_mx(to_numpy(p["w3"][e]))
        q2, e2 = oracle.quantize_mx(to_numpy(p["w2"][e]))
        hq, he = oracle.quantize_mx(oracle.expert_up_mx(xq[ii], xe[ii], q1, e1, q3, e3))
        yacc[ii] += w_np[ii, jj].astype(np.float64)[:, None] * oracle.expert_down_mx(hq, he, q2, e2)
    return oracle.finalize(yacc, np.uint16)


def _fp8_check(cfg, p, w8, x, n_sample, seed):
    sh = moe.shape_of(cfg)
    T, k, d, E = cfg.T, cfg.k, cfg.d, cfg.E
    y = torch.empty((T, d), dtype=torch.bfloat16, device=DEV)
    idx = torch.empty((T, k), dtype=torch.int32, device=DEV)
    w = torch.empty((T, k), dtype=torch.float32, device=DEV)
    counts = torch.empty(E, dtype=torch.int32, device=DEV)
    ws = torch.empty(moe.moe_workspace_size(sh), dtype=torch.uint8, device=DEV)
    moe.moe_layer_forward_fp8(x, p["w_gate"], p["bias"], w8, sh, y, idx, w, counts, ws)
    torch.cuda.synchronize()
    check_status()
    ridx, rw, rcounts, _ = route(sh, x, p["w_gate"], p["bias"], with_aff=False)   # routing is the bf16 path's
    assert torch.equal(ridx, idx) and torch.equal(rw, w) and torch.equal(rcounts, counts)
    tokens = np.sort(np.random.default_rng(seed).choice(T, size=n_sample, replace=False))
    ref = to_f64_rows(_oracle_rows_fp8(p, x, idx, w, tokens, cfg))
    got = as_f64(y[torch.as_tensor(tokens, device=DEV)])
    err = rel_fro(got, ref)
    assert err <= 5e-3, err


def _fp8_projection_checks(cfg, p, w8, x):
    """The E4M3 stages as the bench calls them (quantize x, permute, token tile
    images, gate/up with h quantized in its epilogue, down), at full size.
    For the most-loaded expert, a median one, the last one with rows and the
    shared set: h from moe_ffn_up_fp8 (bf16) element by element against the
    oracle's up projection of the same E4M3 rows and scales; the fused
    launch's codes and tile scales bit for bit against the oracle's
    quantization of that h; y_perm / shared_out element by element against
    the oracle's down projection of the fused launch's own codes and scales
    (each launch checked alone)."""
    from gpu_harness import sf_tokens_to_rows, tile_images_to_rows
    sh = moe.shape_of(cfg)
    T, k, d, E, I, S, Is = cfg.T, cfg.k, cfg.d, cfg.E, cfg.I, cfg.S, cfg.Is
    TOK = moe.MOE_SF_TOKENS
    idx, w, counts, _ = route(sh, x, p["w_gate"], p["bias"], with_aff=False)
    xq = torch.empty((T, d), dtype=torch.uint8, device=DEV)
    xs = moe.fp8_scales(T, d, TOK, DEV)
    moe.moe_quantize_fp8(x, T, d, 1, TOK, xq, xs)
    xq_perm, offsets, perm, inv = permute(sh, xq, idx, counts)
    x_img, xsh_img = moe.fp8_tile_images(T * k, E, d, DEV), moe.fp8_tile_images(T, 1, d, DEV)
    moe.moe_fp8_tile_scales(xs, T, d, perm, k, offsets, E, T * k, x_img)
    moe.moe_fp8_tile_scales(xs, T, d, None, 1, None, 1, T, xsh_img)
    h = torch.empty((T * k, I), dtype=torch.bfloat16, device=DEV)
    hs = torch.empty((T, S * Is), dtype=torch.bfloat16, device=DEV)
    moe.moe_ffn_up_fp8(xq_perm, x_img, offsets, xq, xsh_img, w8, sh, h, hs)
    hq = torch.empty((T * k, I), dtype=torch.uint8, device=DEV)
    hsq = torch.empty((T, S * Is), dtype=torch.uint8, device=DEV)
    h_img, hs_img = moe.fp8_tile_images(T * k, E, I, DEV), moe.fp8_tile_images(T, 1, S * Is, DEV)
    moe.moe_ffn_up_fp8_quant(xq_perm, x_img, offsets, xq, xsh_img, w8, sh, hq, h_img, hsq, hs_img)
    y_perm = torch.empty((T * k, d), dtype=torch.bfloat16, device=DEV)
    shared_out = torch.empty((T, d), dtype=torch.bfloat16, device=DEV)
    moe.moe_ffn_down_fp8(hq, h_img, offsets, hsq, hs_img, w8, sh, y_perm, shared_out)
    torch.cuda.synchronize()
    check_status()
    off = offsets.cpu().numpy()
    xq_o, xe_o = oracle.quantize_mx(to_numpy(x))
    assert np.array_equal(xq.cpu().numpy(), xq_o) and np.array_equal(sf_tokens_to_rows(xs, T, d), xe_o)
    perm_np = perm.cpu().numpy()
    he_all = tile_images_to_rows(h_img, off, T * k, I)
    c = counts.cpu().numpy()
    nz = np.nonzero(c)[0]
    by_load = nz[np.argsort(c[nz], kind="stable")]
    picks = sorted({int(by_load[-1]), int(by_load[len(by_load) // 2]), int(nz[-1])})
    for e in picks:
        r0, r1 = int(off[e]), int(off[e + 1])
        rows = _rows_to_check(r0, r1, 2048)
        fu = np.arange(I) if r1 - r0 <= 512 else _feature_subset(I, 128, UP_OFFS)
        fd = np.arange(d) if r1 - r0 <= 320 else _feature_subset(d, 256, DOWN_OFFS)
        rt = torch.as_tensor(rows, device=DEV)
        tok = perm_np[rows] // k
        q1, e1 = oracle.quantize_mx(to_numpy(p["w1"][e]))
        q3, e3 = oracle.quantize_mx(to_numpy(p["w3"][e]))
        q2, e2 = oracle.quantize_mx(to_numpy(p["w2"][e]))
        h_ref = oracle.expert_up_mx(xq_o[tok], xe_o[tok], q1[fu], e1[fu], q3[fu], e3[fu])
        check_bf16_close(as_f64(h[rt][:, torch.as_tensor(fu, device=DEV)]), to_f64_rows(h_ref),
                         f"{cfg.name} h of expert {e} ({r1 - r0} rows)")
        hq_o, he_o = oracle.quantize_mx(to_numpy(h[rt]))
        assert np.array_equal(hq[rt].cpu().numpy(), hq_o), f"fused h codes of expert {e}"
        assert np.array_equal(he_all[rows], he_o), f"fused h scales of expert {e}"
        o_ref = oracle.expert_down_mx(hq_o, he_o, q2[fd], e2[fd])
        check_bf16_close(as_f64(y_perm[rt][:, torch.as_tensor(fd, device=DEV)]), o_ref,
                         f"{cfg.name} y_perm of expert {e} ({r1 - r0} rows)")
    rows = _rows_to_check(0, T, 640) if T > 640 else np.arange(T)
    rt = torch.as_tensor(rows, device=DEV)
    fu = _feature_subset(S * Is, 128, UP_OFFS)
    fd = _feature_subset(d, 256, DOWN_OFFS)
    q1, e1 = oracle.quantize_mx(to_numpy(p["ws1"]).reshape(S * Is, d))
    q3, e3 = oracle.quantize_mx(to_numpy(p["ws3"]).reshape(S * Is, d))
    q2, e2 = oracle.quantize_mx(to_numpy(p["ws2"]), nseg=S)
    h_ref = oracle.expert_up_mx(xq_o[rows], xe_o[rows], q1[fu], e1[fu], q3[fu], e3[fu])
    check_bf16_close(as_f64(hs[rt][:, torch.as_tensor(fu, device=DEV)]), to_f64_rows(h_ref), f"{cfg.name} hs")
    hsq_o, hse_o = oracle.quantize_mx(to_numpy(hs[rt]))
    assert np.array_equal(hsq[rt].cpu().numpy(), hsq_o), "fused hs codes"
    assert np.array_equal(tile_images_to_rows(hs_img, None, T, S * Is)[rows], hse_o), "fused hs scales"
    o_ref = oracle.expert_down_mx(hsq_o, hse_o, q2[:, fd], e2[fd])   # q2 [S][d][Is], K joined over the blocks
    check_bf16_close(as_f64(shared_out[rt][:, torch.as_tensor(fd, device=DEV)]), o_ref, f"{cfg.name} shared_out")


def test_v3_fp8_prefill_and_decode(v3_layer):
    """V3 prefill (T=8192) and decode calls with per-tile E4M3 experts
    through moe_layer_forward_fp8 (what the bench times); the weights are
    quantized on the device and checked bit for bit (codes and tile
    exponents of W1, W3 and W2) on three sampled experts; the prefill
    batch's stages also expert by expert (_fp8_projection_checks)."""
    from gpu_harness import sf_weights_to_rows
    _, p = v3_layer
    q = moe.quantize_experts_fp8(p)
    w8 = moe.fp8_experts(q)
    torch.cuda.synchronize()
    check_status()
    for n, key, lay in (("w1", "w13s", moe.MOE_SF_GATE), ("w3", "w13s", moe.MOE_SF_UP),
                        ("w2", "w2s", moe.MOE_SF_WEIGHTS)):
        rows, K = p[n].shape[1], p[n].shape[2]
        E = p[n].shape[0]
        ex = sf_weights_to_rows(q[key], E * rows, K, lay)
        for e in (0, 77, 255):
            qo, eo = oracle.quantize_mx(to_numpy(p[n][e]))
            assert np.array_equal(q[n + "q"][e].cpu().numpy(), qo)
            assert np.array_equal(ex[e * rows:(e + 1) * rows], eo)
    cfg = CONFIGS["v3_prefill_fp8"]
    _fp8_check(cfg, p, w8, make_tokens(cfg, DEV), n_sample=16, seed=12)
    _fp8_projection_checks(cfg, p, w8, make_tokens(cfg, DEV))
    cfg = CONFIGS["v3_decode_fp8"]
    for call in (0, 999):
        _fp8_check(cfg, p, w8, make_tokens(cfg, DEV, call), n_sample=8, seed=call)
    del q, w8
    torch.cuda.empty_cache()
