"""GPU parity of the FP8 (E4M3) expert path against the oracle.

Page cited: "DeepSeek V3 Architecture Deep Dive ...", "FP8 Formats" and
"Per-Tensor/Per-Axis Quantization" (E4M3 weights and activations, a scale
per row).

Bars: quantization (codes and scales) bit-exact -- both sides divide in fp32
and round to E4M3 the same way; the permuted E4M3 rows bit-exact; GEMM
outputs against the oracle's double-precision sums of the very same codes and
scales (injected), elementwise within the bf16 rounding of the output plus
the fp32 accumulation error; the whole FP8 layer against the oracle's FP8
layer within 5e-3 relative Frobenius (an h element rounded to the other E4M3
neighbour flips an eighth of its value).
"""
import numpy as np
import pytest
import torch

import fine_grained_moe_gate_b200 as moe
import oracle
from fine_grained_moe_gate_b200.inputs import CONFIGS, make_layer, make_tokens, to_numpy

from gpu_harness import DEV, as_f64, check_status, permute, rel_fro, route, to_f64_rows

pytestmark = pytest.mark.gpu


@pytest.fixture(autouse=True)
def _clean_status():
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    moe.moe_get_last_error()
    yield


def _bits(t: torch.Tensor) -> np.ndarray:
    return to_numpy(t)


def _quant(src: torch.Tensor, rows, kseg, nseg=1):
    q = torch.empty(src.shape, dtype=torch.uint8, device=DEV)
    sc = torch.empty(rows, dtype=torch.float32, device=DEV)
    moe.moe_quantize_fp8(src, rows, kseg, nseg, q, sc)
    torch.cuda.synchronize()
    check_status()
    return q, sc


@pytest.mark.parametrize("rows,K,std", [(37, 200, 0.05), (9, 7168, 1.0), (300, 2048, 3e-3), (1, 8, 100.0),
                                        (5, 10240, 0.5), (3, 4104, 2.0)])
def test_quantize_rows_bit_exact(rows, K, std):
    g = torch.Generator(device=DEV).manual_seed(rows * 31 + K)
    a = (torch.randn((rows, K), generator=g, device=DEV) * std).to(torch.bfloat16)
    a[rows // 2] = 0                                   # an all-zero row
    if rows > 2:
        a[0, :4] = torch.tensor([448.0, -1e4, 3e-8, 0.0])  # saturation-free extremes inside one row
    q, sc = _quant(a, rows, K)
    qo, so = oracle.quantize_rows_fp8(_bits(a))
    assert np.array_equal(sc.cpu().numpy(), so)
    assert np.array_equal(q.cpu().numpy(), qo)


def test_quantize_blocked_layout_bit_exact():
    """Ws2-like [S][d][Is]: one scale per row d across the S blocks."""
    g = torch.Generator(device=DEV).manual_seed(5)
    a = torch.randn((3, 40, 64), generator=g, device=DEV).to(torch.bfloat16)
    a[1] *= 8                                          # the rows' maxima sit in block 1
    q, sc = _quant(a, 40, 64, 3)
    qo, so = oracle.quantize_rows_fp8(_bits(a), nseg=3)
    assert np.array_equal(sc.cpu().numpy(), so)
    assert np.array_equal(q.cpu().numpy(), qo)


def _case(T=333, d=256, E=8, k=2, I=256, S=2, Is=128, seed=0):
    cfg = CONFIGS["small_fp8"].scaled(name="fp8_case", T=T, d=d, E=E, k=k, I=I, S=S, Is=Is, w_std=0.05, seed=seed)
    sh = moe.shape_of(cfg)
    p = make_layer(cfg, DEV)
    x = make_tokens(cfg, DEV)
    q = moe.quantize_experts_fp8(p)
    torch.cuda.synchronize()
    return cfg, sh, p, x, q, moe.fp8_experts(q)


def test_weight_quantization_matches_oracle():
    cfg, sh, p, x, q, _ = _case()
    qo = oracle.quantize_weights_fp8({n: _bits(p[n]) for n in ("w1", "w3", "w2", "ws1", "ws3", "ws2")})
    for n in ("w1", "w3", "w2", "ws1", "ws3", "ws2"):
        assert np.array_equal(q[n + "q"].cpu().numpy(), qo[n + "q"]), n
        assert np.array_equal(q[n + "s"].cpu().numpy(), qo[n + "s"]), n


def _bf16_close(got: torch.Tensor, ref_bits: np.ndarray, atol: float):
    """bf16 outputs from fp32 vs the oracle's bf16 of the double result: at
    most a couple of bf16 ulps apart (2^-7 relative) plus a small absolute
    slack for the fp32 accumulation of large cancelling sums."""
    g = as_f64(got)
    r = to_f64_rows(ref_bits)
    assert np.all(np.abs(g - r) <= np.abs(r) * 2.0 ** -7 + atol), np.max(np.abs(g - r))
    assert rel_fro(g, r) < 2e-3


def _staged(cfg, sh, p, x, q, w8):
    """Route, quantize x, permute, gate/up, quantize h, down -- through the C ABI."""
    T, k, d, I, S, Is = cfg.T, cfg.k, cfg.d, cfg.I, cfg.S, cfg.Is
    idx, w, counts, _ = route(sh, x, p["w_gate"], p["bias"], with_aff=False)
    xq, xs = _quant(x, T, d)
    xq_perm, offsets, perm, inv = permute(sh, xq, idx, counts)
    h = torch.empty((T * k, I), dtype=torch.bfloat16, device=DEV)
    hs = torch.empty((T, S * Is), dtype=torch.bfloat16, device=DEV) if S > 0 else None
    moe.moe_ffn_up_fp8(xq_perm, perm, xs, offsets, xq if S > 0 else None, w8, sh, h, hs)
    torch.cuda.synchronize()
    check_status()
    hq, h_sc = _quant(h, T * k, I)
    hsq, hs_sc = _quant(hs, T, S * Is) if S > 0 else (None, None)
    y_perm = torch.empty((T * k, d), dtype=torch.bfloat16, device=DEV)
    shared_out = torch.empty((T, d), dtype=torch.bfloat16, device=DEV) if S > 0 else None
    moe.moe_ffn_down_fp8(hq, h_sc, offsets, hsq, hs_sc, w8, sh, y_perm, shared_out)
    torch.cuda.synchronize()
    check_status()
    return dict(idx=idx, w=w, counts=counts, xq=xq, xs=xs, xq_perm=xq_perm, offsets=offsets, perm=perm, inv=inv,
                h=h, hs=hs, hq=hq, h_sc=h_sc, hsq=hsq, hs_sc=hs_sc, y_perm=y_perm, shared_out=shared_out)


@pytest.mark.parametrize("shape", [dict(), dict(T=129, E=16, k=4, I=384, S=1, Is=256), dict(T=40, S=0)],
                         ids=["base", "ragged", "no_shared"])
def test_ffn_fp8_stages_against_oracle(shape):
    cfg, sh, p, x, q, w8 = _case(**shape)
    r = _staged(cfg, sh, p, x, q, w8)
    T, k, d, I, S, Is, E = cfg.T, cfg.k, cfg.d, cfg.I, cfg.S, cfg.Is, cfg.E
    # token quantization and the permuted E4M3 rows are exact
    xq_o, xs_o = oracle.quantize_rows_fp8(_bits(x))
    assert np.array_equal(r["xq"].cpu().numpy(), xq_o) and np.array_equal(r["xs"].cpu().numpy(), xs_o)
    inv = r["inv"].cpu().numpy().reshape(T, k)
    xqp = r["xq_perm"].cpu().numpy()
    for j in range(k):
        assert np.array_equal(xqp[inv[:, j]], xq_o)
    # gate/up per expert, from the same codes and scales
    off = r["offsets"].cpu().numpy()
    perm = r["perm"].cpu().numpy()
    wq = {n: q[n].cpu().numpy() for n in q}
    h = r["h"]
    for e in range(E):
        rows = np.arange(off[e], off[e + 1])
        if len(rows) == 0:
            continue
        tok = perm[rows] // k
        ho = oracle.expert_up_fp8(xq_o[tok], xs_o[tok], wq["w1q"][e], wq["w1s"][e * I:(e + 1) * I], wq["w3q"][e],
                                  wq["w3s"][e * I:(e + 1) * I])
        _bf16_close(h[torch.as_tensor(rows, device=DEV)], ho, atol=1e-4)
    if S > 0:
        hso = oracle.expert_up_fp8(xq_o, xs_o, wq["ws1q"].reshape(S * Is, d), wq["ws1s"], wq["ws3q"].reshape(S * Is, d),
                                   wq["ws3s"])
        _bf16_close(r["hs"], hso, atol=1e-4)
    # quantization of the kernel's own h is exact
    hq_o, hsc_o = oracle.quantize_rows_fp8(_bits(h))
    assert np.array_equal(r["hq"].cpu().numpy(), hq_o) and np.array_equal(r["h_sc"].cpu().numpy(), hsc_o)
    # down per expert from the kernel's h codes
    y_perm = r["y_perm"]
    for e in range(E):
        rows = np.arange(off[e], off[e + 1])
        if len(rows) == 0:
            continue
        o = oracle.expert_down_fp8(hq_o[rows], hsc_o[rows], wq["w2q"][e], wq["w2s"][e * d:(e + 1) * d])
        _bf16_close(y_perm[torch.as_tensor(rows, device=DEV)], oracle.finalize(o, np.uint16), atol=1e-4)
    if S > 0:
        hsq_o, hssc_o = oracle.quantize_rows_fp8(_bits(r["hs"]))
        assert np.array_equal(r["hsq"].cpu().numpy(), hsq_o)
        o = oracle.expert_down_fp8(hsq_o, hssc_o, wq["ws2q"], wq["ws2s"])
        _bf16_close(r["shared_out"], oracle.finalize(o, np.uint16), atol=1e-4)


def test_layer_forward_fp8_equals_staged_calls_and_oracle():
    cfg, sh, p, x, q, w8 = _case(T=200, E=16, k=4)
    r = _staged(cfg, sh, p, x, q, w8)
    y_st = torch.empty((cfg.T, cfg.d), dtype=torch.bfloat16, device=DEV)
    moe.moe_combine(r["y_perm"], r["w"], r["inv"], r["shared_out"], sh, y_st)
    y = torch.empty_like(y_st)
    idx = torch.empty((cfg.T, cfg.k), dtype=torch.int32, device=DEV)
    w = torch.empty((cfg.T, cfg.k), dtype=torch.float32, device=DEV)
    counts = torch.empty(cfg.E, dtype=torch.int32, device=DEV)
    ws = torch.empty(moe.moe_workspace_size(sh), dtype=torch.uint8, device=DEV)
    moe.moe_layer_forward_fp8(x, p["w_gate"], p["bias"], w8, sh, y, idx, w, counts, ws)
    torch.cuda.synchronize()
    check_status()
    assert torch.equal(idx, r["idx"]) and torch.equal(counts, r["counts"])
    assert torch.equal(y.view(torch.int16), y_st.view(torch.int16))
    qo = {n: t.cpu().numpy() for n, t in q.items()}
    y_o = oracle.layer_output_fp8(_bits(x), idx.cpu().numpy(), w.cpu().numpy(), qo)
    assert rel_fro(as_f64(y), to_f64_rows(y_o)) < 5e-3


def test_fp8_rejected_by_bf16_weight_calls():
    cfg, sh, p, x, q, w8 = _case(T=16)
    ws = torch.empty(1 << 20, dtype=torch.uint8, device=DEV)
    with pytest.raises(moe.MoEError) as ei:
        moe.moe_layer_forward(x, p["w_gate"], p["bias"], p["w1"], p["w3"], p["w2"], p["ws1"], p["ws3"], p["ws2"], sh,
                              torch.empty_like(x), torch.empty((16, cfg.k), dtype=torch.int32, device=DEV),
                              torch.empty((16, cfg.k), device=DEV), torch.empty(cfg.E, dtype=torch.int32, device=DEV),
                              ws)
    assert ei.value.status == 2          # MOE_ERR_UNSUPPORTED
