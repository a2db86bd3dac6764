"""GPU parity of the FP8 (E4M3) expert path against the oracle.

Pages cited: "DeepSeek V3 From Scratch", "The idea" (FP8 with fine-grained
quantization tiles); crackai.dev "DeepSeek-V3", "How It Works" (per-tile
scaling); "DeepSeek V3 Architecture Deep Dive ...", "FP8 Formats" (E4M3).
Tiles of 32 elements along the contraction, power-of-two scales.

Bars: quantization (codes and tile exponents, both scale layouts)
bit-exact -- both sides take the exponent from the tile maximum exactly and
round v * 2^-e to E4M3 the same way; the permuted E4M3 rows bit-exact; GEMM
outputs against the oracle's double-precision tile-scaled sums of the very
same codes and scales (injected), element by element within the bf16
rounding of the output plus the fp32 accumulation error; the whole FP8 layer
against the oracle's FP8 layer within 5e-3 relative Frobenius.
"""
import numpy as np
import pytest
import torch

import fine_grained_moe_gate_b200 as moe
import oracle
from fine_grained_moe_gate_b200.inputs import CONFIGS, make_layer, make_tokens, to_numpy

from gpu_harness import (DEV, as_f64, check_status, permute, rel_fro, route, sf_tokens_to_rows, sf_weights_to_rows,
                         tile_images_expected, tile_images_to_rows, to_f64_rows)

pytestmark = pytest.mark.gpu

TOK, WGT, GATE, UP = moe.MOE_SF_TOKENS, moe.MOE_SF_WEIGHTS, moe.MOE_SF_GATE, moe.MOE_SF_UP


@pytest.fixture(autouse=True)
def _clean_status():
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    moe.moe_get_last_error()
    yield


def _bits(t: torch.Tensor) -> np.ndarray:
    return to_numpy(t)


def _quant(src: torch.Tensor, rows, kseg, nseg=1, layout=TOK):
    q = torch.empty(src.shape, dtype=torch.uint8, device=DEV)
    sc = moe.fp8_scales(rows, kseg * nseg, layout, DEV)
    moe.moe_quantize_fp8(src, rows, kseg, nseg, layout, q, sc)
    torch.cuda.synchronize()
    check_status()
    return q, sc


def _exps(sc, rows, K, layout):
    return sf_tokens_to_rows(sc, rows, K) if layout == TOK else sf_weights_to_rows(sc, rows, K, layout)


@pytest.mark.parametrize("layout", [TOK, WGT, GATE, UP], ids=["tokens", "weights", "gate", "up"])
@pytest.mark.parametrize("rows,K,std", [(37, 256, 0.05), (9, 7168, 1.0), (300, 2048, 3e-3), (128, 128, 100.0),
                                        (5, 10240, 0.5), (64, 1408, 2.0)])
def test_quantize_tiles_bit_exact(layout, rows, K, std):
    g = torch.Generator(device=DEV).manual_seed(rows * 31 + K)
    a = (torch.randn((rows, K), generator=g, device=DEV) * std).to(torch.bfloat16)
    a[rows // 2] = 0                                   # an all-zero row
    if rows > 2:
        a[0, :4] = torch.tensor([448.0, -1e4, 3e-8, 0.0])  # extremes inside one tile
        a[1, 32:64] = 2.0 ** -120                          # a tile far below 448 * 2^-127 ... clamped exponent
    q, sc = _quant(a, rows, K, layout=layout)
    qo, eo = oracle.quantize_mx(_bits(a))
    assert np.array_equal(_exps(sc, rows, K, layout), eo)
    assert np.array_equal(q.cpu().numpy(), qo)


def test_quantize_blocked_layout_bit_exact():
    """Ws2-like [S][d][Is]: rows d span the S blocks, tiles numbered along the whole row."""
    g = torch.Generator(device=DEV).manual_seed(5)
    a = torch.randn((3, 64, 128), generator=g, device=DEV).to(torch.bfloat16)
    a[1] *= 8
    q, sc = _quant(a, 64, 128, 3, layout=WGT)
    qo, eo = oracle.quantize_mx(_bits(a), nseg=3)
    assert np.array_equal(sf_weights_to_rows(sc, 64, 384), eo)
    assert np.array_equal(q.cpu().numpy(), qo)


def _case(T=333, d=256, E=8, k=2, I=256, S=2, Is=128, seed=0, bias_kind="uniform", tile_pattern=False):
    cfg = CONFIGS["small_fp8"].scaled(name="fp8_case", T=T, d=d, E=E, k=k, I=I, S=S, Is=Is, w_std=0.05, seed=seed,
                                      bias_kind=bias_kind, bias_range=0.02)
    sh = moe.shape_of(cfg)
    p = make_layer(cfg, DEV)
    x = make_tokens(cfg, DEV)
    if tile_pattern:
        # magnitudes that change from tile to tile along K and from row to row, so every
        # tile exponent differs from its neighbours': a scale read for the wrong tile, row,
        # CTA or token column shows as a power-of-two error
        def pat(shape, K):
            c = torch.arange(K, device=DEV) // 32
            f = 2.0 ** ((c % 7) - 3).float()
            r = 2.0 ** ((torch.arange(shape, device=DEV) % 5) - 2).float()
            return r[:, None] * f[None, :]
        x = (x.float() * pat(T, d)).to(torch.bfloat16)
        for n in ("w1", "w3"):
            p[n] = (p[n].float() * pat(I, d)[None]).to(torch.bfloat16)
        p["w2"] = (p["w2"].float() * pat(d, I)[None]).to(torch.bfloat16)
    q = moe.quantize_experts_fp8(p)
    torch.cuda.synchronize()
    return cfg, sh, p, x, q, moe.fp8_experts(q)


def _oracle_weights(p, cfg):
    return oracle.quantize_weights_mx({n: _bits(p[n]) for n in ("w1", "w3", "w2", "ws1", "ws3", "ws2")})


def test_weight_quantization_matches_oracle():
    cfg, sh, p, x, q, _ = _case()
    qo = _oracle_weights(p, cfg)
    E, I, d, S, Is = cfg.E, cfg.I, cfg.d, cfg.S, cfg.Is
    geo = {"w1": (E * I, d, "w13s", GATE), "w3": (E * I, d, "w13s", UP), "w2": (E * d, I, "w2s", WGT),
           "ws1": (S * Is, d, "ws13s", GATE), "ws3": (S * Is, d, "ws13s", UP), "ws2": (d, S * Is, "ws2s", WGT)}
    for n, (rows, K, key, lay) in geo.items():
        assert np.array_equal(q[n + "q"].cpu().numpy(), qo[n + "q"]), n
        assert np.array_equal(sf_weights_to_rows(q[key], rows, K, lay), qo[n + "e"]), n


def _bf16_close(got: torch.Tensor, ref_bits_or_f64: np.ndarray, what: str):
    """bf16 outputs from fp32 accumulation vs the oracle's double result
    (rounded to bf16, or not): at most a couple of bf16 ulps apart (2^-7
    relative) plus 2^-10 of the rows' RMS for the fp32 accumulation of large
    cancelling sums."""
    g = as_f64(got)
    r = to_f64_rows(ref_bits_or_f64) if ref_bits_or_f64.dtype == np.uint16 else ref_bits_or_f64
    rms = float(np.sqrt(np.mean(r * r))) if r.size else 0.0
    bad = np.abs(g - r) > np.abs(r) * 2.0 ** -7 + 2.0 ** -10 * rms + 1e-12
    assert not bad.any(), f"{what}: {int(bad.sum())} of {bad.size} elements off, worst {np.max(np.abs(g - r))}"
    assert rel_fro(g, r) < 2e-3, what


def _images(sc, src_rows, K, rows, offsets=None, groups=1, row_of=None, row_div=1, poison=False):
    """Token tile images of a token-layout scale buffer through moe_fp8_tile_scales."""
    t = moe.fp8_tile_images(rows, groups, K, DEV)
    if poison:
        t.fill_(0xAB)
    moe.moe_fp8_tile_scales(sc, src_rows, K, row_of, row_div, offsets, groups, rows, t)
    return t


def _staged(cfg, sh, p, x, q, w8):
    """Route, quantize x, permute, tile images, gate/up, quantize h, down -- through the C ABI."""
    T, k, d, I, S, Is, E = cfg.T, cfg.k, cfg.d, cfg.I, cfg.S, cfg.Is, cfg.E
    idx, w, counts, _ = route(sh, x, p["w_gate"], p["bias"], with_aff=False)
    xq, xs = _quant(x, T, d)
    xq_perm, offsets, perm, inv = permute(sh, xq, idx, counts)
    x_tiles = _images(xs, T, d, T * k, offsets, E, perm, k, poison=True)
    xsh_tiles = _images(xs, T, d, T, poison=True) if S > 0 else None
    torch.cuda.synchronize()
    check_status()
    # the images hold the unpermuted tokens' words, row by row, zeros elsewhere (every byte written)
    off_np = offsets.cpu().numpy()
    words = xs.view(torch.int32).view(d // 128, T).cpu().numpy().view(np.uint32).T
    exp = tile_images_expected(words[perm.cpu().numpy() // k], off_np, T * k, x_tiles.numel())
    assert np.array_equal(x_tiles.cpu().numpy().view(np.uint32), exp), "routed token images"
    if S > 0:
        assert np.array_equal(xsh_tiles.cpu().numpy().view(np.uint32),
                              tile_images_expected(words, None, T, xsh_tiles.numel())), "shared token images"
    h = torch.empty((T * k, I), dtype=torch.bfloat16, device=DEV)
    hs = torch.empty((T, S * Is), dtype=torch.bfloat16, device=DEV) if S > 0 else None
    moe.moe_ffn_up_fp8(xq_perm, x_tiles, offsets, xq if S > 0 else None, xsh_tiles, w8, sh, h, hs)
    torch.cuda.synchronize()
    check_status()
    hq, h_sc = _quant(h, T * k, I)
    hsq, hs_sc = _quant(hs, T, S * Is) if S > 0 else (None, None)
    h_tiles = _images(h_sc, T * k, I, T * k, offsets, E)
    hs_tiles = _images(hs_sc, T, S * Is, T) if S > 0 else None
    # the same gate/up with h quantized in its epilogue: bit-identical codes, and images holding the same
    # scales at every tile row (buffers poisoned, so every code byte must be written)
    fq = torch.full_like(hq, 0xAB)
    fimg = torch.full_like(h_tiles, 0xAB)
    fsq = torch.full_like(hsq, 0xAB) if S > 0 else None
    fsimg = torch.full_like(hs_tiles, 0xAB) if S > 0 else None
    moe.moe_ffn_up_fp8_quant(xq_perm, x_tiles, offsets, xq if S > 0 else None, xsh_tiles, w8, sh, fq, fimg, fsq,
                             fsimg)
    torch.cuda.synchronize()
    check_status()
    assert torch.equal(fq, hq), "fused h quantization: codes"
    assert np.array_equal(tile_images_to_rows(fimg, off_np, T * k, I, pad_byte=0x7F),
                          sf_tokens_to_rows(h_sc, T * k, I)), "fused h quantization: scales"
    if S > 0:
        assert torch.equal(fsq, hsq), "fused hs quantization: codes"
        assert np.array_equal(tile_images_to_rows(fsimg, None, T, S * Is, pad_byte=0x7F),
                              sf_tokens_to_rows(hs_sc, T, S * Is)), "fused hs quantization: scales"
    y_perm = torch.empty((T * k, d), dtype=torch.bfloat16, device=DEV)
    shared_out = torch.empty((T, d), dtype=torch.bfloat16, device=DEV) if S > 0 else None
    moe.moe_ffn_down_fp8(hq, h_tiles, offsets, hsq, hs_tiles, w8, sh, y_perm, shared_out)
    # the down projection from the fused images (poison past each tile's padded rows) is the same
    y2 = torch.empty_like(y_perm)
    s2 = torch.empty_like(shared_out) if S > 0 else None
    moe.moe_ffn_down_fp8(fq, fimg, offsets, fsq, fsimg, w8, sh, y2, s2)
    torch.cuda.synchronize()
    check_status()
    assert torch.equal(y2, y_perm) and (S == 0 or torch.equal(s2, shared_out)), "down from the fused images"
    return dict(idx=idx, w=w, counts=counts, xq=xq, xs=xs, xq_perm=xq_perm, offsets=offsets, perm=perm, inv=inv,
                h=h, hs=hs, hq=hq, h_sc=h_sc, hsq=hsq, hs_sc=hs_sc, y_perm=y_perm, shared_out=shared_out)


@pytest.mark.parametrize("shape", [
    dict(),
    dict(T=129, E=16, k=4, I=384, S=1, Is=256),
    dict(T=40, S=0),
    # about 250 rows per expert: tiles above 240 tokens (first accumulator only), two-tile experts,
    # and d % 256 == 128 (the last down tile's second CTA has no rows of W2)
    dict(T=1000, d=384, E=4, k=1, I=256, S=1, Is=128, bias_kind="zero"),
    dict(T=300, E=4, k=2, I=256, S=1, Is=128, tile_pattern=True),
], ids=["base", "ragged", "no_shared", "big_tiles", "tile_pattern"])
def test_ffn_fp8_stages_against_oracle(shape):
    cfg, sh, p, x, q, w8 = _case(**shape)
    r = _staged(cfg, sh, p, x, q, w8)
    T, k, d, I, S, Is, E = cfg.T, cfg.k, cfg.d, cfg.I, cfg.S, cfg.Is, cfg.E
    # token quantization and the permuted E4M3 rows are exact
    xq_o, xe_o = oracle.quantize_mx(_bits(x))
    assert np.array_equal(r["xq"].cpu().numpy(), xq_o)
    assert np.array_equal(sf_tokens_to_rows(r["xs"], T, d), xe_o)
    inv = r["inv"].cpu().numpy().reshape(T, k)
    xqp = r["xq_perm"].cpu().numpy()
    for j in range(k):
        assert np.array_equal(xqp[inv[:, j]], xq_o)
    # gate/up per expert, from the same codes and scales
    off = r["offsets"].cpu().numpy()
    perm = r["perm"].cpu().numpy()
    qo = _oracle_weights(p, cfg)
    h = r["h"]
    for e in range(E):
        rows = np.arange(off[e], off[e + 1])
        if len(rows) == 0:
            continue
        tok = perm[rows] // k
        ho = oracle.expert_up_mx(xq_o[tok], xe_o[tok], qo["w1q"][e], qo["w1e"][e * I:(e + 1) * I], qo["w3q"][e],
                                 qo["w3e"][e * I:(e + 1) * I])
        _bf16_close(h[torch.as_tensor(rows, device=DEV)], ho, f"h of expert {e}")
    if S > 0:
        hso = oracle.expert_up_mx(xq_o, xe_o, qo["ws1q"].reshape(S * Is, d), qo["ws1e"], qo["ws3q"].reshape(S * Is, d),
                                  qo["ws3e"])
        _bf16_close(r["hs"], hso, "hs")
    # quantization of the kernel's own h is exact
    hq_o, he_o = oracle.quantize_mx(_bits(h))
    assert np.array_equal(r["hq"].cpu().numpy(), hq_o)
    assert np.array_equal(sf_tokens_to_rows(r["h_sc"], T * k, I), he_o)
    # down per expert from the kernel's h codes
    y_perm = r["y_perm"]
    for e in range(E):
        rows = np.arange(off[e], off[e + 1])
        if len(rows) == 0:
            continue
        o = oracle.expert_down_mx(hq_o[rows], he_o[rows], qo["w2q"][e], qo["w2e"][e * d:(e + 1) * d])
        _bf16_close(y_perm[torch.as_tensor(rows, device=DEV)], o, f"y_perm of expert {e}")
    if S > 0:
        hsq_o, hse_o = oracle.quantize_mx(_bits(r["hs"]))
        assert np.array_equal(r["hsq"].cpu().numpy(), hsq_o)
        assert np.array_equal(sf_tokens_to_rows(r["hs_sc"], T, S * Is), hse_o)
        o = oracle.expert_down_mx(hsq_o, hse_o, qo["ws2q"], qo["ws2e"])
        _bf16_close(r["shared_out"], o, "shared_out")


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
    y_o = oracle.layer_output_mx(_bits(x), idx.cpu().numpy(), w.cpu().numpy(), _oracle_weights(p, cfg))
    assert rel_fro(as_f64(y), to_f64_rows(y_o)) < 5e-3


@pytest.mark.parametrize("sizes", [
    [0, 256, 257, 0, 1, 512, 513, 100],     # empty groups, exactly one and two tiles, a tile of one row
    [3000],                                  # one group of 12 tiles of 250
    [1] * 64,                                # 64 single-row groups
    [255, 0, 0, 767, 1280],                  # tiles of 255, 256 and 256
], ids=["mixed", "one_group", "single_rows", "wide"])
@pytest.mark.parametrize("gather", [False, True], ids=["rows", "gathered"])
def test_token_tile_images_bit_exact(sizes, gather):
    """moe_fp8_tile_scales against images built on the host from the same words and the tile split (a group of n
    rows as ceil(n/256) near-equal tiles), every byte of the buffer; with a row index and a divisor (as perm_tok / k
    for the routed rows) the words come from the indexed source rows."""
    G = len(sizes)
    off = np.concatenate([[0], np.cumsum(sizes)]).astype(np.int32)
    rows = int(off[-1])
    K, k = 384, 3
    src_rows = rows if not gather else (rows + k - 1) // k + 5
    g = np.random.default_rng(rows + G)
    words = g.integers(0, 2 ** 32, size=(K // 128, src_rows), dtype=np.uint64).astype(np.uint32)
    src = torch.as_tensor(words.view(np.int32), device=DEV)
    row_of = None
    src_row = np.arange(rows)
    if gather:
        idx = g.permutation(rows).astype(np.int32) % (src_rows * k)
        row_of = torch.as_tensor(idx, device=DEV)
        src_row = idx // k
    tiles = _images(src, src_rows, K, rows, torch.as_tensor(off, device=DEV), G, row_of, k if gather else 1,
                    poison=True)
    torch.cuda.synchronize()
    check_status()
    exp = tile_images_expected(words.T[src_row], off, rows, tiles.numel())
    assert np.array_equal(tiles.cpu().numpy().view(np.uint32), exp)


def test_token_tile_images_device_check():
    """A group reaching past the operand's rows, or a row index past the source, reports MOE_ERR_DEVICE_CHECK
    (its words stay 0) instead of reading out of bounds."""
    K = 128
    src = torch.zeros((1, 64), dtype=torch.int32, device=DEV)
    off = torch.as_tensor(np.array([0, 40, 80], np.int32), device=DEV)     # 80 rows claimed, 64 given
    t = moe.fp8_tile_images(64, 2, K, DEV)
    moe.moe_fp8_tile_scales(src, 64, K, None, 1, off, 2, 64, t)
    torch.cuda.synchronize()
    assert moe.moe_get_last_error() == 6  # MOE_ERR_DEVICE_CHECK
    bad = torch.as_tensor(np.array([0, 1, 999, 3], np.int32), device=DEV)  # row 2 points past the 64 source rows
    t = moe.fp8_tile_images(4, 1, K, DEV)
    moe.moe_fp8_tile_scales(src, 64, K, bad, 1, None, 1, 4, t)
    torch.cuda.synchronize()
    assert moe.moe_get_last_error() == 6  # MOE_ERR_DEVICE_CHECK
    check_status()


def test_fp8_rejected_by_bf16_weight_calls():
    cfg, sh, p, x, q, w8 = _case(T=16)
    ws = torch.empty(1 << 20, dtype=torch.uint8, device=DEV)
    with pytest.raises(moe.MoEError) as ei:
        moe.moe_layer_forward(x, p["w_gate"], p["bias"], p["w1"], p["w3"], p["w2"], p["ws1"], p["ws3"], p["ws2"], sh,
                              torch.empty_like(x), torch.empty((16, cfg.k), dtype=torch.int32, device=DEV),
                              torch.empty((16, cfg.k), device=DEV), torch.empty(cfg.E, dtype=torch.int32, device=DEV),
                              ws)
    assert ei.value.status == 2          # MOE_ERR_UNSUPPORTED
