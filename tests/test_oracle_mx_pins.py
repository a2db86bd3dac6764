"""Pins for the oracle's per-tile FP8 functions (CPU only).

Pages cited: "DeepSeek V3 From Scratch", "The idea" (FP8 with fine-grained
quantization tiles); crackai.dev "DeepSeek-V3", "How It Works" (per-tile
scaling); "DeepSeek V3 Architecture Deep Dive ...", "FP8 Formats" (E4M3).
Reading: a tile is 32 consecutive elements of a row along the contraction
dimension, scaled by 2^e with e the smallest integer such that the tile's
largest magnitude is at most 448 * 2^e.

Each check compares the oracle with something other than itself: exact
rational arithmetic for the exponent rule, torch's float8_e4m3fn conversion
for the codes, integer matmuls for the tile-scaled sums (with scales that
differ from tile to tile, so a dropped, shifted or transposed tile scale
fails), and the bf16 layer for the overall quantization error.
"""
from fractions import Fraction

import numpy as np
import torch

import oracle


def _bf16_bits(t: torch.Tensor) -> np.ndarray:
    return t.to(torch.bfloat16).contiguous().view(torch.int16).numpy().view(np.uint16)


def test_mx_exponent_is_the_smallest_that_fits(oracle_lib):
    """amax <= 448 * 2^e and amax > 448 * 2^(e-1), checked in exact rationals,
    on the range's edges and on random magnitudes over 60 binades."""
    rng = np.random.default_rng(0)
    vals = [448.0, 449.0, 447.99, 1.0, 0.875, 0.8750001, 1.75, 896.0, 896.5, 2.0 ** -100, 2.0 ** 100, 3.0e38]
    vals += list(np.exp(rng.uniform(-40, 40, 300)))
    for a in vals:
        a = float(np.float32(a))
        e = oracle.mx_exponent(a)
        A = Fraction(a)
        assert A <= 448 * Fraction(2) ** e, (a, e)
        assert A > 448 * Fraction(2) ** (e - 1), (a, e)
    assert oracle.mx_exponent(0.0) == 0
    assert oracle.mx_exponent(1e-45) == -127          # below 448 * 2^-127: clamped


def test_quantize_mx_codes_match_torch_float8(oracle_lib):
    """Every code is torch's float8_e4m3fn conversion of v * 2^-e (exact in
    float32 for bf16 inputs), with e from the tile's own maximum; no code
    saturates and the tile maximum lands in the top binade [256, 448]."""
    g = torch.Generator().manual_seed(1)
    a = torch.randn((7, 96), generator=g) * torch.logspace(-3, 3, 96)[None]   # tiles of very different ranges
    a = a.to(torch.bfloat16)
    q, eb = oracle.quantize_mx(_bf16_bits(a))
    assert q.shape == (7, 96) and eb.shape == (7, 3)
    af = a.float()
    for b in range(3):
        tile = af[:, 32 * b:32 * (b + 1)]
        e = np.array([oracle.mx_exponent(float(m)) for m in tile.abs().max(dim=1).values])
        assert np.array_equal(eb[:, b].astype(int) - 127, e)
        scaled = tile * torch.from_numpy(np.ldexp(1.0, -e)).float()[:, None]
        ref = scaled.to(torch.float8_e4m3fn).view(torch.uint8).numpy()
        assert np.array_equal(q[:, 32 * b:32 * (b + 1)], ref)
        top = oracle.fp8_decode(q[:, 32 * b:32 * (b + 1)]).__abs__().max(axis=1)
        assert np.all((top >= 224.0) & (top <= 448.0))   # RNE can round 255.9 down to 240 but never below 224


def test_quantize_mx_tiles_are_independent(oracle_lib):
    """Scaling one tile by 2^k moves only that tile's exponent, by k, and
    leaves every code unchanged (a tile boundary off by one element fails)."""
    g = torch.Generator().manual_seed(2)
    a = (torch.randn((5, 128), generator=g) * 0.1).to(torch.bfloat16)
    q0, e0 = oracle.quantize_mx(_bf16_bits(a))
    b = a.clone()
    b[:, 64:96] *= 8.0                                     # tile 2, exact in bf16
    q1, e1 = oracle.quantize_mx(_bf16_bits(b))
    assert np.array_equal(q0, q1)
    assert np.array_equal(e1[:, [0, 1, 3]], e0[:, [0, 1, 3]])
    assert np.array_equal(e1[:, 2].astype(int), e0[:, 2].astype(int) + 3)


def test_quantize_mx_blocked_layout_equals_concatenated(oracle_lib):
    g = torch.Generator().manual_seed(3)
    blk = torch.randn((3, 9, 64), generator=g).to(torch.bfloat16)
    qb, eb = oracle.quantize_mx(_bf16_bits(blk), nseg=3)
    qc, ec = oracle.quantize_mx(_bf16_bits(torch.cat(list(blk), dim=1)))
    assert np.array_equal(eb, ec)
    assert np.array_equal(np.concatenate(list(qb), axis=1), qc)


def _tiles(rng, rows, K, lo, hi):
    """Small-integer values (exact in E4M3) and an exponent byte per tile that
    differs from tile to tile."""
    v = rng.integers(lo, hi + 1, (rows, K)).astype(np.float32)
    e = rng.integers(-6, 7, (rows, K // 32))
    return oracle.fp8_encode(v), (e + 127).astype(np.uint8), v.astype(np.int64), e


def _tile_dot(va, ea, vb, eb):
    """sum_b 2^(ea_b + eb_b) * (integer dot of tile b), exact."""
    out = np.zeros((va.shape[0], vb.shape[0]), np.float64)
    for b in range(va.shape[1] // 32):
        s = va[:, 32 * b:32 * (b + 1)] @ vb[:, 32 * b:32 * (b + 1)].T
        out += np.ldexp(s.astype(np.float64), ea[:, b][:, None] + eb[:, b][None, :])
    return out


def test_expert_up_mx_exact_on_representable_inputs(oracle_lib):
    rng = np.random.default_rng(4)
    n, d, I = 5, 96, 7
    xq, xe, xv, xee = _tiles(rng, n, d, -4, 4)
    w1q, w1e, w1v, w1ee = _tiles(rng, I, d, -3, 3)
    w3q, w3e, w3v, w3ee = _tiles(rng, I, d, -3, 3)
    h = oracle.expert_up_mx(xq, xe, w1q, w1e, w3q, w3e)
    a = torch.from_numpy(_tile_dot(xv, xee, w1v, w1ee))
    g = torch.from_numpy(_tile_dot(xv, xee, w3v, w3ee))
    ref = (torch.nn.functional.silu(a) * g).float().to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    assert np.array_equal(h, ref)
    # the scales must follow their own tile: reversing the tile order of W1's scales changes a
    h2 = oracle.expert_up_mx(xq, xe, w1q, np.ascontiguousarray(w1e[:, ::-1]), w3q, w3e)
    assert not np.array_equal(h2, h)


def test_expert_down_mx_exact_and_blocked(oracle_lib):
    rng = np.random.default_rng(5)
    n, d, kseg, nseg = 4, 9, 64, 2
    hq, he, hv, hee = _tiles(rng, n, kseg * nseg, -6, 6)
    wv = rng.integers(-5, 6, (nseg, d, kseg)).astype(np.float32)
    wq = oracle.fp8_encode(wv)
    wee = rng.integers(-6, 7, (d, kseg * nseg // 32))
    o = oracle.expert_down_mx(hq, he, wq, (wee + 127).astype(np.uint8))
    wcat = np.concatenate(list(wv), axis=1).astype(np.int64)
    assert np.array_equal(o, _tile_dot(hv, hee, wcat, wee))


def test_layer_mx_close_to_bf16_layer(oracle_lib):
    """The per-tile FP8 layer departs from the bf16 layer only by E4M3
    rounding: 3 mantissa bits (relative error up to 2^-4, about 3.6% RMS for
    values spread over a binade) on each of x, W and h, so a few percent on
    y; a dropped or misplaced tile scale would be off by factors of 2."""
    from fine_grained_moe_gate_b200.inputs import to_numpy
    g = torch.Generator().manual_seed(7)
    T, d, E, k, I, S, Is = 24, 64, 6, 2, 32, 1, 32
    p = dict(x=torch.randn((T, d), generator=g), w1=torch.randn((E, I, d), generator=g) * 0.1,
             w3=torch.randn((E, I, d), generator=g) * 0.1, w2=torch.randn((E, d, I), generator=g) * 0.1,
             ws1=torch.randn((S, Is, d), generator=g) * 0.1, ws3=torch.randn((S, Is, d), generator=g) * 0.1,
             ws2=torch.randn((S, d, Is), generator=g) * 0.1)
    n = {k_: to_numpy(v.to(torch.bfloat16)) for k_, v in p.items()}
    wg = to_numpy((torch.randn((E, d), generator=g) * 0.1).to(torch.bfloat16))
    idx, w = oracle.select(oracle.affinity(n["x"], wg), np.zeros(E, np.float32), k)
    y16 = oracle.layer_output(n["x"], idx, w, n["w1"], n["w3"], n["w2"], n["ws1"], n["ws3"], n["ws2"])
    q = oracle.quantize_weights_mx(n)
    y8 = oracle.layer_output_mx(n["x"], idx, w, q)
    f = lambda b: torch.from_numpy(b.view(np.int16)).view(torch.bfloat16).double().numpy()
    rel = np.linalg.norm(f(y8) - f(y16)) / np.linalg.norm(f(y16))
    assert 1e-3 < rel < 0.08, rel
