"""Pins for the oracle's FP8 expert functions (CPU only).

Page cited: "DeepSeek V3 Architecture Deep Dive ...", sections "FP8 Formats"
(E4M3 for weights and activations) and "Per-Tensor/Per-Axis Quantization"
(a scale per row/channel).  The E4M3 codec is checked against the format's
own field definition, against torch's float8_e4m3fn conversion, and on ties,
saturation and subnormals; quantization and the expert sums against closed
forms on inputs the format represents exactly.
"""
import numpy as np
import pytest
import torch

import oracle


def _field_value(c: int) -> float:
    """Value of an E4M3 code straight from its sign / exponent / mantissa fields."""
    s, e, m = (c >> 7) & 1, (c >> 3) & 0xF, c & 7
    if e == 0xF and m == 7:
        return float("nan")
    mag = (m / 8.0) * 2.0 ** -6 if e == 0 else (1.0 + m / 8.0) * 2.0 ** (e - 7)
    return -mag if s else mag


def test_e4m3_decode_matches_field_definition(oracle_lib):
    codes = np.arange(256, dtype=np.uint8)
    got = oracle.fp8_decode(codes)
    ref = np.array([_field_value(int(c)) for c in codes])
    nan = np.isnan(ref)
    assert np.array_equal(np.isnan(got), nan) and nan.sum() == 2          # 0x7F and 0xFF
    assert np.array_equal(got[~nan], ref[~nan])
    assert got[0x38] == 1.0 and got[0x7E] == 448.0 and got[0x01] == 2.0 ** -9 and got[0x08] == 2.0 ** -6
    assert np.nanmax(got) == 448.0 and np.nanmin(got) == -448.0


def test_e4m3_encode_inverts_decode_on_every_code(oracle_lib):
    codes = np.arange(256, dtype=np.uint8)
    vals = oracle.fp8_decode(codes)
    fin = ~np.isnan(vals)
    assert np.array_equal(oracle.fp8_encode(vals[fin].astype(np.float32)), codes[fin])


def test_e4m3_ties_saturation_and_subnormals(oracle_lib):
    cases = [
        (1.0625, 0x38),                 # tie between 1.0 (m=0) and 1.125 (m=1): even mantissa
        (1.1875, 0x3A),                 # tie between 1.125 and 1.25 (m=2)
        (0.96875, 0x38),                # tie between 0.9375 (m=7, odd) and 1.0: carries into the next binade
        (0.953125, 0x37),               # 15.25 steps of 2^-4 below 1: down to 0.9375
        (448.0, 0x7E), (450.0, 0x7E), (464.0, 0x7E), (1e30, 0x7E), (-500.0, 0xFE),   # saturation
        (2.0 ** -10, 0x00),             # half a subnormal step: tie to 0
        (3 * 2.0 ** -11, 0x01),         # 0.75 of a step
        (5 * 2.0 ** -11, 0x01),         # 1.25 steps
        (2.0 ** -6 - 2.0 ** -10, 0x08), # 7.5 steps: tie to 8 = the smallest normal
        (0.0, 0x00), (-0.0, 0x80),
    ]
    got = oracle.fp8_encode(np.array([v for v, _ in cases], np.float32))
    assert got.tolist() == [c for _, c in cases]


def test_e4m3_encode_matches_torch_float8_in_range(oracle_lib):
    """Inside the finite range torch's float8_e4m3fn cast is round-to-nearest-even too."""
    g = np.random.default_rng(0)
    x = np.concatenate([g.standard_normal(20000) * 40, g.standard_normal(5000) * 2.0 ** -7,
                        g.uniform(-447.0, 447.0, 5000)]).astype(np.float32)
    ref = torch.from_numpy(x).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    assert np.array_equal(oracle.fp8_encode(x), ref)


def test_e4m3_encode_is_monotone_and_within_half_step(oracle_lib):
    x = np.sort(np.random.default_rng(1).uniform(-460, 460, 50000)).astype(np.float32)
    v = oracle.fp8_decode(oracle.fp8_encode(x))
    assert np.all(np.diff(v) >= 0)
    a = np.abs(x.astype(np.float64))
    inside = a < 448
    binade = np.maximum(np.floor(np.log2(np.maximum(a, 2.0 ** -30))), -6)
    half_step = 2.0 ** (binade - 4)
    assert np.all(np.abs(v - x)[inside] <= half_step[inside])


def test_quantize_rows_scale_and_codes(oracle_lib):
    g = torch.Generator().manual_seed(3)
    a = (torch.randn((37, 200), generator=g) * 0.05).to(torch.bfloat16)
    a[5] = 0                                            # an all-zero row
    bits = a.view(torch.int16).numpy().view(np.uint16)
    q, sc = oracle.quantize_rows_fp8(bits)
    af = a.float().numpy()
    amax = np.abs(af).max(axis=1)
    want_sc = np.where(amax > 0, amax / np.float32(448.0), np.float32(1.0)).astype(np.float32)
    assert np.array_equal(sc, want_sc)
    assert np.all(q[5] == 0) and sc[5] == 1.0
    # codes = encode(v * (448 / amax)) element by element, and the row max maps to +-448
    inv = np.where(amax > 0, np.float32(448.0) / np.where(amax > 0, amax, 1), np.float32(0)).astype(np.float32)
    assert np.array_equal(q, oracle.fp8_encode((af * inv[:, None]).astype(np.float32)))
    dec = oracle.fp8_decode(q)
    nz = amax > 0
    assert np.all(np.abs(dec[nz]).max(axis=1) == 448.0)
    # dequantised error within half an E4M3 step (relative 2^-4) plus the subnormal floor
    err = np.abs(dec * sc[:, None] - af)
    assert np.all(err <= np.abs(af) * 2.0 ** -4 + sc[:, None] * 2.0 ** -10)


def test_quantize_rows_blocked_layout_equals_concatenated(oracle_lib):
    """A matrix stored as [nseg][rows][kseg] is quantized per row across all
    blocks, exactly as the concatenated [rows][nseg*kseg] matrix."""
    g = torch.Generator().manual_seed(4)
    blk = torch.randn((3, 9, 16), generator=g).to(torch.bfloat16)
    cat = torch.cat(list(blk), dim=1)                              # [9][48]
    qb, sb = oracle.quantize_rows_fp8(blk.view(torch.int16).numpy().view(np.uint16), nseg=3)
    qc, sc = oracle.quantize_rows_fp8(cat.contiguous().view(torch.int16).numpy().view(np.uint16))
    assert np.array_equal(sb, sc)
    assert np.array_equal(np.concatenate(list(qb), axis=1), qc)


def _codes_of(vals):
    return oracle.fp8_encode(np.asarray(vals, np.float32))


def test_expert_up_fp8_exact_on_representable_inputs(oracle_lib):
    """Small-integer codes and power-of-two scales make every product and sum
    exact: a = xs*w1s*(xq . w1q) is an integer matmul, and h must equal
    bf16(silu(a) * g) computed from it independently (torch, float64)."""
    g = np.random.default_rng(5)
    n, d, I = 6, 24, 10
    xi = g.integers(-4, 5, (n, d)).astype(np.float32)
    w1i = g.integers(-3, 4, (I, d)).astype(np.float32)
    w3i = g.integers(-3, 4, (I, d)).astype(np.float32)
    xs = (2.0 ** g.integers(-8, -3, n)).astype(np.float32)
    w1s = (2.0 ** g.integers(-6, -2, I)).astype(np.float32)
    w3s = (2.0 ** g.integers(-6, -2, I)).astype(np.float32)
    h = oracle.expert_up_fp8(_codes_of(xi), xs, _codes_of(w1i), w1s, _codes_of(w3i), w3s)
    a = torch.from_numpy((xi.astype(np.int64) @ w1i.T.astype(np.int64)).astype(np.float64)) * \
        torch.from_numpy(xs.astype(np.float64))[:, None] * torch.from_numpy(w1s.astype(np.float64))[None]
    gg = torch.from_numpy((xi.astype(np.int64) @ w3i.T.astype(np.int64)).astype(np.float64)) * \
        torch.from_numpy(xs.astype(np.float64))[:, None] * torch.from_numpy(w3s.astype(np.float64))[None]
    ref = (torch.nn.functional.silu(a) * gg).float().to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    assert np.array_equal(h, ref)


def test_expert_down_fp8_exact_and_blocked(oracle_lib):
    g = np.random.default_rng(6)
    n, d, kseg, nseg = 5, 12, 8, 2
    hi = g.integers(-6, 7, (n, kseg * nseg)).astype(np.float32)
    wi = g.integers(-5, 6, (nseg, d, kseg)).astype(np.float32)
    hs = (2.0 ** g.integers(-9, -4, n)).astype(np.float32)
    ws = (2.0 ** g.integers(-7, -3, d)).astype(np.float32)
    o = oracle.expert_down_fp8(_codes_of(hi), hs, _codes_of(wi), ws)
    wcat = np.concatenate(list(wi), axis=1)                          # [d][K]
    ref = (hi.astype(np.int64) @ wcat.T.astype(np.int64)).astype(np.float64) * hs[:, None] * ws[None]
    assert np.array_equal(o, ref)


def test_layer_fp8_close_to_bf16_layer(oracle_lib):
    """The FP8 layer departs from the bf16 layer only by E4M3 rounding (3
    mantissa bits on x, W and h): the relative error of y stays at the few-
    percent level and shrinks to 0 where quantization is lossless."""
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
    q = oracle.quantize_weights_fp8(n)
    y8 = oracle.layer_output_fp8(n["x"], idx, w, q)
    f = lambda b: torch.from_numpy(b.view(np.int16)).view(torch.bfloat16).double().numpy()
    rel = np.linalg.norm(f(y8) - f(y16)) / np.linalg.norm(f(y16))
    assert 1e-3 < rel < 0.08, rel
