"""Pins for the oracle's E4M3 codec (CPU only); the per-tile quantization
and the FP8 expert sums built on it are pinned in test_oracle_mx_pins.py.

Page cited: "DeepSeek V3 Architecture Deep Dive ...", section "FP8 Formats"
(E4M3 for weights and activations).  The codec is checked against the
format's own field definition, against torch's float8_e4m3fn conversion, and
on ties, saturation and subnormals.
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
