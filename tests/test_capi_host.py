"""Host-side checks of the C ABI that need no GPU: the library loads, it
exports every entry point include/moe_gate.h declares, and argument
validation rejects bad calls before anything reaches the device."""
import ctypes
import os
import re

import pytest

import fine_grained_moe_gate_b200 as moe

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "moe_gate.h")

INVALID, UNSUPPORTED, ALIGN, WORKSPACE = 1, 2, 3, 4


def declared_entry_points():
    text = open(HEADER).read()
    return sorted(set(re.findall(r"MOE_API\s+[\w\s\*]+?\b(moe_\w+)\s*\(", text)))


@pytest.fixture(scope="module")
def L():
    if not os.path.exists(moe.LIB_PATH):
        from fine_grained_moe_gate_b200 import build
        build.build()
    return moe.lib()


def test_header_declares_the_abi():
    names = declared_entry_points()
    for required in ("moe_route", "moe_load_and_bias_update", "moe_permute", "moe_grouped_swiglu", "moe_combine",
                     "moe_layer_forward", "moe_workspace_size", "moe_get_last_error"):
        assert required in names


def test_library_exports_every_declared_symbol(L):
    for name in declared_entry_points():
        assert hasattr(L, name), name
    assert set(moe.EXPORTS) == set(declared_entry_points())


def test_abi_version_and_strings(L):
    assert moe.moe_abi_version() == 100
    assert moe.moe_status_string(0) == "ok"
    assert "workspace" in moe.moe_status_string(WORKSPACE)


def shape(**kw):
    base = dict(T=128, d=256, E=16, k=4, I=64, S=1, Is=64, dtype=moe.MOE_F32)
    base.update(kw)
    return moe.MoEShape(*[base[n] for n, _ in moe.MoEShape._fields_])


def test_workspace_sizes(L):
    sh = shape()
    ws = moe.moe_workspace_size(sh)
    assert ws > 0 and ws % 256 == 0
    assert moe.moe_permute_workspace_size(sh) == 256          # one chunk x 16 experts x int32, rounded
    eb = 4
    swg = ((128 * 4 * 64 * eb + 255) // 256 * 256) + ((128 * 1 * 64 * eb + 255) // 256 * 256)
    assert moe.moe_grouped_swiglu_workspace_size(sh) == swg
    # invalid shapes report 0
    assert moe.moe_workspace_size(shape(k=17, E=16)) == 0
    # bf16 needs tensor-core friendly sizes
    assert moe.moe_workspace_size(shape(dtype=moe.MOE_BF16, d=256, I=128, Is=128)) > 0
    assert moe.moe_workspace_size(shape(dtype=moe.MOE_BF16, d=96, I=128, Is=128)) == 0
    assert moe.moe_workspace_size(shape(dtype=moe.MOE_BF16, d=256, I=96, Is=128)) == 0


FAKE = 1 << 20  # a 16-byte aligned non-null "pointer" never dereferenced


def _route(L, sh, **ptr):
    p = dict(x=FAKE, wg=FAKE, bias=FAKE, idx=FAKE, w=FAKE, counts=FAKE, aff=None)
    p.update(ptr)
    c = lambda v: None if v is None else ctypes.c_void_p(v)
    return L.moe_route(c(p["x"]), c(p["wg"]), c(p["bias"]), sh, c(p["idx"]), c(p["w"]), c(p["counts"]), c(p["aff"]),
                       None)


@pytest.mark.parametrize("bad,code", [
    (dict(k=0), INVALID), (dict(k=17, E=32), UNSUPPORTED), (dict(k=5, E=4), INVALID), (dict(E=300), UNSUPPORTED),
    (dict(T=-1), INVALID), (dict(d=12), UNSUPPORTED), (dict(dtype=7), INVALID), (dict(S=1, Is=0), INVALID),
    (dict(dtype=moe.MOE_BF16, d=256, I=64), UNSUPPORTED),
])
def test_route_rejects_bad_shapes(L, bad, code):
    assert _route(L, shape(**bad)) == code


def test_route_rejects_null_and_misaligned(L):
    assert _route(L, shape(), wg=None) == INVALID
    assert _route(L, shape(), counts=None) == INVALID
    assert _route(L, shape(), x=FAKE + 4) == ALIGN
    assert _route(L, shape(), aff=FAKE + 8) == ALIGN


def test_permute_workspace_checks(L):
    sh = shape()
    c = ctypes.c_void_p
    ws_need = moe.moe_permute_workspace_size(sh)
    r = L.moe_permute(c(FAKE), c(FAKE), c(FAKE), sh, c(FAKE), c(FAKE), c(FAKE), c(FAKE), c(FAKE), ws_need - 1, None)
    assert r == WORKSPACE
    r = L.moe_permute(c(FAKE), c(FAKE), c(FAKE), sh, c(FAKE), c(FAKE), c(FAKE), c(FAKE), c(FAKE + 16), ws_need, None)
    assert r == ALIGN


def test_layer_forward_checks(L):
    sh = shape()
    c = ctypes.c_void_p
    need = moe.moe_workspace_size(sh)
    args = [c(FAKE)] * 9
    r = L.moe_layer_forward(*args, sh, c(FAKE), c(FAKE), c(FAKE), c(FAKE), c(FAKE), need - 256, None)
    assert r == WORKSPACE
    args_noshared = [c(FAKE)] * 6 + [None, None, None]
    r = L.moe_layer_forward(*args_noshared, sh, c(FAKE), c(FAKE), c(FAKE), c(FAKE), c(FAKE), need, None)
    assert r == INVALID  # S = 1 needs the shared weights


def test_ffn_checks(L):
    sh = shape()
    c = ctypes.c_void_p
    # up: x_perm, offsets, w1, w3, x, ws1, ws3, sh, h, hs
    assert L.moe_ffn_up(c(FAKE), None, c(FAKE), c(FAKE), None, None, None, sh, c(FAKE), None, None) == INVALID
    assert L.moe_ffn_up(c(FAKE), c(FAKE), c(FAKE), c(FAKE), c(FAKE), None, c(FAKE), sh, c(FAKE), c(FAKE),
                        None) == INVALID                                    # x given: shared weights needed
    assert L.moe_ffn_up(c(FAKE), c(FAKE), c(FAKE), c(FAKE), c(FAKE), c(FAKE), c(FAKE), sh, c(FAKE), None,
                        None) == INVALID                                    # ... and hs
    assert L.moe_ffn_up(c(FAKE), c(FAKE), c(FAKE), c(FAKE), None, None, None, sh, c(FAKE + 4), None,
                        None) == ALIGN
    # down: h, offsets, w2, hs, ws2, sh, y_perm, shared_out
    assert L.moe_ffn_down(c(FAKE), c(FAKE), None, None, None, sh, c(FAKE), None, None) == INVALID
    assert L.moe_ffn_down(c(FAKE), c(FAKE), c(FAKE), c(FAKE), c(FAKE), sh, c(FAKE), None, None) == INVALID
    assert L.moe_ffn_down(c(FAKE), c(FAKE), c(FAKE), c(FAKE), None, sh, c(FAKE), c(FAKE), None) == INVALID
    assert L.moe_ffn_down(c(FAKE), c(FAKE), c(FAKE), None, None, shape(k=17, E=32), c(FAKE), None,
                          None) == UNSUPPORTED


def test_ep_checks(L):
    c = ctypes.c_void_p
    sh = shape(E=16, k=4)
    peers = (ctypes.c_void_p * 4)(FAKE, FAKE, FAKE, FAKE)
    assert moe.moe_ep_plan_size(4, sh) > 0 and moe.moe_ep_plan_size(3, sh) == 0        # E % W != 0
    assert L.moe_ep_dispatch(c(FAKE), c(FAKE), c(FAKE), 3, 0, sh, peers, None) == INVALID
    assert L.moe_ep_dispatch(c(FAKE), c(FAKE), c(FAKE), 4, 4, sh, peers, None) == INVALID   # rank out of range
    assert L.moe_ep_dispatch(c(FAKE), c(FAKE), c(FAKE), 4, 0, shape(E=16, k=4, dtype=moe.MOE_FP8_E4M3, d=256,
                                                                          I=128, Is=128), peers, None) == UNSUPPORTED
    bad = (ctypes.c_void_p * 4)(FAKE, None, FAKE, FAKE)
    assert L.moe_ep_dispatch(c(FAKE), c(FAKE), c(FAKE), 4, 0, sh, bad, None) == INVALID
    odd = (ctypes.c_void_p * 4)(FAKE, FAKE + 8, FAKE, FAKE)
    assert L.moe_ep_return(c(FAKE), c(FAKE), 4, 1, sh, odd, None) == ALIGN
    assert L.moe_ep_plan(c(FAKE), 4, 5, sh, 1024, c(FAKE), None, None) == INVALID          # rank out of range
    assert L.moe_ep_plan(c(FAKE), 4, 1, sh, 0, c(FAKE), None, None) == INVALID             # no receive capacity
    assert L.moe_ep_plan(c(FAKE), 4, 1, sh, 1 << 31, c(FAKE), None, None) == INVALID       # beyond int32 rows


def test_bias_update_checks(L):
    c = ctypes.c_void_p
    assert L.moe_load_and_bias_update(c(FAKE), shape(T=0), ctypes.c_float(1e-3), None, c(FAKE), None, None) == INVALID
    assert L.moe_load_and_bias_update(None, shape(), ctypes.c_float(1e-3), None, c(FAKE), None, None) == INVALID
    assert L.moe_load_and_bias_update(c(FAKE), shape(), ctypes.c_float(float("nan")), None, c(FAKE), None,
                                      None) == INVALID


def test_binding_raises_on_error(L):
    with pytest.raises(moe.MoEError) as ei:
        moe.moe_route(FAKE, None, FAKE, shape(), FAKE, FAKE, FAKE, stream=0)
    assert ei.value.status == INVALID


def test_backward_checks(L):
    """moe_layer_backward validates before touching the device."""
    c = ctypes.c_void_p
    F = ctypes.c_float
    sh = shape()
    need = moe.moe_backward_workspace_size(sh, 0)
    assert need > 0 and need % 256 == 0
    assert moe.moe_backward_workspace_size(sh, 32) > need          # per-sequence buffers
    assert moe.moe_backward_workspace_size(shape(dtype=moe.MOE_FP8_E4M3, d=256, I=128, Is=128), 0) == 0

    def call(sh=sh, x=FAKE, ws1=FAKE, dy=FAKE, dx=FAKE, alpha=0.0, L_=0, ws=FAKE, nbytes=None):
        w = [c(x), c(FAKE), c(FAKE), c(FAKE), c(FAKE), c(ws1), c(FAKE), c(FAKE)]
        return L.moe_layer_backward(*w, sh, c(FAKE), c(FAKE), c(FAKE), c(FAKE), c(dy), F(alpha), L_, c(dx), c(FAKE),
                                    c(FAKE), c(FAKE), c(FAKE), c(FAKE), c(FAKE), c(FAKE), None, c(ws),
                                    need if nbytes is None else nbytes, None)

    assert call(sh=shape(dtype=moe.MOE_FP8_E4M3, d=256, I=128, Is=128)) == UNSUPPORTED
    assert call(dy=None) == INVALID
    assert call(ws1=None) == INVALID                  # S = 1 needs the shared weights
    assert call(alpha=-1.0) == INVALID
    assert call(alpha=float("nan")) == INVALID
    assert call(alpha=0.01, L_=0) == INVALID          # a balance loss needs a sequence length
    assert call(alpha=0.01, L_=48) == INVALID         # that divides T = 128
    assert call(sh=shape(T=65536 * 2), alpha=0.01, L_=1) == UNSUPPORTED   # more than 65535 sequences
    assert call(dx=FAKE + 4) == ALIGN
    assert call(nbytes=need - 256) == WORKSPACE
    assert call(alpha=0.01, L_=32) == WORKSPACE       # the sequences' buffers are not in `need`
    assert call(ws=FAKE + 128) == ALIGN


def test_backward_binding_marshals_and_raises(L):
    """The Python wrapper passes its 28 arguments in header order: a call
    whose only fault is a missing dy comes back as MOE_ERR_INVALID_ARG."""
    import torch
    sh = shape()
    ws = torch.empty(256, dtype=torch.uint8)   # never reached: validation fails first
    with pytest.raises(moe.MoEError) as ei:
        moe.moe_layer_backward(FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, sh, FAKE, FAKE, FAKE, FAKE, None, 0.0,
                               0, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, None, ws, stream=0)
    assert ei.value.status == INVALID
    with pytest.raises(moe.MoEError) as ei:   # every pointer given, alpha negative
        moe.moe_layer_backward(FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, sh, FAKE, FAKE, FAKE, FAKE, FAKE, -1.0,
                               0, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, None, ws, stream=0)
    assert ei.value.status == INVALID


def test_fp8_scale_and_fused_up_checks(L):
    """The FP8 scale helpers and the fused gate/up validate before touching the device."""
    c = ctypes.c_void_p
    sh8 = shape(d=256, I=128, Is=128, dtype=moe.MOE_FP8_E4M3)
    # scale buffer sizes: token words, 128-row atoms, the joint gate/up units, token tile images
    assert moe.moe_fp8_scale_bytes(200, 256, moe.MOE_SF_TOKENS) == 200 * 2 * 4
    assert moe.moe_fp8_scale_bytes(200, 256, moe.MOE_SF_WEIGHTS) == 2 * 2 * 512
    assert moe.moe_fp8_scale_bytes(200, 256, moe.MOE_SF_GATE) == moe.moe_fp8_scale_bytes(200, 256, moe.MOE_SF_UP) \
        == 4 * 2 * 512
    assert moe.moe_fp8_scale_bytes(200, 256, 4) == 0 and moe.moe_fp8_scale_bytes(200, 200, moe.MOE_SF_TOKENS) == 0
    assert moe.moe_fp8_tile_scale_bytes(1000, 8, 256) == (1000 // 256 + 8) * 2 * 1024
    assert moe.moe_fp8_tile_scale_bytes(1000, 0, 256) == 0 and moe.moe_fp8_tile_scale_bytes(1000, 257, 256) == 0
    assert moe.moe_fp8_tile_scale_bytes(1000, 8, 200) == 0
    # moe_fp8_tile_scales(src, src_rows, K, row_of, row_div, offsets, groups, rows, tiles, stream)
    tiles = L.moe_fp8_tile_scales
    assert tiles(c(FAKE), 100, 256, None, 1, None, 2, 100, c(FAKE), None) == INVALID       # groups need offsets
    assert tiles(c(FAKE), 100, 256, c(FAKE), 2, c(FAKE), 257, 100, c(FAKE), None) == INVALID  # more than 256 groups
    assert tiles(c(FAKE), 100, 256, None, 0, None, 1, 100, c(FAKE), None) == INVALID       # row_div 0
    assert tiles(None, 100, 256, None, 1, None, 1, 100, c(FAKE), None) == INVALID
    assert tiles(c(FAKE), 100, 200, None, 1, None, 1, 100, c(FAKE), None) == UNSUPPORTED   # K % 128 != 0
    assert tiles(c(FAKE), 100, 256, None, 1, None, 1, 100, c(FAKE + 4), None) == ALIGN
    # moe_ffn_up_fp8_quant(xq_perm, x_tiles, offsets, xq, xsh_tiles, w, sh, hq, h_tiles, hsq, hs_tiles, stream)
    w8 = moe.MoEFp8Experts()
    assert L.moe_ffn_up_fp8_quant(c(FAKE), c(FAKE), c(FAKE), None, None, ctypes.byref(w8), shape(), c(FAKE), c(FAKE),
                                  None, None, None) == INVALID                              # not an E4M3 shape
    assert L.moe_ffn_up_fp8_quant(c(FAKE), c(FAKE), c(FAKE), None, None, ctypes.byref(w8), sh8, c(FAKE), c(FAKE),
                                  None, None, None) == INVALID                              # no expert weights
