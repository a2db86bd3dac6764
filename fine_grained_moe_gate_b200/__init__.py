"""B200 (sm_100a) fine-grained MoE layer forward -- Python binding.

A thin ctypes binding over ``libmoe_gate.so`` (the C ABI in
``include/moe_gate.h``): each function has the C entry point's name and
arguments, takes torch tensors (or raw device pointers as ints) and raises
``MoEError`` on a non-OK status.  Every step of the layer runs in the
library's CUDA kernels; PyTorch only provides device memory and streams.
There is no CPU fallback: if the library is missing, every call raises.
"""
from __future__ import annotations

import ctypes
import os

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "libmoe_gate.so")

MOE_F32, MOE_BF16 = 0, 1

STATUS = {
    0: "MOE_OK",
    1: "MOE_ERR_INVALID_ARG",
    2: "MOE_ERR_UNSUPPORTED",
    3: "MOE_ERR_ALIGNMENT",
    4: "MOE_ERR_WORKSPACE",
    5: "MOE_ERR_CUDA",
    6: "MOE_ERR_DEVICE_CHECK",
    7: "MOE_ERR_TIMEOUT",
}

EXPORTS = (
    "moe_route", "moe_load_and_bias_update", "moe_permute", "moe_permute_workspace_size", "moe_permute_noalloc",
    "moe_grouped_swiglu", "moe_grouped_swiglu_workspace_size", "moe_expert_up", "moe_expert_down", "moe_ffn_up",
    "moe_ffn_down", "moe_ffn_down_combine", "moe_combine_finish", "moe_combine", "moe_layer_forward",
    "moe_workspace_size", "moe_get_last_error",
    "moe_kernel_launch_count", "moe_selftest_bounded_wait", "moe_status_string", "moe_abi_version",
    "moe_quantize_fp8", "moe_fp8_scale_bytes", "moe_fp8_tile_scales", "moe_fp8_tile_scale_bytes", "moe_ffn_up_fp8",
    "moe_ffn_up_fp8_quant", "moe_ffn_down_fp8",
    "moe_layer_forward_fp8",
    "moe_ep_plan_size", "moe_ep_plan", "moe_ep_dispatch", "moe_ep_return",
    "moe_layer_backward", "moe_backward_workspace_size",
)

MOE_ROUTED, MOE_SHARED = 0, 1
MOE_F32, MOE_BF16, MOE_FP8_E4M3 = 0, 1, 2


class MoEError(RuntimeError):
    def __init__(self, status: int, where: str):
        self.status = status
        super().__init__(f"{where}: {STATUS.get(status, status)}")


class MoEShape(ctypes.Structure):
    _fields_ = [("T", ctypes.c_int32), ("d", ctypes.c_int32), ("E", ctypes.c_int32), ("k", ctypes.c_int32),
                ("I", ctypes.c_int32), ("S", ctypes.c_int32), ("Is", ctypes.c_int32), ("dtype", ctypes.c_int32)]

    def __repr__(self):
        return "MoEShape(" + ", ".join(f"{n}={getattr(self, n)}" for n, _ in self._fields_) + ")"


def shape_of(cfg, T: int | None = None) -> MoEShape:
    """MoEShape from a workload config (``inputs.MoEConfig``)."""
    return MoEShape(cfg.T if T is None else T, cfg.d, cfg.E, cfg.k, cfg.I, cfg.S, cfg.Is,
                    {"bf16": MOE_BF16, "fp8": MOE_FP8_E4M3}.get(cfg.dtype, MOE_F32))


class MoEFp8Experts(ctypes.Structure):
    """moe_fp8_experts: E4M3 expert weights and their 1x32-tile power-of-two
    scales (W1/W3 scales in one gate/up buffer, W2 in 128-row atoms)."""
    _fields_ = [(n, ctypes.c_void_p) for n in ("w1", "w3", "w13_scale", "w2", "w2_scale",
                                               "ws1", "ws3", "ws13_scale", "ws2", "ws2_scale")]


def fp8_experts(q: dict) -> MoEFp8Experts:
    """MoEFp8Experts from a dict of device tensors with keys w1q, w3q, w13s,
    w2q, w2s, ... (the layout of ``quantize_experts_fp8``).  The tensors must
    outlive its use."""
    f = {n: _p(q.get(n + "q")) for n in ("w1", "w3", "w2", "ws1", "ws3", "ws2")}
    for n in ("w13", "w2", "ws13", "ws2"):
        f[n + "_scale"] = _p(q.get(n + "s"))
    return MoEFp8Experts(**f)


_lib = None


def lib() -> ctypes.CDLL:
    """The loaded library; raises MoEError-free ImportError if it is not built."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise ImportError(f"{LIB_PATH} is missing: build it with `python -m fine_grained_moe_gate_b200.build`")
        L = ctypes.CDLL(LIB_PATH)
        P, S, F = ctypes.c_void_p, MoEShape, ctypes.c_float
        sz = ctypes.c_size_t
        sig = {
            "moe_route": [P, P, P, S, P, P, P, P, P],
            "moe_load_and_bias_update": [P, S, F, P, P, P, P],
            "moe_permute": [P, P, P, S, P, P, P, P, P, sz, P],
            "moe_permute_noalloc": [P, P, P, S, P, P, P, P, P],
            "moe_grouped_swiglu": [P, P, P, P, P, P, P, P, P, S, P, P, P, sz, P],
            "moe_expert_up": [P, P, P, P, P, S, ctypes.c_int32, P, P],
            "moe_expert_down": [P, P, P, S, ctypes.c_int32, P, P],
            "moe_ffn_up": [P, P, P, P, P, P, P, S, P, P, P],
            "moe_ffn_down": [P, P, P, P, P, S, P, P, P],
            "moe_combine": [P, P, P, P, S, P, P],
            "moe_ffn_down_combine": [P, P, P, P, P, P, P, S, P, P],
            "moe_combine_finish": [P, S, P, P],
            "moe_layer_forward": [P, P, P, P, P, P, P, P, P, S, P, P, P, P, P, sz, P],
            "moe_get_last_error": [P],
            "moe_quantize_fp8": [P, ctypes.c_int64, ctypes.c_int32, ctypes.c_int32, ctypes.c_int32, P, P, P],
            "moe_ffn_up_fp8": [P, P, P, P, P, ctypes.POINTER(MoEFp8Experts), S, P, P, P],
            "moe_ffn_up_fp8_quant": [P, P, P, P, P, ctypes.POINTER(MoEFp8Experts), S, P, P, P, P, P],
            "moe_fp8_tile_scales": [P, ctypes.c_int64, ctypes.c_int32, P, ctypes.c_int32, P, ctypes.c_int32,
                                    ctypes.c_int64, P, P],
            "moe_ffn_down_fp8": [P, P, P, P, P, ctypes.POINTER(MoEFp8Experts), S, P, P, P],
            "moe_layer_forward_fp8": [P, P, P, ctypes.POINTER(MoEFp8Experts), S, P, P, P, P, P, sz, P],
            "moe_ep_plan": [P, ctypes.c_int32, ctypes.c_int32, S, ctypes.c_int64, P, P, P],
            "moe_ep_dispatch": [P, P, P, ctypes.c_int32, ctypes.c_int32, S, P, P],
            "moe_ep_return": [P, P, ctypes.c_int32, ctypes.c_int32, S, P, P],
            "moe_selftest_bounded_wait": [ctypes.c_uint32, P],
            "moe_layer_backward": [P, P, P, P, P, P, P, P, S, P, P, P, P, P, F, ctypes.c_int32, P, P, P, P, P, P, P,
                                   P, P, P, sz, P],
        }
        for name, args in sig.items():
            fn = getattr(L, name)
            fn.argtypes = args
            fn.restype = ctypes.c_int
        for name in ("moe_workspace_size", "moe_permute_workspace_size", "moe_grouped_swiglu_workspace_size"):
            fn = getattr(L, name)
            fn.argtypes = [S]
            fn.restype = sz
        L.moe_backward_workspace_size.argtypes = [S, ctypes.c_int32]
        L.moe_backward_workspace_size.restype = sz
        L.moe_fp8_scale_bytes.argtypes = [ctypes.c_int64, ctypes.c_int32, ctypes.c_int32]
        L.moe_fp8_scale_bytes.restype = sz
        L.moe_fp8_tile_scale_bytes.argtypes = [ctypes.c_int64, ctypes.c_int32, ctypes.c_int32]
        L.moe_fp8_tile_scale_bytes.restype = sz
        L.moe_ep_plan_size.argtypes = [ctypes.c_int32, S]
        L.moe_ep_plan_size.restype = sz
        L.moe_kernel_launch_count.argtypes = []
        L.moe_kernel_launch_count.restype = ctypes.c_uint64
        L.moe_status_string.argtypes = [ctypes.c_int]
        L.moe_status_string.restype = ctypes.c_char_p
        L.moe_abi_version.argtypes = []
        L.moe_abi_version.restype = ctypes.c_int
        _lib = L
    return _lib


def _p(t):
    """Device pointer of a tensor (None -> NULL; an int is taken as a pointer)."""
    if t is None:
        return None
    if isinstance(t, int):
        return ctypes.c_void_p(t)
    return ctypes.c_void_p(t.data_ptr())


def _stream(stream):
    if stream is None:
        import torch
        return ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    if isinstance(stream, int):
        return ctypes.c_void_p(stream)
    return ctypes.c_void_p(stream.cuda_stream)


def _check(status: int, where: str):
    if status != 0:
        raise MoEError(status, where)


def _nbytes(t) -> int:
    return 0 if t is None else t.numel() * t.element_size()


# ---- entry points (same names and argument order as moe_gate.h) -----------

def moe_route(x, w_gate, bias, shape, topk_idx, topk_w, counts, affinity_out=None, stream=None):
    _check(lib().moe_route(_p(x), _p(w_gate), _p(bias), shape, _p(topk_idx), _p(topk_w), _p(counts),
                           _p(affinity_out), _stream(stream)), "moe_route")


def moe_load_and_bias_update(counts, shape, step, target, bias, load_out=None, stream=None):
    _check(lib().moe_load_and_bias_update(_p(counts), shape, ctypes.c_float(step), _p(target), _p(bias), _p(load_out),
                                          _stream(stream)), "moe_load_and_bias_update")


def moe_permute(x, topk_idx, counts, shape, x_perm, offsets, perm_tok, inv_row, workspace, stream=None):
    _check(lib().moe_permute(_p(x), _p(topk_idx), _p(counts), shape, _p(x_perm), _p(offsets), _p(perm_tok),
                             _p(inv_row), _p(workspace), _nbytes(workspace), _stream(stream)), "moe_permute")


def moe_permute_noalloc(x, topk_idx, counts, shape, x_perm, offsets, perm_tok, inv_row, stream=None):
    """moe_permute for callers that cannot provide scratch memory: the
    library uses a fixed array in its own device image instead (see
    moe_gate.h for the size limit and the sharing rules)."""
    _check(lib().moe_permute_noalloc(_p(x), _p(topk_idx), _p(counts), shape, _p(x_perm), _p(offsets), _p(perm_tok),
                                     _p(inv_row), _stream(stream)), "moe_permute_noalloc")


def moe_grouped_swiglu(x_perm, offsets, w1, w3, w2, x, ws1, ws3, ws2, shape, y_perm, shared_out, workspace,
                       stream=None):
    _check(lib().moe_grouped_swiglu(_p(x_perm), _p(offsets), _p(w1), _p(w3), _p(w2), _p(x), _p(ws1), _p(ws3),
                                    _p(ws2), shape, _p(y_perm), _p(shared_out), _p(workspace), _nbytes(workspace),
                                    _stream(stream)), "moe_grouped_swiglu")


def moe_expert_up(a, gather_idx, offsets, w1, w3, shape, expert_set, h, stream=None):
    _check(lib().moe_expert_up(_p(a), _p(gather_idx), _p(offsets), _p(w1), _p(w3), shape, expert_set, _p(h),
                               _stream(stream)), "moe_expert_up")


def moe_expert_down(h, offsets, w2, shape, expert_set, y, stream=None):
    _check(lib().moe_expert_down(_p(h), _p(offsets), _p(w2), shape, expert_set, _p(y), _stream(stream)),
           "moe_expert_down")


def moe_ffn_up(x_perm, offsets, w1, w3, x, ws1, ws3, shape, h, hs, stream=None):
    _check(lib().moe_ffn_up(_p(x_perm), _p(offsets), _p(w1), _p(w3), _p(x), _p(ws1), _p(ws3), shape, _p(h), _p(hs),
                            _stream(stream)), "moe_ffn_up")


def moe_ffn_down(h, offsets, w2, hs, ws2, shape, y_perm, shared_out, stream=None):
    _check(lib().moe_ffn_down(_p(h), _p(offsets), _p(w2), _p(hs), _p(ws2), shape, _p(y_perm), _p(shared_out),
                              _stream(stream)), "moe_ffn_down")


def moe_ffn_down_combine(h, offsets, w2, hs, ws2, perm_tok, topk_w, shape, y_acc, stream=None):
    _check(lib().moe_ffn_down_combine(_p(h), _p(offsets), _p(w2), _p(hs), _p(ws2), _p(perm_tok), _p(topk_w), shape,
                                      _p(y_acc), _stream(stream)), "moe_ffn_down_combine")


def moe_combine_finish(y_acc, shape, y, stream=None):
    _check(lib().moe_combine_finish(_p(y_acc), shape, _p(y), _stream(stream)), "moe_combine_finish")


def moe_combine(y_perm, topk_w, inv_row, shared_out, shape, y, stream=None):
    _check(lib().moe_combine(_p(y_perm), _p(topk_w), _p(inv_row), _p(shared_out), shape, _p(y), _stream(stream)),
           "moe_combine")


def moe_layer_forward(x, w_gate, bias, w1, w3, w2, ws1, ws3, ws2, shape, y, topk_idx, topk_w, counts, workspace,
                      stream=None):
    _check(lib().moe_layer_forward(_p(x), _p(w_gate), _p(bias), _p(w1), _p(w3), _p(w2), _p(ws1), _p(ws3), _p(ws2),
                                   shape, _p(y), _p(topk_idx), _p(topk_w), _p(counts), _p(workspace),
                                   _nbytes(workspace), _stream(stream)), "moe_layer_forward")


def moe_workspace_size(shape) -> int:
    return lib().moe_workspace_size(shape)


def moe_layer_backward(x, w_gate, w1, w3, w2, ws1, ws3, ws2, shape, topk_idx, topk_w, counts, affinity, dy, alpha,
                       seq_len, dx, dw_gate, dw1, dw3, dw2, dws1, dws3, dws2, balance_loss, workspace, stream=None):
    _check(lib().moe_layer_backward(_p(x), _p(w_gate), _p(w1), _p(w3), _p(w2), _p(ws1), _p(ws3), _p(ws2), shape,
                                    _p(topk_idx), _p(topk_w), _p(counts), _p(affinity), _p(dy), float(alpha),
                                    int(seq_len), _p(dx), _p(dw_gate), _p(dw1), _p(dw3), _p(dw2), _p(dws1), _p(dws3),
                                    _p(dws2), _p(balance_loss), _p(workspace), _nbytes(workspace), _stream(stream)),
           "moe_layer_backward")


def moe_backward_workspace_size(shape, seq_len: int = 0) -> int:
    return lib().moe_backward_workspace_size(shape, int(seq_len))


def moe_permute_workspace_size(shape) -> int:
    return lib().moe_permute_workspace_size(shape)


def moe_grouped_swiglu_workspace_size(shape) -> int:
    return lib().moe_grouped_swiglu_workspace_size(shape)


def moe_get_last_error(stream=None) -> int:
    return lib().moe_get_last_error(_stream(stream))


def moe_selftest_bounded_wait(limit_us: int, stream=None):
    _check(lib().moe_selftest_bounded_wait(limit_us, _stream(stream)), "moe_selftest_bounded_wait")


def moe_kernel_launch_count() -> int:
    return lib().moe_kernel_launch_count()


def moe_status_string(status: int) -> str:
    return lib().moe_status_string(status).decode()


def moe_abi_version() -> int:
    return lib().moe_abi_version()


# ---- FP8 experts -------------------------------------------------------------

MOE_SF_TOKENS, MOE_SF_WEIGHTS, MOE_SF_GATE, MOE_SF_UP = 0, 1, 2, 3


def moe_fp8_scale_bytes(rows, K, layout) -> int:
    return lib().moe_fp8_scale_bytes(rows, K, layout)


def moe_quantize_fp8(src, rows, kseg, nseg, layout, q, scales, stream=None):
    _check(lib().moe_quantize_fp8(_p(src), rows, kseg, nseg, layout, _p(q), _p(scales), _stream(stream)),
           "moe_quantize_fp8")


def fp8_scales(rows, K, layout, device):
    """An uninitialised device buffer for the tile scales of a [rows][K] matrix
    in the given layout (uint8, moe_fp8_scale_bytes long)."""
    import torch
    n = moe_fp8_scale_bytes(rows, K, layout)
    if n == 0:
        raise MoEError(1, "moe_fp8_scale_bytes: K must be a multiple of 128")
    return torch.empty(n, dtype=torch.uint8, device=device)


def moe_fp8_tile_scale_bytes(rows, groups, K) -> int:
    return lib().moe_fp8_tile_scale_bytes(rows, groups, K)


def fp8_tile_images(rows, groups, K, device):
    """An uninitialised device buffer for the token tile images of `rows`
    operand rows in `groups` groups with K columns (uint8)."""
    import torch
    n = moe_fp8_tile_scale_bytes(rows, groups, K)
    if n == 0:
        raise MoEError(1, "moe_fp8_tile_scale_bytes: K must be a multiple of 128, 1 <= groups <= 256")
    return torch.empty(n, dtype=torch.uint8, device=device)


def moe_fp8_tile_scales(src, src_rows, K, row_of, row_div, offsets, groups, rows, tiles, stream=None):
    _check(lib().moe_fp8_tile_scales(_p(src), src_rows, K, _p(row_of), row_div, _p(offsets), groups, rows, _p(tiles),
                                     _stream(stream)), "moe_fp8_tile_scales")


def moe_ffn_up_fp8(xq_perm, x_tiles, offsets, xq, xsh_tiles, experts, shape, h, hs, stream=None):
    _check(lib().moe_ffn_up_fp8(_p(xq_perm), _p(x_tiles), _p(offsets), _p(xq), _p(xsh_tiles), ctypes.byref(experts),
                                shape, _p(h), _p(hs), _stream(stream)), "moe_ffn_up_fp8")


def moe_ffn_up_fp8_quant(xq_perm, x_tiles, offsets, xq, xsh_tiles, experts, shape, hq, h_tiles, hsq, hs_tiles,
                         stream=None):
    _check(lib().moe_ffn_up_fp8_quant(_p(xq_perm), _p(x_tiles), _p(offsets), _p(xq), _p(xsh_tiles),
                                      ctypes.byref(experts), shape, _p(hq), _p(h_tiles), _p(hsq), _p(hs_tiles),
                                      _stream(stream)), "moe_ffn_up_fp8_quant")


def moe_ffn_down_fp8(hq, h_tiles, offsets, hsq, hs_tiles, experts, shape, y_perm, shared_out, stream=None):
    _check(lib().moe_ffn_down_fp8(_p(hq), _p(h_tiles), _p(offsets), _p(hsq), _p(hs_tiles), ctypes.byref(experts),
                                  shape, _p(y_perm), _p(shared_out), _stream(stream)), "moe_ffn_down_fp8")


def moe_layer_forward_fp8(x, w_gate, bias, experts, shape, y, topk_idx, topk_w, counts, workspace, stream=None):
    _check(lib().moe_layer_forward_fp8(_p(x), _p(w_gate), _p(bias), ctypes.byref(experts), shape, _p(y),
                                       _p(topk_idx), _p(topk_w), _p(counts), _p(workspace), _nbytes(workspace),
                                       _stream(stream)), "moe_layer_forward_fp8")


def quantize_experts_fp8(p: dict, stream=None) -> dict:
    """E4M3 copies of a layer's bf16 expert weights (device tensors) through
    moe_quantize_fp8: W1 and W3 (Ws1 and Ws3) with their scales in one gate/up
    buffer (MOE_SF_GATE, MOE_SF_UP), W2 in 128-row atoms (MOE_SF_WEIGHTS), the
    shared Ws2 [S][d][Is] as d rows across its S blocks.  Returns uint8 codes
    (the weights' own shapes) under w1q, w3q, w2q, ... and scale buffers under
    w13s, w2s, ws13s, ws2s."""
    import torch
    out = {}
    for a, b in (("w1", "w3"), ("ws1", "ws3")):
        w1, w3 = p.get(a), p.get(b)
        if w1 is None or w1.numel() == 0:
            continue
        rows, K = w1.numel() // w1.shape[-1], w1.shape[-1]
        sc = fp8_scales(rows, K, MOE_SF_GATE, w1.device)
        for n, w, lay in ((a, w1, MOE_SF_GATE), (b, w3, MOE_SF_UP)):
            q = torch.empty(w.shape, dtype=torch.uint8, device=w.device)
            moe_quantize_fp8(w, rows, K, 1, lay, q, sc, stream)
            out[n + "q"] = q
        out[a[:-1] + "13s"] = sc
    w = p["w2"]
    rows, K = w.numel() // w.shape[-1], w.shape[-1]
    q = torch.empty(w.shape, dtype=torch.uint8, device=w.device)
    sc = fp8_scales(rows, K, MOE_SF_WEIGHTS, w.device)
    moe_quantize_fp8(w, rows, K, 1, MOE_SF_WEIGHTS, q, sc, stream)
    out["w2q"], out["w2s"] = q, sc
    w = p.get("ws2")
    if w is not None and w.numel() > 0:
        S, d, Is = w.shape
        q = torch.empty(w.shape, dtype=torch.uint8, device=w.device)
        sc = fp8_scales(d, S * Is, MOE_SF_WEIGHTS, w.device)
        moe_quantize_fp8(w, d, Is, S, MOE_SF_WEIGHTS, q, sc, stream)
        out["ws2q"], out["ws2s"] = q, sc
    return out


# ---- expert parallelism --------------------------------------------------------

def _ptr_array(bufs):
    arr = (ctypes.c_void_p * len(bufs))()
    for i, b in enumerate(bufs):
        arr[i] = b if isinstance(b, int) else b.data_ptr()
    return arr


def moe_ep_plan_size(world, shape) -> int:
    return lib().moe_ep_plan_size(world, shape)


def moe_ep_plan(counts_all, world, rank, shape, recv_capacity, plan, recv_offsets, stream=None):
    _check(lib().moe_ep_plan(_p(counts_all), world, rank, shape, recv_capacity, _p(plan), _p(recv_offsets),
                             _stream(stream)),
           "moe_ep_plan")


def moe_ep_dispatch(x, perm_tok, plan, world, rank, shape, recv_bufs, stream=None):
    """recv_bufs: per rank, its receive buffer (tensor or device pointer valid here)."""
    _check(lib().moe_ep_dispatch(_p(x), _p(perm_tok), _p(plan), world, rank, shape, _ptr_array(recv_bufs),
                                 _stream(stream)), "moe_ep_dispatch")


def moe_ep_return(y_recv, plan, world, rank, shape, back_bufs, stream=None):
    """back_bufs: per rank, its return buffer (tensor or device pointer valid here)."""
    _check(lib().moe_ep_return(_p(y_recv), _p(plan), world, rank, shape, _ptr_array(back_bufs), _stream(stream)),
           "moe_ep_return")
