"""CPU oracle for the fine-grained MoE layer forward -- TEST INFRASTRUCTURE.

Only the tests, the package smoke check and the bench's CPU-baseline leg may
import this module.  The CUDA library never calls it and shares no code with it.

The arithmetic lives in ``moe_oracle.c`` (plain C, double accumulation); this
module only builds it with gcc and marshals numpy arrays.  bf16 tensors are
passed as ``uint16`` arrays holding the raw bf16 bits.

Sources, by page title and section:
  * "DeepSeek V3 From Scratch" -- "The idea", "Worked example", "In code".
  * "Scaling Efficiency: A Deep Dive into the DeepSeek-V3 Architecture" --
    the DeepSeekMoE module sketch.
  * kbwen.com DeepSeek tag page -- "A bias term for each expert".
  * "DeepSeek V3 Architecture Deep Dive ..." -- "FP8 Formats" (E4M3).
  * "DeepSeek V3 From Scratch", "The idea", and crackai.dev "DeepSeek-V3",
    "How It Works" -- FP8 with per-tile scaling (the *_mx functions).
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "moe_oracle.c")
_LIB = os.path.join(_HERE, "liboracle.so")

F32 = 0
BF16 = 1

_lib = None


def build(force: bool = False) -> str:
    """Compile moe_oracle.c into liboracle.so next to it (gcc, OpenMP)."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        tmp = _LIB + f".tmp{os.getpid()}"
        subprocess.check_call(
            ["gcc", "-O2", "-fopenmp", "-ffp-contract=off", "-fno-fast-math", "-shared", "-fPIC",
             "-o", tmp, _SRC, "-lm"])
        os.replace(tmp, _LIB)
    return _LIB


def _load():
    global _lib
    if _lib is None:
        build()
        lib = ctypes.CDLL(_LIB)
        P = ctypes.c_void_p
        i = ctypes.c_int
        lib.orc_affinity.argtypes = [P, P, i, i, i, i, P]
        lib.orc_select.argtypes = [P, P, i, i, i, P, P]
        lib.orc_select.restype = i
        lib.orc_histogram.argtypes = [P, i, i, i, P]
        lib.orc_histogram.restype = i
        lib.orc_bias_update.argtypes = [P, i, i, i, ctypes.c_float, P, P, P]
        lib.orc_permute.argtypes = [P, i, i, i, P, P, P]
        lib.orc_permute.restype = i
        lib.orc_expert_accumulate.argtypes = [P, i, P, P, P, P, P, i, i, i, P]
        lib.orc_finalize.argtypes = [P, ctypes.c_size_t, i, P]
        lib.orc_expert_up.argtypes = [P, i, P, P, i, i, i, P]
        lib.orc_expert_down.argtypes = [P, i, P, i, i, i, P]
        lib.orc_layer_output.argtypes = [P, P, P, P, P, P, P, P, P, i, i, i, i, i, i, i, i, P]
        lib.orc_e4m3_encode_array.argtypes = [P, ctypes.c_size_t, P]
        lib.orc_e4m3_decode_array.argtypes = [P, ctypes.c_size_t, P]
        lib.orc_mx_exponent.argtypes = [ctypes.c_double]
        lib.orc_mx_exponent.restype = i
        lib.orc_quantize_mx.argtypes = [P, i, ctypes.c_long, i, i, P, P]
        lib.orc_expert_up_mx.argtypes = [P, P, i, P, P, P, P, i, i, P]
        lib.orc_expert_down_mx.argtypes = [P, P, i, P, P, i, i, i, P]
        _lib = lib
    return _lib


def _ptr(a):
    return None if a is None else a.ctypes.data_as(ctypes.c_void_p)


def _dtype_code(a: np.ndarray) -> int:
    if a.dtype == np.float32:
        return F32
    if a.dtype == np.uint16:
        return BF16
    raise TypeError(f"oracle takes float32 or bf16-as-uint16 arrays, got {a.dtype}")


def _c(a, dtype=None):
    a = np.ascontiguousarray(a if dtype is None else a.astype(dtype, copy=False))
    return a


def affinity(x: np.ndarray, w_gate: np.ndarray) -> np.ndarray:
    """s = sigmoid(x @ W_g^T), double inside, fp32 out.  x [T][d], W_g [E][d]."""
    x, w_gate = _c(x), _c(w_gate)
    dt = _dtype_code(x)
    assert _dtype_code(w_gate) == dt
    T, d = x.shape
    E = w_gate.shape[0]
    s = np.empty((T, E), np.float32)
    _load().orc_affinity(_ptr(x), _ptr(w_gate), dt, T, d, E, _ptr(s))
    return s


def select(s: np.ndarray, bias: np.ndarray, k: int):
    """Top-k of fl32(s + b) by rank counting; weights from the unbiased s.

    Returns (idx int32 [T][k], w float32 [T][k])."""
    s, bias = _c(s, np.float32), _c(bias, np.float32)
    T, E = s.shape
    idx = np.empty((T, k), np.int32)
    w = np.empty((T, k), np.float32)
    rc = _load().orc_select(_ptr(s), _ptr(bias), T, E, k, _ptr(idx), _ptr(w))
    if rc != 0:
        raise ValueError("oracle select: a row did not fill k slots (non-finite scores)")
    return idx, w


def histogram(idx: np.ndarray, E: int) -> np.ndarray:
    idx = _c(idx, np.int32)
    T, k = idx.shape
    counts = np.empty(E, np.int32)
    if _load().orc_histogram(_ptr(idx), T, k, E, _ptr(counts)) != 0:
        raise ValueError("oracle histogram: expert index out of range")
    return counts


def bias_update(counts: np.ndarray, bias: np.ndarray, T: int, k: int, step: float = 1e-3, target=None):
    """Returns (new_bias, load) -- the sign-step update, fp32 throughout."""
    counts = _c(counts, np.int32)
    E = counts.shape[0]
    b = np.array(bias, np.float32, copy=True)
    load = np.empty(E, np.float32)
    tgt = None if target is None else _c(target, np.float32)
    _load().orc_bias_update(_ptr(counts), T, E, k, ctypes.c_float(step), _ptr(tgt), _ptr(b), _ptr(load))
    return b, load


def permute(idx: np.ndarray, E: int):
    """Returns (offsets [E+1], perm_tok [T*k], inv_row [T*k]), all int32."""
    idx = _c(idx, np.int32)
    T, k = idx.shape
    offsets = np.empty(E + 1, np.int32)
    perm = np.empty(T * k, np.int32)
    inv = np.empty(T * k, np.int32)
    if _load().orc_permute(_ptr(idx), T, k, E, _ptr(offsets), _ptr(perm), _ptr(inv)) != 0:
        raise ValueError("oracle permute: expert index out of range")
    return offsets, perm, inv


def expert_accumulate(x_rows, dest, wts, w1, w3, w2, yacc):
    """yacc[dest[r]] += wts[r] * W2 (round(silu(W1 x) * W3 x)) for each row r."""
    x_rows = _c(x_rows)
    dt = _dtype_code(x_rows)
    n, d = x_rows.shape
    I = w1.shape[0]
    dest = _c(dest, np.int32)
    wts = _c(wts, np.float64)
    w1, w3, w2 = _c(w1), _c(w3), _c(w2)
    assert yacc.dtype == np.float64 and yacc.flags.c_contiguous
    _load().orc_expert_accumulate(_ptr(x_rows), n, _ptr(dest), _ptr(wts), _ptr(w1), _ptr(w3), _ptr(w2),
                                  d, I, dt, _ptr(yacc))


def expert_up(x_rows, w1, w3) -> np.ndarray:
    """h [n][I] = round(silu(x W1^T) * (x W3^T)), the dot products in double,
    rounded once to x's dtype (float32, or bf16 bits as uint16)."""
    x_rows, w1, w3 = _c(x_rows), _c(w1), _c(w3)
    dt = _dtype_code(x_rows)
    assert _dtype_code(w1) == dt and _dtype_code(w3) == dt
    n, d = x_rows.shape
    I = w1.shape[0]
    h = np.empty((n, I), x_rows.dtype)
    _load().orc_expert_up(_ptr(x_rows), n, _ptr(w1), _ptr(w3), d, I, dt, _ptr(h))
    return h


def expert_down(h_rows, w2) -> np.ndarray:
    """o [n][d] = h W2^T in double (not rounded); h [n][K], W2 [d][K]."""
    h_rows, w2 = _c(h_rows), _c(w2)
    dt = _dtype_code(h_rows)
    assert _dtype_code(w2) == dt
    n, K = h_rows.shape
    d = w2.shape[0]
    o = np.empty((n, d), np.float64)
    _load().orc_expert_down(_ptr(h_rows), n, _ptr(w2), d, K, dt, _ptr(o))
    return o


def finalize(yacc: np.ndarray, like_dtype) -> np.ndarray:
    out = np.empty(yacc.shape, like_dtype)
    _load().orc_finalize(_ptr(np.ascontiguousarray(yacc)), yacc.size, _dtype_code(out), _ptr(out))
    return out


def layer_output(x, idx, w, w1, w3, w2, ws1, ws3, ws2) -> np.ndarray:
    """Whole layer output y [T][d] (same dtype as x) for given routing."""
    x = _c(x)
    dt = _dtype_code(x)
    T, d = x.shape
    E, I, _ = w1.shape
    S, Is, _ = ws1.shape
    k = idx.shape[1]
    idx = _c(idx, np.int32)
    w = _c(w, np.float32)
    arrs = [_c(a) for a in (w1, w3, w2, ws1, ws3, ws2)]
    for a in arrs:
        assert _dtype_code(a) == dt
    y = np.empty((T, d), x.dtype)
    _load().orc_layer_output(_ptr(x), _ptr(idx), _ptr(w), *[_ptr(a) for a in arrs], T, d, E, k, I, S, Is, dt,
                             _ptr(y))
    return y


def route(x, w_gate, bias, k):
    """The pages' route(): returns (weights, idx, s) computed entirely here."""
    s = affinity(x, w_gate)
    idx, w = select(s, bias, k)
    return w, idx, s


# ------------------------------------------------- FP8 experts, per-tile scales
#
# E4M3 codes ("DeepSeek V3 Architecture Deep Dive ...", "FP8 Formats") with
# tiles of 32 consecutive elements of a row along the contraction dimension,
# each with a power-of-two scale 2^e (e the smallest integer with
# amax <= 448 * 2^e), stored as the byte e + 127; codes E4M3(v * 2^-e).
# Pages: "DeepSeek V3 From Scratch", "The idea" (fine-grained quantization
# tiles); crackai.dev "DeepSeek-V3", "How It Works" (per-tile scaling).

MX_TILE = 32


def fp8_encode(x) -> np.ndarray:
    """E4M3 codes (uint8) of fp32 values: nearest, ties to even, +-448 saturation."""
    x = np.ascontiguousarray(x, np.float32)
    q = np.empty(x.shape, np.uint8)
    _load().orc_e4m3_encode_array(_ptr(x), x.size, _ptr(q))
    return q


def fp8_decode(q) -> np.ndarray:
    """Values (float64) of E4M3 codes."""
    q = np.ascontiguousarray(q, np.uint8)
    x = np.empty(q.shape, np.float64)
    _load().orc_e4m3_decode_array(_ptr(q), q.size, _ptr(x))
    return x


def mx_exponent(amax: float) -> int:
    """Smallest e in [-127, 127] with amax <= 448 * 2^e (0 for amax = 0)."""
    return int(_load().orc_mx_exponent(float(amax)))


def quantize_mx(a: np.ndarray, nseg: int = 1):
    """Per-tile E4M3 quantization.  ``a`` is [rows][K] (bf16 bits as uint16,
    or float32) or [nseg][rows][kseg] (rows span all blocks, K = nseg*kseg).
    Returns (codes with a's shape, exponent bytes uint8 [rows][K/32])."""
    a = _c(a)
    dt = _dtype_code(a)
    if a.ndim == 3:
        if a.shape[0] != nseg:
            raise ValueError("nseg must equal the number of column blocks")
        rows, kseg = a.shape[1], a.shape[2]
    else:
        if nseg != 1:
            raise ValueError("a blocked matrix is passed as [nseg][rows][kseg]")
        rows, kseg = a.shape
    if kseg % MX_TILE:
        raise ValueError("the row length of each block must be a multiple of 32")
    q = np.empty(a.shape, np.uint8)
    eb = np.empty((rows, nseg * kseg // MX_TILE), np.uint8)
    _load().orc_quantize_mx(_ptr(a), dt, rows, kseg, nseg, _ptr(q), _ptr(eb))
    return q, eb


def mx_dequantize(q: np.ndarray, eb: np.ndarray) -> np.ndarray:
    """Values (float64) of row-major codes [rows][K] with exponent bytes [rows][K/32]."""
    v = fp8_decode(q)
    scale = np.ldexp(1.0, eb.astype(np.int64) - 127)
    return v * np.repeat(scale, MX_TILE, axis=1)


def expert_up_mx(xq, xe, w1q, w1e, w3q, w3e) -> np.ndarray:
    """h = bf16(silu(a) * g), a and g tile-scaled E4M3 dot products; bf16 bits [n][I]."""
    xq, w1q, w3q = _c(xq, np.uint8), _c(w1q, np.uint8), _c(w3q, np.uint8)
    xe, w1e, w3e = _c(xe, np.uint8), _c(w1e, np.uint8), _c(w3e, np.uint8)
    n, d = xq.shape
    I = w1q.shape[0]
    h = np.empty((n, I), np.uint16)
    _load().orc_expert_up_mx(_ptr(xq), _ptr(xe), n, _ptr(w1q), _ptr(w1e), _ptr(w3q), _ptr(w3e), d, I, _ptr(h))
    return h


def expert_down_mx(hq, he, w2q, w2e) -> np.ndarray:
    """o [n][d] (float64), tile-scaled E4M3 products of h rows and W2 rows.
    w2q is [d][K] or [nseg][d][kseg] (blocks joined along K) with w2e [d][K/32]."""
    hq, w2q = _c(hq, np.uint8), _c(w2q, np.uint8)
    he, w2e = _c(he, np.uint8), _c(w2e, np.uint8)
    n = hq.shape[0]
    if w2q.ndim == 3:
        nseg, d, kseg = w2q.shape
    else:
        nseg, (d, kseg) = 1, w2q.shape
    o = np.empty((n, d), np.float64)
    _load().orc_expert_down_mx(_ptr(hq), _ptr(he), n, _ptr(w2q), _ptr(w2e), d, kseg, nseg, _ptr(o))
    return o


def quantize_weights_mx(p: dict) -> dict:
    """Per-tile quantization of a layer's expert weights (numpy, bf16 bits):
    W1/W3 [E][I][d] and W2 [E][d][I] per row, shared Ws1/Ws3 [S][Is][d] per
    row, Ws2 [S][d][Is] per row d across the S blocks.  Codes under w1q, ...
    exponent bytes under w1e, ... ([rows][K/32], rows = E*I, E*d, ...)."""
    out = {}
    for key in ("w1", "w3", "w2", "ws1", "ws3"):
        a = p[key]
        q, eb = quantize_mx(a.reshape(-1, a.shape[-1]))
        out[key + "q"], out[key + "e"] = q.reshape(a.shape), eb
    ws2 = p["ws2"]
    q, eb = quantize_mx(ws2, nseg=ws2.shape[0])
    out["ws2q"], out["ws2e"] = q, eb
    return out


def layer_output_mx(x, idx, w, q: dict) -> np.ndarray:
    """Whole layer with tile-scaled FP8 experts for given routing: x (bf16
    bits) [T][d] quantized by tiles; each routed expert e: h = up(x rows), h
    quantized by tiles, o = down(h), y += w * o; shared: h over the S*Is
    concatenated features, quantized by tiles, o = down over the concatenated
    K.  y in bf16 bits."""
    T, d = x.shape
    E, I, _ = q["w1q"].shape
    S, Is, _ = q["ws1q"].shape
    xq, xe = quantize_mx(x)
    yacc = np.zeros((T, d), np.float64)
    if S > 0:
        hs = expert_up_mx(xq, xe, q["ws1q"].reshape(S * Is, d), q["ws1e"], q["ws3q"].reshape(S * Is, d), q["ws3e"])
        hq, he = quantize_mx(hs)
        yacc += expert_down_mx(hq, he, q["ws2q"], q["ws2e"])
    for e in range(E):
        t, j = np.nonzero(idx == e)
        if len(t) == 0:
            continue
        h = expert_up_mx(xq[t], xe[t], q["w1q"][e], q["w1e"][e * I:(e + 1) * I], q["w3q"][e],
                         q["w3e"][e * I:(e + 1) * I])
        hq, he = quantize_mx(h)
        o = expert_down_mx(hq, he, q["w2q"][e], q["w2e"][e * d:(e + 1) * d])
        yacc[t] += w[t, j].astype(np.float64)[:, None] * o
    return finalize(yacc, x.dtype)
