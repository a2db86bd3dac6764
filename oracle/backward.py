"""CPU oracle for the backward of the MoE layer forward -- TEST INFRASTRUCTURE.

Only the tests, the package smoke check and the bench's CPU-baseline leg may
import this module.  The CUDA library never calls it and shares no code with it.

Plain numpy in float64; a matrix product is the only library step.  bf16
tensors arrive as uint16 arrays of raw bf16 bits.

What is differentiated, by page title and section:
  * "DeepSeek V3 From Scratch", "In code" (route): s = sigmoid(x W_g^T), the
    top-k chosen on s + b, weights w_j = s_{idx_j} / sum_j' s_{idx_j'} from the
    unbiased scores.  The bias and the selection carry no gradient (the
    selection is piecewise constant; the bias enters only the choice).
  * "Scaling Efficiency: A Deep Dive into the DeepSeek-V3 Architecture", the
    DeepSeekMoE sketch: y_t = sum_s shared_s(x_t) + sum_j w_j expert_{idx_j}(x_t),
    each expert SwiGLU: W2 (silu(W1 x) * (W3 x)).
  * kbwen.com DeepSeek tag page, "A bias term for each expert": a
    complementary sequence-wise balance loss of weight 0.0001 is kept.  The
    pages give no formula; the one used here is the DeepSeek-V3 technical
    report's (restated, not printed on the pages -- parity unpinned by the
    pages; pinned by finite differences and a closed form only):
        per sequence of L tokens:  f_i = E / (k L) * #{t : i in top-k(t)}
                                   P_i = 1/L * sum_t s_it / sum_j s_jt
                                   L_seq = alpha * sum_i f_i P_i
        balance loss = the mean of L_seq over the batch's T / L sequences.
    f_i is a count (no gradient); the gradient reaches s through P_i.

Rounding points of the forward that the backward treats as identity: the
bf16 rounding of h (the recomputed h is rounded the same way before it is
used), the output dtype rounding of y.
"""
from __future__ import annotations

import numpy as np


def to_f64(a: np.ndarray) -> np.ndarray:
    """float32 values, or uint16 raw bf16 bits, as float64."""
    a = np.asarray(a)
    if a.dtype == np.uint16:
        return (a.astype(np.uint32) << 16).view(np.float32).astype(np.float64)
    if a.dtype in (np.float32, np.float64):
        return a.astype(np.float64)
    raise TypeError(f"expected float32 or bf16-as-uint16, got {a.dtype}")


def _round_f32(v: np.ndarray) -> np.ndarray:
    return v.astype(np.float32).astype(np.float64)


def _round_bf16(v: np.ndarray) -> np.ndarray:
    """float64 -> float32 -> bf16 (round to nearest, ties to even) -> float64."""
    u = v.astype(np.float32).view(np.uint32).astype(np.uint64)
    u = (u + 0x7FFF + ((u >> 16) & 1)) >> 16
    return (u.astype(np.uint32) << 16).view(np.float32).astype(np.float64)


def round_like(v: np.ndarray, bf16: bool) -> np.ndarray:
    return _round_bf16(v) if bf16 else _round_f32(v)


def _sigmoid(z):
    return 1.0 / (1.0 + np.exp(-z))


def balance_loss(s: np.ndarray, idx: np.ndarray, alpha: float, seq_len: int):
    """Sequence-wise balance loss and its gradient with respect to s.

    s [T][E] affinities, idx [T][k] the chosen experts.  Returns (loss, ds)."""
    s = np.asarray(s, np.float64)
    T, E = s.shape
    k = idx.shape[1]
    L = seq_len
    assert L > 0 and T % L == 0
    nb = T // L
    ds = np.zeros_like(s)
    loss = 0.0
    for b in range(nb):
        rows = slice(b * L, (b + 1) * L)
        sb = s[rows]
        cnt = np.zeros(E)
        np.add.at(cnt, idx[rows].ravel(), 1.0)
        f = cnt * E / (k * L)
        tot = sb.sum(axis=1, keepdims=True)          # sum over all experts, per token
        sn = sb / tot
        P = sn.mean(axis=0)
        loss += alpha * float(f @ P)
        # d(f . P)/d s_ti = 1/L * (f_i - sum_j f_j sn_tj) / tot_t
        ds[rows] = alpha / L * (f[None, :] - (sn @ f)[:, None]) / tot
    return loss / nb, ds / nb


def layer_forward_f64(x, w_gate, idx, w1, w3, w2, ws1, ws3, ws2, round_h=None):
    """Differentiable restatement of the forward for a FIXED selection idx:
    w comes from s(x) renormalised over idx.  round_h: None (no rounding) or
    'bf16' / 'f32' (the forward's rounding of h).  Returns (y, s, w)."""
    X, Wg = to_f64(x), to_f64(w_gate)
    W1, W3, W2 = to_f64(w1), to_f64(w3), to_f64(w2)
    T, d = X.shape
    k = idx.shape[1]
    s = _sigmoid(X @ Wg.T)
    sel = np.take_along_axis(s, idx, axis=1)
    w = sel / sel.sum(axis=1, keepdims=True)
    rnd = (lambda v: v) if round_h is None else (lambda v: round_like(v, round_h == "bf16"))
    y = np.zeros((T, d))
    if ws1 is not None and np.asarray(ws1).size:
        Ws1, Ws3, Ws2 = to_f64(ws1), to_f64(ws3), to_f64(ws2)
        for j in range(Ws1.shape[0]):
            a, g = X @ Ws1[j].T, X @ Ws3[j].T
            y += rnd(a * _sigmoid(a) * g) @ Ws2[j].T
    for t in range(T):
        for j in range(k):
            e = idx[t, j]
            a, g = W1[e] @ X[t], W3[e] @ X[t]
            y[t] += w[t, j] * (W2[e] @ rnd(a * _sigmoid(a) * g))
    return y, s, w


def layer_backward(x, w_gate, idx, w, s, w1, w3, w2, ws1, ws3, ws2, dy, alpha=0.0, seq_len=0, round_h=None):
    """Gradients of <dy, y> (+ the balance loss when alpha > 0) for the layer
    forward with the given selection idx, weights w [T][k] and affinities
    s [T][E] (both as the forward produced them).

    Returns a dict: dx [T][d], dw_gate [E][d], dw1, dw3 [E][I][d], dw2
    [E][d][I], dws1, dws3 [S][Is][d], dws2 [S][d][Is], balance_loss, and the
    intermediates dw [T][k] (gradient of the combine weights) and ds [T][E]."""
    X, Wg = to_f64(x), to_f64(w_gate)
    W1, W3, W2 = to_f64(w1), to_f64(w3), to_f64(w2)
    dY = np.asarray(dy, np.float64)
    s = np.asarray(s, np.float64)
    w = np.asarray(w, np.float64)
    idx = np.asarray(idx)
    T, d = X.shape
    E, I, _ = W1.shape
    k = idx.shape[1]
    rnd = (lambda v: v) if round_h is None else (lambda v: round_like(v, round_h == "bf16"))

    dX = np.zeros((T, d))
    dW1, dW3, dW2 = np.zeros_like(W1), np.zeros_like(W3), np.zeros_like(W2)
    dw = np.zeros((T, k))
    # routed experts, one expert's rows at a time
    for e in range(E):
        tt, jj = np.nonzero(idx == e)
        if tt.size == 0:
            continue
        Xe = X[tt]                                   # [n][d]
        a, g = Xe @ W1[e].T, Xe @ W3[e].T            # [n][I]
        sa = _sigmoid(a)
        h = rnd(a * sa * g)
        o = h @ W2[e].T                              # [n][d]
        dw[tt, jj] = np.einsum("nd,nd->n", dY[tt], o)
        do = w[tt, jj][:, None] * dY[tt]             # [n][d]
        dW2[e] = do.T @ h
        dh = do @ W2[e]                              # [n][I]
        da = dh * g * sa * (1.0 + a * (1.0 - sa))
        dg = dh * a * sa
        dW1[e] = da.T @ Xe
        dW3[e] = dg.T @ Xe
        np.add.at(dX, tt, da @ W1[e] + dg @ W3[e])
    # shared experts (weight 1)
    out = {}
    if ws1 is not None and np.asarray(ws1).size:
        Ws1, Ws3, Ws2 = to_f64(ws1), to_f64(ws3), to_f64(ws2)
        dWs1, dWs3, dWs2 = np.zeros_like(Ws1), np.zeros_like(Ws3), np.zeros_like(Ws2)
        for j in range(Ws1.shape[0]):
            a, g = X @ Ws1[j].T, X @ Ws3[j].T
            sa = _sigmoid(a)
            h = rnd(a * sa * g)
            dWs2[j] = dY.T @ h
            dh = dY @ Ws2[j]
            da = dh * g * sa * (1.0 + a * (1.0 - sa))
            dg = dh * a * sa
            dWs1[j] = da.T @ X
            dWs3[j] = dg.T @ X
            dX += da @ Ws1[j] + dg @ Ws3[j]
        out.update(dws1=dWs1, dws3=dWs3, dws2=dWs2)
    # router: w_j = s_{idx_j} / S_t, S_t the sum over the chosen experts
    ds = np.zeros((T, E))
    sel = np.take_along_axis(s, idx, axis=1)
    S_t = sel.sum(axis=1, keepdims=True)
    wn = sel / S_t
    dsel = (dw - (dw * wn).sum(axis=1, keepdims=True)) / S_t
    np.put_along_axis(ds, idx, dsel, axis=1)
    loss = 0.0
    if alpha > 0.0:
        loss, dsb = balance_loss(s, idx, alpha, seq_len)
        ds += dsb
    dz = ds * s * (1.0 - s)
    dX += dz @ Wg
    dWg = dz.T @ X
    out.update(dx=dX, dw_gate=dWg, dw1=dW1, dw3=dW3, dw2=dW2, balance_loss=loss, dw=dw, ds=ds)
    return out
