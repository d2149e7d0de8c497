"""fp64 CPU oracle of the routed MoE layer -- TEST INFRASTRUCTURE ONLY.

Only the tests, the smoke check and the bench's CPU-baseline leg may import this
module.  The CUDA library never calls it and shares no code with it.

What it computes is the plain definition of a routed mixture-of-experts layer as the
Olmo-core 3 write-ups describe it: every token is sent to a few of many expert
sub-networks (deniz.in, "Hedeflediği kapasite sorunu"); routing metadata (expert
indices, per-expert counts and offsets) is produced on the device
(deniz.in, "Yeni stack nasıl çalışıyor"); each selected token row is written into
its expert's contiguous input buffer (unite.ai, "पैरालेलिज़्म, प्रिसीजन, और मेमोरी
तकनीकें"; donmalab.com, "擴展與最佳化手段"); the grouped GEMM runs the ragged
per-expert shapes (deniz.in, "Yeni stack nasıl çalışıyor").  A grouped GEMM is not
an approximation: it equals one dense matmul per expert over that expert's rows,
which is how it is written here.

The pages give no formulas.  The readings used where they are silent:
  * router: softmax over all experts, keep the top k, renormalise over the kept set;
    this equals a softmax over the k kept logits, which is what is computed.
  * selection is on the fp32 logits, ordered by (logit descending, expert index
    ascending); topk_idx lists the kept experts in that order.
  * permutation: a stable counting sort of the (token, j) pairs keyed by expert, so an
    expert's rows are in token order.
  * expert FFN: SwiGLU, a = silu(x W1^T) * (x W3^T), y = a W2^T, with W13 = [W1; W3].
  * the gate is applied at the combine: y_t = sum_j g_tj * y_perm[slot[t, j]].
  * backward: the chain rule through the above, written out by hand.

All floating point work is fp64; inputs (bf16 or fp32) are upcast exactly.
Parity for every function here is pinned by tests that do not retype these formulas:
a brute-force per-token loop, invariants, the identical-experts identity (a dense
SwiGLU FFN), k = E (full softmax) and k = 1 (unit gates), central finite differences
and fp64 torch.autograd.
"""
from __future__ import annotations

import numpy as np

from .mx import bf16_round, mx_quantize_dequantize


def _f64(a) -> np.ndarray:
    return np.asarray(a, dtype=np.float64)


def _sigmoid(z: np.ndarray) -> np.ndarray:
    with np.errstate(over="ignore"):
        return 1.0 / (1.0 + np.exp(-z))


def silu(z: np.ndarray) -> np.ndarray:
    """silu(z) = z * sigmoid(z)."""
    return z * _sigmoid(z)


# --------------------------------------------------------------------------- routing

def router_logits(x, Wr) -> np.ndarray:
    """Router projection L = x . Wr  ([T,d] x [d,E] -> [T,E])."""
    return _f64(x) @ _f64(Wr)


def topk_gates(logits, k: int):
    """Top-k selection and renormalised softmax gates per token.

    Experts are ordered by (logit descending, index ascending) and the first k kept.
    Gates g = exp(L_sel - max) / sum exp(L_sel - max) over the kept logits.
    Returns (topk_idx int32 [T,k], gates fp64 [T,k]).
    """
    L = _f64(logits)
    T, E = L.shape
    if not 1 <= k <= E:
        raise ValueError("need 1 <= k <= E")
    # stable sort of -L keeps equal logits in index order (lower index first)
    order = np.argsort(-L, axis=1, kind="stable")[:, :k]
    sel = np.take_along_axis(L, order, axis=1)
    z = np.exp(sel - sel[:, :1])
    gates = z / z.sum(axis=1, keepdims=True)
    return order.astype(np.int32), gates


def counts_offsets(topk_idx, E: int):
    """Per-expert row counts and their exclusive prefix sum (offsets[E] = T*k)."""
    idx = np.asarray(topk_idx)
    counts = np.bincount(idx.ravel(), minlength=E).astype(np.int64)
    offsets = np.zeros(E + 1, dtype=np.int64)
    offsets[1:] = np.cumsum(counts)
    return counts, offsets


def permutation(topk_idx, gates, E: int):
    """Expert-sorted order of the (token, j) pairs.

    slot[t, j] is the row of pair (t, j) in the expert-contiguous buffers:
    slot[t, j] = offsets[e] + #{t' < t : e in sel(t')} with e = topk_idx[t, j].
    row_token[s] and row_gate[s] are the token and gate of row s.
    """
    idx = np.asarray(topk_idx)
    T, k = idx.shape
    R = T * k
    flat = idx.ravel()
    order = np.argsort(flat, kind="stable")       # pairs by expert, then by t*k + j
    slot = np.empty(R, dtype=np.int64)
    slot[order] = np.arange(R, dtype=np.int64)
    row_token = (order // k).astype(np.int64)
    row_gate = _f64(gates).ravel()[order]
    return slot.reshape(T, k), row_token, row_gate


def route(logits, k: int, E: int) -> dict:
    """All routing metadata of one batch (steps in the order the layer runs them)."""
    idx, gates = topk_gates(logits, k)
    counts, offsets = counts_offsets(idx, E)
    slot, row_token, row_gate = permutation(idx, gates, E)
    return dict(topk_idx=idx, gates=gates, counts=counts, offsets=offsets, slot=slot,
                row_token=row_token, row_gate=row_gate)


# --------------------------------------------------------------------------- dispatch / combine

def dispatch(x, slot) -> np.ndarray:
    """x_perm[slot[t, j]] = x[t]."""
    X = _f64(x)
    slot = np.asarray(slot)
    T, k = slot.shape
    out = np.empty((T * k, X.shape[1]), dtype=np.float64)
    out[slot.ravel()] = np.repeat(X, k, axis=0)
    return out


def combine(y_perm, gates, slot) -> np.ndarray:
    """y[t] = sum_j gates[t, j] * y_perm[slot[t, j]]."""
    Y = _f64(y_perm)
    g = _f64(gates)
    slot = np.asarray(slot)
    T, k = slot.shape
    y = np.zeros((T, Y.shape[1]), dtype=np.float64)
    for j in range(k):
        y += g[:, j:j + 1] * Y[slot[:, j]]
    return y


def combine_bwd(dy, y_perm, gates, topk_idx, slot, E: int):
    """Backward of the combine and of the selected-logit softmax.

    dy_perm[slot[t, j]] = g_tj * dy[t]
    dg_tj = <dy[t], y_perm[slot[t, j]]>
    dL_tj = g_tj * (dg_tj - sum_i g_ti dg_ti) on the selected experts, 0 elsewhere.
    Returns (dy_perm [R,d], d_logits [T,E]).
    """
    dY = _f64(dy)
    Y = _f64(y_perm)
    g = _f64(gates)
    idx = np.asarray(topk_idx)
    slot = np.asarray(slot)
    T, k = slot.shape
    dy_perm = np.empty((T * k, dY.shape[1]), dtype=np.float64)
    dg = np.empty((T, k), dtype=np.float64)
    for j in range(k):
        dy_perm[slot[:, j]] = g[:, j:j + 1] * dY
        dg[:, j] = np.einsum("td,td->t", dY, Y[slot[:, j]])
    dsel = g * (dg - (g * dg).sum(axis=1, keepdims=True))
    d_logits = np.zeros((T, E), dtype=np.float64)
    np.put_along_axis(d_logits, idx.astype(np.int64), dsel, axis=1)
    return dy_perm, d_logits


def dispatch_bwd(dx_perm, slot) -> np.ndarray:
    """dx[t] = sum_j dx_perm[slot[t, j]]."""
    D = _f64(dx_perm)
    slot = np.asarray(slot)
    T, k = slot.shape
    dx = np.zeros((T, D.shape[1]), dtype=np.float64)
    for j in range(k):
        dx += D[slot[:, j]]
    return dx


# --------------------------------------------------------------------------- expert FFN

def _mx(a, axis, mx: bool):
    """An MXFP8 GEMM operand: the operand as the BF16 tensor the GEMM reads (BF16 I/O),
    quantised with blocks of 32 along ``axis``.  Without ``mx``, ``a`` unchanged."""
    return mx_quantize_dequantize(bf16_round(a), axis=axis) if mx else a


def experts_fwd(x_perm, offsets, W13, W2, mx: bool = False):
    """Per-expert SwiGLU FFN over each expert's contiguous rows.

    H_e = X_e W13_e^T, a_e = silu(H_e[:, :f]) * H_e[:, f:], Y_e = a_e W2_e^T.
    With ``mx`` the GEMM operands are MX-quantised (E4M3 + E8M0 per 32 along the
    GEMM's K) at the points the MXFP8 path quantises them, each taken as the BF16
    tensor the GEMM reads; the rest stays fp64.
    Returns (H13 [R,2f], a [R,f], y_perm [R,d]).
    """
    X = _f64(x_perm)
    off = np.asarray(offsets, dtype=np.int64)
    E = len(off) - 1
    f2 = W13.shape[1]
    f = f2 // 2
    d = W2.shape[1]
    R = X.shape[0]
    H13 = np.zeros((R, f2))
    A = np.zeros((R, f))
    Y = np.zeros((R, d))
    for e in range(E):
        r0, r1 = int(off[e]), int(off[e + 1])
        if r1 == r0:
            continue
        Xe = X[r0:r1]
        W13e = _f64(W13[e])
        W2e = _f64(W2[e])
        H = _mx(Xe, 1, mx) @ _mx(W13e, 1, mx).T
        a = silu(H[:, :f]) * H[:, f:]
        H13[r0:r1] = H
        A[r0:r1] = a
        Y[r0:r1] = _mx(a, 1, mx) @ _mx(W2e, 1, mx).T
    return H13, A, Y


def swiglu_bwd(dA, H13):
    """dH1 = dA * H3 * s * (1 + H1 * (1 - s)), dH3 = dA * silu(H1), s = sigmoid(H1)."""
    H = _f64(H13)
    f = H.shape[1] // 2
    H1, H3 = H[:, :f], H[:, f:]
    s = _sigmoid(H1)
    dH1 = dA * H3 * s * (1.0 + H1 * (1.0 - s))
    dH3 = dA * H1 * s
    return np.concatenate([dH1, dH3], axis=1)


def experts_bwd(dy_perm, x_perm, H13, a, offsets, W13, W2, mx: bool = False):
    """Backward of ``experts_fwd``.

    dA_e = dY_e W2_e ; dH13_e = swiglu_bwd(dA_e, H13_e)
    dW2_e = dY_e^T a_e ; dW13_e = dH13_e^T X_e ; dX_e = dH13_e W13_e
    An expert with no rows gets dW = 0 exactly.
    Returns (dH13 [R,2f], dx_perm [R,d], dW13 [E,2f,d], dW2 [E,d,f]).
    """
    dY = _f64(dy_perm)
    X = _f64(x_perm)
    H = _f64(H13)
    A = _f64(a)
    off = np.asarray(offsets, dtype=np.int64)
    E = len(off) - 1
    f2, d = W13.shape[1], W13.shape[2]
    f = f2 // 2
    R = X.shape[0]
    dH13 = np.zeros((R, f2))
    dX = np.zeros((R, d))
    dW13 = np.zeros((E, f2, d))
    dW2 = np.zeros((E, d, f))
    for e in range(E):
        r0, r1 = int(off[e]), int(off[e + 1])
        if r1 == r0:
            continue
        W13e = _f64(W13[e])
        W2e = _f64(W2[e])
        dYe = dY[r0:r1]
        # dgrad of FC2: contraction over d
        dAe = _mx(dYe, 1, mx) @ _mx(W2e, 0, mx)
        dHe = swiglu_bwd(dAe, H[r0:r1])
        dH13[r0:r1] = dHe
        # wgrad: contraction over this expert's tokens
        dW2[e] = _mx(dYe, 0, mx).T @ _mx(A[r0:r1], 0, mx)
        dW13[e] = _mx(dHe, 0, mx).T @ _mx(X[r0:r1], 0, mx)
        # dgrad of FC1: contraction over 2f
        dX[r0:r1] = _mx(dHe, 1, mx) @ _mx(W13e, 0, mx)
    return dH13, dX, dW13, dW2


# --------------------------------------------------------------------------- whole layer

def layer_fwd(x, W13, W2, logits=None, Wr=None, k: int = 2, mx: bool = False,
              shared: bool = False) -> dict:
    """Forward of the routed MoE layer; returns every intermediate by name.

    ``shared``: W13 / W2 hold one more expert than the router chooses from; that last
    one is the shared expert (the write-ups' production rows use one: bigchange.ai
    pt-BR, last section), a SwiGLU FFN applied to every token with weight 1 and added
    to y: y_t = sum_j g_tj FFN_{e_tj}(x_t) + FFN_shared(x_t).
    """
    E = W13.shape[0] - (1 if shared else 0)
    if logits is None:
        if Wr is None:
            raise ValueError("need logits or Wr")
        L = router_logits(x, Wr)
    else:
        L = _f64(logits)
    r = route(L, k, E)
    x_perm = dispatch(x, r["slot"])
    H13, A, Yp = experts_fwd(x_perm, r["offsets"], W13[:E], W2[:E], mx=mx)
    y = combine(Yp, r["gates"], r["slot"])
    r.update(logits=L, x_perm=x_perm, H13=H13, a=A, y_perm=Yp)
    if shared:
        # one expert over all T tokens in token order: a dense SwiGLU FFN
        T = _f64(x).shape[0]
        Hs, As, Ys = experts_fwd(_f64(x), [0, T], W13[E:], W2[E:], mx=mx)
        y = y + Ys
        r.update(H13_shared=Hs, a_shared=As, y_shared=Ys)
    r["y"] = y
    return r


def layer_bwd(fwd: dict, dy, x, W13, W2, Wr=None, mx: bool = False) -> dict:
    """Backward of ``layer_fwd`` for upstream gradient ``dy``.

    Returns dx, d_logits, dW13, dW2 and, when the router ran (``Wr`` given), dWr.
    With the router, dx includes d_logits . Wr^T and dWr = x^T . d_logits.  With a
    shared expert (the forward ran with ``shared``), dW13 / dW2 have its gradient as
    their last expert and dx includes its input gradient.
    """
    shared = "y_shared" in fwd
    E = W13.shape[0] - (1 if shared else 0)
    dy_perm, d_logits = combine_bwd(dy, fwd["y_perm"], fwd["gates"], fwd["topk_idx"],
                                    fwd["slot"], E)
    dH13, dx_perm, dW13, dW2 = experts_bwd(dy_perm, fwd["x_perm"], fwd["H13"], fwd["a"],
                                           fwd["offsets"], W13[:E], W2[:E], mx=mx)
    dx = dispatch_bwd(dx_perm, fwd["slot"])
    if shared:
        T = _f64(dy).shape[0]
        _, dXs, dW13s, dW2s = experts_bwd(_f64(dy), _f64(x), fwd["H13_shared"], fwd["a_shared"],
                                          [0, T], W13[E:], W2[E:], mx=mx)
        dx = dx + dXs
        dW13 = np.concatenate([dW13, dW13s])
        dW2 = np.concatenate([dW2, dW2s])
    out = dict(dy_perm=dy_perm, dH13=dH13, dx_perm=dx_perm, dW13=dW13, dW2=dW2,
               d_logits=d_logits)
    if Wr is not None:
        dx = dx + d_logits @ _f64(Wr).T
        out["dWr"] = _f64(x).T @ d_logits
    out["dx"] = dx
    return out


def load_stats(counts) -> dict:
    """Expert load statistics of one routing: the measurable side of the imbalance the
    write-ups call "Token Gerrymandering" (deniz.in, "Ekibin reddettiği yaklaşımlar"; they
    give no formula, so these are the plain definitions).  counts [E] >= 0."""
    c = np.asarray(counts, dtype=np.int64)
    E = len(c)
    total = int(c.sum())
    mean = total / E
    out = dict(total=total, max_count=int(c.max()), min_count=int(c.min()),
               num_empty=int((c == 0).sum()), num_experts=E, mean=mean,
               max_over_mean=0.0, cv=0.0)
    if total > 0:
        out["max_over_mean"] = float(c.max()) / mean
        out["cv"] = float(np.sqrt(np.mean((c.astype(np.float64) - mean) ** 2))) / mean
    return out


def rel_fro(a, b) -> float:
    """Relative Frobenius error ||a - b|| / ||b||  (0 when both are zero)."""
    a = _f64(a)
    b = _f64(b)
    nb = np.linalg.norm(b)
    na = np.linalg.norm(a - b)
    if nb == 0.0:
        return 0.0 if na == 0.0 else float("inf")
    return float(na / nb)
