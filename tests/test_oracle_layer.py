"""Pins of the oracle's layer forward and backward.

Each pin reaches the oracle's numbers another way: a per-token brute-force loop,
a reduction to a dense SwiGLU FFN, fp64 torch.autograd, and central finite
differences.
"""
import math

import numpy as np
import pytest
import torch
import torch.nn.functional as F

import oracle
from routing_grouped_gemm_route_b200.inputs import Workload, make_inputs


def tiny(T=8, d=16, E=4, k=2, f=8, router=False, seed=0, dtype="fp32"):
    w = Workload("t", T, d, E, k, f, dtype, router=router, skew=False, seed=seed)
    inp = make_inputs(w)
    return w, {n: (None if v is None else v.double().numpy()) for n, v in inp.items()}


def brute_fwd(x, W13, W2, L, k):
    """y_t = sum over the token's experts of gate * SwiGLU_e(x_t), one token at a time."""
    T, E = L.shape
    f = W13.shape[1] // 2
    y = np.zeros((T, W2.shape[1]))
    for t in range(T):
        sel = sorted(range(E), key=lambda e: (-L[t, e], e))[:k]
        z = np.array([math.exp(L[t, e] - L[t, sel[0]]) for e in sel])
        g = z / z.sum()
        for j, e in enumerate(sel):
            h1 = W13[e, :f] @ x[t]
            h3 = W13[e, f:] @ x[t]
            a = np.array([v / (1.0 + math.exp(-v)) for v in h1]) * h3
            y[t] += g[j] * (W2[e] @ a)
    return y


@pytest.mark.parametrize("T,d,E,k,f,router", [(8, 16, 4, 2, 8, False), (13, 32, 5, 3, 16, False),
                                              (9, 16, 3, 3, 8, True), (6, 8, 6, 1, 4, True)])
def test_fwd_matches_per_token_brute_force(T, d, E, k, f, router):
    w, t = tiny(T, d, E, k, f, router=router, seed=T + d)
    L = t["x"] @ t["Wr"] if router else t["logits"]
    out = oracle.layer_fwd(t["x"], t["W13"], t["W2"], logits=None if router else t["logits"],
                           Wr=t["Wr"], k=k)
    ref = brute_fwd(t["x"], t["W13"], t["W2"], L, k)
    assert np.allclose(out["y"], ref, rtol=1e-12, atol=1e-14)


def test_identical_experts_reduce_to_dense_swiglu():
    w, t = tiny(T=24, d=16, E=6, k=3, f=8, seed=3)
    W13 = np.repeat(t["W13"][:1], 6, axis=0)
    W2 = np.repeat(t["W2"][:1], 6, axis=0)
    fwd = oracle.layer_fwd(t["x"], W13, W2, logits=t["logits"], k=3)
    x = torch.tensor(t["x"], requires_grad=True)
    w13 = torch.tensor(W13[0], requires_grad=True)
    w2 = torch.tensor(W2[0], requires_grad=True)
    h = x @ w13.T
    y = (F.silu(h[:, :8]) * h[:, 8:]) @ w2.T
    assert np.allclose(fwd["y"], y.detach().numpy(), rtol=1e-12, atol=1e-14)
    # backward: sum_e dW_e equals the dense FFN's dW, d_logits vanish, dx equals dense dx
    (y * torch.tensor(t["dy"])).sum().backward()
    bwd = oracle.layer_bwd(fwd, t["dy"], t["x"], W13, W2)
    assert np.allclose(bwd["dW13"].sum(0), w13.grad.numpy(), rtol=1e-11, atol=1e-13)
    assert np.allclose(bwd["dW2"].sum(0), w2.grad.numpy(), rtol=1e-11, atol=1e-13)
    assert np.allclose(bwd["dx"], x.grad.numpy(), rtol=1e-11, atol=1e-13)
    assert np.abs(bwd["d_logits"]).max() < 1e-12


def torch_layer(x, W13, W2, L, idx, dy, Wr=None):
    """The same layer in fp64 torch with the selection fixed; autograd gives the grads."""
    x = torch.tensor(x, requires_grad=True)
    W13 = torch.tensor(W13, requires_grad=True)
    W2 = torch.tensor(W2, requires_grad=True)
    if Wr is not None:
        Wr = torch.tensor(Wr, requires_grad=True)
        Lt = x @ Wr
    else:
        Lt = torch.tensor(L, requires_grad=True)
    idx = torch.tensor(idx, dtype=torch.long)
    g = torch.softmax(Lt.gather(1, idx), dim=1)
    f = W13.shape[1] // 2
    h = torch.einsum("tkfd,td->tkf", W13[idx], x)
    a = F.silu(h[..., :f]) * h[..., f:]
    yk = torch.einsum("tkdf,tkf->tkd", W2[idx], a)
    y = (g[..., None] * yk).sum(1)
    (y * torch.tensor(dy)).sum().backward()
    grads = dict(dx=x.grad.numpy(), dW13=W13.grad.numpy(), dW2=W2.grad.numpy())
    if Wr is not None:
        grads["dWr"] = Wr.grad.numpy()
    else:
        grads["d_logits"] = Lt.grad.numpy()
    return y.detach().numpy(), grads


@pytest.mark.parametrize("router", [False, True])
def test_bwd_matches_torch_autograd(router):
    w, t = tiny(T=16, d=16, E=5, k=2, f=8, router=router, seed=7)
    fwd = oracle.layer_fwd(t["x"], t["W13"], t["W2"], logits=t["logits"], Wr=t["Wr"], k=2)
    bwd = oracle.layer_bwd(fwd, t["dy"], t["x"], t["W13"], t["W2"], Wr=t["Wr"])
    y, grads = torch_layer(t["x"], t["W13"], t["W2"], t["logits"], fwd["topk_idx"], t["dy"], t["Wr"])
    assert np.allclose(fwd["y"], y, rtol=1e-12, atol=1e-14)
    for name, ref in grads.items():
        assert np.allclose(bwd[name], ref, rtol=1e-10, atol=1e-13), name


def _loss(x, W13, W2, L, Wr, dy, k):
    out = oracle.layer_fwd(x, W13, W2, logits=L, Wr=Wr, k=k)
    return float((out["y"] * dy).sum()), out["topk_idx"]


def _fd_check(name, arr, grad, fn, idx0, rng, n=60, eps=1e-6):
    flat = arr.reshape(-1)
    picks = rng.choice(flat.size, size=min(n, flat.size), replace=False)
    for p in picks:
        old = flat[p]
        flat[p] = old + eps
        lp, ip = fn()
        flat[p] = old - eps
        lm, im = fn()
        flat[p] = old
        assert np.array_equal(ip, idx0) and np.array_equal(im, idx0), "selection moved"
        fd = (lp - lm) / (2 * eps)
        g = grad.reshape(-1)[p]
        assert abs(fd - g) <= 1e-6 * max(1.0, abs(g)), (name, p, fd, g)


@pytest.mark.parametrize("router", [False, True])
def test_bwd_central_finite_differences(router):
    w, t = tiny(T=8, d=16, E=4, k=2, f=8, router=router, seed=21)
    x, W13, W2, dy = t["x"].copy(), t["W13"].copy(), t["W2"].copy(), t["dy"]
    L = None if router else t["logits"].copy()
    Wr = t["Wr"].copy() if router else None
    fwd = oracle.layer_fwd(x, W13, W2, logits=L, Wr=Wr, k=2)
    # the selection must not move under the perturbation
    Ls = np.sort(fwd["logits"], axis=1)[:, ::-1]
    assert np.min(Ls[:, 1] - Ls[:, 2]) > 1e-4
    bwd = oracle.layer_bwd(fwd, dy, x, W13, W2, Wr=Wr)
    idx0 = fwd["topk_idx"]
    rng = np.random.default_rng(0)
    fn = lambda: _loss(x, W13, W2, L, Wr, dy, 2)
    _fd_check("x", x, bwd["dx"], fn, idx0, rng)
    _fd_check("W13", W13, bwd["dW13"], fn, idx0, rng)
    _fd_check("W2", W2, bwd["dW2"], fn, idx0, rng)
    if router:
        _fd_check("Wr", Wr, bwd["dWr"], fn, idx0, rng)
    else:
        _fd_check("logits", L, bwd["d_logits"], fn, idx0, rng, n=L.size)


def test_empty_expert_has_exactly_zero_weight_grad():
    w, t = tiny(T=32, d=16, E=5, k=2, f=8, seed=9)
    L = t["logits"].copy()
    L[:, 3] -= 100.0                        # expert 3 is never selected
    fwd = oracle.layer_fwd(t["x"], t["W13"], t["W2"], logits=L, k=2)
    assert fwd["counts"][3] == 0
    bwd = oracle.layer_bwd(fwd, t["dy"], t["x"], t["W13"], t["W2"])
    assert np.all(bwd["dW13"][3] == 0.0) and np.all(bwd["dW2"][3] == 0.0)
    assert np.all(bwd["d_logits"][:, 3] == 0.0)


def test_dispatch_combine_identities():
    rng = np.random.default_rng(1)
    T, k, E, d = 30, 3, 7, 12
    L = rng.standard_normal((T, E)).astype(np.float32)
    r = oracle.route(L, k, E)
    x = rng.standard_normal((T, d))
    xp = oracle.dispatch(x, r["slot"])
    assert np.array_equal(xp, x[r["row_token"]])                  # gather form of the same copy
    assert np.allclose(oracle.dispatch_bwd(xp, r["slot"]), k * x, rtol=1e-15, atol=0)
    # combining copies of x with gates that sum to 1 returns x
    assert np.allclose(oracle.combine(xp, r["gates"], r["slot"]), x, rtol=1e-14, atol=1e-15)


def test_combine_bwd_softmax_jacobian_rows_sum_to_zero():
    rng = np.random.default_rng(2)
    T, k, E, d = 40, 4, 9, 8
    L = rng.standard_normal((T, E)).astype(np.float32)
    r = oracle.route(L, k, E)
    yp = rng.standard_normal((T * k, d))
    dy = rng.standard_normal((T, d))
    dyp, dL = oracle.combine_bwd(dy, yp, r["gates"], r["topk_idx"], r["slot"], E)
    # softmax is invariant to adding a constant to all logits, so each row of dL sums to 0
    assert np.allclose(dL.sum(axis=1), 0.0, atol=1e-13)
    assert np.allclose(dyp[r["slot"][:, 0]], r["gates"][:, :1] * dy, rtol=1e-15, atol=0)


# --------------------------------------------------------------- shared expert

def tiny_shared(T=12, d=16, E=4, k=2, f=8, router=False, seed=0):
    w = Workload("ts", T, d, E, k, f, "fp32", router=router, skew=False, seed=seed, shared=True)
    inp = make_inputs(w)
    return w, {n: (None if v is None else v.double().numpy()) for n, v in inp.items()}


def test_shared_expert_identical_weights_double_the_dense_ffn():
    # all routed experts and the shared one equal: gates sum to 1, so y = 2 * FFN(x)
    w, t = tiny_shared(T=20, d=16, E=5, k=3, f=8, seed=4)
    W13 = np.repeat(t["W13"][:1], 6, axis=0)
    W2 = np.repeat(t["W2"][:1], 6, axis=0)
    fwd = oracle.layer_fwd(t["x"], W13, W2, logits=t["logits"], k=3, shared=True)
    x = torch.tensor(t["x"])
    h = x @ torch.tensor(W13[0]).T
    dense = ((F.silu(h[:, :8]) * h[:, 8:]) @ torch.tensor(W2[0]).T).numpy()
    assert np.allclose(fwd["y"], 2 * dense, rtol=1e-12, atol=1e-14)


@pytest.mark.parametrize("router", [False, True])
def test_shared_expert_bwd_matches_torch_autograd(router):
    w, t = tiny_shared(T=14, d=16, E=4, k=2, f=8, router=router, seed=9)
    E = 4
    fwd = oracle.layer_fwd(t["x"], t["W13"], t["W2"], logits=t["logits"], Wr=t["Wr"], k=2,
                           shared=True)
    bwd = oracle.layer_bwd(fwd, t["dy"], t["x"], t["W13"], t["W2"], Wr=t["Wr"])
    # torch: the routed layer on the first E experts plus a dense SwiGLU FFN on the last
    x = torch.tensor(t["x"], requires_grad=True)
    W13 = torch.tensor(t["W13"], requires_grad=True)
    W2 = torch.tensor(t["W2"], requires_grad=True)
    Wr = torch.tensor(t["Wr"], requires_grad=True) if router else None
    Lt = x @ Wr if router else torch.tensor(t["logits"], requires_grad=True)
    idx = torch.tensor(fwd["topk_idx"], dtype=torch.long)
    g = torch.softmax(Lt.gather(1, idx), dim=1)
    h = torch.einsum("tkfd,td->tkf", W13[:E][idx], x)
    yk = torch.einsum("tkdf,tkf->tkd", W2[:E][idx], F.silu(h[..., :8]) * h[..., 8:])
    hs = x @ W13[E].T
    y = (g[..., None] * yk).sum(1) + (F.silu(hs[:, :8]) * hs[:, 8:]) @ W2[E].T
    (y * torch.tensor(t["dy"])).sum().backward()
    assert np.allclose(fwd["y"], y.detach().numpy(), rtol=1e-12, atol=1e-14)
    assert np.allclose(bwd["dx"], x.grad.numpy(), rtol=1e-10, atol=1e-13)
    assert np.allclose(bwd["dW13"], W13.grad.numpy(), rtol=1e-10, atol=1e-13)
    assert np.allclose(bwd["dW2"], W2.grad.numpy(), rtol=1e-10, atol=1e-13)
    if router:
        assert np.allclose(bwd["dWr"], Wr.grad.numpy(), rtol=1e-10, atol=1e-13)
    else:
        assert np.allclose(bwd["d_logits"], Lt.grad.numpy(), rtol=1e-10, atol=1e-13)
