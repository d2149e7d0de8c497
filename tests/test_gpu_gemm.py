"""Grouped GEMM forward and backward on the GPU against the oracle, stage by stage:
each GEMM is compared with the oracle applied to that GEMM's actual GPU inputs, so a
rounding difference upstream is not charged to the stage downstream."""
import numpy as np
import pytest
import torch

import oracle
from routing_grouped_gemm_route_b200 import lib
from routing_grouped_gemm_route_b200.inputs import normal_tensor, random_logits

from helpers import TOL, f64, npi, rel, row_rel, run_route

pytestmark = pytest.mark.gpu

# (T, d, d_ff, E, k, dtype, logit bias mode)
CASES = [
    (300, 256, 128, 5, 2, "bf16", None),        # ragged tails in every expert
    (512, 128, 256, 8, 2, "fp32", None),        # the tiny fp32 workload's shape (TF32 MMA)
    (1000, 512, 192, 8, 4, "bf16", None),       # d_ff not a multiple of 128
    (700, 384, 64, 12, 3, "fp32", None),
    (2048, 256, 128, 33, 4, "bf16", "empty"),   # several experts with no rows
    (1500, 256, 128, 6, 1, "bf16", "one"),      # nearly all rows on one expert
    (96, 256, 128, 4, 4, "bf16", None),         # k = E, fewer rows than one tile
    (4096, 1024, 512, 16, 4, "bf16", None),
    (300, 256, 256, 5, 2, "bf16", None),        # d_ff % 256 == 0: every GEMM with tokens as N
    (2048, 512, 256, 33, 4, "bf16", "empty"),   # ... with empty experts and short tails
    (700, 256, 128, 1024, 8, "bf16", None),     # the largest E: ~5 rows per expert, many empty
]


def make(T, d, f, E, k, dt, mode, seed=0):
    act = torch.float32 if dt == "fp32" else torch.bfloat16
    desc = lib.make_desc(T, d, f, E, k, dt)
    L = random_logits(T, E, seed=seed + 11)
    if mode == "empty":
        L[:, ::3] -= 50.0                          # experts 0, 3, 6, ... never chosen
    elif mode == "one":
        L[: T - 3, 2] += 50.0
    r = run_route(desc, L.cuda())
    x = normal_tensor((T, d), seed=seed + 12, dtype=act).cuda()
    W13 = normal_tensor((E, 2 * f, d), seed=seed + 13, std=0.02, dtype=act).cuda()
    W2 = normal_tensor((E, d, f), seed=seed + 14, std=0.02, dtype=act).cuda()
    ws = lib.alloc_workspace(desc)
    R = T * k
    xp = torch.empty(R, d, dtype=act, device="cuda")
    lib.moe_dispatch(desc, x, r["slot"], xp, ws)
    return desc, act, r, x, W13, W2, ws, xp


def fwd(desc, act, r, W13, W2, ws, xp):
    R, d, f = desc.T * desc.k, desc.d, desc.d_ff
    H13 = torch.full((R, 2 * f), float("nan"), dtype=act, device="cuda")
    a = torch.full((R, f), float("nan"), dtype=act, device="cuda")
    yp = torch.full((R, d), float("nan"), dtype=act, device="cuda")
    lib.moe_grouped_gemm_fwd(desc, xp, W13, W2, r["offsets"], H13, a, yp, ws)
    torch.cuda.synchronize()
    assert lib.moe_read_device_status(ws) == 0
    return H13, a, yp


@pytest.mark.parametrize("T,d,f,E,k,dt,mode", CASES)
def test_grouped_gemm_fwd(cuda_lib, T, d, f, E, k, dt, mode):
    desc, act, r, x, W13, W2, ws, xp = make(T, d, f, E, k, dt, mode)
    H13, a, yp = fwd(desc, act, r, W13, W2, ws, xp)
    off = npi(r["offsets"])
    W13h, W2h = f64(W13), f64(W2)
    # FC1 (+ SwiGLU) from the GPU's x_perm
    refH, refA, _ = oracle.experts_fwd(f64(xp), off, W13h, W2h)
    assert rel(H13, refH) < TOL
    assert rel(a, refA) < TOL
    # FC2 from the GPU's a
    refY = np.zeros((T * k, d))
    for e in range(E):
        refY[off[e]:off[e + 1]] = f64(a)[off[e]:off[e + 1]] @ W2h[e].T
    assert rel(yp, refY) < TOL
    # every row written (no NaN left from the fill)
    assert not torch.isnan(H13).any() and not torch.isnan(a).any() and not torch.isnan(yp).any()
    # per-expert check so one bad expert cannot hide in the global norm
    for e in range(E):
        if off[e + 1] > off[e]:
            assert rel(yp[off[e]:off[e + 1]], refY[off[e]:off[e + 1]]) < 2 * TOL, e
    # and per row: what remains is fp32 accumulation (TF32 operand rounding) and the
    # output's own rounding, so one wrong row (a tile edge, a ragged tail) fails this
    assert row_rel(H13, refH).max() < 1e-2
    assert row_rel(yp, refY).max() < 1e-2


@pytest.mark.parametrize("dw_fp32", [False, True])
@pytest.mark.parametrize("T,d,f,E,k,dt,mode", CASES)
def test_grouped_gemm_bwd(cuda_lib, T, d, f, E, k, dt, mode, dw_fp32):
    desc, act, r, x, W13, W2, ws, xp = make(T, d, f, E, k, dt, mode, seed=1)
    H13, a, yp = fwd(desc, act, r, W13, W2, ws, xp)
    if dw_fp32:
        desc = lib.make_desc(T, d, f, E, k, dt, lib.MOE_FLAG_DW_FP32)
    R = T * k
    dyp = normal_tensor((R, d), seed=21, dtype=act).cuda()
    dH13 = torch.full((R, 2 * f), float("nan"), dtype=act, device="cuda")
    dxp = torch.full((R, d), float("nan"), dtype=act, device="cuda")
    dw_dt = torch.float32 if dw_fp32 else act
    dW13 = torch.full((E, 2 * f, d), float("nan"), dtype=dw_dt, device="cuda")
    dW2 = torch.full((E, d, f), float("nan"), dtype=dw_dt, device="cuda")
    lib.moe_grouped_gemm_bwd(desc, dyp, xp, H13, a, W13, W2, r["offsets"], dH13, dxp, dW13, dW2, ws)
    torch.cuda.synchronize()
    assert lib.moe_read_device_status(ws) == 0
    off = npi(r["offsets"])
    W13h, W2h = f64(W13), f64(W2)
    dY, A, X, H, dHg = f64(dyp), f64(a), f64(xp), f64(H13), f64(dH13)
    ref_dH = np.zeros((R, 2 * f))
    ref_dX = np.zeros((R, d))
    for e in range(E):
        s = slice(off[e], off[e + 1])
        if off[e + 1] == off[e]:
            # an expert with no rows has exactly zero weight gradients
            assert torch.all(dW13[e] == 0) and torch.all(dW2[e] == 0), e
            continue
        ref_dH[s] = oracle.swiglu_bwd(dY[s] @ W2h[e], H[s])
        ref_dX[s] = dHg[s] @ W13h[e]
        assert rel(dW2[e], dY[s].T @ A[s]) < TOL, ("dW2", e)
        assert rel(dW13[e], dHg[s].T @ X[s]) < TOL, ("dW13", e)
    assert rel(dH13, ref_dH) < TOL
    assert rel(dxp, ref_dX) < TOL
    assert not torch.isnan(dH13).any() and not torch.isnan(dxp).any()
    # the references start from the GPU's own bf16 H13 and dH13, so per row only
    # accumulation and output rounding remain
    assert row_rel(dH13, ref_dH).max() < 1e-2
    assert row_rel(dxp, ref_dX).max() < 1e-2


def test_accumulate_dw(cuda_lib):
    T, d, f, E, k = 600, 256, 128, 6, 2
    desc, act, r, x, W13, W2, ws, xp = make(T, d, f, E, k, "bf16", "empty", seed=2)
    H13, a, yp = fwd(desc, act, r, W13, W2, ws, xp)
    R = T * k
    dyp = normal_tensor((R, d), seed=31).cuda()
    dH13 = torch.empty(R, 2 * f, dtype=act, device="cuda")
    dxp = torch.empty(R, d, dtype=act, device="cuda")
    base13 = normal_tensor((E, 2 * f, d), seed=32, dtype=torch.float32).cuda()
    base2 = normal_tensor((E, d, f), seed=33, dtype=torch.float32).cuda()
    dW13, dW2 = base13.clone(), base2.clone()
    acc = lib.make_desc(T, d, f, E, k, "bf16", lib.MOE_FLAG_DW_FP32 | lib.MOE_FLAG_ACCUM_DW)
    lib.moe_grouped_gemm_bwd(acc, dyp, xp, H13, a, W13, W2, r["offsets"], dH13, dxp, dW13, dW2, ws)
    one13 = torch.empty_like(base13)
    one2 = torch.empty_like(base2)
    plain = lib.make_desc(T, d, f, E, k, "bf16", lib.MOE_FLAG_DW_FP32)
    lib.moe_grouped_gemm_bwd(plain, dyp, xp, H13, a, W13, W2, r["offsets"], dH13, dxp, one13, one2,
                             ws)
    torch.cuda.synchronize()
    assert torch.allclose(dW13, base13 + one13, rtol=0, atol=1e-6)
    assert torch.allclose(dW2, base2 + one2, rtol=0, atol=1e-6)
    off = npi(r["offsets"])
    empty = [e for e in range(E) if off[e + 1] == off[e]]
    assert empty and all(torch.equal(dW13[e], base13[e]) for e in empty)


def test_bad_offsets_set_status_and_write_nothing(cuda_lib):
    T, d, f, E, k = 256, 128, 64, 4, 2
    desc, act, r, x, W13, W2, ws, xp = make(T, d, f, E, k, "bf16", None)
    bad = r["offsets"].clone()
    bad[2] = bad[1] - 1                                   # not monotone
    R = T * k
    H13 = torch.zeros(R, 2 * f, dtype=act, device="cuda")
    a = torch.zeros(R, f, dtype=act, device="cuda")
    yp = torch.zeros(R, d, dtype=act, device="cuda")
    lib.moe_grouped_gemm_fwd(desc, xp, W13, W2, bad, H13, a, yp, ws)
    bits = lib.moe_read_device_status(ws)
    assert bits & lib.MOE_DEV_BAD_OFFSETS
    assert torch.all(yp == 0) and torch.all(H13 == 0)
    bad2 = r["offsets"].clone()
    bad2[E] = R + 5                                       # does not end at R
    lib.moe_workspace_init(ws)
    lib.moe_grouped_gemm_fwd(desc, xp, W13, W2, bad2, H13, a, yp, ws)
    assert lib.moe_read_device_status(ws) & lib.MOE_DEV_BAD_OFFSETS


@pytest.mark.parametrize("dt", ["bf16", "fp32", "mxfp8"])
def test_bounded_waits_run_out_and_the_next_call_succeeds(cuda_lib, dt):
    """The bounded-wait path, without faulting anything: with the test hook the GEMMs'
    producers load nothing, so the MMA and epilogue waits give up after 10 ms.  The call
    must report MOE_DEV_TIMEOUT, write none of its outputs and leave the context usable:
    its tensor memory freed (an allocation left behind would stall the next GEMM on that
    SM) and the next normal call on the same workspace correct against the oracle."""
    T, d, f, E, k = 256, 128, 128, 4, 2
    desc, act, r, x, W13, W2, ws, xp = make(T, d, f, E, k, dt, None, seed=5)
    R = T * k
    stall = lib.make_desc(T, d, f, E, k, dt, lib.MOE_FLAG_TEST_WAIT_TIMEOUT)
    H13 = torch.full((R, 2 * f), float("nan"), dtype=act, device="cuda")
    a = torch.full((R, f), float("nan"), dtype=act, device="cuda")
    yp = torch.full((R, d), float("nan"), dtype=act, device="cuda")
    lib.moe_grouped_gemm_fwd(stall, xp, W13, W2, r["offsets"], H13, a, yp, ws)
    bits = lib.moe_read_device_status(ws)
    assert bits & lib.MOE_DEV_TIMEOUT
    assert torch.isnan(H13).all() and torch.isnan(a).all() and torch.isnan(yp).all()
    lib.moe_workspace_init(ws)
    H13, a, yp = fwd(desc, act, r, W13, W2, ws, xp)     # asserts a clear status word
    mx = dt == "mxfp8"
    refH, refA, refY = oracle.experts_fwd(f64(xp), npi(r["offsets"]), f64(W13), f64(W2), mx=mx)
    tol = 3e-2 if mx else TOL
    assert rel(H13, refH) < tol
    assert rel(yp, refY) < tol
