"""Dispatch, combine and their backward on the GPU against the oracle, each stage fed
the GPU's own routing.  Dispatch is a copy and must be bit-exact (for fp32, a copy of x
rounded to TF32, the precision the GEMMs read it in; likewise fp32 dy_perm)."""
import numpy as np
import pytest
import torch

import oracle
from routing_grouped_gemm_route_b200 import lib
from routing_grouped_gemm_route_b200.inputs import normal_tensor, random_logits

from helpers import TOL, f64, npi, rel, run_route

pytestmark = pytest.mark.gpu

CASES = [(1, 128, 8, 2, "bf16"), (300, 256, 8, 2, "bf16"), (1000, 384, 37, 3, "fp32"),
         (4096, 2048, 128, 4, "bf16"), (777, 128, 16, 8, "fp32"), (513, 1024, 64, 32, "bf16")]


def setup(T, d, E, k, dt, seed=0):
    desc = lib.make_desc(T, d, 64, E, k, dt)
    act = torch.float32 if dt == "fp32" else torch.bfloat16
    L = random_logits(T, E, seed=seed + 1)
    r = run_route(desc, L.cuda())
    ws = lib.alloc_workspace(desc)
    return desc, act, r, ws


@pytest.mark.parametrize("T,d,E,k,dt", CASES)
def test_dispatch_is_an_exact_copy(cuda_lib, T, d, E, k, dt):
    desc, act, r, ws = setup(T, d, E, k, dt)
    x = normal_tensor((T, d), seed=2, dtype=act)
    xp = torch.full((T * k, d), float("nan"), dtype=act, device="cuda")
    lib.moe_dispatch(desc, x.cuda(), r["slot"], xp, ws)
    torch.cuda.synchronize()
    assert lib.moe_read_device_status(ws) == 0
    # fp32: x_perm holds x rounded to TF32 (the precision the GEMMs read it in)
    xs = oracle.tf32_round(x.numpy()) if dt == "fp32" else f64(x)
    ref = oracle.dispatch(np.asarray(xs, dtype=np.float64), npi(r["slot"]))
    assert np.array_equal(f64(xp), ref)


@pytest.mark.parametrize("T,d,E,k,dt", CASES)
def test_combine(cuda_lib, T, d, E, k, dt):
    desc, act, r, ws = setup(T, d, E, k, dt)
    yp = normal_tensor((T * k, d), seed=3, dtype=act)
    y = torch.empty(T, d, dtype=act, device="cuda")
    lib.moe_combine(desc, yp.cuda(), r["gates"], r["slot"], y, ws)
    torch.cuda.synchronize()
    ref = oracle.combine(f64(yp), f64(r["gates"]), npi(r["slot"]))
    assert rel(y, ref) < (2e-6 if dt == "fp32" else TOL)


@pytest.mark.parametrize("T,d,E,k,dt", CASES)
def test_combine_bwd(cuda_lib, T, d, E, k, dt):
    desc, act, r, ws = setup(T, d, E, k, dt)
    yp = normal_tensor((T * k, d), seed=4, dtype=act)
    dy = normal_tensor((T, d), seed=5, dtype=act)
    dyp = torch.empty(T * k, d, dtype=act, device="cuda")
    dl = torch.full((T, E), float("nan"), dtype=torch.float32, device="cuda")
    lib.moe_combine_bwd(desc, dy.cuda(), yp.cuda(), r["gates"], r["topk_idx"], r["slot"], dyp, dl,
                        ws)
    torch.cuda.synchronize()
    assert lib.moe_read_device_status(ws) == 0
    ref_dyp, ref_dl = oracle.combine_bwd(f64(dy), f64(yp), f64(r["gates"]), npi(r["topk_idx"]),
                                         npi(r["slot"]), E)
    if dt == "fp32":
        # dy_perm[slot] = g * dy in fp32, rounded to TF32: bit-exact
        g32 = r["gates"].cpu().numpy().astype(np.float32)
        d32 = dy.numpy().astype(np.float32)
        want = np.empty((T * k, d), dtype=np.float32)
        for j in range(k):
            want[npi(r["slot"])[:, j]] = oracle.tf32_round(g32[:, j:j + 1] * d32)
        assert np.array_equal(dyp.cpu().numpy().view(np.uint32), want.view(np.uint32))
    assert rel(dyp, ref_dyp) < (6e-4 if dt == "fp32" else TOL)
    assert rel(dl, ref_dl) < 1e-4
    # experts that were not selected get exactly zero
    mask = np.ones((T, E), bool)
    np.put_along_axis(mask, npi(r["topk_idx"]), False, axis=1)
    assert np.all(f64(dl)[mask] == 0.0)


@pytest.mark.parametrize("T,d,E,k,dt", CASES)
def test_dispatch_bwd(cuda_lib, T, d, E, k, dt):
    desc, act, r, ws = setup(T, d, E, k, dt)
    dxp = normal_tensor((T * k, d), seed=6, dtype=act)
    dx = torch.empty(T, d, dtype=act, device="cuda")
    lib.moe_dispatch_bwd(desc, dxp.cuda(), r["slot"], dx, ws)
    torch.cuda.synchronize()
    ref = oracle.dispatch_bwd(f64(dxp), npi(r["slot"]))
    assert rel(dx, ref) < (2e-6 if dt == "fp32" else TOL)


def test_bad_slot_sets_status_and_is_skipped(cuda_lib):
    T, d, E, k = 64, 128, 8, 2
    desc = lib.make_desc(T, d, 64, E, k, "bf16")
    ws = lib.alloc_workspace(desc)
    slot = torch.arange(T * k, dtype=torch.int32).view(T, k)
    slot[5, 1] = T * k + 7                                  # out of range
    slot[9, 0] = -3
    x = normal_tensor((T, d), seed=1).cuda()
    xp = torch.zeros(T * k, d, dtype=torch.bfloat16, device="cuda")
    lib.moe_dispatch(desc, x, slot.cuda(), xp, ws)
    bits = lib.moe_read_device_status(ws)
    assert bits & lib.MOE_DEV_BAD_INDEX
    good = slot.clone()
    assert torch.equal(xp[good[0, 0].item()], x[0])
    assert torch.all(xp[int(slot[9, 1])] == x[9])
    lib.moe_workspace_init(ws)
    assert lib.moe_read_device_status(ws) == 0
