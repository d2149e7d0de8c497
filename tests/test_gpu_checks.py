"""The MOE_CHECKS switch: whole-layout verification of the routing on the device.

With MOE_CHECKS set, the calls that produce the expert-sorted layout (moe_route,
moe_layer_fwd) verify it, and moe_dispatch / moe_grouped_gemm_fwd verify what they are
given: slot maps the T*k pairs to distinct rows inside their experts' ranges,
row_token[slot[t,j]] == t, offsets are a monotone scan ending at R (or the capacity
multiples).  A failure sets MOE_DEV_CHECK_FAILED."""
import numpy as np
import pytest
import torch

from routing_grouped_gemm_route_b200 import lib
from routing_grouped_gemm_route_b200.inputs import Workload, make_inputs, normal_tensor

from helpers import run_layer, run_route

pytestmark = pytest.mark.gpu


@pytest.fixture
def checks_on(monkeypatch):
    monkeypatch.setenv("MOE_CHECKS", "1")


@pytest.mark.parametrize("skew,capacity_extra", [(False, None), (True, None), (False, 5),
                                                 (True, 0)])
def test_checks_pass_on_the_routing_the_library_produces(cuda_lib, checks_on, skew,
                                                         capacity_extra):
    w = Workload("chk", 3000, 256, 16, 4, 128, "bf16", router=False, skew=skew, seed=41)
    inp = make_inputs(w)
    cap = 0
    if capacity_extra is not None:
        desc = lib.make_desc(w.T, w.d, w.d_ff, w.E, w.k, "bf16")
        cap = int(run_route(desc, inp["logits"].cuda())["counts"].max()) + capacity_extra
    desc, layer, dv, y, g, status = run_layer(w, inp, capacity=cap)
    assert status == 0


def _dispatch_status(slot):
    T, k = slot.shape
    desc = lib.make_desc(T, 128, 64, 8, k, "bf16")
    ws = lib.alloc_workspace(desc)
    x = normal_tensor((T, 128), seed=3).cuda()
    xp = torch.zeros(T * k, 128, dtype=torch.bfloat16, device="cuda")
    lib.moe_dispatch(desc, x, slot.cuda(), xp, ws)
    return lib.moe_read_device_status(ws)


def test_checks_catch_a_duplicated_slot(cuda_lib, checks_on):
    T, k = 300, 2
    perm = torch.randperm(T * k, generator=torch.Generator().manual_seed(2)).to(torch.int32)
    assert _dispatch_status(perm.view(T, k)) == 0          # a permutation passes
    dup = perm.clone()
    dup[17] = dup[250]                                      # two pairs on one row, one row empty
    bits = _dispatch_status(dup.view(T, k))
    assert bits & lib.MOE_DEV_CHECK_FAILED
    assert not bits & lib.MOE_DEV_BAD_INDEX                 # every slot was in range


def test_checks_are_off_by_default(cuda_lib, monkeypatch):
    monkeypatch.delenv("MOE_CHECKS", raising=False)
    T, k = 300, 2
    dup = torch.randperm(T * k, generator=torch.Generator().manual_seed(2)).to(torch.int32)
    dup[17] = dup[250]
    assert _dispatch_status(dup.view(T, k)) == 0


def test_checks_catch_offsets_that_are_not_a_scan(cuda_lib, checks_on):
    T, d, f, E, k = 256, 128, 64, 4, 2
    desc = lib.make_desc(T, d, f, E, k, "bf16")
    ws = lib.alloc_workspace(desc)
    R = T * k
    off = torch.tensor([0, 200, 150, 400, R], dtype=torch.int32, device="cuda")   # not monotone
    z = lambda *s: torch.zeros(*s, dtype=torch.bfloat16, device="cuda")   # noqa: E731
    lib.moe_grouped_gemm_fwd(desc, z(R, d), z(E, 2 * f, d), z(E, d, f), off, z(R, 2 * f), z(R, f),
                             z(R, d), ws)
    bits = lib.moe_read_device_status(ws)
    assert bits & lib.MOE_DEV_CHECK_FAILED and bits & lib.MOE_DEV_BAD_OFFSETS
