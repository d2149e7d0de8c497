"""moe_route_noalloc: routing for callers that cannot give the library a workspace.

Some callers own every device buffer themselves (a host framework or plugin that plans
its memory ahead and passes only inputs and outputs) or must not call cudaMalloc on a
latency-critical path, since it synchronises the device.  For them the library keeps
the routing scratch in a fixed static device array.  This file checks, through the C
ABI, that two calls in a row give exactly what moe_route gives with a workspace and
what the fp64 oracle gives, that a problem too large for the static array is refused
before anything runs, and that the capacity-padded layout (whose overflow it could not
report) is refused too.  It is collected last so a failure here never hides the other
tests.
"""
import ctypes

import numpy as np
import pytest
import torch

import oracle
from routing_grouped_gemm_route_b200 import lib
from routing_grouped_gemm_route_b200.inputs import random_logits

pytestmark = pytest.mark.gpu


def _outputs(T, E, k):
    dev = "cuda"
    return dict(topk_idx=torch.empty(T, k, dtype=torch.int32, device=dev),
                gates=torch.empty(T, k, dtype=torch.float32, device=dev),
                counts=torch.empty(E, dtype=torch.int32, device=dev),
                offsets=torch.empty(E + 1, dtype=torch.int32, device=dev),
                slot=torch.empty(T, k, dtype=torch.int32, device=dev),
                row_token=torch.empty(T * k, dtype=torch.int32, device=dev),
                row_gate=torch.empty(T * k, dtype=torch.float32, device=dev))


def _args(o):
    return (o["topk_idx"], o["gates"], o["counts"], o["offsets"], o["slot"], o["row_token"],
            o["row_gate"])


@pytest.mark.parametrize("T,E,k,skew", [(16384, 128, 4, False), (3001, 37, 3, True)])
def test_noalloc_route_matches_workspace_route_twice(cuda_lib, T, E, k, skew):
    desc = lib.make_desc(T, 128, 64, E, k, "bf16")
    ws = lib.alloc_workspace(desc)
    for call, seed in enumerate((11, 12)):        # two calls in a row, different logits
        L = random_logits(T, E, seed=seed + T, skew=skew).cuda()
        ref, got = _outputs(T, E, k), _outputs(T, E, k)
        lib.moe_route(desc, L, *_args(ref), ws)
        lib.moe_route_noalloc(desc, L, *_args(got))
        torch.cuda.synchronize()
        for name in ("topk_idx", "counts", "offsets", "slot", "row_token"):
            assert torch.equal(got[name], ref[name]), (call, name)
        # same tolerance as the routing parity tests (the kernels are the same)
        assert torch.max(torch.abs(got["gates"] - ref["gates"])).item() < 2e-6
        assert torch.max(torch.abs(got["row_gate"] - ref["row_gate"])).item() < 2e-6
        assert int(got["counts"].sum()) == T * k
        assert lib.moe_read_device_status(ws) == 0
        # and against the oracle: indices, counts, offsets and the permutation bit-exact
        ref = oracle.route(L.cpu().numpy().astype(np.float64), k, E)
        for name in ("topk_idx", "counts", "offsets", "slot", "row_token"):
            assert np.array_equal(got[name].cpu().numpy().astype(np.int64),
                                  np.asarray(ref[name]).reshape(got[name].shape)), (call, name)
        assert np.max(np.abs(got["gates"].cpu().double().numpy() - ref["gates"])) < 2e-6


def test_noalloc_route_refuses_problems_beyond_its_scratch(cuda_lib):
    # (ceil(T/64) + ceil(T/256)) * E * 4 bytes (20 * E per 256 tokens) above the fixed
    # array: refused before any launch
    E = 1024
    T = 256 * (lib.MOE_ROUTE_NOALLOC_SCRATCH_BYTES // (20 * E) + 1)
    desc = lib.make_desc(T, 128, 64, E, 2, "bf16")
    small = _outputs(1, E, 2)
    logits = torch.zeros(1, E, device="cuda")
    # the library itself refuses (buffers sized for one token: nothing may run) ...
    st = lib.load().moe_route_noalloc(ctypes.byref(desc), logits.data_ptr(),
                                      *[t.data_ptr() for t in _args(small)], lib._stream())
    assert st == lib.MOE_EWORKSPACE
    # ... and the binding does not let buffers this short through in the first place
    with pytest.raises(ValueError):
        lib.moe_route_noalloc(desc, logits, *_args(small))


def test_noalloc_route_refuses_the_padded_layout(cuda_lib):
    # capacity > 0 can overflow an expert; with no status word to report it, the call
    # refuses the layout before any launch instead of dropping tokens silently
    T, E, k = 1000, 16, 2
    desc = lib.make_desc(T, 128, 64, E, k, "bf16", capacity=(T * k) // E)
    o = _outputs(T, E, k)
    o["row_token"] = torch.empty(E * desc.capacity, dtype=torch.int32, device="cuda")
    o["row_gate"] = torch.empty(E * desc.capacity, dtype=torch.float32, device="cuda")
    L = random_logits(T, E, seed=5).cuda()
    with pytest.raises(lib.MoEError) as err:
        lib.moe_route_noalloc(desc, L, *_args(o))
    assert err.value.status == lib.MOE_EUNSUPPORTED
