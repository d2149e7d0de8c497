"""Shared helpers of the GPU parity tests (device runs through the C ABI, comparisons
against the fp64 oracle)."""
import numpy as np
import torch

import oracle
from routing_grouped_gemm_route_b200 import lib
from routing_grouped_gemm_route_b200.inputs import Workload, make_inputs

# Relative Frobenius bound of every floating-point output against the fp64 oracle.
# bf16: storage of x_perm/H13/a/y_perm/dH13 in bf16 (2^-9 relative rounding each)
# compounds to ~2-4e-3 at the layer output, under this bar.  fp32 storage with TF32
# tensor-core products (10 explicit mantissa bits, ~2^-11 per product) lands near
# 5e-4, also under it.
TOL = 5e-3


def f64(t) -> np.ndarray:
    if isinstance(t, np.ndarray):
        return t.astype(np.float64)
    return t.detach().to("cpu", torch.float64).numpy()


def npi(t) -> np.ndarray:
    return t.detach().cpu().numpy().astype(np.int64)


def row_rel(got, ref) -> np.ndarray:
    """Per-row relative error ||got - ref|| / ||ref|| of a GPU tensor against fp64 rows."""
    g = f64(got)
    return np.linalg.norm(g - ref, axis=1) / np.maximum(np.linalg.norm(ref, axis=1), 1e-30)


def rel(a, b) -> float:
    return oracle.rel_fro(f64(a), f64(b))


def workload(T, d, E, k, f, dtype="bf16", router=False, skew=False, seed=0):
    return Workload(f"t{T}_{d}_{E}_{k}_{f}", T, d, E, k, f, dtype, router=router, skew=skew,
                    seed=seed)


def desc_of(w: Workload, flags=0):
    if w.router:
        flags |= lib.MOE_FLAG_ROUTER
    if w.shared:
        flags |= lib.MOE_FLAG_SHARED_EXPERT
    return lib.make_desc(w.T, w.d, w.d_ff, w.E, w.k, w.dtype, flags)


def to_dev(inp: dict, device="cuda") -> dict:
    return {k: (None if v is None else v.to(device)) for k, v in inp.items()}


def run_route(desc, logits_dev):
    T, E, k = desc.T, desc.E, desc.k
    dev = logits_dev.device
    out = dict(topk_idx=torch.empty(T, k, dtype=torch.int32, device=dev),
               gates=torch.empty(T, k, dtype=torch.float32, device=dev),
               counts=torch.empty(E, dtype=torch.int32, device=dev),
               offsets=torch.empty(E + 1, dtype=torch.int32, device=dev),
               slot=torch.empty(T, k, dtype=torch.int32, device=dev),
               row_token=torch.empty(lib.rows_of(desc), dtype=torch.int32, device=dev),
               row_gate=torch.empty(lib.rows_of(desc), dtype=torch.float32, device=dev))
    ws = lib.alloc_workspace(desc)
    lib.moe_route(desc, logits_dev, out["topk_idx"], out["gates"], out["counts"], out["offsets"],
                  out["slot"], out["row_token"], out["row_gate"], ws)
    torch.cuda.synchronize()
    assert lib.moe_read_device_status(ws) == 0
    return out


def assert_route_equal(gpu: dict, ref: dict, k: int):
    assert np.array_equal(npi(gpu["topk_idx"]), ref["topk_idx"])
    assert np.array_equal(npi(gpu["counts"]), ref["counts"])
    assert np.array_equal(npi(gpu["offsets"]), ref["offsets"])
    assert np.array_equal(npi(gpu["slot"]), ref["slot"])
    assert np.array_equal(npi(gpu["row_token"]), ref["row_token"])
    g = f64(gpu["gates"])
    assert np.max(np.abs(g - ref["gates"])) < 2e-6
    # row_gate is a copy of the gate of each sorted row
    assert np.array_equal(f64(gpu["row_gate"])[npi(gpu["slot"])], g)


def run_layer(w: Workload, inp: dict, flags=0, capacity=0):
    """Layer fwd+bwd through moe_layer_fwd / moe_layer_bwd on the device."""
    desc = desc_of(w, flags)
    desc.capacity = capacity
    layer = lib.Layer(desc)
    dv = to_dev(inp)
    y = layer.fwd(dv["x"], dv["W13"], dv["W2"], logits=dv["logits"], Wr=dv["Wr"])
    g = layer.bwd(dv["dy"], dv["W13"], dv["W2"], x=dv["x"], Wr=dv["Wr"])
    torch.cuda.synchronize()
    status = lib.moe_read_device_status(layer.ws)
    return desc, layer, dv, y, g, status
