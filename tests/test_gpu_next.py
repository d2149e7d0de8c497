"""Device load statistics (moe_load_stats) against the oracle's definitions, and the
layer with activation recompute (MOE_FLAG_RECOMPUTE) against the layer without it."""
import numpy as np
import pytest
import torch

import oracle
from routing_grouped_gemm_route_b200 import lib
from routing_grouped_gemm_route_b200.inputs import Workload, make_inputs, random_logits

from helpers import TOL, f64, npi, rel, run_layer, run_route

pytestmark = pytest.mark.gpu


def gpu_stats(counts_dev, status=None):
    out = torch.zeros(64, dtype=torch.uint8, device="cuda")
    lib.moe_load_stats(counts_dev, out, status)
    torch.cuda.synchronize()
    return lib.decode_load_stats(out)


def assert_stats_equal(got, want):
    for key in ("total", "max_count", "min_count", "num_empty", "num_experts"):
        assert got[key] == want[key], key
    for key in ("mean", "max_over_mean", "cv"):
        assert abs(got[key] - want[key]) <= 1e-12 * max(1.0, abs(want[key])), key


@pytest.mark.parametrize("T,E,k,skew", [(16384, 128, 4, False), (16384, 128, 4, True),
                                        (4096, 8, 2, False), (1000, 1024, 8, True),
                                        (300, 1, 1, False)])
def test_load_stats_of_routing(cuda_lib, T, E, k, skew):
    L = random_logits(T, E, seed=T + E)
    if skew:
        # Zipf-like bias over a seeded permutation of the experts
        g = np.random.default_rng(E)
        rank = g.permutation(E) + 1
        L = L + torch.tensor(-1.8 * np.log(rank), dtype=torch.float32)[None, :]
    desc = lib.make_desc(T, 128, 64, E, k, "bf16")
    r = run_route(desc, L.cuda())
    want = oracle.load_stats(npi(r["counts"]))
    assert_stats_equal(gpu_stats(r["counts"]), want)


def test_load_stats_edge_cases(cuda_lib):
    for counts in ([0, 0, 0, 0], [5], [0] * 1023 + [77], list(range(1024))):
        c = torch.tensor(counts, dtype=torch.int32, device="cuda")
        assert_stats_equal(gpu_stats(c), oracle.load_stats(counts))
    # a negative count is reported and read as 0
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    c = torch.tensor([3, -2, 5], dtype=torch.int32, device="cuda")
    st = gpu_stats(c, status)
    assert int(status.item()) & lib.MOE_DEV_BAD_OFFSETS
    assert_stats_equal(st, oracle.load_stats([3, 0, 5]))


@pytest.mark.parametrize("T,d,E,k,f,dt,router", [
    (3000, 256, 16, 4, 128, "bf16", False),
    (2000, 256, 8, 2, 256, "bf16", True),
    (1500, 256, 8, 4, 128, "mxfp8", False),
    (512, 128, 8, 2, 256, "fp32", True),
    (0, 256, 8, 2, 128, "bf16", False),
])
def test_recompute_is_bit_identical(cuda_lib, T, d, E, k, f, dt, router):
    w = Workload("rc", T, d, E, k, f, dt, router=router, skew=False, seed=T + 3)
    inp = make_inputs(w)
    _, lay0, _, y0, g0, st0 = run_layer(w, inp)
    _, lay1, _, y1, g1, st1 = run_layer(w, inp, flags=lib.MOE_FLAG_RECOMPUTE)
    assert st0 == 0 and st1 == 0
    assert lay1.saved.numel() < lay0.saved.numel() or T == 0
    assert torch.equal(y0, y1)
    for name in ("dx", "d_logits", "dW13", "dW2") + (("dWr",) if router else ()):
        assert torch.equal(g0[name], g1[name]), name
    if T and dt == "bf16":
        # and against the oracle, as the plain layer is
        x, dy = f64(inp["x"]), f64(inp["dy"])
        W13, W2 = inp["W13"].float().numpy(), inp["W2"].float().numpy()
        L = None if router else f64(inp["logits"])
        Wr = inp["Wr"].float().numpy() if router else None
        if router:
            L = f64(lay1.views()["logits"])
        fwd = oracle.layer_fwd(x, W13, W2, logits=L, k=k)
        bwd = oracle.layer_bwd(fwd, dy, x, W13, W2, Wr=Wr)
        assert rel(y1, fwd["y"]) < TOL
        assert rel(g1["dW13"], bwd["dW13"]) < TOL


# ------------------------------------------------------------------- shared expert

@pytest.mark.parametrize("T,d,E,k,f,dt,router,flags", [
    (3000, 256, 16, 4, 128, "bf16", False, 0),
    (1000, 512, 64, 4, 256, "bf16", True, 0),
    (700, 256, 8, 2, 128, "bf16", False, lib.MOE_FLAG_RECOMPUTE),
    (333, 384, 12, 3, 192, "fp32", True, 0),
    (1200, 256, 8, 2, 128, "bf16", False, lib.MOE_FLAG_DW_FP32),
])
def test_shared_expert_layer_matches_oracle(cuda_lib, T, d, E, k, f, dt, router, flags):
    w = Workload("sh", T, d, E, k, f, dt, router=router, skew=False, seed=T + 5, shared=True)
    inp = make_inputs(w)
    desc, layer, dv, y, g, status = run_layer(w, inp, flags=flags)
    assert status == 0
    assert g["dW13"].shape[0] == E + 1
    v = layer.views()
    x, dy = f64(inp["x"]), f64(inp["dy"])
    W13, W2 = inp["W13"].float().numpy(), inp["W2"].float().numpy()
    L = f64(v["logits"]) if router else f64(inp["logits"])
    Wr = inp["Wr"].float().numpy() if router else None
    fwd = oracle.layer_fwd(x, W13, W2, logits=L, k=k, shared=True)
    bwd = oracle.layer_bwd(fwd, dy, x, W13, W2, Wr=Wr)
    assert np.array_equal(npi(v["topk_idx"]), fwd["topk_idx"])
    assert rel(y, fwd["y"]) < TOL
    for name in ("dx", "d_logits", "dW13", "dW2") + (("dWr",) if router else ()):
        assert rel(g[name], bwd[name]) < TOL, name
    # the shared expert's own slices, on their own
    assert rel(g["dW13"][E], bwd["dW13"][E]) < TOL
    assert rel(g["dW2"][E], bwd["dW2"][E]) < TOL
    if not flags & lib.MOE_FLAG_RECOMPUTE:
        assert rel(v["a_shared"], fwd["a_shared"]) < TOL


def test_shared_expert_recompute_is_bit_identical(cuda_lib):
    w = Workload("shrc", 2000, 256, 16, 4, 128, "bf16", router=True, skew=False, seed=77,
                 shared=True)
    inp = make_inputs(w)
    _, lay0, _, y0, g0, st0 = run_layer(w, inp)
    _, lay1, _, y1, g1, st1 = run_layer(w, inp, flags=lib.MOE_FLAG_RECOMPUTE)
    assert st0 == 0 and st1 == 0
    assert torch.equal(y0, y1)
    for name in ("dx", "d_logits", "dW13", "dW2", "dWr"):
        assert torch.equal(g0[name], g1[name]), name


def test_shared_expert_no_tokens(cuda_lib):
    w = Workload("sh0", 0, 256, 8, 2, 128, "bf16", router=False, skew=False, seed=1, shared=True)
    inp = make_inputs(w)
    _, layer, _, y, g, status = run_layer(w, inp)
    assert status == 0
    assert torch.all(g["dW13"] == 0) and torch.all(g["dW2"] == 0)


# ------------------------------------------------------- capacity-padded comparator

def max_count(w, inp):
    desc = lib.make_desc(w.T, w.d, w.d_ff, w.E, w.k, w.dtype)
    L = inp["logits"] if inp["logits"] is not None else None
    r = run_route(desc, L.cuda())
    return int(r["counts"].max().item()), r


def test_padded_routing_layout(cuda_lib):
    w = Workload("cap", 3000, 256, 16, 4, 128, "bf16", router=False, skew=True, seed=11)
    inp = make_inputs(w)
    C, rr = max_count(w, inp)
    desc = lib.make_desc(w.T, w.d, w.d_ff, w.E, w.k, "bf16", capacity=C + 5)
    rp = run_route(desc, inp["logits"].cuda())
    E, Cp = w.E, C + 5
    assert torch.equal(rp["counts"], rr["counts"])
    assert np.array_equal(npi(rp["offsets"]), np.arange(E + 1) * Cp)
    idx, off = npi(rr["topk_idx"]), npi(rr["offsets"])
    # slot = e*C + (the token's rank in e), the rank being the ragged slot minus offsets[e]
    assert np.array_equal(npi(rp["slot"]), idx * Cp + npi(rr["slot"]) - off[idx])
    rt = npi(rp["row_token"]).reshape(E, Cp)
    cnt = npi(rr["counts"])
    for e in range(E):
        assert np.array_equal(rt[e, :cnt[e]], npi(rr["row_token"])[off[e]:off[e + 1]])
        assert np.all(rt[e, cnt[e]:] == -1)


@pytest.mark.parametrize("T,d,E,k,f,dt,skew,router,shared", [
    (3000, 256, 16, 4, 128, "bf16", False, False, False),
    (3000, 256, 16, 4, 128, "bf16", True, False, False),
    (1500, 256, 8, 4, 128, "mxfp8", False, False, False),
    (333, 384, 12, 3, 192, "fp32", False, False, False),
    (1000, 256, 64, 4, 128, "bf16", False, True, True),
])
def test_padded_layer_is_bit_identical_to_ragged(cuda_lib, T, d, E, k, f, dt, skew, router,
                                                 shared):
    w = Workload("pad", T, d, E, k, f, dt, router=router, skew=skew, seed=T + 9, shared=shared)
    inp = make_inputs(w)
    _, lay0, _, y0, g0, st0 = run_layer(w, inp)
    C = int(lay0.views()["counts"].max().item())
    _, lay1, _, y1, g1, st1 = run_layer(w, inp, capacity=C)
    assert st0 == 0 and st1 == 0
    assert torch.equal(y0, y1)
    for name in ("dx", "d_logits", "dW13", "dW2") + (("dWr",) if router else ()):
        assert torch.equal(g0[name], g1[name]), name


@pytest.mark.parametrize("T,d,E,k,f,dt,skew,extra", [
    (3000, 256, 16, 4, 128, "bf16", False, 0),
    (3000, 256, 16, 4, 128, "bf16", True, 37),
    (2000, 256, 128, 4, 128, "bf16", False, 3),
    (333, 384, 12, 3, 192, "fp32", False, 11),
])
def test_padded_layer_matches_oracle(cuda_lib, T, d, E, k, f, dt, skew, extra):
    """The capacity-padded layout against the fp64 oracle, not only against the ragged
    layer: every expert owns C rows (deniz.in, "Yeni stack nasil calisiyor": padding
    every expert group to a common capacity), offsets are e*C, a token's slot is
    e*C + its rank among the expert's tokens, padding rows of x_perm are zero and
    marked row_token = -1, and the layer's outputs match the oracle's."""
    w = Workload("padx", T, d, E, k, f, dt, router=False, skew=skew, seed=T + 31)
    inp = make_inputs(w)
    C = max_count(w, inp)[0] + extra
    desc, layer, dv, y, g, status = run_layer(w, inp, capacity=C)
    assert status == 0
    v = layer.views()
    x, dy = f64(inp["x"]), f64(inp["dy"])
    W13, W2 = inp["W13"].float().numpy(), inp["W2"].float().numpy()
    fwd = oracle.layer_fwd(x, W13, W2, logits=f64(inp["logits"]), k=k)
    bwd = oracle.layer_bwd(fwd, dy, x, W13, W2)
    idx = fwd["topk_idx"].astype(np.int64)
    assert np.array_equal(npi(v["topk_idx"]), idx)
    assert np.array_equal(npi(v["counts"]), fwd["counts"])
    assert np.array_equal(npi(v["offsets"]), np.arange(E + 1) * C)
    rank = fwd["slot"] - fwd["offsets"][idx]
    assert np.array_equal(npi(v["slot"]), idx * C + rank)
    rt = npi(v["row_token"]).reshape(E, C)
    xp = f64(v["x_perm"]).reshape(E, C, d)
    # (fp32: x_perm holds x rounded to TF32, the precision the GEMMs read it in)
    xr = np.asarray(oracle.tf32_round(inp["x"].numpy()), dtype=np.float64) if dt == "fp32" else x
    for e in range(E):
        c = int(fwd["counts"][e])
        o = int(fwd["offsets"][e])
        assert np.array_equal(rt[e, :c], fwd["row_token"][o:o + c])
        assert np.all(rt[e, c:] == -1)
        assert np.array_equal(xp[e, :c], xr[fwd["row_token"][o:o + c]])
        assert np.all(xp[e, c:] == 0)
    assert rel(y, fwd["y"]) < TOL
    for name in ("dx", "d_logits", "dW13", "dW2"):
        assert rel(g[name], bwd[name]) < TOL, name


def test_capacity_below_the_largest_count_is_reported(cuda_lib):
    w = Workload("capx", 2000, 256, 16, 4, 128, "bf16", router=False, skew=True, seed=3)
    inp = make_inputs(w)
    C, _ = max_count(w, inp)
    desc, layer, dv, y, g, status = run_layer(w, inp, capacity=C - 1)
    assert status & lib.MOE_DEV_BAD_INDEX


# ------------------------------------------------------------------- CUDA graphs

def _graph_matches_eager(w, flags=0, capacity=0):
    """Capture fwd+bwd of the layer in one CUDA graph, replay it with new logits, and
    compare against an uncaptured run on the same inputs (bit-identical)."""
    inp = make_inputs(w)
    desc = lib.make_desc(w.T, w.d, w.d_ff, w.E, w.k, w.dtype, flags, capacity)
    if w.shared:
        desc.flags |= lib.MOE_FLAG_SHARED_EXPERT
    layer = lib.Layer(desc)
    dv = {k: (None if v is None else v.cuda()) for k, v in inp.items()}
    y = torch.empty(w.T, w.d, dtype=torch.bfloat16, device="cuda")
    out = dict(dx=torch.empty_like(y), d_logits=torch.empty(w.T, w.E, device="cuda"),
               dW13=torch.empty_like(dv["W13"]), dW2=torch.empty_like(dv["W2"]))
    run = lambda: (layer.fwd(dv["x"], dv["W13"], dv["W2"], logits=dv["logits"], y=y),  # noqa: E731
                   layer.bwd(dv["dy"], dv["W13"], dv["W2"], x=dv["x"], out=out))
    run()                                   # warm-up (kernel attributes, descriptor caches)
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        run()
    newL = random_logits(w.T, w.E, seed=w.seed + 1000)
    dv["logits"].copy_(newL)
    g.replay()
    torch.cuda.synchronize()
    got = {k: v.clone() for k, v in dict(out, y=y).items()}
    run()                                   # the same inputs, uncaptured
    torch.cuda.synchronize()
    for k, v in dict(out, y=y).items():
        assert torch.equal(got[k], v), k
    assert lib.moe_read_device_status(layer.ws) == 0


def test_mxfp8_layer_replays_in_a_cuda_graph(cuda_lib):
    _graph_matches_eager(Workload("gmx", 2000, 512, 16, 4, 256, "mxfp8", router=False,
                                  skew=False, seed=21))


def test_recompute_shared_padded_layer_replays_in_a_cuda_graph(cuda_lib):
    w = Workload("gall", 2000, 256, 16, 4, 128, "bf16", router=False, skew=True, seed=22,
                 shared=True)
    _graph_matches_eager(w, flags=lib.MOE_FLAG_RECOMPUTE, capacity=2000)
