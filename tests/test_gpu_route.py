"""GPU routing (top-k, gates, counts, offsets, slots) against the oracle: indices,
counts, offsets and the permutation bit-exact; gates to fp32 rounding."""
import numpy as np
import pytest
import torch

import oracle
from routing_grouped_gemm_route_b200 import lib
from routing_grouped_gemm_route_b200.inputs import random_logits

from helpers import assert_route_equal, run_route

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("T,E,k,skew", [
    (1, 1, 1, False), (1, 8, 2, False), (255, 8, 2, False), (257, 8, 2, False),
    (512, 8, 2, False), (1000, 37, 3, False), (4096, 128, 4, False), (8192, 8, 4, False),
    (16384, 128, 4, False), (16384, 128, 4, True), (513, 64, 32, False), (700, 1024, 8, False),
    (300, 5, 5, False), (2049, 33, 32, False), (32768, 128, 8, False)])
def test_route_matches_oracle(cuda_lib, T, E, k, skew):
    L = random_logits(T, E, seed=T + E + k, skew=skew)
    desc = lib.make_desc(T, 128, 64, E, k, "bf16")
    gpu = run_route(desc, L.cuda())
    ref = oracle.route(L.numpy(), k, E)
    assert_route_equal(gpu, ref, k)


@pytest.mark.parametrize("E,k", [(8, 2), (128, 4), (40, 7)])
def test_route_ties_break_to_lower_index(cuda_lib, E, k):
    # logits on a coarse grid: many exact ties, including across the k-th position
    T = 3000
    L = torch.round(random_logits(T, E, seed=99) * 2.0) / 2.0
    L[:17] = 0.0                                      # whole rows equal
    L[17:40, ::2] = 1.0                               # half the experts tied at the top
    desc = lib.make_desc(T, 128, 64, E, k, "bf16")
    gpu = run_route(desc, L.cuda())
    ref = oracle.route(L.numpy(), k, E)
    assert_route_equal(gpu, ref, k)
    assert np.array_equal(ref["topk_idx"][0], np.arange(k))


def test_all_tokens_to_one_expert(cuda_lib):
    T, E, k = 5000, 16, 1
    L = random_logits(T, E, seed=3)
    L[:, 11] += 100.0
    desc = lib.make_desc(T, 128, 64, E, k, "bf16")
    gpu = run_route(desc, L.cuda())
    ref = oracle.route(L.numpy(), k, E)
    assert_route_equal(gpu, ref, k)
    assert ref["counts"][11] == T


def test_route_replays_in_a_cuda_graph_with_new_logits(cuda_lib):
    """No host round trip: the routing captures in a CUDA graph and replays correctly
    for logits written after capture."""
    T, E, k = 4096, 128, 4
    desc = lib.make_desc(T, 128, 64, E, k, "bf16")
    logits = random_logits(T, E, seed=1).cuda()
    outs = dict(topk_idx=torch.empty(T, k, dtype=torch.int32, device="cuda"),
                gates=torch.empty(T, k, dtype=torch.float32, device="cuda"),
                counts=torch.empty(E, dtype=torch.int32, device="cuda"),
                offsets=torch.empty(E + 1, dtype=torch.int32, device="cuda"),
                slot=torch.empty(T, k, dtype=torch.int32, device="cuda"),
                row_token=torch.empty(T * k, dtype=torch.int32, device="cuda"),
                row_gate=torch.empty(T * k, dtype=torch.float32, device="cuda"))
    ws = lib.alloc_workspace(desc)
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        lib.moe_route(desc, logits, outs["topk_idx"], outs["gates"], outs["counts"],
                      outs["offsets"], outs["slot"], outs["row_token"], outs["row_gate"], ws)
    for seed in (5, 6):
        Lh = random_logits(T, E, seed=seed)
        logits.copy_(Lh)
        g.replay()
        torch.cuda.synchronize()
        assert_route_equal(outs, oracle.route(Lh.numpy(), k, E), k)


@pytest.mark.parametrize("E,k", [(40, 7), (128, 4)])
def test_nan_logits_rank_as_minus_infinity(cuda_lib, E, k):
    """A NaN logit ranks as -inf: every token still gets k distinct experts in range,
    and the routing equals the oracle's on the logits with NaN replaced by -inf (the
    reading the library documents; a row of NaNs gets NaN gates)."""
    T = 3000
    L = random_logits(T, E, seed=E + k)
    g = torch.Generator().manual_seed(1)
    L[0] = float("nan")                                        # a whole row
    L[1:200][torch.rand(199, E, generator=g) < 0.3] = float("nan")
    L[200:260, :k + 1] = float("nan")                          # NaN where the top would be
    desc = lib.make_desc(T, 128, 64, E, k, "bf16")
    gpu = run_route(desc, L.cuda())
    Lr = L.clone()
    Lr[torch.isnan(Lr)] = float("-inf")
    ref = oracle.route(Lr.numpy(), k, E)
    idx = gpu["topk_idx"].cpu().numpy()
    assert idx.min() >= 0 and idx.max() < E
    assert all(len(set(r)) == k for r in idx.tolist())
    for name in ("topk_idx", "counts", "offsets", "slot", "row_token"):
        assert np.array_equal(gpu[name].cpu().numpy().astype(np.int64),
                              np.asarray(ref[name]).reshape(gpu[name].shape)), name
    gg = gpu["gates"].cpu().double().numpy()
    assert np.array_equal(np.isnan(gg), np.isnan(ref["gates"]))
    fin = ~np.isnan(ref["gates"])
    assert np.max(np.abs(gg[fin] - ref["gates"][fin])) < 2e-6
