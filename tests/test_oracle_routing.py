"""Pins of the oracle's routing: brute force, closed forms, invariants, library softmax."""
import math

import numpy as np
import pytest
import torch

import oracle
from routing_grouped_gemm_route_b200.inputs import random_logits


def brute_route(L, k):
    """Per-token python loops: order experts by (-logit, index), keep k, softmax over kept."""
    T, E = len(L), len(L[0])
    idx, gates = [], []
    for t in range(T):
        sel = sorted(range(E), key=lambda e: (-float(L[t][e]), e))[:k]
        m = max(float(L[t][e]) for e in sel)
        z = [math.exp(float(L[t][e]) - m) for e in sel]
        s = sum(z)
        idx.append(sel)
        gates.append([v / s for v in z])
    counts = [0] * E
    for t in range(T):
        for e in idx[t]:
            counts[e] += 1
    offsets = [0]
    for c in counts:
        offsets.append(offsets[-1] + c)
    seen = [0] * E
    slot = [[0] * k for _ in range(T)]
    for t in range(T):                      # tokens in order: an expert's rows are in token order
        for j, e in enumerate(idx[t]):
            slot[t][j] = offsets[e] + seen[e]
            seen[e] += 1
    return idx, gates, counts, offsets, slot


@pytest.mark.parametrize("T,E,k,seed", [(1, 1, 1, 0), (7, 5, 2, 1), (33, 8, 2, 2), (64, 16, 4, 3),
                                        (40, 6, 6, 4), (50, 37, 3, 5)])
def test_route_matches_brute_force(T, E, k, seed):
    L = random_logits(T, E, seed).numpy()
    r = oracle.route(L, k, E)
    idx, gates, counts, offsets, slot = brute_route(L.tolist(), k)
    assert np.array_equal(r["topk_idx"], np.array(idx))
    assert np.allclose(r["gates"], np.array(gates), rtol=1e-14, atol=0)
    assert np.array_equal(r["counts"], counts)
    assert np.array_equal(r["offsets"], offsets)
    assert np.array_equal(r["slot"], np.array(slot))


def test_route_ties_choose_lower_index():
    # every logit equal: experts 0..k-1 in order, uniform gates
    L = np.zeros((3, 6), dtype=np.float32)
    r = oracle.route(L, 4, 6)
    assert np.array_equal(r["topk_idx"], np.tile(np.arange(4), (3, 1)))
    assert np.allclose(r["gates"], 0.25, rtol=0, atol=1e-16)
    # a tie across the k boundary: logits [1, 3, 1, 3, 0] top-3 -> 1, 3, 0
    L = np.array([[1, 3, 1, 3, 0]], dtype=np.float32)
    r = oracle.route(L, 3, 5)
    assert r["topk_idx"].tolist() == [[1, 3, 0]]
    # +0 and -0 are equal logits: the lower index wins
    L = np.array([[-0.0, 0.0, -1.0]], dtype=np.float32)
    assert oracle.route(L, 1, 3)["topk_idx"].tolist() == [[0]]


def test_route_closed_form_two_of_three():
    # L = [1, 2, 0], k = 2: experts [1, 0]; gates are sigmoid(+-1)
    r = oracle.route(np.array([[1.0, 2.0, 0.0]], dtype=np.float32), 2, 3)
    assert r["topk_idx"].tolist() == [[1, 0]]
    s = 1.0 / (1.0 + math.exp(-1.0))
    assert np.allclose(r["gates"], [[s, 1.0 - s]], rtol=1e-15, atol=0)
    assert r["counts"].tolist() == [1, 1, 0]
    assert r["offsets"].tolist() == [0, 1, 2, 2]
    assert r["slot"].tolist() == [[1, 0]]
    assert r["row_token"].tolist() == [0, 0]


def test_k_equals_E_is_full_softmax():
    L = random_logits(20, 7, 11).double()
    r = oracle.route(L.numpy(), 7, 7)
    ref = torch.softmax(L, dim=1).numpy()
    got = np.zeros_like(ref)
    np.put_along_axis(got, r["topk_idx"].astype(np.int64), r["gates"], axis=1)
    assert np.allclose(got, ref, rtol=1e-13, atol=1e-16)
    assert np.array_equal(r["counts"], np.full(7, 20))


def test_k1_gates_are_one():
    L = random_logits(50, 9, 12).numpy()
    r = oracle.route(L, 1, 9)
    assert np.array_equal(r["gates"], np.ones((50, 1)))
    assert np.array_equal(r["topk_idx"][:, 0], np.argmax(L, axis=1))


@pytest.mark.parametrize("T,E,k,skew", [(512, 8, 2, False), (2048, 128, 4, False),
                                        (2048, 128, 4, True), (999, 13, 5, False)])
def test_route_invariants(T, E, k, skew):
    L = random_logits(T, E, 5, skew=skew).numpy()
    r = oracle.route(L, k, E)
    R = T * k
    idx, slot, off = r["topk_idx"], r["slot"], r["offsets"]
    assert r["counts"].sum() == R
    assert off[0] == 0 and off[-1] == R and np.all(np.diff(off) == r["counts"])
    assert np.allclose(r["gates"].sum(axis=1), 1.0, rtol=0, atol=1e-14)
    assert np.all(r["gates"] > 0)
    assert all(len(set(row)) == k for row in idx.tolist())            # distinct experts
    assert np.array_equal(np.sort(slot.ravel()), np.arange(R))       # bijection onto [0, R)
    assert np.array_equal(r["row_token"][slot], np.repeat(np.arange(T)[:, None], k, 1))
    assert np.array_equal(r["row_gate"][slot], r["gates"])
    for e in range(E):                                                 # rows in [off_e, off_e+1)
        rows = slot[idx == e]
        assert np.all((rows >= off[e]) & (rows < off[e + 1]))
        toks = r["row_token"][off[e]:off[e + 1]]
        assert np.all(np.diff(toks) > 0)                               # token order inside an expert
    # gates are non-increasing along j (logits listed in descending order)
    assert np.all(np.diff(r["gates"], axis=1) <= 0)


def test_skewed_routing_is_imbalanced():
    # the Zipf bias leaves experts empty and one expert far above the mean
    L = random_logits(16384, 128, 0, skew=True).numpy()
    c = oracle.route(L, 4, 128)["counts"]
    assert (c == 0).sum() >= 40
    assert c.max() > 10 * c.mean()


# ------------------------------------------------------------------- load statistics

def test_load_stats_hand_example():
    # mean 3; deviations -3, -1, 1, 3 -> mean square 5
    st = oracle.load_stats([0, 2, 4, 6])
    assert (st["total"], st["max_count"], st["min_count"], st["num_empty"]) == (12, 6, 0, 1)
    assert st["mean"] == 3.0 and st["max_over_mean"] == 2.0
    assert abs(st["cv"] - np.sqrt(5.0) / 3.0) < 1e-15


def test_load_stats_balanced_and_one_hot():
    st = oracle.load_stats([7] * 8)
    assert st["max_over_mean"] == 1.0 and st["cv"] == 0.0 and st["num_empty"] == 0
    # everything on one of E experts: max/mean = E, E-1 empty, cv = sqrt(E-1)
    st = oracle.load_stats([0] * 7 + [40])
    assert st["max_over_mean"] == 8.0 and st["num_empty"] == 7
    assert abs(st["cv"] - np.sqrt(7.0)) < 1e-14


def test_load_stats_no_tokens():
    st = oracle.load_stats([0, 0, 0])
    assert st["total"] == 0 and st["num_empty"] == 3
    assert st["max_over_mean"] == 0.0 and st["cv"] == 0.0


def test_route_matches_brute_force_with_many_ties():
    """Random small routings whose logits come from a 4-value set, so most tokens have
    tied logits at the top-k boundary: the oracle must still equal the brute-force
    reading (ties to the lower expert index) in every output."""
    from hypothesis import given, settings, strategies as st

    @settings(max_examples=80, deadline=None)
    @given(st.data())
    def check(data):
        T = data.draw(st.integers(1, 12))
        E = data.draw(st.integers(1, 10))
        k = data.draw(st.integers(1, E))
        vals = data.draw(st.lists(st.lists(st.sampled_from([-1.0, 0.0, 0.5, 1.0]),
                                           min_size=E, max_size=E), min_size=T, max_size=T))
        L = np.array(vals, dtype=np.float32)
        r = oracle.route(L, k, E)
        idx, gates, counts, offsets, slot = brute_route(L.tolist(), k)
        assert np.array_equal(r["topk_idx"], np.array(idx))
        assert np.allclose(r["gates"], np.array(gates), rtol=1e-14, atol=0)
        assert np.array_equal(r["counts"], counts)
        assert np.array_equal(r["offsets"], offsets)
        assert np.array_equal(r["slot"], np.array(slot))

    check()
