"""Pins of where the oracle's MXFP8 layer quantises each grouped-GEMM operand.

The write-ups offer MXFP8 for selected operations (bigchange.ai pt-BR, opening section;
"Três números, três denominadores") and the workload fixes E4M3 elements with one E8M0
scale per 32-element block, BF16 in and out.  The oracle's reading: every block runs
along the contraction (K) of the GEMM that reads the operand --
    FC1 / FC2 forward   X, W13 / a, W2 along their rows (d / d_ff);
    FC2 dgrad           dY along its rows (d), W2 along its d rows (axis 0);
    FC1 dgrad           dH13 along its rows (2 d_ff), W13 along its 2 d_ff rows (axis 0);
    wgrads              dY, a, dH13, X along tokens, blocks restarting at the expert's
                        first row (an expert segment that starts mid-block does not
                        share a block with the previous expert).
The quantiser itself is pinned elsewhere (hand blocks, the E4M3 grid, torch's fp8 cast).
Here the question is only which axis and which block boundaries each operand gets.

Method.  Operands are built so that MX quantisation along the prescribed axis, with
the prescribed block boundaries, is exact (every value already lies on the block's
E4M3 grid: 3-bit mantissas and a dynamic range well inside one block's span), while
any other axis or boundary mixes values 2^18 apart in one block and rounds the small
ones.  Then the MX oracle must return exactly what the unquantised oracle returns
(1e-12 relative, summation order only), and each plausible mistake, planted in the
oracle one call site at a time (the axis of one operand flipped, or one wgrad
operand's blocks aligned to global rows instead of to its expert's first row), must
make them differ.  Intermediate GEMM operands (a, dA, dH13) are made exact through the
inputs: silu(H1) = H1 for H1 >= 256 in fp64, sigmoid(0) = 1/2, and weight matrices with
one power-of-two entry per contraction column.
"""
from contextlib import contextmanager

import numpy as np
import pytest

import oracle
import oracle.moe_oracle as om

BIG = 2.0 ** 18          # ratio that no MX block can span exactly (E4M3 covers ~2^17)
MANT = np.array([1.0, 1.25, 1.5, 1.75])
D, F = 64, 64            # d_model, d_ff: two 32-blocks along d, four along 2*d_ff
OFF = [0, 40, 40, 100]   # expert 0: 40 rows, expert 1 empty, expert 2 starts mid-block
R = OFF[-1]
E = len(OFF) - 1
SEG2_HI = 72             # expert 2's second block (relative to its first row) starts here

# _mx call sites per non-empty expert, in the order experts_fwd / experts_bwd make them
FWD_SITES = ["X", "W13", "a", "W2"]
BWD_SITES = ["dY_dgrad", "W2_dgrad", "dY_wgrad", "a_wgrad", "dH13_wgrad", "X_wgrad",
             "dH13_dgrad", "W13_dgrad"]


def _small(rng, shape):
    """Positive values with 3-bit mantissas over 2^-2 .. 2^2: exact in any MX block."""
    return rng.choice(MANT, size=shape) * 2.0 ** rng.integers(-2, 3, size=shape)


def _alternating(n):
    """1, BIG, 1, BIG, ... (one line in two 2^18 larger)."""
    return np.where(np.arange(n) % 2 == 0, 1.0, BIG)


def _row_structured_column(rng, n_rows, col, base):
    """`base` with column `col` BIG times larger on expert 2's second block of rows."""
    out = base.copy()
    out[SEG2_HI:OFF[3], col] *= BIG
    return out


def _exact_along(a, axis):
    return np.array_equal(oracle.mx_quantize_dequantize(a, axis=axis), a)


@contextmanager
def planted(sites, target, kind):
    """Plant one mistake in the oracle's quantisation: at call site `target`, either
    flip the axis (kind "axis") or align the blocks to global rows instead of to the
    expert's first row (kind "phase": the segment is quantised as if preceded by the
    rows that fill its first block up to a multiple of 32)."""
    real = om._mx
    starts = [OFF[e] for e in range(E) if OFF[e + 1] > OFF[e]]
    calls = [0]

    def fake(a, axis, mx):
        i = calls[0]
        calls[0] += 1
        e_i, s = divmod(i, len(sites))
        if mx and sites[s] == target:
            if kind == "axis":
                return real(a, 1 - axis, mx)
            phase = starts[e_i] % 32
            pad = np.zeros((phase,) + a.shape[1:])
            return real(np.concatenate([pad, a]), axis, mx)[phase:]
        return real(a, axis, mx)

    om._mx = fake
    try:
        yield calls
    finally:
        om._mx = real


def _close(a, b):
    return np.allclose(a, b, rtol=1e-12, atol=0.0)


# ------------------------------------------------------------------ forward

def fwd_inputs(seed=0):
    rng = np.random.default_rng(seed)
    s = _alternating(R)                               # row scales of x
    x = _small(rng, (R, D)) * s[:, None]
    x[:, 0] = s                                       # H1 = x[:,0] * W1[:,0] >= 256
    t = _alternating(F)                               # row scales of W1 (W3 the inverse)
    W13 = np.zeros((E, 2 * F, D))
    W2 = np.zeros((E, D, F))
    for e in range(E):
        W13[e, :F, 0] = 256.0 * t
        kj = rng.integers(1, D, size=F)               # W3 row j: one power of two at kj
        W13[e, F + np.arange(F), kj] = 2.0 ** rng.integers(-2, 3, size=F) / t
        W2[e] = _small(rng, (D, F)) * _alternating(D)[:, None]
    return x, W13, W2


def test_forward_inputs_separate_the_axes():
    x, W13, W2 = fwd_inputs()
    for e in range(E):
        assert _exact_along(W13[e], 1) and not _exact_along(W13[e], 0)
        assert _exact_along(W2[e], 1) and not _exact_along(W2[e], 0)
    assert _exact_along(x, 1) and not _exact_along(x, 0)
    H13, a, _ = oracle.experts_fwd(x, OFF, W13, W2)
    assert np.all(H13[:, :F] >= 256.0)                 # silu(H1) = H1 exactly
    assert _exact_along(a, 1) and not _exact_along(a, 0)


def test_mx_forward_quantises_along_each_gemms_k():
    x, W13, W2 = fwd_inputs()
    ref = oracle.experts_fwd(x, OFF, W13, W2, mx=False)
    got = oracle.experts_fwd(x, OFF, W13, W2, mx=True)
    for r, g in zip(ref, got):
        assert _close(g, r)


@pytest.mark.parametrize("site", FWD_SITES)
def test_mx_forward_catches_a_flipped_axis(site):
    x, W13, W2 = fwd_inputs()
    ref = oracle.experts_fwd(x, OFF, W13, W2, mx=False)
    with planted(FWD_SITES, site, "axis") as calls:
        got = oracle.experts_fwd(x, OFF, W13, W2, mx=True)
    assert calls[0] == len(FWD_SITES) * 2              # two non-empty experts
    assert not all(_close(g, r) for g, r in zip(got, ref))


# ------------------------------------------------------------------ backward, dgrads

def bwd_common(rng, w2_odd=1.0 / BIG, w13_odd=1.0 / BIG):
    """W2 with one power-of-two entry per column j (row j // 2) and W13 with one per
    column i (row i // 2, in the dH1 half): exact along their contraction axis 0; the
    `*_odd` factors on odd columns make their rows span 2^18 (inexact along axis 1)."""
    W2 = np.zeros((E, D, F))
    W13 = np.zeros((E, 2 * F, D))
    j = np.arange(F)
    i = np.arange(D)
    for e in range(E):
        W2[e, j // 2, j] = np.where(j % 2 == 0, 1.0, w2_odd)
        W13[e, i // 2, i] = np.where(i % 2 == 0, 1.0, w13_odd)
    return W2, W13


def dgrad_inputs(seed=1):
    rng = np.random.default_rng(seed)
    s = _alternating(R)
    dy = _small(rng, (R, D)) * s[:, None]             # rows exact, columns span 2^18
    W2, W13 = bwd_common(rng)
    # H1 = 0 (sigmoid = 1/2, silu = 0): dH1 = dA * H3 / 2, dH3 = 0; H3 undoes W2's
    # column factors so every dH13 row keeps its dY row's scale
    j = np.arange(F)
    w2col = np.where(j % 2 == 0, 1.0, 1.0 / BIG)
    H13 = np.zeros((R, 2 * F))
    H13[:, F:] = (2.0 ** rng.integers(-1, 2, size=(R, F))) / w2col
    x = _small(rng, (R, D))
    a = _small(rng, (R, F))
    return dy, x, H13, a, W13, W2


def test_dgrad_inputs_separate_the_axes():
    dy, x, H13, a, W13, W2 = dgrad_inputs()
    assert _exact_along(dy, 1) and not _exact_along(dy, 0)
    for e in range(E):
        assert _exact_along(W2[e], 0) and not _exact_along(W2[e], 1)
        assert _exact_along(W13[e], 0) and not _exact_along(W13[e], 1)
    dH13 = oracle.experts_bwd(dy, x, H13, a, OFF, W13, W2)[0]
    assert _exact_along(dH13, 1) and not _exact_along(dH13, 0)


def test_mx_dgrads_quantise_along_each_gemms_k():
    args = dgrad_inputs()
    ref = oracle.experts_bwd(*args[:4], OFF, *args[4:], mx=False)
    got = oracle.experts_bwd(*args[:4], OFF, *args[4:], mx=True)
    assert _close(got[0], ref[0])                      # dH13
    assert _close(got[1], ref[1])                      # dx_perm


@pytest.mark.parametrize("site", ["dY_dgrad", "W2_dgrad", "dH13_dgrad", "W13_dgrad"])
def test_mx_dgrads_catch_a_flipped_axis(site):
    args = dgrad_inputs()
    ref = oracle.experts_bwd(*args[:4], OFF, *args[4:], mx=False)
    with planted(BWD_SITES, site, "axis") as calls:
        got = oracle.experts_bwd(*args[:4], OFF, *args[4:], mx=True)
    assert calls[0] == len(BWD_SITES) * 2
    assert not (_close(got[0], ref[0]) and _close(got[1], ref[1]))


# ------------------------------------------------------------------ backward, wgrads

def wgrad2_inputs(seed=2):
    """FC2 wgrad: dY column 5 and a column 7 are 2^18 larger on expert 2's second
    32-row block: exact with blocks counted from the expert's first row (row 40),
    inexact with blocks at global multiples of 32 (block [64, 96) spans both)."""
    rng = np.random.default_rng(seed)
    dy = _row_structured_column(rng, R, 5, _small(rng, (R, D)))
    a = _row_structured_column(rng, R, 7, _small(rng, (R, F)))
    x = _small(rng, (R, D))
    W2, W13 = bwd_common(rng, 1.0, 1.0)
    H13 = np.zeros((R, 2 * F))
    H13[:, F:] = 1.0
    return dy, x, H13, a, W13, W2


def wgrad1_inputs(seed=3):
    """FC1 wgrad: dY exact both ways, so dH13 = [dA * H3 / 2, 0] is computed exactly; H3
    column 9 and x column 11 carry the same expert-2 block structure as above."""
    rng = np.random.default_rng(seed)
    dy = _small(rng, (R, D))
    x = _row_structured_column(rng, R, 11, _small(rng, (R, D)))
    a = _small(rng, (R, F))
    W2, W13 = bwd_common(rng, 1.0, 1.0)
    H13 = np.zeros((R, 2 * F))
    H13[:, F:] = 1.0
    H13[SEG2_HI:OFF[3], F + 9] = BIG
    return dy, x, H13, a, W13, W2


def _seg(a, e):
    return a[OFF[e]:OFF[e + 1]]


def test_wgrad_inputs_separate_block_boundaries():
    for make, names in ((wgrad2_inputs, ("dy", "a")), (wgrad1_inputs, ("x",))):
        dy, x, H13, a, W13, W2 = make()
        ops = dict(dy=dy, x=x, a=a)
        for n in names:
            op = ops[n]
            # expert 2's segment: exact with blocks from its own first row, not with
            # blocks at global row multiples of 32, nor along the rows
            seg = _seg(op, 2)
            phase = OFF[2] % 32
            glob = oracle.mx_quantize_dequantize(
                np.concatenate([np.zeros((phase, op.shape[1])), seg]), axis=0)[phase:]
            assert _exact_along(seg, 0) and not np.array_equal(glob, seg), n
            assert not _exact_along(seg, 1), n
    dH13 = oracle.experts_bwd(*wgrad1_inputs()[:4], OFF, *wgrad1_inputs()[4:])[0]
    assert _exact_along(_seg(dH13, 2), 0) and not _exact_along(_seg(dH13, 2), 1)


def test_mx_wgrads_quantise_along_tokens_from_each_experts_first_row():
    a2 = wgrad2_inputs()
    ref = oracle.experts_bwd(*a2[:4], OFF, *a2[4:], mx=False)
    got = oracle.experts_bwd(*a2[:4], OFF, *a2[4:], mx=True)
    assert _close(got[3], ref[3])                      # dW2
    a1 = wgrad1_inputs()
    ref = oracle.experts_bwd(*a1[:4], OFF, *a1[4:], mx=False)
    got = oracle.experts_bwd(*a1[:4], OFF, *a1[4:], mx=True)
    assert _close(got[2], ref[2])                      # dW13
    assert np.all(got[2][1] == 0) and np.all(got[3][1] == 0)   # the empty expert


@pytest.mark.parametrize("site,kind", [("dY_wgrad", "axis"), ("a_wgrad", "axis"),
                                       ("dY_wgrad", "phase"), ("a_wgrad", "phase")])
def test_mx_fc2_wgrad_catches_misplaced_blocks(site, kind):
    args = wgrad2_inputs()
    ref = oracle.experts_bwd(*args[:4], OFF, *args[4:], mx=False)
    with planted(BWD_SITES, site, kind):
        got = oracle.experts_bwd(*args[:4], OFF, *args[4:], mx=True)
    assert not _close(got[3][2], ref[3][2])


@pytest.mark.parametrize("site,kind", [("dH13_wgrad", "axis"), ("X_wgrad", "axis"),
                                       ("dH13_wgrad", "phase"), ("X_wgrad", "phase")])
def test_mx_fc1_wgrad_catches_misplaced_blocks(site, kind):
    args = wgrad1_inputs()
    ref = oracle.experts_bwd(*args[:4], OFF, *args[4:], mx=False)
    with planted(BWD_SITES, site, kind):
        got = oracle.experts_bwd(*args[:4], OFF, *args[4:], mx=True)
    assert not _close(got[2][2], ref[2][2])
