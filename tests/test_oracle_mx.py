"""Pins of the oracle's MXFP8 quantiser: hand-computed blocks, the E4M3 grid, torch's fp8 cast."""
import numpy as np
import pytest
import torch

import oracle
from oracle import mx


def test_unit_block():
    # amax = 1 -> s = 0 - 8 = -8 (byte 119); 1 * 2**8 = 256 = 2**8 * 1.0 -> E=15, m=0 -> 0x78
    codes, sb, deq = oracle.mx_quantize(np.ones(32))
    assert sb.tolist() == [119]
    assert np.all(codes == 0x78)
    assert np.all(deq == 1.0)


def test_powers_of_two_round_trip():
    vals = 2.0 ** np.arange(-8, 0)                    # 2**-8 .. 2**-1, amax 0.5 -> s = -9
    x = np.concatenate([vals, -vals, vals, -vals])
    codes, sb, deq = oracle.mx_quantize(x)
    assert sb.tolist() == [127 - 9 - 1 + 1]           # byte = s + 127 = 118
    assert np.array_equal(deq, x)


def test_saturation():
    # amax = 1.9 -> s = -8; 1.9 * 256 = 486.4 > 448 -> saturates to 448 -> 1.75
    x = np.zeros(32)
    x[0] = 1.9
    x[1] = -1.9
    codes, sb, deq = oracle.mx_quantize(x)
    assert deq[0] == 1.75 and deq[1] == -1.75
    assert codes[0] == 0x7E and codes[1] == 0xFE


def test_all_zero_block_and_signed_zero():
    x = np.zeros(64)
    x[40] = -0.0
    codes, sb, deq = oracle.mx_quantize(x)
    assert sb.tolist() == [0, 0]
    assert np.all(codes[:40] == 0) and codes[40] == 0x80
    assert np.all(deq == 0.0)


def test_ties_round_to_even():
    x = np.zeros(32)
    x[0] = 1.0                                          # fixes s = -8
    x[1] = 1.0625 / 256                                 # 1.0625 halfway 1.0|1.125 -> 1.0
    x[2] = 1.1875 / 256                                 # halfway 1.125|1.25 -> 1.25
    x[3] = 2.0 ** -10 / 256                             # halfway 0|2**-9 -> 0
    x[4] = 3 * 2.0 ** -10 / 256                         # halfway 2**-9|2**-8 -> 2**-8 (even)
    deq = oracle.mx_quantize(x)[2] * 256
    assert deq[1] == 1.0 and deq[2] == 1.25 and deq[3] == 0.0 and deq[4] == 2.0 ** -8


def test_e4m3_grid():
    codes = np.arange(256, dtype=np.uint8)
    v = mx.e4m3_decode(codes)
    finite = ~np.isnan(v)
    assert finite.sum() == 254                          # 0x7F and 0xFF are NaN
    pos = np.sort(v[(codes < 0x80) & finite])
    assert pos[0] == 0.0 and pos[1] == 2.0 ** -9 and pos[-1] == 448.0
    assert np.all(np.diff(pos) > 0) and len(pos) == 127
    # every finite code is a fixed point of round and re-encodes to itself
    c = codes[finite]
    assert np.array_equal(mx.e4m3_round(v[finite]), v[finite])
    assert np.array_equal(mx.e4m3_encode(v[finite]), c)


def test_e4m3_round_matches_torch_float8_cast():
    # torch's float8_e4m3fn cast rounds to nearest even; inside +-448 it needs no saturation
    rng = np.random.default_rng(0)
    v = np.concatenate([rng.standard_normal(20000) * s for s in (1e-3, 0.05, 1.0, 30.0, 150.0)])
    v = np.clip(v, -448, 448).astype(np.float32).astype(np.float64)
    ref = torch.tensor(v, dtype=torch.float32).to(torch.float8_e4m3fn).to(torch.float64).numpy()
    assert np.array_equal(mx.e4m3_round(v), ref)
    bits = torch.tensor(v, dtype=torch.float32).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    assert np.array_equal(mx.e4m3_encode(mx.e4m3_round(v)), bits)


@pytest.mark.parametrize("n", [32, 33, 95])
def test_partial_block_and_axis(n):
    rng = np.random.default_rng(n)
    x = rng.standard_normal((3, n))
    c1, s1, d1 = oracle.mx_quantize(x, axis=1)
    c0, s0, d0 = oracle.mx_quantize(x.T.copy(), axis=0)
    assert s1.shape == (3, -(-n // 32))
    assert np.array_equal(c1, c0.T) and np.array_equal(s1, s0.T) and np.array_equal(d1, d0.T)
    # the last partial block takes its own amax
    tail = x[:, (n // 32) * 32:]
    if tail.shape[1]:
        amax = np.abs(tail).max(axis=1)
        assert np.array_equal(s1[:, -1].astype(int) - 127, np.floor(np.log2(amax)).astype(int) - 8)
    # per element, by region of v = x / 2**s: saturated to 448 above 448; within E4M3's
    # half-ulp (2**-4 relative) in the normal range; within half the subnormal step below
    s = (s1.astype(np.int64) - 127).repeat(32, axis=1)[:, :n]
    v = np.ldexp(x, -s)
    dv = np.ldexp(d1, -s)
    sat = np.abs(v) > 448
    nrm = ~sat & (np.abs(v) >= 2.0 ** -6)
    sub = ~sat & ~nrm
    assert np.all(dv[sat] == np.sign(v[sat]) * 448)
    assert np.all(np.abs(dv - v)[nrm] <= 2.0 ** -4 * np.abs(v)[nrm])
    assert np.all(np.abs(dv - v)[sub] <= 2.0 ** -10)


# ---------------------------------------------------------------- bf16 rounding (BF16 I/O)

def test_bf16_round_hand_cases():
    r = oracle.bf16_round
    # bf16 spacing at 1 is 2**-7: 1 + 2**-8 is a tie -> even (1.0); 1 + 3*2**-8 -> 1 + 2**-6
    assert r(1.0 + 2.0 ** -8) == 1.0
    assert r(1.0 + 3 * 2.0 ** -8) == 1.0 + 2.0 ** -6
    assert r(-(1.0 + 3 * 2.0 ** -8)) == -(1.0 + 2.0 ** -6)
    # just above the tie rounds up even where an fp32 intermediate would land on the tie
    assert r(1.0 + 2.0 ** -8 + 2.0 ** -40) == 1.0 + 2.0 ** -7
    assert r(3.0) == 3.0 and r(0.0) == 0.0 and np.signbit(r(-0.0))
    # smallest subnormal 2**-133; half of it is a tie -> 0
    assert r(2.0 ** -133) == 2.0 ** -133
    assert r(2.0 ** -134) == 0.0
    assert r(1.5 * 2.0 ** -133) == 2.0 ** -132
    # largest finite 2**128 - 2**120; the tie above it overflows
    assert r(2.0 ** 128 - 2.0 ** 120) == 2.0 ** 128 - 2.0 ** 120
    assert np.isinf(r(2.0 ** 128 - 2.0 ** 119))


def test_bf16_round_matches_torch_cast_of_fp32():
    # values exact in fp32, so torch's fp32 -> bf16 cast is one rounding of the same number
    g = np.random.default_rng(5)
    v = (g.standard_normal(200000) * np.exp(g.uniform(-95, 85, 200000))).astype(np.float32)
    v[:50] = np.float32(1.0) + np.float32(2.0 ** -8) * np.arange(50, dtype=np.float32)   # ties
    want = torch.from_numpy(v).to(torch.bfloat16).double().numpy()
    got = oracle.bf16_round(v.astype(np.float64))
    assert np.array_equal(got, want)
    # idempotent
    assert np.array_equal(oracle.bf16_round(got), got)


def test_mx_operand_of_layer_oracle_is_bf16_rounded():
    # a layer whose activation "a" is not bf16-representable: the MX oracle quantises
    # bf16(a), so its output equals the one computed from bf16-rounded a
    from oracle.moe_oracle import _mx
    g = np.random.default_rng(1)
    a = g.standard_normal((64, 128))
    assert np.array_equal(_mx(a, 1, True), mx.mx_quantize_dequantize(oracle.bf16_round(a), axis=1))
    assert _mx(a, 1, False) is a


def test_tf32_round_hand_values():
    # TF32 keeps 10 mantissa bits: the spacing at 1 is 2**-10, ties go away from zero
    # subnormals keep 10 bits too: 2**-136 is the smallest TF32 step, 2**-137 a tie that
    # goes to it, 2**-140 below half of it goes to 0
    x = np.array([1 + 2.0 ** -11, 1 + 2.0 ** -12, 1 + 3 * 2.0 ** -11, -(1 + 2.0 ** -11),
                  1 + 2.0 ** -10, 3.0, 2.0 ** -136, 2.0 ** -137, 2.0 ** -140, 0.0, -0.0],
                 dtype=np.float32)
    want = np.array([1 + 2.0 ** -10, 1.0, 1 + 2.0 ** -9, -(1 + 2.0 ** -10),
                     1 + 2.0 ** -10, 3.0, 2.0 ** -136, 2.0 ** -136, 0.0, 0.0, -0.0],
                    dtype=np.float32)
    got = oracle.tf32_round(x)
    assert np.array_equal(got.view(np.uint32), want.view(np.uint32))


def test_tf32_round_properties():
    rng = np.random.default_rng(3)
    x = (rng.standard_normal(100000) * 10.0 ** rng.integers(-8, 8, 100000)).astype(np.float32)
    r = oracle.tf32_round(x)
    assert np.all((r.view(np.uint32) & 0x1FFF) == 0)            # 10 mantissa bits left
    assert np.array_equal(oracle.tf32_round(r), r)               # idempotent
    assert np.array_equal(np.signbit(r), np.signbit(x))
    # nearest: within half a TF32 spacing (2**(e-10) in the binade of |x|)
    _, e = np.frexp(x.astype(np.float64))
    half = np.ldexp(1.0, e - 12)
    assert np.all(np.abs(r.astype(np.float64) - x.astype(np.float64)) <= half)
    # unbiased on random data, unlike dropping the 13 bits (which always shrinks |x|)
    rel = (r.astype(np.float64) - x) / x
    assert abs(rel.mean()) < 2e-6
    trunc = (x.view(np.uint32) & np.uint32(0xFFFFE000)).view(np.float32)
    assert ((trunc.astype(np.float64) - x) / x).mean() < -1e-4
