"""MX (microscaling) FP8 quantiser of the oracle -- TEST INFRASTRUCTURE ONLY.

The Olmo-core 3 write-ups offer MXFP8 "for selected operations"
(bigchange.ai pt-BR, opening section; "Três números, três denominadores") and name no
block or scale rule.  This oracle follows the OCP Microscaling Formats (MX) v1.0
definition for MXFP8 with E4M3 elements:

  * blocks of 32 consecutive elements along the quantised axis (a last partial block
    takes its amax over the elements it has);
  * one shared E8M0 scale per block, X = 2**s with
        s = floor(log2(amax)) - 8      (8 = exponent of E4M3's largest normal, 448)
    clamped to [-127, 127]; stored as the byte s + 127 (0xFF, NaN, is never produced);
    an all-zero block gets s = -127 (byte 0);
  * each element is v / X rounded to the nearest E4M3 value, ties to even, with
    results above 448 in magnitude saturated to +-448.  The sign of zero is kept.

E4M3 ("FN" variant): 1 sign bit, 4 exponent bits with bias 7, 3 mantissa bits;
normals 2**(E-7) * (1 + m/8) for E in 1..15 (E=15, m=7 is NaN, so the largest
normal is 448); subnormals 2**-6 * m/8.

The MXFP8 workload keeps BF16 inputs and outputs around its block-scaled GEMMs ("fp32
accumulate, BF16 I/O"), so the tensor a quantiser sees is a BF16 tensor: ``bf16_round``
gives that rounding (IEEE round to nearest even, 8 significant bits) for the layer
oracle to apply before quantising an operand.
"""
from __future__ import annotations

import numpy as np

BLOCK = 32
E4M3_MAX = 448.0
E4M3_EMAX = 8
E4M3_EMIN = -6


def bf16_round(v) -> np.ndarray:
    """fp64 values rounded once to the nearest bfloat16 value (ties to even).

    bfloat16 has 8 significant bits and the exponent range of fp32: the spacing of
    values in the binade [2**(e-1), 2**e) is 2**(e-8), down to 2**-133 for the
    subnormals below 2**-126.  Magnitudes that round above the largest finite value
    (2**128 - 2**120) become infinite.
    """
    v = np.asarray(v, dtype=np.float64)
    _, ex = np.frexp(v)
    spacing = np.ldexp(1.0, np.maximum(ex, -125) - 8)
    r = np.rint(v / spacing) * spacing          # np.rint rounds halves to even
    big = np.abs(r) > np.ldexp(255.0, 120)
    return np.where(big, np.copysign(np.inf, v), r)


def tf32_round(v) -> np.ndarray:
    """fp32 values rounded to the nearest TF32 value, ties away from zero (fp32 result).

    TF32 keeps fp32's sign and 8 exponent bits and 10 of its 23 mantissa bits: the value
    is the fp32 bit pattern with the low 13 bits cleared after adding half of their
    range to the magnitude.  This is the precision the fp32 layer's tensor-core GEMMs
    read their operands in; the layer rounds each operand once where it is produced.
    """
    a = np.asarray(v, dtype=np.float32)
    bits = a.view(np.uint32)
    mag = bits & np.uint32(0x7FFFFFFF)
    sign = bits & np.uint32(0x80000000)
    finite = mag < np.uint32(0x7F800000)
    rounded = (mag + np.uint32(0x1000)) & np.uint32(0xFFFFE000)
    out = np.where(finite, sign | rounded, bits).astype(np.uint32)
    return out.view(np.float32)


def _floor_log2(a: np.ndarray) -> np.ndarray:
    """floor(log2(a)) for a > 0, exact (from the binary exponent)."""
    _, ex = np.frexp(a)
    return ex.astype(np.int64) - 1


def e4m3_round(v: np.ndarray) -> np.ndarray:
    """Round fp64 values to the nearest E4M3 value (ties to even), saturating to +-448."""
    v = np.asarray(v, dtype=np.float64)
    a = np.abs(v)
    out = np.zeros_like(a)
    nz = a > 0
    e = np.maximum(_floor_log2(np.where(nz, a, 1.0)), E4M3_EMIN)
    # quantum of the binade is 2**(e-3); a / quantum is exact (power-of-two scaling)
    n = np.ldexp(a, (3 - e).astype(np.int64))
    r = np.rint(n)                       # round half to even
    q = np.ldexp(r, (e - 3).astype(np.int64))
    q = np.minimum(q, E4M3_MAX)
    out = np.where(nz, q, 0.0)
    return np.copysign(out, v)


def e4m3_encode(q: np.ndarray) -> np.ndarray:
    """Bit pattern (uint8) of values that are already on the E4M3 grid."""
    q = np.asarray(q, dtype=np.float64)
    sign = np.signbit(q).astype(np.uint8) << 7
    a = np.abs(q)
    code = np.zeros(a.shape, dtype=np.int64)
    sub = (a > 0) & (a < 2.0 ** E4M3_EMIN)
    code = np.where(sub, np.rint(np.ldexp(a, 9)).astype(np.int64), code)
    nrm = a >= 2.0 ** E4M3_EMIN
    e = _floor_log2(np.where(nrm, a, 1.0))
    m = np.rint(np.ldexp(a, (3 - e).astype(np.int64)) - 8.0).astype(np.int64)
    code = np.where(nrm, ((e + 7) << 3) | m, code)
    return (code.astype(np.uint8) | sign).astype(np.uint8)


def e4m3_decode(codes: np.ndarray) -> np.ndarray:
    """Value of E4M3 bit patterns (NaN pattern 0x7F/0xFF decodes to NaN)."""
    c = np.asarray(codes, dtype=np.int64)
    s = np.where(c & 0x80, -1.0, 1.0)
    E = (c >> 3) & 0xF
    m = c & 0x7
    val = np.where(E == 0, np.ldexp(m.astype(np.float64), -9),
                   np.ldexp(1.0 + m / 8.0, (E - 7).astype(np.int64)))
    val = np.where((E == 15) & (m == 7), np.nan, val)
    return s * val


def _blocks_last(a: np.ndarray):
    n = a.shape[-1]
    nb = -(-n // BLOCK)
    pad = nb * BLOCK - n
    if pad:
        a = np.concatenate([a, np.zeros(a.shape[:-1] + (pad,), dtype=a.dtype)], axis=-1)
    return a.reshape(a.shape[:-1] + (nb, BLOCK)), n


def mx_quantize(x, axis: int = -1):
    """MXFP8 (E4M3 + E8M0 per 32) quantisation of ``x`` along ``axis``.

    Returns (codes uint8 with x's shape, scale bytes uint8 whose ``axis`` extent is
    ceil(n/32), element values fp64 before scaling back).
    """
    x = np.asarray(x, dtype=np.float64)
    xm = np.moveaxis(x, axis, -1)
    blk, n = _blocks_last(xm)
    amax = np.abs(blk).max(axis=-1)
    s = np.where(amax > 0, _floor_log2(np.where(amax > 0, amax, 1.0)) - E4M3_EMAX, -127)
    s = np.clip(s, -127, 127).astype(np.int64)
    v = np.ldexp(blk, -s[..., None])
    q = e4m3_round(v)
    codes = e4m3_encode(q).reshape(blk.shape[:-2] + (-1,))[..., :n]
    deq = np.ldexp(q, s[..., None]).reshape(blk.shape[:-2] + (-1,))[..., :n]
    sbytes = (s + 127).astype(np.uint8)
    return (np.moveaxis(codes, -1, axis), np.moveaxis(sbytes, -1, axis),
            np.moveaxis(deq, -1, axis))


def mx_quantize_dequantize(x, axis: int = -1) -> np.ndarray:
    """x rounded through MXFP8 along ``axis`` (fp64 result)."""
    return mx_quantize(x, axis)[2]
