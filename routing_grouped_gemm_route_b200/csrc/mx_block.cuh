// The MX (microscaling) block rule shared by the standalone quantiser and the GEMM
// epilogues that quantise their own bf16 outputs: OCP MX v1.0, E4M3 elements with one
// E8M0 scale per 32 (the write-ups offer MXFP8 and give no rule of their own:
// bigchange.ai pt-BR, opening section).  Per block, s = floor(log2(amax)) - 8 clamped to
// [-127, 127] (-127 for an all-zero block), stored as the byte s + 127; each element is
// x / 2^s rounded to nearest-even E4M3, saturated to +-448.
#pragma once

#include <cuda_bf16.h>
#include <cuda_fp8.h>
#include <stdint.h>

namespace moe {
namespace mxb {

// Shared exponent of a block whose largest magnitude has the bf16 bit pattern `b`
// (sign cleared).  For a normal value with exponent field E, floor(log2) = E - 127, so
// s = E - 135; anything at or below 2^-119 (E <= 8, subnormals and zero) clamps to -127.
// Non-finite blocks: infinity gives 127, NaN -127.
__device__ __forceinline__ int exponent_bits(uint32_t b) {
  const int e = static_cast<int>((b >> 7) & 0xffu);
  if (e == 0xff) return (b & 0x7fu) ? -127 : 127;
  return (e < 8 ? 8 : e) - 135;
}
// 2^-s as a float, exactly (2^-127 is the subnormal 0x00400000).  Multiplying by it is
// the same IEEE operation as scaling the exponent: exact, or one round to nearest even.
__device__ __forceinline__ float exp2_neg(int s) {
  return s <= 126 ? __int_as_float((127 - s) << 23) : __int_as_float(0x00400000);
}
// Two E4M3 codes (round to nearest even, saturating to +-448) of a and b; a in the low byte.
__device__ __forceinline__ uint32_t e4m3x2(float a, float b) {
  return static_cast<uint32_t>(
      __nv_cvt_float2_to_fp8x2(make_float2(a, b), __NV_SATFINITE, __NV_E4M3));
}
// Byte of (MN index i, block b) in scale chunk `chunk`: 512-byte chunks of 128 indices x
// 4 blocks, laid out as byte 16*(i%32) + 4*((i%128)/32) + b (the order in which a
// tcgen05.cp of 32 rows x 16 bytes puts them where the block-scaled MMA reads them).
__device__ __forceinline__ size_t sf_byte(int64_t chunk, int i, int block) {
  return (size_t)chunk * 512 + 16 * (i & 31) + 4 * ((i & 127) >> 5) + block;
}
__device__ __forceinline__ float bf_lo(uint32_t w) { return __uint_as_float(w << 16); }
__device__ __forceinline__ float bf_hi(uint32_t w) { return __uint_as_float(w & 0xffff0000u); }
// |x| of both bf16 halves (the sign bits cleared).  Non-negative IEEE values order like
// their bit patterns, so a per-half unsigned max of |x| bits is the exact max |x|.
__device__ __forceinline__ uint32_t abs2(uint32_t w) { return w & 0x7fff7fffu; }

// One block held by one thread: 32 bf16 packed two to a word (w[i] = elements 2i, 2i+1
// in its low and high halves) -> 32 codes written to dst (16-byte aligned); returns s.
__device__ __forceinline__ int quantise_block32(const uint32_t* w, uint8_t* dst) {
  uint32_t m = 0u;
#pragma unroll
  for (int i = 0; i < 16; ++i) m = __vmaxu2(m, abs2(w[i]));
  const int s = exponent_bits(max(m & 0xffffu, m >> 16));
  const float mul = exp2_neg(s);
  uint32_t o[8];
#pragma unroll
  for (int j = 0; j < 8; ++j)
    o[j] = e4m3x2(bf_lo(w[2 * j]) * mul, bf_hi(w[2 * j]) * mul) |
           (e4m3x2(bf_lo(w[2 * j + 1]) * mul, bf_hi(w[2 * j + 1]) * mul) << 16);
  uint4* d = reinterpret_cast<uint4*>(dst);
  d[0] = make_uint4(o[0], o[1], o[2], o[3]);
  d[1] = make_uint4(o[4], o[5], o[6], o[7]);
  return s;
}

}  // namespace mxb
}  // namespace moe
