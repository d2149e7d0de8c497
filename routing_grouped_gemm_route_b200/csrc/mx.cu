// MX (microscaling) FP8 quantisers: E4M3 elements with one E8M0 scale per 32 elements.
//
// The write-ups offer MXFP8 for selected operations and credit most of its gain to the
// FFN and expert data movement (bigchange.ai pt-BR, opening section and "Três números,
// três denominadores"; unite.ai, "पैरालेलिज़्म, प्रिसीजन, और मेमोरी तकनीकें").  They give no
// rule; this follows the OCP MX v1.0 definition: per block of 32 the shared exponent is
// s = floor(log2(amax)) - 8 (8 = exponent of E4M3's largest normal) clamped to
// [-127, 127] (an all-zero block gets -127), stored as the byte s + 127; each element is
// x / 2^s rounded to nearest-even E4M3 with saturation to +-448.
//
// Layout.  Codes keep the bf16 tensor's [rows, cols] layout, one byte per element.
// Rows come in segments (one per expert); `p` is a row's index inside its segment.
// Scales are stored in 512-byte chunks, each holding 128 "MN" indices x 4 blocks along
// the quantised axis as byte 16*(i%32) + 4*(i/32) + block -- the order in which a
// tcgen05.cp of 32 rows x 16 bytes (replicated to the four lane quadrants) puts them
// where the block-scaled MMA reads them.  Chunk numbering, with tile_pref[e] the prefix
// over segments of ceil(rows/128):
//   rowwise (blocks of 32 along cols):  chunk (tile_pref[e] + p/128) * (cols/128) + col/128,
//                                        MN index p % 128, block (col % 128) / 32;
//   colwise (blocks of 32 along rows inside the segment, starting at its first row):
//                                        chunk (tile_pref[e] + p/128) * (cols/128) + col/128,
//                                        MN index col % 128, block (p % 128) / 32.
// A 128-row tile of a segment (or 128 rows of K of a wgrad stage) thus finds its scales
// in whole chunks.
#include <cuda_runtime.h>
#include <cuda_bf16.h>
#include <cuda_fp8.h>
#include <math.h>

#include "common.cuh"
#include "internal.h"

namespace moe {
namespace {

// Shared exponent of a block with max magnitude `amax` (>= 0).
__device__ __forceinline__ int mx_exponent(float amax) {
  if (!(amax > 0.f)) return -127;
  int s = ilogbf(amax) - 8;          // floor(log2(amax)) for finite non-zero amax
  return s < -127 ? -127 : (s > 127 ? 127 : s);
}
__device__ __forceinline__ uint8_t e4m3(float v) {
  return static_cast<uint8_t>(__nv_cvt_float_to_fp8(v, __NV_SATFINITE, __NV_E4M3));
}
__device__ __forceinline__ size_t sf_byte(int64_t chunk, int i, int block) {
  return (size_t)chunk * 512 + 16 * (i & 31) + 4 * ((i & 127) >> 5) + block;
}

// Segment of row r: the e with seg_off[e] <= r < seg_off[e+1] (skipping empty ones).
__device__ __forceinline__ int segment_of(const int32_t* seg_off, int E, int r) {
  int lo = 0, hi = E;
  while (hi - lo > 1) {
    const int mid = (lo + hi) >> 1;
    if (seg_off[mid] <= r) lo = mid; else hi = mid;
  }
  return lo;
}

// tile_pref[e] = sum_{e'<e} ceil(rows_e'/128); blk_pref[e] = sum_{e'<e} ceil(rows_e'/32).
__global__ void seg_prefix_kernel(const int32_t* __restrict__ seg_off, int E,
                                  int32_t* __restrict__ tile_pref, int32_t* __restrict__ blk_pref) {
  if (threadIdx.x != 0 || blockIdx.x != 0) return;
  int t = 0, b = 0;
  for (int e = 0; e < E; ++e) {
    tile_pref[e] = t;
    blk_pref[e] = b;
    const int c = seg_off[e + 1] - seg_off[e];
    t += (c + 127) / 128;
    b += (c + 31) / 32;
  }
  tile_pref[E] = t;
  blk_pref[E] = b;
}

// Rowwise: one warp per row, lane l handles blocks l, l+32, ... (64 contiguous bytes each).
// perm_f > 0 (SwiGLU weights [W1; W3], d_ff = perm_f rows each): the scale of row p is
// filed under the row order gate[0:64], up[0:64], gate[64:128], up[64:128], ..., the order
// in which a 128-row B tile of the fused SwiGLU GEMM takes 64 gate and 64 up rows.
__global__ void __launch_bounds__(256) quant_rows_kernel(
    const __nv_bfloat16* __restrict__ x, int R, int C, const int32_t* __restrict__ seg_off, int E,
    const int32_t* __restrict__ tile_pref, int perm_f, uint8_t* __restrict__ codes,
    uint8_t* __restrict__ sf) {
  const int r = blockIdx.x * 8 + (threadIdx.x >> 5);
  const int lane = threadIdx.x & 31;
  if (r >= R) return;
  const int e = segment_of(seg_off, E, r);
  int p = r - seg_off[e];
  if (perm_f > 0) p = p < perm_f ? (p / 64) * 128 + (p % 64) : ((p - perm_f) / 64) * 128 + 64 + (p - perm_f) % 64;
  const int64_t group = (int64_t)tile_pref[e] + p / 128;
  const int nb = C / 32;
  const __nv_bfloat16* row = x + (int64_t)r * C;
  for (int b = lane; b < nb; b += 32) {
    float v[32];
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      Vec16<__nv_bfloat16> pk;
      pk.raw = *reinterpret_cast<const uint4*>(row + b * 32 + j * 8);
      pk.to_float(v + j * 8);
    }
    float amax = 0.f;
#pragma unroll
    for (int j = 0; j < 32; ++j) amax = fmaxf(amax, fabsf(v[j]));
    const int s = mx_exponent(amax);
    uint32_t w[8];
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      w[j] = (uint32_t)e4m3(scalbnf(v[4 * j], -s)) | ((uint32_t)e4m3(scalbnf(v[4 * j + 1], -s)) << 8) |
             ((uint32_t)e4m3(scalbnf(v[4 * j + 2], -s)) << 16) |
             ((uint32_t)e4m3(scalbnf(v[4 * j + 3], -s)) << 24);
    }
    uint4* dst = reinterpret_cast<uint4*>(codes + (int64_t)r * C + b * 32);   // codes stay in x's row order
    dst[0] = make_uint4(w[0], w[1], w[2], w[3]);
    dst[1] = make_uint4(w[4], w[5], w[6], w[7]);
    const int64_t chunk = group * (C / 128) + (b * 32) / 128;
    sf[sf_byte(chunk, p, b & 3)] = static_cast<uint8_t>(s + 127);
  }
}

// Colwise: one CTA per (32-row block of a segment, 256 columns); thread = column.
__global__ void __launch_bounds__(256) quant_cols_kernel(
    const __nv_bfloat16* __restrict__ x, int R, int C, const int32_t* __restrict__ seg_off, int E,
    const int32_t* __restrict__ tile_pref, const int32_t* __restrict__ blk_pref,
    uint8_t* __restrict__ codes, uint8_t* __restrict__ sf) {
  const int blk = blockIdx.y;                 // global 32-row block index over all segments
  if (blk >= blk_pref[E]) return;
  int lo = 0, hi = E;                         // segment: blk_pref[lo] <= blk < blk_pref[lo+1]
  while (hi - lo > 1) {
    const int mid = (lo + hi) >> 1;
    if (blk_pref[mid] <= blk) lo = mid; else hi = mid;
  }
  const int e = lo;
  const int p0 = (blk - blk_pref[e]) * 32;    // first row of the block inside the segment
  const int r0 = seg_off[e] + p0;
  const int nrows = min(32, seg_off[e + 1] - r0);
  const int c = blockIdx.x * 256 + threadIdx.x;
  if (c >= C) return;
  float v[32];
  float amax = 0.f;
#pragma unroll
  for (int j = 0; j < 32; ++j) {
    v[j] = j < nrows ? __bfloat162float(x[(int64_t)(r0 + j) * C + c]) : 0.f;
    amax = fmaxf(amax, fabsf(v[j]));
  }
  const int s = mx_exponent(amax);
#pragma unroll
  for (int j = 0; j < 32; ++j)
    if (j < nrows) codes[(int64_t)(r0 + j) * C + c] = e4m3(scalbnf(v[j], -s));
  const int64_t chunk = ((int64_t)tile_pref[e] + p0 / 128) * (C / 128) + c / 128;
  sf[sf_byte(chunk, c, (p0 & 127) >> 5)] = static_cast<uint8_t>(s + 127);
  // The segment's last chunk may hold fewer than four blocks.  A K-stage of a wgrad GEMM
  // still reads all four scales (its rows past the segment are zero codes), so the absent
  // blocks get the finite scale 2^-127 rather than whatever the buffer held (0xFF = NaN).
  if (p0 + 32 >= seg_off[e + 1] - seg_off[e])
    for (int b = ((p0 & 127) >> 5) + 1; b < 4; ++b) sf[sf_byte(chunk, c, b)] = 0;
}

// seg_off[e] = e * rows (uniform segments: one per expert's weight matrix)
__global__ void uniform_offsets_kernel(int32_t* seg_off, int E, int rows) {
  const int e = blockIdx.x * blockDim.x + threadIdx.x;
  if (e <= E) seg_off[e] = e * rows;
}

}  // namespace

cudaError_t launch_uniform_offsets(int32_t* seg_off, int E, int rows, cudaStream_t s) {
  uniform_offsets_kernel<<<(E + 1 + 255) / 256, 256, 0, s>>>(seg_off, E, rows);
  return cudaGetLastError();
}

size_t mx_sf_bytes(int64_t R, int C, int E) {
  // chunks: (sum_e ceil(rows_e/128)) * (C/128) <= (R/128 + E) * (C/128)
  return (size_t)((R + 127) / 128 + E) * (size_t)(C / 128) * 512;
}

cudaError_t launch_mx_quantize(const void* x, int64_t R, int C, const int32_t* seg_off, int E,
                               bool colwise, uint8_t* codes, uint8_t* sf, int32_t* scratch,
                               cudaStream_t s, int perm_f) {
  if (R == 0) return cudaSuccess;
  int32_t* tile_pref = scratch;               // [E+1]
  int32_t* blk_pref = scratch + (E + 1);      // [E+1]
  seg_prefix_kernel<<<1, 32, 0, s>>>(seg_off, E, tile_pref, blk_pref);
  cudaError_t err = cudaGetLastError();
  if (err != cudaSuccess) return err;
  const __nv_bfloat16* xb = reinterpret_cast<const __nv_bfloat16*>(x);
  if (!colwise) {
    quant_rows_kernel<<<(unsigned)((R + 7) / 8), 256, 0, s>>>(xb, (int)R, C, seg_off, E, tile_pref,
                                                            perm_f, codes, sf);
  } else {
    // one CTA row per possible 32-row block: sum_e ceil(rows_e/32) <= R/32 + E
    dim3 grid((C + 255) / 256, (unsigned)((R + 31) / 32 + E));
    quant_cols_kernel<<<grid, 256, 0, s>>>(xb, (int)R, C, seg_off, E, tile_pref, blk_pref, codes,
                                           sf);
  }
  return cudaGetLastError();
}

}  // namespace moe
