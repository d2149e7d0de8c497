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

#include <algorithm>

#include "common.cuh"
#include "internal.h"
#include "mx_block.cuh"
#include "sm100.cuh"

namespace moe {
namespace {

using namespace sm100;

using mxb::exp2_neg;
using mxb::e4m3x2;
using mxb::sf_byte;
using mxb::bf_lo;
using mxb::bf_hi;
using mxb::abs2;
__device__ __forceinline__ int mx_exponent_bits(uint32_t b) { return mxb::exponent_bits(b); }

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

// One tile = one 32-row block of a segment (its rows p0 .. p0+nrows-1, starting at row r0
// of the tensor) x 128 columns.
struct TilePos {
  int e, p0, r0, nrows;
};
__device__ __forceinline__ bool tile_pos(const MxSegs& g, int blk, TilePos& o) {
  if (g.rows > 0) {
    const int per = (g.rows + 31) / 32;
    const int e = blk / per;
    if (e >= g.E) return false;
    o.e = e;
    o.p0 = (blk - e * per) * 32;
    o.r0 = e * g.rows + o.p0;
    o.nrows = min(32, g.rows - o.p0);
    return true;
  }
  if (blk >= g.blk_pref[g.E]) return false;
  int lo = 0, hi = g.E;                       // largest e with blk_pref[e] <= blk
  while (hi - lo > 1) {
    const int mid = (lo + hi) >> 1;
    if (g.blk_pref[mid] <= blk) lo = mid; else hi = mid;
  }
  o.e = lo;
  o.p0 = (blk - g.blk_pref[lo]) * 32;
  o.r0 = g.off[lo] + o.p0;
  o.nrows = min(32, g.off[lo + 1] - o.r0);
  return true;
}
__device__ __forceinline__ int seg_rows(const MxSegs& g, int e) {
  return g.rows > 0 ? g.rows : g.off[e + 1] - g.off[e];
}
__device__ __forceinline__ int64_t seg_tile0(const MxSegs& g, int e) {
  return g.rows > 0 ? (int64_t)e * ((g.rows + 127) / 128) : (int64_t)g.tile_pref[e];
}

// A lane's CPL consecutive bf16 of one row (CPL = 4: two words) and what is done with
// them: the per-half max of |x|, the codes (one multiplier per column), stores.
template <int CPL> struct Lane;
template <> struct Lane<4> {
  using V = uint2;
  static __device__ __forceinline__ V load(const __nv_bfloat16* p) { return __ldg(reinterpret_cast<const uint2*>(p)); }
  static __device__ __forceinline__ V zero() { return make_uint2(0u, 0u); }
  static __device__ __forceinline__ uint32_t absmax(V v) { return __vmaxu2(abs2(v.x), abs2(v.y)); }
  static __device__ __forceinline__ void absmax_cols(uint32_t* m, V v) {
    m[0] = __vmaxu2(m[0], abs2(v.x));
    m[1] = __vmaxu2(m[1], abs2(v.y));
  }
  static __device__ __forceinline__ void store(uint8_t* p, V v, const float* m) {
    *reinterpret_cast<uint32_t*>(p) = e4m3x2(bf_lo(v.x) * m[0], bf_hi(v.x) * m[1]) |
                                      (e4m3x2(bf_lo(v.y) * m[2], bf_hi(v.y) * m[3]) << 16);
  }
};

// One level of the rowwise reduce-scatter over the lanes of a 32-column block: lanes
// whose bit M is set keep the upper half of the CPL*2*M rows still held and take the
// partner's (lane ^ M) maxima of them; the others keep the lower half.  Levels M, M/2,
// .., 1 leave lane j with rows CPL*j .. CPL*j+CPL-1.
template <int CPL, int M>
__device__ __forceinline__ void row_reduce_scatter(uint32_t (&a)[32], int sub) {
  constexpr int N = CPL * M;
  const bool up = (sub & M) != 0;
#pragma unroll
  for (int i = 0; i < N; ++i) {
    const uint32_t send = up ? a[i] : a[i + N];
    const uint32_t keep = up ? a[i + N] : a[i];
    a[i] = __vmaxu2(keep, __shfl_xor_sync(0xffffffffu, send, M));
  }
  if constexpr (M > 1) row_reduce_scatter<CPL, M / 2>(a, sub);
}

constexpr int kQWarps = 4;                   // warps per CTA
// CTAs per SM: 4 (16 warps, <= 128 registers) for one direction; 3 (12 warps) when a
// tile is quantised both ways, whose live set does not fit 128 registers
template <int CPL> constexpr int q_ctas_per_sm(bool both) { return both ? 3 : 4; }

// Persistent quantiser; one warp per tile, no shared memory, no barriers.  A tile is one
// 32-row block of a segment x 32*CPL columns; lane L holds columns CPL*L .. CPL*L+CPL-1
// of all 32 rows in registers (each load instruction of the warp reads 64*CPL contiguous
// bytes of one row; all 32 rows' loads are in flight together), so
//   ROW (blocks of 32 along columns): a row's block spans G = 32/CPL lanes.  A butterfly
//        reduce-scatter over them leaves lane j of the group with the maxima of rows
//        CPL*j .. CPL*j+CPL-1 (each step halves the rows a lane keeps); it derives
//        those rows' exponents and scale bytes, and shuffles return the multipliers;
//   COL (blocks of 32 along the segment's rows; the tile is exactly one block per
//        column): each lane's running max over its 32 rows, no communication.
// Codes leave as CPL-byte stores, 32*CPL contiguous bytes per row and instruction.
// perm_f > 0 (SwiGLU weights [W1; W3], d_ff = perm_f rows each): the rowwise scale of
// row p is filed under the row order gate[0:128], up[0:128], gate[128:256], ..., the
// order in which a 256-column tile of the fused SwiGLU GEMM takes 128 gate and 128 up
// rows of B.
template <int CPL, bool ROW, bool COL>
__global__ void __launch_bounds__(kQWarps * 32, q_ctas_per_sm<CPL>(ROW && COL)) quant_warp_kernel(
    const __nv_bfloat16* __restrict__ x, int C, const MxSegs g, int perm_f,
    uint8_t* __restrict__ codes_r, uint8_t* __restrict__ sf_r, uint8_t* __restrict__ codes_c,
    uint8_t* __restrict__ sf_c) {
  using LN = Lane<CPL>;
  using V = typename LN::V;
  constexpr int TC = 32 * CPL;               // tile columns
  constexpr int G = 32 / CPL;                // lanes of one 32-column block
  const int lane = threadIdx.x & 31;
  const int ctiles = C / TC;
  const int W = C / 128;
  const int nblk = g.rows > 0 ? g.E * ((g.rows + 31) / 32) : g.blk_pref[g.E];
  const int ntiles = nblk * ctiles;
  const int stride = static_cast<int>(gridDim.x) * kQWarps;
  for (int tile = static_cast<int>(blockIdx.x) * kQWarps + static_cast<int>(threadIdx.x >> 5);
       tile < ntiles; tile += stride) {
    TilePos tp;
    tile_pos(g, tile / ctiles, tp);
    const int c0 = (tile % ctiles) * TC;
    const int col = c0 + CPL * lane;          // my first column
    const int nrows = tp.nrows;               // warp-uniform
    const __nv_bfloat16* src = x + (int64_t)tp.r0 * C + col;
    V v[32];
#pragma unroll
    for (int r = 0; r < 32; ++r)
      v[r] = r < nrows ? LN::load(src + (int64_t)r * C) : LN::zero();   // past the segment: 0
    const int64_t tile0 = seg_tile0(g, tp.e);
    if (COL) {
      uint32_t mc[CPL / 2] = {};              // column maxima (|x| bits, two per word)
#pragma unroll
      for (int r = 0; r < 32; ++r) LN::absmax_cols(mc, v[r]);
      int sc[CPL];
      float mul[CPL];
#pragma unroll
      for (int i = 0; i < CPL; ++i) {
        sc[i] = mx_exponent_bits((i & 1) ? mc[i / 2] >> 16 : mc[i / 2] & 0xffffu);
        mul[i] = exp2_neg(sc[i]);
      }
      uint8_t* dst = codes_c + (int64_t)tp.r0 * C + col;
#pragma unroll
      for (int r = 0; r < 32; ++r)
        if (r < nrows) LN::store(dst + (int64_t)r * C, v[r], mul);
      const int64_t chunk = (tile0 + tp.p0 / 128) * W + c0 / 128;
      const int blk = (tp.p0 & 127) >> 5;
#pragma unroll
      for (int i = 0; i < CPL; ++i) sf_c[sf_byte(chunk, col + i, blk)] = static_cast<uint8_t>(sc[i] + 127);
      // The segment's last chunk may hold fewer than four blocks.  A K-stage of a wgrad
      // GEMM still reads all four scales (its rows past the segment are zero codes), so
      // the absent blocks get the finite scale 2^-127 rather than whatever the buffer
      // held (0xFF = NaN).
      if (tp.p0 + 32 >= seg_rows(g, tp.e))
        for (int k = blk + 1; k < 4; ++k)
#pragma unroll
          for (int i = 0; i < CPL; ++i) sf_c[sf_byte(chunk, col + i, k)] = 0;
    }
    if (ROW) {
      const int sub = lane & (G - 1);
      uint32_t a[32];
#pragma unroll
      for (int r = 0; r < 32; ++r) a[r] = LN::absmax(v[r]);
      row_reduce_scatter<CPL, G / 2>(a, sub);
      // rows CPL*sub + i (i < CPL) are mine; the segment's row p0 + r maps to the scale
      // MN index pp0 + r (a 32-row block never straddles a 128-row gate/up group)
      int pp0 = tp.p0;
      if (perm_f > 0)
        pp0 = pp0 < perm_f ? (pp0 / 128) * 256 + (pp0 % 128)
                           : ((pp0 - perm_f) / 128) * 256 + 128 + (pp0 - perm_f) % 128;
      const int blk = (c0 & 127) / 32 + lane / G;
      uint8_t* sf = sf_r + sf_byte((tile0 + pp0 / 128) * W + c0 / 128, pp0, blk);
      float mine[CPL];
#pragma unroll
      for (int i = 0; i < CPL; ++i) {
        const int s = mx_exponent_bits(max(a[i] & 0xffffu, a[i] >> 16));
        mine[i] = exp2_neg(s);
        if (CPL * sub + i < nrows) sf[16 * (CPL * sub + i)] = static_cast<uint8_t>(s + 127);
      }
      uint8_t* dst = codes_r + (int64_t)tp.r0 * C + col;
#pragma unroll
      for (int r = 0; r < 32; ++r) {
        float m[CPL];
        m[0] = __shfl_sync(0xffffffffu, mine[r % CPL], (lane & ~(G - 1)) | (r / CPL));
#pragma unroll
        for (int i = 1; i < CPL; ++i) m[i] = m[0];
        if (r < nrows) LN::store(dst + (int64_t)r * C, v[r], m);
      }
    }
  }
}

}  // namespace

size_t mx_sf_bytes(int64_t R, int C, int E) {
  // chunks: (sum_e ceil(rows_e/128)) * (C/128) <= (R/128 + E) * (C/128)
  return (size_t)((R + 127) / 128 + E) * (size_t)(C / 128) * 512;
}

cudaError_t launch_mx_prefix(const int32_t* seg_off, int E, int32_t* tile_pref, int32_t* blk_pref,
                             cudaStream_t s) {
  seg_prefix_kernel<<<1, 32, 0, s>>>(seg_off, E, tile_pref, blk_pref);
  return cudaGetLastError();
}

template <int CPL>
static cudaError_t launch_quant(const __nv_bfloat16* x, int64_t tiles, int C, const MxSegs& g,
                                int perm_f, uint8_t* codes_r, uint8_t* sf_r, uint8_t* codes_c,
                                uint8_t* sf_c, cudaStream_t s) {
  const bool row = codes_r != nullptr, col = codes_c != nullptr;
  const int64_t grid = std::min<int64_t>((tiles + kQWarps - 1) / kQWarps,
                                         (int64_t)num_sms() * q_ctas_per_sm<CPL>(row && col));
  auto kern = row && col ? quant_warp_kernel<CPL, true, true>
              : row      ? quant_warp_kernel<CPL, true, false>
                         : quant_warp_kernel<CPL, false, true>;
  kern<<<(unsigned)grid, kQWarps * 32, 0, s>>>(x, C, g, row ? perm_f : 0, codes_r, sf_r, codes_c,
                                              sf_c);
  return cudaGetLastError();
}

constexpr int kQCpl = 4;   // columns per lane

cudaError_t launch_mx_quant(const void* x, int64_t R, int C, const MxSegs& g, int perm_f,
                            uint8_t* codes_r, uint8_t* sf_r, uint8_t* codes_c, uint8_t* sf_c,
                            int* status, cudaStream_t s) {
  (void)status;   // no waits, no data-dependent failure
  if (R == 0 || (codes_r == nullptr && codes_c == nullptr)) return cudaSuccess;
  // tiles: sum_e ceil(rows_e/32) <= R/32 + E row blocks, times the column tiles
  const int64_t blocks = g.rows > 0 ? (int64_t)g.E * ((g.rows + 31) / 32) : (R + 31) / 32 + g.E;
  const int64_t tiles = blocks * (C / (32 * kQCpl));
  if (tiles > 0x7fffffffLL) return cudaErrorInvalidValue;
  return launch_quant<kQCpl>(reinterpret_cast<const __nv_bfloat16*>(x), tiles, C, g, perm_f,
                             codes_r, sf_r, codes_c, sf_c, s);
}

cudaError_t launch_mx_quantize(const void* x, int64_t R, int C, const int32_t* seg_off, int E,
                               bool colwise, uint8_t* codes, uint8_t* sf, int32_t* scratch,
                               int* status, cudaStream_t s) {
  if (R == 0) return cudaSuccess;
  MxSegs g;
  g.off = seg_off;
  g.tile_pref = scratch;               // [E+1]
  g.blk_pref = scratch + (E + 1);      // [E+1]
  g.E = E;
  cudaError_t err = launch_mx_prefix(seg_off, E, scratch, scratch + (E + 1), s);
  if (err != cudaSuccess) return err;
  return colwise ? launch_mx_quant(x, R, C, g, 0, nullptr, nullptr, codes, sf, status, s)
                 : launch_mx_quant(x, R, C, g, 0, codes, sf, nullptr, nullptr, status, s);
}

}  // namespace moe
