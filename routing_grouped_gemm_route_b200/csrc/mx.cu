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
#include "sm100.cuh"

namespace moe {
namespace {

using namespace sm100;

// Shared exponent of a block with max magnitude `amax` (>= 0).
__device__ __forceinline__ int mx_exponent(float amax) {
  if (!(amax > 0.f)) return -127;
  int s = ilogbf(amax) - 8;          // floor(log2(amax)) for finite non-zero amax
  return s < -127 ? -127 : (s > 127 ? 127 : s);
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
__device__ __forceinline__ size_t sf_byte(int64_t chunk, int i, int block) {
  return (size_t)chunk * 512 + 16 * (i & 31) + 4 * ((i & 127) >> 5) + block;
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

constexpr int kQRows = 32, kQCols = 128;
constexpr int kQThreads = kQCols;            // one warp per 32-column block
constexpr int kQCtasPerSm = 8;
constexpr int kQPitch = kQCols * 2 + 16;     // bytes per staged row (16-byte skew: no bank conflicts)
constexpr int kQBufs = 2;                    // tiles in flight per CTA (one being quantised)
constexpr int kQBufBytes = kQRows * kQPitch;
constexpr size_t kQSmem = 128 + (size_t)kQBufs * kQBufBytes;

// 32 bf16 of a staged row (64 contiguous bytes), kept packed: w[i] holds elements
// 2i (low half) and 2i+1 (high half).
__device__ __forceinline__ void staged32(const uint8_t* p, uint32_t* w) {
#pragma unroll
  for (int j = 0; j < 4; ++j) {
    const uint4 u = *reinterpret_cast<const uint4*>(p + 16 * j);
    w[4 * j] = u.x;
    w[4 * j + 1] = u.y;
    w[4 * j + 2] = u.z;
    w[4 * j + 3] = u.w;
  }
}
__device__ __forceinline__ float bf_lo(uint32_t w) { return __uint_as_float(w << 16); }
__device__ __forceinline__ float bf_hi(uint32_t w) { return __uint_as_float(w & 0xffff0000u); }
// |x| of both bf16 halves (the sign bits cleared).  Non-negative IEEE values order like
// their bit patterns, so a per-half unsigned max of |x| bits is the exact max |x|.
__device__ __forceinline__ uint32_t abs2(uint32_t w) { return w & 0x7fff7fffu; }
__device__ __forceinline__ float amax32(const uint32_t* w) {
  uint32_t m = 0u;
#pragma unroll
  for (int i = 0; i < 16; ++i) m = __vmaxu2(m, abs2(w[i]));
  return fmaxf(bf_lo(m), bf_hi(m));
}

// 32 codes of the packed bf16 w[] times m[j] (PER_ELEM) or m[0] -> two 16-byte stores
template <bool PER_ELEM>
__device__ __forceinline__ void store_codes32(uint8_t* dst, const uint32_t* w, const float* m) {
  uint32_t o[8];
#pragma unroll
  for (int j = 0; j < 8; ++j) {
    const int i = 4 * j;
    const float m0 = m[PER_ELEM ? i : 0], m1 = m[PER_ELEM ? i + 1 : 0];
    const float m2 = m[PER_ELEM ? i + 2 : 0], m3 = m[PER_ELEM ? i + 3 : 0];
    o[j] = e4m3x2(bf_lo(w[2 * j]) * m0, bf_hi(w[2 * j]) * m1) |
           (e4m3x2(bf_lo(w[2 * j + 1]) * m2, bf_hi(w[2 * j + 1]) * m3) << 16);
  }
  uint4* d = reinterpret_cast<uint4*>(dst);
  d[0] = make_uint4(o[0], o[1], o[2], o[3]);
  d[1] = make_uint4(o[4], o[5], o[6], o[7]);
}

// Persistent quantiser.  A tile is one 32-row block of a segment x 128 columns; each CTA
// walks tiles blockIdx.x, +gridDim.x, ... with kQBufs shared-memory buffers: while it
// quantises one tile, the next ones' rows stream in by 1-D bulk copies (so the bytes in
// flight do not depend on registers).  Per tile it writes the rowwise codes/scales (ROW:
// blocks of 32 along columns) and/or the colwise ones (COL: blocks of 32 along the
// segment's rows; the tile is exactly one such block per column).
// perm_f > 0 (SwiGLU weights [W1; W3], d_ff = perm_f rows each): the rowwise scale of
// row p is filed under the row order gate[0:128], up[0:128], gate[128:256], ..., the
// order in which a 256-column tile of the fused SwiGLU GEMM takes 128 gate and 128 up
// rows of B.
template <bool ROW, bool COL>
__global__ void __launch_bounds__(kQThreads, kQCtasPerSm) quant_tile_kernel(
    const __nv_bfloat16* __restrict__ x, int C, const MxSegs g, int perm_f,
    uint8_t* __restrict__ codes_r, uint8_t* __restrict__ sf_r, uint8_t* __restrict__ codes_c,
    uint8_t* __restrict__ sf_c, int* status) {
  extern __shared__ uint8_t q_smem_raw[];
  uint8_t* bufs = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(q_smem_raw) + 127) &
                                             ~uintptr_t(127));
  __shared__ float col_m[kQCols];
  __shared__ uint64_t bar[kQBufs];
  __shared__ TilePos pos[kQBufs];
  __shared__ int abort_flag;
  const int t = threadIdx.x;
  const int ctiles = (C + kQCols - 1) / kQCols;
  const int nblk = g.rows > 0 ? g.E * ((g.rows + 31) / 32) : g.blk_pref[g.E];
  const int ntiles = nblk * ctiles;
  if ((int)blockIdx.x >= ntiles) return;      // uniform over the CTA
  if (t == 0) {
    for (int i = 0; i < kQBufs; ++i) mbar_init(&bar[i], 1);
    abort_flag = 0;
    fence_mbar_init();
  }
  __syncthreads();
  // warp 0 loads tile `tile` into buffer `b`: lane 0 arms the barrier with the byte count,
  // lane r copies row r (the phase cannot complete before lane 0's arrival)
  auto issue = [&](int tile, int b) {
    TilePos tp;
    tile_pos(g, tile / ctiles, tp);
    const int c0 = (tile % ctiles) * kQCols;
    const int ncols = min(kQCols, C - c0);
    if (t == 0) {
      pos[b] = tp;
      fence_proxy_async_smem();               // earlier generic reads of buf[b] before the copies
      mbar_arrive_expect_tx(&bar[b], static_cast<uint32_t>(tp.nrows * ncols * 2));
    }
    __syncwarp();
    if (t < tp.nrows)
      bulk_load(bufs + b * kQBufBytes + t * kQPitch, x + (int64_t)(tp.r0 + t) * C + c0,
                static_cast<uint32_t>(ncols * 2), &bar[b]);
  };
  // prologue: the first kQBufs-1 tiles
  for (int i = 0; i < kQBufs - 1; ++i) {
    const int tile = blockIdx.x + i * gridDim.x;
    if (t < 32 && tile < ntiles) issue(tile, i);
  }
  const int W = C / 128;
  const int row = t & 31, q = t >> 5;         // this thread's row and 32-column block
  const int lane = t & 31;
  int it = 0;
  for (int tile = blockIdx.x; tile < ntiles; tile += gridDim.x, ++it) {
    const int b = it % kQBufs;
    // the buffer of iteration it-1 was released by the barrier that ended it
    const int ahead = tile + (kQBufs - 1) * gridDim.x;
    if (t < 32 && ahead < ntiles) issue(ahead, (it + kQBufs - 1) % kQBufs);
    const bool ok = mbar_wait(&bar[b], (it / kQBufs) & 1u,
                              reinterpret_cast<volatile int*>(&abort_flag), status);
    // every step below is warp-local; the barrier at the end releases the buffer (and
    // agrees on an abort)
    if (ok) {
    const TilePos tp = pos[b];
    const int c0 = (tile % ctiles) * kQCols;
    const int ncols = min(kQCols, C - c0);
    const int64_t tile0 = seg_tile0(g, tp.e);
    const uint8_t* tb = bufs + b * kQBufBytes;
    const bool active = row < tp.nrows && q * 32 < ncols;
    uint32_t v[16];
    if (active) staged32(tb + row * kQPitch + q * 64, v);
    if (ROW && active) {
      const int s = mx_exponent(amax32(v));
      const float m = exp2_neg(s);
      store_codes32<false>(codes_r + (int64_t)(tp.r0 + row) * C + c0 + q * 32, v, &m);
      int p = tp.p0 + row;
      if (perm_f > 0)
        p = p < perm_f ? (p / 128) * 256 + (p % 128)
                       : ((p - perm_f) / 128) * 256 + 128 + (p - perm_f) % 128;
      const int col = c0 + q * 32;
      sf_r[sf_byte((tile0 + p / 128) * W + col / 128, p, (col & 127) >> 5)] =
          static_cast<uint8_t>(s + 127);
    }
    if (COL && q * 32 < ncols) {   // warp-uniform: this warp's 32-column block exists
      // The warp holds the block's 32 rows (one per lane; rows past the segment's end
      // are masked to zero).  A butterfly reduce-scatter of |x| over the lanes leaves
      // lane L with the max of column L: each step halves the words a lane keeps.
      uint32_t a[16];
#pragma unroll
      for (int i = 0; i < 16; ++i) a[i] = active ? abs2(v[i]) : 0u;
#pragma unroll
      for (int m = 16; m >= 2; m >>= 1) {
        const bool up = (lane & m) != 0;
#pragma unroll
        for (int i = 0; i < m / 2; ++i) {
          const uint32_t send = up ? a[i] : a[i + m / 2];
          const uint32_t keep = up ? a[i + m / 2] : a[i];
          a[i] = __vmaxu2(keep, __shfl_xor_sync(0xffffffffu, send, m));
        }
      }
      const uint32_t mm = __vmaxu2(a[0], __shfl_xor_sync(0xffffffffu, a[0], 1));
      const int s = mx_exponent((lane & 1) ? bf_hi(mm) : bf_lo(mm));
      const int col = c0 + q * 32 + lane;
      col_m[q * 32 + lane] = exp2_neg(s);
      const int64_t chunk = (tile0 + tp.p0 / 128) * W + col / 128;
      const int blk = (tp.p0 & 127) >> 5;
      sf_c[sf_byte(chunk, col, blk)] = static_cast<uint8_t>(s + 127);
      // The segment's last chunk may hold fewer than four blocks.  A K-stage of a wgrad
      // GEMM still reads all four scales (its rows past the segment are zero codes), so
      // the absent blocks get the finite scale 2^-127 rather than whatever the buffer
      // held (0xFF = NaN).
      if (tp.p0 + 32 >= seg_rows(g, tp.e))
        for (int k = blk + 1; k < 4; ++k) sf_c[sf_byte(chunk, col, k)] = 0;
      __syncwarp();
      if (active)
        store_codes32<true>(codes_c + (int64_t)(tp.r0 + row) * C + c0 + q * 32, v, col_m + q * 32);
    }
    }
    if (__syncthreads_or(!ok)) break;   // this buffer and col_m free for reuse
  }
  // After an abort, the copies still in flight (iterations it .. it+kQBufs-1 that have a
  // tile) must land before the CTA exits.
  if (t == 0 && abort_flag) {
    for (int j = it; j < it + kQBufs; ++j)
      if (blockIdx.x + j * gridDim.x < ntiles)
        mbar_wait_teardown(&bar[j % kQBufs], (j / kQBufs) & 1u);
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

cudaError_t launch_mx_quant(const void* x, int64_t R, int C, const MxSegs& g, int perm_f,
                            uint8_t* codes_r, uint8_t* sf_r, uint8_t* codes_c, uint8_t* sf_c,
                            int* status, cudaStream_t s) {
  if (R == 0) return cudaSuccess;
  // tiles: sum_e ceil(rows_e/32) <= R/32 + E row blocks, times the column tiles
  const int64_t blocks = g.rows > 0 ? (int64_t)g.E * ((g.rows + 31) / 32) : (R + 31) / 32 + g.E;
  const int64_t tiles = blocks * ((C + kQCols - 1) / kQCols);
  if (tiles > 0x7fffffffLL) return cudaErrorInvalidValue;
  const int64_t grid = std::min<int64_t>(tiles, (int64_t)num_sms() * kQCtasPerSm);
  const __nv_bfloat16* xb = reinterpret_cast<const __nv_bfloat16*>(x);
  const bool row = codes_r != nullptr, col = codes_c != nullptr;
  auto kern = row && col ? quant_tile_kernel<true, true>
              : row      ? quant_tile_kernel<true, false>
                         : quant_tile_kernel<false, true>;
  if (!row && !col) return cudaSuccess;
  cudaError_t err =
      cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)kQSmem);
  if (err != cudaSuccess) return err;
  kern<<<(unsigned)grid, kQThreads, kQSmem, s>>>(xb, C, g, row ? perm_f : 0, codes_r, sf_r, codes_c,
                                           sf_c, status);
  return cudaGetLastError();
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
