// Device-scheduled grouped GEMM of the SwiGLU experts on sm_100a tensor cores.
//
// The write-ups describe grouped GEMMs scheduled on the device that run the
// imbalanced per-expert shapes routing produces, measured against padding every
// expert to a common capacity (deniz.in, "Ai2, Olmo-core 3'ü Apache 2.0 ile
// yayınladı", section "Yeni stack nasıl çalışıyor").  Here one persistent kernel
// covers all experts of one GEMM: every CTA reads the expert offsets from device
// memory, builds the tile list itself and walks it; the host never learns the
// per-expert sizes.
//
// Kernel structure (one CTA per SM; the 16-bit and MXFP8 kernels run as CTA pairs,
// cta_group::2, on 256-row tiles):
//   warp 0      TMA producer: 128-byte-swizzled operand tiles into a ring of stages
//               (MXFP8: plus each stage's 512-byte scale chunks)
//   warp 1      tcgen05.mma issuer (one thread of the pair's first CTA) + tensor-memory
//               allocation
//   warps 2..   epilogue (4 warps; 8 for the math-heavy SwiGLU backward and for
//               single-accumulator tiles: two per tensor-memory lane quadrant,
//               splitting the columns): tensor memory -> registers -> fused math ->
//               swizzled shared memory -> TMA bulk tensor stores, one 32x32 chunk at a
//               time
// Two fp32 accumulators of 128 x BN live in tensor memory so the epilogue of one
// tile overlaps the main loop of the next (MXFP8 256-column tiles: one, beside the
// scale columns, released before the stores).
//
// Two groupings:
//   RAGGED_M  forward and dgrad: expert e owns rows [off_e, off_e+1) of the routed
//             activations; tiles of 128 (pairs: 256) rows start at off_e and rows
//             past the expert's end are computed but never stored (a 32-row slice
//             that ends inside the expert is written with plain stores, row by row).
//             Without offsets (null) the whole R rows form one segment.
//   RAGGED_K  wgrad: dW_e = G_e^T . X_e sums over the expert's rows.  G is read
//             through a per-expert tensor map whose row extent ends at the
//             expert's last row (built on the device from the offsets), so the
//             last, partial K-block arrives with its foreign rows zero-filled by
//             the TMA unit.  An expert with no rows writes dW_e = 0.
#include <cuda.h>
#include <cuda_runtime.h>
#include <cuda_bf16.h>
#include <cuda_fp8.h>

#include <mutex>
#include <type_traits>

#include "common.cuh"
#include "internal.h"
#include "mx_block.cuh"
#include "sm100.cuh"

namespace moe {
namespace gemm {

using bf16 = __nv_bfloat16;
using fp8 = __nv_fp8_e4m3;     // MXFP8 operand codes (with E8M0 scales per 32 along K)
using namespace moe::sm100;

enum { RAGGED_M = 0, RAGGED_K = 1 };
enum { EPI_STORE = 0, EPI_SWIGLU_FWD = 1, EPI_SWIGLU_BWD = 2 };

constexpr int BM = 128;
constexpr int kMaxE = 1024;

struct Params {
  const int32_t* offsets;  // [E+1]
  int E, R;
  int M;                   // RAGGED_K: rows of dW_e
  int N;                   // width of the accumulator grid (columns of the output per expert)
  int K;                   // RAGGED_M: reduction length
  int b_rows_per_expert;   // expert e's rows start at e * b_rows_per_expert in B's tensor map
  int f;                   // d_ff (SwiGLU epilogues)
  void* out;               // main output (plain-store path of partial row slices)
  int64_t ldo;             // its row stride in elements
  void* out_a;             // SwiGLU forward: a [R, f]
  int accumulate;          // RAGGED_K: dW += result (float dW only)
  const CUtensorMap* a_maps;  // RAGGED_K: per-expert maps of G (row extent = off_e+1)
  // MXFP8: where each operand's 512-byte scale chunks are (see csrc/mx.cu for the
  // layout).  Chunk of (expert e, M/N index mn, K-stage kb):
  //   k_major: (seg(e) + mn/128) * W + kb     otherwise: (seg(e) + kb) * W + mn/128
  // with seg(e) = e * seg_uniform, or tile_pref[e] when seg_uniform is 0.
  struct Sf {
    const uint8_t* base;
    int seg_uniform;
    int k_major;
    int W;
  } sfa, sfb;
  const int32_t* tile_pref;  // [E+1] prefix of ceil(count_e / 128)
  // MXFP8 SwiGLU forward: also quantise the bf16 a that FC2 reads along its rows into
  // E4M3 codes [R, q_ld] and scale chunks in the quantiser's rowwise layout (null: not
  // asked for)
  uint8_t* q_codes;
  uint8_t* q_sf;
  int q_ld;
  int* status;
  // Test hook (MOE_FLAG_TEST_WAIT_TIMEOUT): the producers issue no loads, so every wait
  // for operands runs out after wait_ns and the kernel takes its abort path.
  int stall;
  uint64_t wait_ns;        // limit of each bounded wait (2 s; 10 ms with the hook)
};

__device__ __forceinline__ int64_t sf_chunk(const Params::Sf& f, const int32_t* tile_pref, int e,
                                            int mn, int kb) {
  const int64_t seg = f.seg_uniform > 0 ? (int64_t)e * f.seg_uniform : (int64_t)tile_pref[e];
  return f.k_major ? (seg + mn / 128) * f.W + kb : (seg + kb) * f.W + mn / 128;
}

// PAIR: a cluster of two CTAs on two SMs computes 256-row tiles with cta_group::2 MMAs;
// each CTA loads its 128 rows of A and half of the BN rows of B, so each SM moves a
// third fewer operand bytes per MMA flop than a lone CTA with a 128 x BN tile.
// KAT: 128-byte K atoms per stage.  Two for the 16-bit ragged-M pair GEMMs whose K allows
// it: a stage then carries eight MMAs instead of four for the same per-stage cost (the
// barrier round trip and the TMA issue of each stage weigh as much as its bytes).
template <typename T, typename OutT, int BN, int EPI, bool PAIR = false, int MODE = RAGGED_M,
          int KAT = 1>
struct Cfg {
  static constexpr int ES = sizeof(T);
  static constexpr int KA = 128 / ES;     // K elements of one 128-byte swizzle row (an atom)
  static constexpr int KB = KA * KAT;     // K elements per stage
  static constexpr int MNB = 128 / ES;    // M/N elements per 128-byte block (M/N-major tiles)
  static constexpr int UK = 32 / ES;      // K of one MMA instruction
  static constexpr int TM = PAIR ? 2 * BM : BM;     // tile rows (M) of the whole cluster
  static constexpr int BNC = PAIR ? BN / 2 : BN;    // rows of B held by one CTA
  static constexpr int A_ATOM = BM * 128;           // one K atom of A (K-major)
  static constexpr int B_ATOM = BNC * 128;          // one K atom of B (K-major)
  static constexpr int A_BYTES = A_ATOM * KAT;
  static constexpr int B_BYTES = B_ATOM * KAT;
  static constexpr int STAGE = A_BYTES + B_BYTES;
  // MXFP8: per stage, one 512-byte scale chunk for this CTA's 128 rows of A and one per
  // 128 rows of the whole BN of B (in a pair each CTA's MMA half reads all of B's scales
  // from its own TMEM)
  static constexpr bool MX = ES == 1;
  static constexpr int SF_CHUNKS_B = MX ? BN / 128 : 0;
  static constexpr int SF_STAGE = MX ? 512 * (1 + SF_CHUNKS_B) : 0;
  static constexpr int SFC = MX ? 4 * (1 + SF_CHUNKS_B) : 0;      // TMEM columns per stage
  // accumulator buffers in TMEM: two (the epilogue drains one while the MMAs fill the
  // other), except for MXFP8 256-column tiles, where the scale columns leave room for one
  static constexpr int NACC = MX && BN == 256 ? 1 : 2;
  static constexpr int TMEM_COLS = MX ? 512 : 2 * BN;
  // 8 epilogue warps for the math-heavy SwiGLU backward (4 leave the MMA waiting there),
  // for single-accumulator tiles (the MMAs wait for the whole epilogue, so it is split
  // over two warps per lane quadrant) and for the wgrads (~8 K-stages a tile leave the
  // epilogue the bottleneck: with 4 warps the MMAs waited on it ~20% of the time);
  // elsewhere 4 warps keep up and leave more shared memory to the operand ring
  static constexpr int EPI_WARPS = EPI == EPI_SWIGLU_BWD || NACC == 1 || MODE == RAGGED_K ? 8 : 4;
  static constexpr int THREADS = 64 + 32 * EPI_WARPS;
  static constexpr int COLGRP = EPI_WARPS / 4;          // warps sharing one lane quadrant
  static constexpr int NCH = BN / 32;                   // 32-column chunks per tile
  static constexpr int WCH = NCH / COLGRP;              // chunks per epilogue warp
  // epilogue shared memory per warp: output staging chunks of 32 rows x 32 columns
  static constexpr int CH = 32 * 32 * sizeof(OutT);
  // (the wgrads' 8 warps take one staging chunk each, so the operand ring keeps 6 stages)
  static constexpr int NBUF = EPI == EPI_SWIGLU_FWD ? 3 : EPI == EPI_SWIGLU_BWD ? 0 : MODE == RAGGED_K ? 1 : 2;
  // SwiGLU backward: slots of prefetched H1/H3 input chunks (32 x 32 each, in the
  // activation type: bf16 for the 16-bit and MXFP8 kernels); the dH1/dH3 results are
  // staged in place in the slot they were computed from
  static constexpr int AES = ES == 4 ? 4 : 2;
  // (one slot per warp: each warp's H1/H3 chunk loads overlap its previous chunk's math,
  // and the 32 KB saved buy the operand ring a fifth stage, which the main loop needs
  // more -- with four it waits on its loads a third of the time)
  static constexpr int IN_SLOTS = EPI == EPI_SWIGLU_BWD ? 1 : 0;
  static constexpr int IN_CH = 2 * 32 * 32 * AES;
  static constexpr int EPI_WARP = ((NBUF * CH + IN_SLOTS * IN_CH) + 1023) / 1024 * 1024;
  static constexpr int EPI_BYTES = EPI_WARPS * EPI_WARP;
  static constexpr int BAR_BYTES = 512;
  static constexpr int BUDGET =
      227 * 1024 - 1024 /*alignment*/ - BAR_BYTES - (2 * (kMaxE + 1) + 8) * 4 - EPI_BYTES;
  static constexpr int STAGES =
      BUDGET / (STAGE + SF_STAGE) > 8 ? 8 : BUDGET / (STAGE + SF_STAGE);
  static_assert(STAGES >= 2, "shared memory budget");
  static_assert(!MX || NACC * BN + STAGES * SFC <= 512, "tensor memory budget");
  static constexpr int SF_COL0 = NACC * BN;                       // first scale column
  static constexpr size_t smem_bytes(int E) {
    return 1024 + size_t(STAGES) * (STAGE + SF_STAGE) + EPI_BYTES + BAR_BYTES +
           size_t(2 * (E + 1) + 8) * 4;
  }
};

struct Tile {
  int e, n0, m0, row0, rows_end, kb, cnt;
};

template <int MODE, int BN, int KB, int TM>
__device__ __forceinline__ Tile decode_tile(int t, int n_tiles, int m_tiles, const int* s_off,
                                            const int* s_mt, int E, int K) {
  Tile tl;
  if (MODE == RAGGED_M) {
    const int mtg = t / n_tiles;
    const int nt = t - mtg * n_tiles;
    int lo = 0, hi = E;                    // s_mt[lo] <= mtg < s_mt[hi]
    while (hi - lo > 1) {
      const int mid = (lo + hi) >> 1;
      if (s_mt[mid] <= mtg) lo = mid; else hi = mid;
    }
    tl.e = lo;
    tl.m0 = (mtg - s_mt[lo]) * TM;
    tl.row0 = s_off[lo] + tl.m0;
    tl.rows_end = s_off[lo + 1];
    tl.n0 = nt * BN;
    tl.kb = K / KB;
    tl.cnt = 0;
  } else {
    const int per = m_tiles * n_tiles;
    const int slot = t / per;
    tl.e = s_mt[slot];               // RAGGED_K: s_mt holds the experts, longest K first
    const int r = t - slot * per;
    const int mt = r / n_tiles;
    tl.m0 = mt * TM;
    tl.n0 = (r - mt * n_tiles) * BN;
    tl.row0 = s_off[tl.e];
    tl.rows_end = s_off[tl.e + 1];
    tl.cnt = tl.rows_end - tl.row0;
    tl.kb = (tl.cnt + KB - 1) / KB;
  }
  return tl;
}

template <typename T>
__device__ __forceinline__ void store32(T* dst, const float* v) {
  constexpr int PER = 16 / sizeof(T);
#pragma unroll
  for (int i = 0; i < 32; i += PER) {
    Vec16<T> pk;
    pk.from_float(v + i);
    stg16(dst + i, pk.raw);
  }
}

// One row of a 32 x 32 staging chunk in shared memory, laid out for a TMA box of
// 32 x 32 elements: 64-byte rows with the 64-byte swizzle (16-bit elements) or 128-byte
// rows with the 128-byte swizzle (32-bit elements).  Thread `r` owns row r; the XOR
// spreads the 32 rows' 16-byte pieces over all banks.
template <typename T>
__device__ __forceinline__ int swz_chunk(int j, int r) {
  return sizeof(T) == 4 ? (j ^ (r & 7)) : (j ^ ((r >> 1) & 3));
}
template <typename T>
__device__ __forceinline__ void stage_row(uint8_t* buf, int r, const float* v) {
  constexpr int RB = 32 * sizeof(T);
  constexpr int PER = 16 / sizeof(T);
  uint8_t* row = buf + r * RB;
#pragma unroll
  for (int j = 0; j < RB / 16; ++j) {
    Vec16<T> pk;
    pk.from_float(v + j * PER);
    *reinterpret_cast<uint4*>(row + swz_chunk<T>(j, r) * 16) = pk.raw;
  }
}
template <typename T>
__device__ __forceinline__ void unstage_row(const uint8_t* buf, int r, float* v) {
  constexpr int RB = 32 * sizeof(T);
  constexpr int PER = 16 / sizeof(T);
  const uint8_t* row = buf + r * RB;
#pragma unroll
  for (int j = 0; j < RB / 16; ++j) {
    Vec16<T> pk;
    pk.raw = *reinterpret_cast<const uint4*>(row + swz_chunk<T>(j, r) * 16);
    pk.to_float(v + j * PER);
  }
}

// Logistic function with the fast exponential and fast division intrinsics; the exponent
// is capped at 80 so the denominator stays finite (the result is then below 1e-34).
__device__ __forceinline__ float sigmoid_f(float z) {
  return __fdividef(1.0f, 1.0f + __expf(fminf(-z, 80.0f)));
}

__device__ __forceinline__ void bits_to_f32(const uint32_t* v, float* f) {
#pragma unroll
  for (int i = 0; i < 32; ++i) f[i] = __uint_as_float(v[i]);
}

// Writes the 32 x 32 chunk held one row per lane through staging buffer `buf` with a TMA
// store (or reduce-add) at (x, y).  `lane 0` owns the bulk groups; before refilling a
// buffer it waits until at most NBUF-1 earlier groups still read shared memory.
template <typename OutT, int NBUF>
__device__ __forceinline__ void staged_store(uint8_t* buf, const float* v, int lane,
                                             const void* tmap, int x, int y, bool reduce) {
  if (lane == 0) bulk_wait_read<NBUF - 1>();
  __syncwarp();
  stage_row<OutT>(buf, lane, v);
  fence_proxy_async_smem();
  __syncwarp();
  if (lane == 0) {
    if (reduce) tma_reduce_add_2d(tmap, buf, x, y);
    else tma_store_2d(tmap, buf, x, y);
    bulk_commit();
  }
}

// The same for a chunk row already packed to bf16 (16 words = 32 values).
template <int NBUF>
__device__ __forceinline__ void staged_store_packed(uint8_t* buf, const uint32_t* w, int lane,
                                                    const void* tmap, int x, int y) {
  if (lane == 0) bulk_wait_read<NBUF - 1>();
  __syncwarp();
  uint8_t* row = buf + lane * 64;
#pragma unroll
  for (int j = 0; j < 4; ++j)
    *reinterpret_cast<uint4*>(row + swz_chunk<bf16>(j, lane) * 16) =
        make_uint4(w[4 * j], w[4 * j + 1], w[4 * j + 2], w[4 * j + 3]);
  fence_proxy_async_smem();
  __syncwarp();
  if (lane == 0) {
    tma_store_2d(tmap, buf, x, y);
    bulk_commit();
  }
}
// 32 floats rounded to bf16 (nearest even), packed two to a word.
__device__ __forceinline__ void pack_bf16x32(const float* v, uint32_t* w) {
#pragma unroll
  for (int j = 0; j < 4; ++j) {
    Vec16<bf16> pk;
    pk.from_float(v + 8 * j);
    w[4 * j] = pk.raw.x;
    w[4 * j + 1] = pk.raw.y;
    w[4 * j + 2] = pk.raw.z;
    w[4 * j + 3] = pk.raw.w;
  }
}
// Rowwise MX block of an epilogue's output row: codes at (row, col) of q_codes and the
// scale in the chunk of (expert e, row p of its segment, column col); col % 32 == 0.
__device__ __forceinline__ void quantise_out_block(const Params& p, int e, int p_seg, int64_t row,
                                                   int col, const uint32_t* w) {
  const int s = mxb::quantise_block32(w, p.q_codes + row * p.q_ld + col);
  const int64_t chunk = ((int64_t)p.tile_pref[e] + p_seg / 128) * (p.q_ld / 128) + col / 128;
  p.q_sf[mxb::sf_byte(chunk, p_seg, (col & 127) >> 5)] = static_cast<uint8_t>(s + 127);
}
__device__ __forceinline__ void store_packed32(bf16* dst, const uint32_t* w) {
#pragma unroll
  for (int j = 0; j < 4; ++j) stg16(dst + 8 * j, make_uint4(w[4 * j], w[4 * j + 1], w[4 * j + 2], w[4 * j + 3]));
}

template <typename T, typename OutT, int BN, bool A_MN, bool B_MN, int MODE, int EPI, bool PAIR,
          int KAT>
__global__ void __launch_bounds__(Cfg<T, OutT, BN, EPI, PAIR, MODE, KAT>::THREADS, 1)
grouped_gemm_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
                    const __grid_constant__ CUtensorMap tmO, const __grid_constant__ CUtensorMap tmO2,
                    const __grid_constant__ CUtensorMap tmI, const __grid_constant__ CUtensorMap tmSA,
                    const __grid_constant__ CUtensorMap tmSB, const Params p) {
  using C = Cfg<T, OutT, BN, EPI, PAIR, MODE, KAT>;
  using ActT = typename std::conditional<sizeof(T) == 4, float, bf16>::type;  // epilogue inputs
  constexpr bool kTF32 = sizeof(T) == 4;
  constexpr bool kMX = C::MX;
  constexpr uint32_t IDESC = kMX ? idesc_mxf8(C::TM, BN, A_MN, B_MN)
                                 : idesc_f32acc(C::TM, BN, kTF32 ? 2u : 1u, A_MN, B_MN);
  static_assert(!(kMX && EPI == EPI_SWIGLU_FWD && !PAIR), "MXFP8 SwiGLU forward: pair tiles");
  static_assert(!PAIR || !kTF32, "CTA pairs run the 16-bit kernels");
  static_assert(!B_MN || C::BNC % C::MNB == 0, "an M/N-major B half is whole 128-byte blocks");
  static_assert(BN == 64 || BN == 128 || BN == 256, "tile width");
  static_assert(MODE == RAGGED_M || (A_MN && B_MN && EPI == EPI_STORE), "wgrad layout");
  static_assert(KAT == 1 || (MODE == RAGGED_M && PAIR && !A_MN && !kMX), "two-atom stages");
  static_assert(KAT == 1 || C::STAGES >= 3, "two-atom stages need a ring of three");

  // a programmatic dependent of the previous kernel: its writes are visible from here on
  pdl_wait();
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~uintptr_t(1023));
  uint8_t* tiles = smem;
  uint8_t* sf_smem = tiles + C::STAGES * C::STAGE;                 // MXFP8 scale chunks
  uint8_t* epi_smem = sf_smem + C::STAGES * C::SF_STAGE;
  uint64_t* full = reinterpret_cast<uint64_t*>(epi_smem + C::EPI_BYTES);
  uint64_t* empty = full + C::STAGES;
  uint64_t* tfull = empty + C::STAGES;
  uint64_t* tempty = tfull + 2;
  uint64_t* fin = tempty + 2;
  uint64_t* in_full = fin + 1;                                   // [EPI_WARPS][IN_SLOTS]
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(full) + C::BAR_BYTES / 4 - 4;
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
  int* s_total = reinterpret_cast<int*>(tmem_slot + 2);
  int* s_off = reinterpret_cast<int*>(reinterpret_cast<uint8_t*>(full) + C::BAR_BYTES);
  int* s_mt = s_off + (p.E + 1);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int E = p.E;
  const int n_tiles = p.N / BN;
  const int m_tiles = MODE == RAGGED_K ? p.M / C::TM : 0;
  // CTA pair: rank 0 (leader) issues the MMAs and owns the shared full/tempty barriers
  const uint32_t rank = PAIR ? cluster_ctarank() : 0u;
  const int unit = PAIR ? static_cast<int>(blockIdx.x >> 1) : static_cast<int>(blockIdx.x);
  const int n_units = PAIR ? static_cast<int>(gridDim.x >> 1) : static_cast<int>(gridDim.x);

  // no offsets: one segment of all R rows (the router GEMMs)
  for (int i = threadIdx.x; i <= E; i += C::THREADS)
    s_off[i] = p.offsets ? p.offsets[i] : (i == 0 ? 0 : p.R);
  __syncthreads();

  if (warp == 0) {
    // Validate the offsets and build the per-expert m-tile prefix (warp scan).
    int ok = 1, carry = 0;
    for (int base = 0; base < E; base += 32) {
      const int e = base + lane;
      int mt = 0;
      if (e < E) {
        const int c = s_off[e + 1] - s_off[e];
        if (c < 0) ok = 0;
        mt = c > 0 ? (c + C::TM - 1) / C::TM : 0;
      }
      int incl = mt;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const int v = __shfl_up_sync(0xffffffffu, incl, o);
        if (lane >= o) incl += v;
      }
      if (e < E) s_mt[e] = carry + incl - mt;
      carry += __shfl_sync(0xffffffffu, incl, 31);
    }
    ok = __all_sync(0xffffffffu, ok);
    if (lane == 0) {
      if (s_off[0] != 0 || s_off[E] != p.R) ok = 0;
      s_mt[E] = carry;
      int total = 0;
      if (ok) total = MODE == RAGGED_M ? carry * n_tiles : E * m_tiles * n_tiles;
      s_total[0] = total;
      if (!ok) set_status(p.status, MOE_DEV_BAD_OFFSETS);
      *abort_flag = 0;
      for (int s = 0; s < C::STAGES; ++s) {
        mbar_init(&full[s], 1);
        mbar_init(&empty[s], 1);
      }
      for (int a = 0; a < 2; ++a) {
        mbar_init(&tfull[a], 1);
        mbar_init(&tempty[a], C::EPI_WARPS * (PAIR ? 2 : 1));
      }
      mbar_init(fin, 1);
      for (int i = 0; i < C::EPI_WARPS * C::IN_SLOTS; ++i) mbar_init(&in_full[i], 1);
      fence_mbar_init();
    }
  }
  __syncthreads();
  if (MODE == RAGGED_K) {
    // Tiles are dealt to the CTAs round-robin, expert by expert.  When the experts' row
    // counts are skewed (the largest above twice the mean), ordering the experts by row
    // count (longest K first, ties to the lower index) keeps the long tiles of hot experts
    // from piling up on a few CTAs; otherwise the experts keep their own order (the
    // layout order of their rows and weights).  (s_mt, the ragged-M tile prefix, is not
    // used by the ragged-K tiles: it holds the order instead.)
    for (int e = threadIdx.x; e < E; e += C::THREADS) {
      const int c = s_off[e + 1] - s_off[e];
      int rank = 0, mx = 0;
      for (int o = 0; o < E; ++o) {
        const int co = s_off[o + 1] - s_off[o];
        rank += co > c || (co == c && o < e);
        mx = co > mx ? co : mx;
      }
      const bool skewed = (int64_t)mx * E > 2 * (int64_t)(s_off[E] - s_off[0]);
      s_mt[skewed ? rank : e] = e;
    }
    __syncthreads();
  }
  const int total = s_total[0];
  if (unit >= total) return;   // uniform over the CTA (and over a CTA pair)

  if (warp == 1) {
    if (PAIR) tmem_alloc_pair(tmem_slot, C::TMEM_COLS);
    else tmem_alloc(tmem_slot, C::TMEM_COLS);
  }
  tc_fence_before();
  if (PAIR) cluster_sync();   // barriers of both CTAs initialised, TMEM allocated
  else __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;
  const bool leader = rank == 0;

  if (warp == 0) {
    // ------------------------------------------------------------------ TMA producer
    if (lane == 0) {
      tma_prefetch_desc(&tmA);
      tma_prefetch_desc(&tmB);
      int acquired_e = -1;   // RAGGED_K: expert whose A tensor map was last acquired
      int stage = 0;
      uint32_t phase = 0;
      uint32_t armed = 0, armed_par = 0;
      bool stop = false;
      // In a pair, both CTAs' loads complete on the leader's full barrier; only the
      // leader arms it (with both CTAs' bytes).  The follower may land its bytes before
      // the leader arms the phase: the transaction count goes transiently negative and
      // the phase still waits for the leader's arrival.
      const uint32_t full_leader = PAIR ? map_to_rank(smem_u32(full), 0) : 0u;
      const int arow = PAIR ? static_cast<int>(rank) * BM : 0;         // my rows of A
      const int bcol = PAIR ? static_cast<int>(rank) * C::BNC : 0;     // my rows of B
      if (p.stall) stop = true;   // test hook: nothing is loaded, nothing is in flight
      for (int t = unit; t < total && !stop; t += n_units) {
        const Tile tl = decode_tile<MODE, BN, C::KB, C::TM>(t, n_tiles, m_tiles, s_off, s_mt, E, p.K);
        for (int kb = 0; kb < tl.kb; ++kb) {
          if (!mbar_wait(&empty[stage], phase ^ 1u, abort_flag, p.status, p.wait_ns)) { stop = true; break; }
          uint8_t* sA = tiles + stage * C::STAGE;
          uint8_t* sB = sA + C::A_BYTES;
          if (leader) {
            mbar_arrive_expect_tx(&full[stage], (C::STAGE + C::SF_STAGE) * (PAIR ? 2 : 1));
            armed |= 1u << stage;
            armed_par = (armed_par & ~(1u << stage)) | (phase << stage);
          }
          const uint32_t fb = full_leader + static_cast<uint32_t>(stage) * 8u;
          auto load = [&](void* dst, const CUtensorMap* tm, int x, int y) {
            if (PAIR) tma_load_2d_pair(dst, tm, fb, x, y);
            else tma_load_2d(dst, tm, &full[stage], x, y);
          };
          const int k0 = kb * C::KB;
          if constexpr (kMX) {
            // this stage's scale chunks (one 512-byte row of a scale map each): my 128 rows
            // of A, then all of B's rows 128 at a time
            uint8_t* sfs = sf_smem + stage * C::SF_STAGE;
            load(sfs, &tmSA, 0, static_cast<int>(sf_chunk(p.sfa, p.tile_pref, tl.e, tl.m0 + arow, kb)));
#pragma unroll
            for (int j = 0; j < C::SF_CHUNKS_B; ++j)
              load(sfs + 512 * (1 + j), &tmSB, 0,
                   static_cast<int>(sf_chunk(p.sfb, p.tile_pref, tl.e, tl.n0 + 128 * j, kb)));
          }
          if (MODE == RAGGED_M) {
#pragma unroll
            for (int at = 0; at < KAT; ++at)
              load(sA + at * C::A_ATOM, &tmA, k0 + at * C::KA, tl.row0 + arow);
            const int brow = tl.e * p.b_rows_per_expert;
            if (!B_MN) {
#pragma unroll
              for (int at = 0; at < KAT; ++at) {
                uint8_t* sBa = sB + at * C::B_ATOM;
                const int ka = k0 + at * C::KA;
                if (EPI == EPI_SWIGLU_FWD) {
                  // B rows: the gate block W1[h0, h0+BN/2) then the up block W3[h0, ...)
                  const int h0 = tl.n0 / 2;
                  if (PAIR) {
                    load(sBa, &tmB, ka, brow + (rank ? p.f : 0) + h0);
                  } else {
                    load(sBa, &tmB, ka, brow + h0);
                    load(sBa + (BN / 2) * 128, &tmB, ka, brow + p.f + h0);
                  }
                } else {
                  load(sBa, &tmB, ka, brow + tl.n0 + bcol);
                }
              }
            } else {
#pragma unroll
              for (int i = 0; i < C::BNC / C::MNB; ++i)
                load(sB + i * C::KB * 128, &tmB, tl.n0 + bcol + i * C::MNB, brow + k0);
            }
          } else {
            const CUtensorMap* am = p.a_maps + tl.e;
            // written by the map-building kernel: acquired once per expert (consecutive
            // tiles share it)
            if (kb == 0 && tl.e != acquired_e) {
              fence_tmap_acquire(am);
              acquired_e = tl.e;
            }
            if constexpr (!kMX) {
              // one request per operand: the maps' third dimension steps through the
              // 128-byte column blocks, so A's (and B's) blocks arrive as consecutive
              // [KB rows x 128 B] slices, the layout of separate 2-D loads
              if (PAIR) {
                tma_load_3d_pair(sA, am, fb, 0, tl.row0 + k0, (tl.m0 + arow) / C::MNB);
                tma_load_3d_pair(sB, &tmB, fb, 0, tl.row0 + k0, (tl.n0 + bcol) / C::MNB);
              } else {
                tma_load_3d(sA, am, &full[stage], 0, tl.row0 + k0, (tl.m0 + arow) / C::MNB);
                tma_load_3d(sB, &tmB, &full[stage], 0, tl.row0 + k0, (tl.n0 + bcol) / C::MNB);
              }
            } else {
#pragma unroll
              for (int i = 0; i < BM / C::MNB; ++i)
                load(sA + i * C::KB * 128, am, tl.m0 + arow + i * C::MNB, tl.row0 + k0);
#pragma unroll
              for (int i = 0; i < C::BNC / C::MNB; ++i)
                load(sB + i * C::KB * 128, &tmB, tl.n0 + bcol + i * C::MNB, tl.row0 + k0);
            }
          }
          if (++stage == C::STAGES) { stage = 0; phase ^= 1u; }
        }
      }
      // Teardown: every armed stage's bytes must have landed before the CTA exits.
      for (int s = 0; s < C::STAGES; ++s)
        if (armed & (1u << s)) mbar_wait_teardown(&full[s], (armed_par >> s) & 1u);
    }
    __syncwarp();
  } else if (warp == 1 && leader) {
    // ------------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      // Descriptors of stage 0; a stage or K step only moves the start-address field
      // (bits [0,14) in 16-byte units; shared addresses stay below 256 KB).
      constexpr uint32_t MN_LAYOUT = kTF32 ? kLayoutSW128Atom32 : kLayoutSW128;
      constexpr uint32_t MN_SBO = kTF32 ? 512 : 1024;   // M/N-major TF32: 4-row K groups
      const uint32_t a0 = smem_u32(tiles);
      const uint64_t a_desc0 = A_MN ? sdesc(a0, C::KB * 128, MN_SBO, MN_LAYOUT)
                                    : sdesc(a0, 16, 1024, kLayoutSW128);
      const uint64_t b_desc0 = B_MN ? sdesc(a0 + C::A_BYTES, C::KB * 128, MN_SBO, MN_LAYOUT)
                                    : sdesc(a0 + C::A_BYTES, 16, 1024, kLayoutSW128);
      constexpr uint32_t A_STEP = (A_MN ? C::UK * 128 : 32) >> 4;   // per MMA along K
      constexpr uint32_t B_STEP = (B_MN ? C::UK * 128 : 32) >> 4;
      int stage = 0;
      uint32_t phase = 0;
      int acc = 0;
      uint32_t acc_phase = 0;
      bool stop = false;
      for (int t = unit; t < total && !stop; t += n_units) {
        const Tile tl =
            decode_tile<MODE, BN, C::KB, C::TM>(t, n_tiles, m_tiles, s_off, s_mt, E, p.K);
        if (!mbar_wait(&tempty[acc], acc_phase ^ 1u, abort_flag, p.status, p.wait_ns)) break;
        tc_fence_after();
        const uint32_t d_tmem = tmem_base + static_cast<uint32_t>(acc * BN);
        for (int kb = 0; kb < tl.kb; ++kb) {
          if (!mbar_wait(&full[stage], phase, abort_flag, p.status, p.wait_ns)) { stop = true; break; }
          tc_fence_after();
          const uint32_t so = static_cast<uint32_t>(stage * C::STAGE) >> 4;
          uint32_t sfa_t = 0, sfb_t = 0;
          if constexpr (kMX) {
            // scales of this stage into its TMEM slot (4 columns per 512-byte chunk); the
            // MMAs below run after these copies (same issuing thread)
            const uint32_t col = static_cast<uint32_t>(C::SF_COL0 + stage * C::SFC);
            const uint32_t src = smem_u32(sf_smem + stage * C::SF_STAGE);
            sfa_t = tmem_base + col;
            sfb_t = tmem_base + col + 4;
#pragma unroll
            for (int j = 0; j <= C::SF_CHUNKS_B; ++j) {
              if (PAIR) tmem_cp_scales_pair(tmem_base + col + 4 * j, sdesc(src + 512 * j, 128, 128, 0));
              else tmem_cp_scales(tmem_base + col + 4 * j, sdesc(src + 512 * j, 128, 128, 0));
            }
          }
          // K-major operands: MMA kk reads atom kk / KPA at K offset kk % KPA; M/N-major
          // ones hold the stage's K rows contiguously in each 128-byte block
          constexpr int KPA = C::KA / C::UK;
#pragma unroll
          for (int kk = 0; kk < C::KB / C::UK; ++kk) {
            const uint32_t a_off = A_MN ? kk * A_STEP
                                        : (kk / KPA) * (C::A_ATOM >> 4) + (kk % KPA) * A_STEP;
            const uint32_t b_off = B_MN ? kk * B_STEP
                                        : (kk / KPA) * (C::B_ATOM >> 4) + (kk % KPA) * B_STEP;
            const uint64_t ad = a_desc0 + so + a_off;
            const uint64_t bd = b_desc0 + so + b_off;
            const uint32_t accum = (kb | kk) != 0 ? 1u : 0u;
            if constexpr (kMX) {
              if (PAIR) umma_mx_pair(d_tmem, ad, bd, IDESC | idesc_sf_ids(kk, kk), sfa_t, sfb_t, accum);
              else umma_mx(d_tmem, ad, bd, IDESC | idesc_sf_ids(kk, kk), sfa_t, sfb_t, accum);
            } else if (PAIR) umma_pair(d_tmem, ad, bd, IDESC, accum);
            else umma<kTF32>(d_tmem, ad, bd, IDESC, accum);
          }
          if (PAIR) umma_commit_pair(&empty[stage], 3);   // frees the stage in both CTAs
          else umma_commit(&empty[stage]);
          if (++stage == C::STAGES) { stage = 0; phase ^= 1u; }
        }
        // an aborted tile is never handed to the epilogue (its accumulator is incomplete);
        // the epilogue warps see the abort flag or time out themselves
        if (stop) break;
        if (PAIR) umma_commit_pair(&tfull[acc], 3);
        else umma_commit(&tfull[acc]);
        if (++acc == C::NACC) { acc = 0; acc_phase ^= 1u; }
      }
      // (a kernel's tcgen05 instructions all use one cta_group)
      if (PAIR) umma_commit_pair(fin, 1);
      else umma_commit(fin);
      mbar_wait_teardown(fin, 0);
    }
    __syncwarp();
  } else if (warp >= 2) {
    // ------------------------------------------------------------------ epilogue
    const int q = warp & 3;                 // tensor-memory lane quadrant of this warp
    const int ew = warp - 2;                // epilogue warp index (shared-memory slice)
    const int cg = ew >> 2;                 // column group: chunks [cg*WCH, (cg+1)*WCH)
    uint8_t* stage_buf = epi_smem + ew * C::EPI_WARP;
    uint8_t* in_buf = stage_buf + C::NBUF * C::CH;
    constexpr int INS = C::IN_SLOTS > 0 ? C::IN_SLOTS : 1;   // slot-ring modulus
    uint64_t* my_in_full = in_full + ew * INS;
    int sbuf = 0;
    uint32_t in_issued = 0, in_used = 0;    // SwiGLU-backward input chunks
    int acc = 0;
    uint32_t acc_phase = 0;
    uint32_t v[32];
    float fv[32];
    const uint32_t tempty_leader = PAIR ? map_to_rank(smem_u32(tempty), 0) : 0u;
    const int myrow = PAIR ? static_cast<int>(rank) * BM : 0;      // my 128 rows of the tile
    for (int t = unit; t < total; t += n_units) {
      const Tile tl = decode_tile<MODE, BN, C::KB, C::TM>(t, n_tiles, m_tiles, s_off, s_mt, E, p.K);
      const int rbase = MODE == RAGGED_M ? tl.row0 + myrow + q * 32 : 0;   // first row of my slice
      int nvalid = 32;
      if (MODE == RAGGED_M) {
        nvalid = tl.rows_end - rbase;
        nvalid = nvalid < 0 ? 0 : (nvalid > 32 ? 32 : nvalid);
      }
      const bool whole = nvalid == 32;
      const int cfirst = cg * C::WCH;       // my first 32-column chunk
      if (EPI == EPI_SWIGLU_BWD && nvalid > 0) {
        // prefetch this slice's H1/H3 chunks while the main loop still runs (the slots'
        // previous results must have been read out by their TMA stores first)
        if (lane == 0) {
          bulk_wait_read<0>();
          for (int i = 0; i < C::WCH && i < C::IN_SLOTS; ++i) {
            const int slot = in_issued % INS;
            const int x = tl.n0 + (cfirst + i) * 32;
            uint8_t* dst = in_buf + slot * C::IN_CH;
            mbar_arrive_expect_tx(&my_in_full[slot], C::IN_CH);
            tma_load_2d(dst, &tmI, &my_in_full[slot], x, rbase);
            tma_load_2d(dst + C::IN_CH / 2, &tmI, &my_in_full[slot], p.f + x, rbase);
            ++in_issued;
          }
        }
        in_issued = __shfl_sync(0xffffffffu, in_issued, 0);
      }
      if (!mbar_wait_warp(&tfull[acc], acc_phase, abort_flag, p.status, p.wait_ns)) break;
      tc_fence_after();
      const uint32_t tb = tmem_base + (static_cast<uint32_t>(q * 32) << 16) +
                          static_cast<uint32_t>(acc * BN);
      if constexpr (C::NACC == 1 && EPI != EPI_SWIGLU_BWD && sizeof(OutT) == 2) {
        // One accumulator: the next tile's MMAs wait for it.  Pull this warp's columns
        // into registers (rounded to the bf16 outputs), free the accumulator, and only
        // then stage and store them, so the stores overlap the next tile's main loop.
        constexpr int RCH = EPI == EPI_SWIGLU_FWD ? (BN / 2 / C::COLGRP) / 32 : C::WCH;
        uint32_t pk[EPI == EPI_SWIGLU_FWD ? 3 : 1][RCH][16];
        const int c_sw = cg * RCH * 32;     // SwiGLU: my first gate (and up) column
        bool any = true;                    // RAGGED_K: this tile has rows (else dW = 0)
        if (MODE == RAGGED_K) any = tl.kb > 0;
#pragma unroll
        for (int i = 0; i < RCH; ++i) {
          if (EPI == EPI_SWIGLU_FWD) {
            uint32_t v3[32];
            float h3[32], av[32];
            tmem_ld32(tb + c_sw + 32 * i, v);
            tmem_ld32(tb + BN / 2 + c_sw + 32 * i, v3);
            tmem_ld_wait();
            reg_fence32(v);
            reg_fence32(v3);
            bits_to_f32(v, fv);
            bits_to_f32(v3, h3);
#pragma unroll
            for (int j = 0; j < 32; ++j) av[j] = fv[j] * sigmoid_f(fv[j]) * h3[j];
            pack_bf16x32(fv, pk[0][i]);
            pack_bf16x32(h3, pk[EPI == EPI_SWIGLU_FWD ? 1 : 0][i]);
            pack_bf16x32(av, pk[EPI == EPI_SWIGLU_FWD ? 2 : 0][i]);
          } else {
            if (any) {
              tmem_ld32(tb + (cfirst + i) * 32, v);
              tmem_ld_wait();
              reg_fence32(v);
              bits_to_f32(v, fv);
            } else {
#pragma unroll
              for (int j = 0; j < 32; ++j) fv[j] = 0.f;
            }
            pack_bf16x32(fv, pk[0][i]);
          }
        }
        tc_fence_before();
        __syncwarp();
        if (lane == 0) {
          if (PAIR) mbar_arrive_remote(tempty_leader + static_cast<uint32_t>(acc) * 8u);
          else mbar_arrive(&tempty[acc]);
        }
        if (MODE == RAGGED_M) {
          const int64_t grow = rbase + lane;
          const bool valid = lane < nvalid;
          if (nvalid > 0) {
#pragma unroll
            for (int i = 0; i < RCH; ++i) {
              if (EPI == EPI_SWIGLU_FWD) {
                const int hc = tl.n0 / 2 + c_sw + 32 * i;   // H1/a column
                if (whole) {
                  staged_store_packed<C::NBUF>(stage_buf + 0 * C::CH, pk[0][i], lane, &tmO, hc, rbase);
                  staged_store_packed<C::NBUF>(stage_buf + 1 * C::CH, pk[EPI == EPI_SWIGLU_FWD ? 1 : 0][i],
                                               lane, &tmO, p.f + hc, rbase);
                  staged_store_packed<C::NBUF>(stage_buf + 2 * C::CH, pk[EPI == EPI_SWIGLU_FWD ? 2 : 0][i],
                                               lane, &tmO2, hc, rbase);
                } else if (valid) {
                  bf16* h13 = reinterpret_cast<bf16*>(p.out) + grow * (2 * (int64_t)p.f) + hc;
                  store_packed32(h13, pk[0][i]);
                  store_packed32(h13 + p.f, pk[EPI == EPI_SWIGLU_FWD ? 1 : 0][i]);
                  store_packed32(reinterpret_cast<bf16*>(p.out_a) + grow * (int64_t)p.f + hc,
                                 pk[EPI == EPI_SWIGLU_FWD ? 2 : 0][i]);
                }
                if (kMX && p.q_codes && valid)
                  quantise_out_block(p, tl.e, tl.m0 + myrow + q * 32 + lane, grow, hc,
                                     pk[EPI == EPI_SWIGLU_FWD ? 2 : 0][i]);
              } else {
                const int c = (cfirst + i) * 32;
                if (whole) {
                  staged_store_packed<C::NBUF>(stage_buf + sbuf * C::CH, pk[0][i], lane, &tmO,
                                               tl.n0 + c, rbase);
                  sbuf = sbuf + 1 == C::NBUF ? 0 : sbuf + 1;
                } else if (valid) {
                  store_packed32(reinterpret_cast<bf16*>(p.out) + grow * p.ldo + tl.n0 + c, pk[0][i]);
                }
              }
            }
          }
        } else {
          const int y = tl.e * p.M + tl.m0 + myrow + q * 32;
#pragma unroll
          for (int i = 0; i < RCH; ++i) {
            staged_store_packed<C::NBUF>(stage_buf + sbuf * C::CH, pk[0][i], lane, &tmO,
                                         tl.n0 + (cfirst + i) * 32, y);
            sbuf = sbuf + 1 == C::NBUF ? 0 : sbuf + 1;
          }
        }
        if (++acc == C::NACC) { acc = 0; acc_phase ^= 1u; }
        continue;
      }
      if (MODE == RAGGED_M) {
        const int64_t grow = rbase + lane;
        const bool valid = lane < nvalid;
        if (nvalid > 0) {
          if (EPI == EPI_STORE) {
#pragma unroll 1
            for (int c = cfirst * 32; c < (cfirst + C::WCH) * 32; c += 32) {
              tmem_ld32(tb + c, v);
              tmem_ld_wait();
              reg_fence32(v);
              bits_to_f32(v, fv);
              if (whole) {
                staged_store<OutT, C::NBUF>(stage_buf + sbuf * C::CH, fv, lane, &tmO, tl.n0 + c,
                                            rbase, false);
                sbuf = sbuf + 1 == C::NBUF ? 0 : sbuf + 1;
              } else if (valid) {
                store32<OutT>(reinterpret_cast<OutT*>(p.out) + grow * p.ldo + tl.n0 + c, fv);
              }
            }
          } else if (EPI == EPI_SWIGLU_FWD) {
            const int h0 = tl.n0 / 2;
            uint32_t v3[32];
            float h3[32], av[32];
            constexpr int HW = BN / 2 / C::COLGRP;   // gate (and up) columns of this warp
#pragma unroll 1
            for (int c = cg * HW; c < (cg + 1) * HW; c += 32) {
              tmem_ld32(tb + c, v);
              tmem_ld32(tb + BN / 2 + c, v3);
              tmem_ld_wait();
              reg_fence32(v);
              reg_fence32(v3);
              bits_to_f32(v, fv);
              bits_to_f32(v3, h3);
#pragma unroll
              for (int i = 0; i < 32; ++i) av[i] = fv[i] * sigmoid_f(fv[i]) * h3[i];
              if constexpr (kTF32) {
                // a feeds TF32 GEMMs only (FC2, FC2 wgrad): stored rounded to TF32
#pragma unroll
                for (int i = 0; i < 32; ++i) av[i] = tf32_round(av[i]);
              }
              if (whole) {
                staged_store<OutT, C::NBUF>(stage_buf + 0 * C::CH, fv, lane, &tmO, h0 + c, rbase,
                                            false);
                staged_store<OutT, C::NBUF>(stage_buf + 1 * C::CH, h3, lane, &tmO, p.f + h0 + c,
                                            rbase, false);
                staged_store<OutT, C::NBUF>(stage_buf + 2 * C::CH, av, lane, &tmO2, h0 + c, rbase,
                                            false);
              } else if (valid) {
                OutT* h13 = reinterpret_cast<OutT*>(p.out) + grow * (2 * (int64_t)p.f) + h0 + c;
                store32<OutT>(h13, fv);
                store32<OutT>(h13 + p.f, h3);
                store32<OutT>(reinterpret_cast<OutT*>(p.out_a) + grow * (int64_t)p.f + h0 + c, av);
              }
            }
          } else {  // EPI_SWIGLU_BWD: accumulator = dA; H1/H3 prefetched in in_buf
            float h1[32], h3[32], d3[32];
#pragma unroll 1
            for (int i = 0; i < C::WCH; ++i) {
              const int c = (cfirst + i) * 32;
              const int slot = in_used % INS;
              const uint32_t par = (in_used / INS) & 1u;
              tmem_ld32(tb + c, v);
              tmem_ld_wait();
              reg_fence32(v);
              bits_to_f32(v, fv);
              if (!mbar_wait_warp(&my_in_full[slot], par, abort_flag, p.status, p.wait_ns)) break;
              uint8_t* sl = in_buf + slot * C::IN_CH;
              unstage_row<ActT>(sl, lane, h1);
              unstage_row<ActT>(sl + C::IN_CH / 2, lane, h3);
              ++in_used;
#pragma unroll
              for (int j = 0; j < 32; ++j) {
                const float sg = sigmoid_f(h1[j]);
                const float da = fv[j];
                d3[j] = da * h1[j] * sg;
                fv[j] = da * h3[j] * sg * (1.0f + h1[j] * (1.0f - sg));
                if constexpr (kTF32) {
                  // dH13 feeds TF32 GEMMs only (FC1 dgrad, FC1 wgrad): rounded to TF32
                  d3[j] = tf32_round(d3[j]);
                  fv[j] = tf32_round(fv[j]);
                }
              }
              if (whole) {
                // each lane rewrites only the row it read, so no barrier is needed first
                stage_row<OutT>(sl, lane, fv);
                stage_row<OutT>(sl + C::IN_CH / 2, lane, d3);
                fence_proxy_async_smem();
                __syncwarp();
                if (lane == 0) {
                  tma_store_2d(&tmO, sl, tl.n0 + c, rbase);
                  tma_store_2d(&tmO, sl + C::IN_CH / 2, p.f + tl.n0 + c, rbase);
                  bulk_commit();
                }
              } else if (valid) {
                OutT* dh = reinterpret_cast<OutT*>(p.out) + grow * (2 * (int64_t)p.f) + tl.n0 + c;
                store32<OutT>(dh, fv);
                store32<OutT>(dh + p.f, d3);
              }
              if (i + C::IN_SLOTS < C::WCH) {
                // refill the slot with the chunk IN_SLOTS ahead once its stores read it out
                __syncwarp();
                if (lane == 0) {
                  bulk_wait_read<0>();
                  const int x = tl.n0 + (cfirst + i + C::IN_SLOTS) * 32;
                  mbar_arrive_expect_tx(&my_in_full[slot], C::IN_CH);
                  tma_load_2d(sl, &tmI, &my_in_full[slot], x, rbase);
                  tma_load_2d(sl + C::IN_CH / 2, &tmI, &my_in_full[slot], p.f + x, rbase);
                }
                ++in_issued;
              }
            }
          }
        }
      } else {
        // RAGGED_K: dW_e[m0 + 32q .. +32, n0 .. n0 + BN), a [E*M, N] tensor
        const bool has = tl.kb > 0;
        const int y = tl.e * p.M + tl.m0 + myrow + q * 32;
        if (has || !p.accumulate) {
#pragma unroll 1
          for (int c = cfirst * 32; c < (cfirst + C::WCH) * 32; c += 32) {
            if (has) {
              tmem_ld32(tb + c, v);
              tmem_ld_wait();
              reg_fence32(v);
              bits_to_f32(v, fv);
            } else {
#pragma unroll
              for (int i = 0; i < 32; ++i) fv[i] = 0.f;
            }
            staged_store<OutT, C::NBUF>(stage_buf + sbuf * C::CH, fv, lane, &tmO, tl.n0 + c, y,
                                        p.accumulate != 0);
            sbuf = sbuf + 1 == C::NBUF ? 0 : sbuf + 1;
          }
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) {
        if (PAIR) mbar_arrive_remote(tempty_leader + static_cast<uint32_t>(acc) * 8u);
        else mbar_arrive(&tempty[acc]);
      }
      if (++acc == C::NACC) { acc = 0; acc_phase ^= 1u; }
    }
    if (lane == 0) {
      bulk_wait_all();
      // input chunks still in flight (only after an abort) must land before exit
      for (; in_used < in_issued; ++in_used)
        mbar_wait_teardown(&my_in_full[in_used % INS], (in_used / INS) & 1u);
    }
    __syncwarp();
  }

  pdl_trigger();   // this CTA's tiles are done
  // A pair's leader reads the follower's shared memory and writes its TMEM until its
  // last MMA completes (the leader waited for that above): neither CTA leaves before.
  tc_fence_before();
  if (PAIR) cluster_sync();
  else __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    if (PAIR) tmem_dealloc_pair(tmem_base, C::TMEM_COLS);
    else tmem_dealloc(tmem_base, C::TMEM_COLS);
  }
}

// Per-expert views of G [R, M] for the ragged-K wgrad: maps[e] = tmpl with its row
// extent cut at off_e+1, so TMA zero-fills every row past expert e's last one.  (A view
// needs at least one row; an expert with no rows never loads through its map.)
__global__ void expert_maps_kernel(const __grid_constant__ CUtensorMap tmpl0,
                                   const __grid_constant__ CUtensorMap tmpl1,
                                   const int32_t* __restrict__ offsets, int E, int R,
                                   CUtensorMap* maps) {
  pdl_wait();
  const int i = blockIdx.x * blockDim.x + threadIdx.x;
  if (i >= 2 * E) return;
  const int e = i < E ? i : i - E;
  const uint4* src = reinterpret_cast<const uint4*>(i < E ? &tmpl0 : &tmpl1);
  uint4* dst = reinterpret_cast<uint4*>(maps + i);
#pragma unroll
  for (int j = 0; j < 8; ++j) dst[j] = src[j];
  const int rows = offsets ? offsets[e + 1] : R;   // no offsets: one segment of R rows
  tmap_replace_row_dim(maps + i, static_cast<uint32_t>(rows > 0 ? rows : 1));
  fence_tmap_release();
  pdl_trigger();
}

// =============================================================================== host side

typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                  const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                  const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                  CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

static EncodeTiledFn encode_fn() {
  static EncodeTiledFn fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* ptr = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(ptr);
  });
  return fn;
}

enum class Box { KMajor, MNMajor, Chunk };

// MXFP8 scale chunks as a 2-D map of `chunks` rows of 512 bytes (128 x uint32), one row
// per box: a scale load is a TMA load of row `chunk` (x = 0), so it can complete on the
// pair leader's barrier like the operand tiles.
static bool make_sf_map(CUtensorMap* m, const void* base, int64_t chunks) {
  EncodeTiledFn enc = encode_fn();
  if (!enc || chunks < 1) return false;
  cuuint64_t dims[2] = {128, static_cast<cuuint64_t>(chunks)};
  cuuint64_t strides[1] = {512};
  cuuint32_t box[2] = {128, 1};
  cuuint32_t estr[2] = {1, 1};
  return enc(m, CU_TENSOR_MAP_DATA_TYPE_UINT32, 2, const_cast<void*>(base), dims, strides, box,
             estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE,
             CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// 2-D row-major tensor [rows, cols] of bf16 or fp32 with box [box_rows, box_cols]:
//   KMajor / MNMajor operand tiles: 128-byte rows, 128-byte swizzle (M/N-major fp32
//   tiles: the 32-byte-atom variant, the layout the tensor core takes for M/N-major
//   TF32 operands);
//   Chunk: 32 x 32 epilogue chunks, 64-byte swizzle for 16-bit, 128-byte for 32-bit.
static bool make_tmap(CUtensorMap* m, const void* base, int es_, uint64_t cols, uint64_t rows,
                      uint32_t box_cols, uint32_t box_rows, Box kind) {
  EncodeTiledFn enc = encode_fn();
  if (!enc) return false;
  const uint64_t es = static_cast<uint64_t>(es_);
  const bool fp32 = es == 4;
  cuuint64_t dims[2] = {cols, rows};
  cuuint64_t strides[1] = {cols * es};
  cuuint32_t box[2] = {box_cols, box_rows};
  cuuint32_t estr[2] = {1, 1};
  CUtensorMapSwizzle swz = CU_TENSOR_MAP_SWIZZLE_128B;
  if (kind == Box::MNMajor && fp32) swz = CU_TENSOR_MAP_SWIZZLE_128B_ATOM_32B;
  if (kind == Box::Chunk && !fp32) swz = CU_TENSOR_MAP_SWIZZLE_64B;
  const CUtensorMapDataType dt = es == 4   ? CU_TENSOR_MAP_DATA_TYPE_FLOAT32
                                 : es == 2 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16
                                           : CU_TENSOR_MAP_DATA_TYPE_UINT8;
  CUresult r = enc(m, dt, 2,
                   const_cast<void*>(base), dims, strides, box, estr,
                   CU_TENSOR_MAP_INTERLEAVE_NONE, swz, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                   CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

// M/N-major operand [rows, cols] (bf16 or fp32, cols a multiple of 128 bytes) as a 3-D
// map {128-byte column block, rows, blocks}: strides {cols * es, 128 B}, box {one block,
// box_rows, nblk}.  One load brings nblk consecutive column blocks of box_rows rows,
// each as its own [box_rows x 128 B] slice, swizzled like the 2-D M/N-major tiles.
static bool make_tmap_mn3(CUtensorMap* m, const void* base, int es_, uint64_t cols,
                          uint64_t rows, uint32_t box_rows, uint32_t nblk) {
  EncodeTiledFn enc = encode_fn();
  if (!enc) return false;
  const uint64_t es = static_cast<uint64_t>(es_);
  const uint64_t blk = 128 / es;                       // elements per column block
  cuuint64_t dims[3] = {blk, rows, cols / blk};
  cuuint64_t strides[2] = {cols * es, 128};
  cuuint32_t box[3] = {static_cast<cuuint32_t>(blk), box_rows, nblk};
  cuuint32_t estr[3] = {1, 1, 1};
  const bool fp32 = es == 4;
  const CUtensorMapSwizzle swz =
      fp32 ? CU_TENSOR_MAP_SWIZZLE_128B_ATOM_32B : CU_TENSOR_MAP_SWIZZLE_128B;
  const CUtensorMapDataType dt =
      fp32 ? CU_TENSOR_MAP_DATA_TYPE_FLOAT32 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16;
  return enc(m, dt, 3, const_cast<void*>(base), dims, strides, box, estr,
             CU_TENSOR_MAP_INTERLEAVE_NONE, swz, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
             CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

template <typename T, typename OutT, int BN, bool A_MN, bool B_MN, int MODE, int EPI, bool PAIR,
          int KAT = 1>
static moe_status launch(const CUtensorMap& ta, const CUtensorMap& tb, const CUtensorMap& to,
                         const CUtensorMap& to2, const CUtensorMap& ti, const CUtensorMap& tsa,
                         const CUtensorMap& tsb, const Params& p, int max_tiles, cudaStream_t s) {
  using C = Cfg<T, OutT, BN, EPI, PAIR, MODE, KAT>;
  auto kern = grouped_gemm_kernel<T, OutT, BN, A_MN, B_MN, MODE, EPI, PAIR, KAT>;
  const size_t smem = C::smem_bytes(p.E);
  if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           static_cast<int>(smem)) != cudaSuccess)
    return MOE_ECUDA;
  cudaLaunchConfig_t cfg = {};
  cudaLaunchAttribute attr[2];
  cfg.blockDim = dim3(C::THREADS, 1, 1);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = s;
  cfg.attrs = attr;
  int units = num_sms();
  if (PAIR) {
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = 2;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.numAttrs = 1;
    // how many CTA pairs fit at once (one CTA per SM: the shared memory takes it all)
    static int max_pairs[64] = {0};
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return MOE_ECUDA;
    if (max_pairs[dev] == 0) {
      cfg.gridDim = dim3(2, 1, 1);
      int n = 0;
      if (cudaOccupancyMaxActiveClusters(&n, kern, &cfg) != cudaSuccess || n < 1) n = num_sms() / 2;
      max_pairs[dev] = n;
    }
    units = max_pairs[dev];
  }
  if (max_tiles < units) units = max_tiles;
  if (units < 1) return MOE_OK;
  // a programmatic dependent of the previous kernel (the kernel waits for it itself)
  attr[cfg.numAttrs].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[cfg.numAttrs].val.programmaticStreamSerializationAllowed = 1;
  ++cfg.numAttrs;
  cfg.gridDim = dim3(PAIR ? 2 * units : units, 1, 1);
  if (cudaLaunchKernelEx(&cfg, kern, ta, tb, to, to2, ti, tsa, tsb, p) != cudaSuccess)
    return MOE_ECUDA;
  return cudaGetLastError() == cudaSuccess ? MOE_OK : MOE_ECUDA;
}

static int pick_bn(int n) { return n % 256 == 0 ? 256 : n % 128 == 0 ? 128 : 64; }

// Upper bound of the ragged-M tile count: sum_e ceil(cnt_e / TM) <= R / TM + E.
static int ragged_m_tiles(const GemmShape& g, int n_tiles, int tm) {
  const long long mt = (long long)g.R / tm + g.E;
  const long long t = mt * n_tiles;
  return t > (1 << 30) ? (1 << 30) : static_cast<int>(t);
}

// RAGGED_M GEMM, A K-major [R, K] act, B K-major weights [E*N_rows, K] (B_MN = false)
// or M/N-major weights [E*K, N] (B_MN = true).  Output `out` [R, out_cols]; SwiGLU
// forward also writes out_a [R, f]; SwiGLU backward reads aux [R, 2f].
struct MxRefs {             // MXFP8 scale chunks of both operands (unused otherwise)
  Params::Sf a{}, b{};
  int64_t a_chunks = 0, b_chunks = 0;   // sizes of the two scale buffers in chunks
  const int32_t* tile_pref = nullptr;
  uint8_t* q_codes = nullptr;           // SwiGLU forward: rowwise codes of a
  uint8_t* q_sf = nullptr;
  int q_ld = 0;
};

// Scale maps of an MXFP8 GEMM (copies of `dummy` for the other kernels, which never
// read them).
static bool sf_maps(const MxRefs& mx, bool is_mx, const CUtensorMap& dummy, CUtensorMap* tsa,
                    CUtensorMap* tsb) {
  if (!is_mx) {
    *tsa = dummy;
    *tsb = dummy;
    return true;
  }
  return make_sf_map(tsa, mx.a.base, mx.a_chunks) && make_sf_map(tsb, mx.b.base, mx.b_chunks);
}

template <typename T, bool B_MN, int EPI, int BN, bool PAIR, typename OutT = T, int KAT = 1>
static moe_status run_m(const GemmShape& g, const void* A, int K, const void* B, int N,
                        int b_rows_per_expert, int b_cols, void* out, int out_cols, void* out_a,
                        const void* aux, const int32_t* offsets, int* status, cudaStream_t s,
                        const MxRefs& mx = MxRefs()) {
  using C = Cfg<T, OutT, BN, EPI, PAIR, RAGGED_M, KAT>;
  constexpr int ES = sizeof(T);
  constexpr int OES = sizeof(OutT);
  if (K % C::KB != 0) return MOE_EINVAL;
  CUtensorMap ta, tb, to, to2, ti;
  if (!make_tmap(&ta, A, ES, K, g.R, C::KA, BM, Box::KMajor)) return MOE_ECUDA;
  if (!B_MN) {
    const int box_rows = EPI == EPI_SWIGLU_FWD ? BN / 2 : C::BNC;
    if (!make_tmap(&tb, B, ES, K, (uint64_t)g.E * b_rows_per_expert, C::KA, box_rows,
                   Box::KMajor))
      return MOE_ECUDA;
  } else {
    if (!make_tmap(&tb, B, ES, b_cols, (uint64_t)g.E * b_rows_per_expert, C::MNB, C::KB,
                   Box::MNMajor))
      return MOE_ECUDA;
  }
  if (!make_tmap(&to, out, OES, out_cols, g.R, 32, 32, Box::Chunk)) return MOE_ECUDA;
  to2 = to;
  ti = to;
  if (EPI == EPI_SWIGLU_FWD && !make_tmap(&to2, out_a, OES, g.f, g.R, 32, 32, Box::Chunk))
    return MOE_ECUDA;
  if (EPI == EPI_SWIGLU_BWD && !make_tmap(&ti, aux, OES, 2 * (uint64_t)g.f, g.R, 32, 32,
                                          Box::Chunk))
    return MOE_ECUDA;
  Params p{};
  p.offsets = offsets;
  p.E = g.E;
  p.R = g.R;
  p.N = N;
  p.K = K;
  p.b_rows_per_expert = b_rows_per_expert;
  p.f = g.f;
  p.out = out;
  p.ldo = out_cols;
  p.out_a = out_a;
  p.sfa = mx.a;
  p.sfb = mx.b;
  p.tile_pref = mx.tile_pref;
  p.q_codes = mx.q_codes;
  p.q_sf = mx.q_sf;
  p.q_ld = mx.q_ld;
  p.status = status;
  p.stall = g.test_stall ? 1 : 0;
  p.wait_ns = g.test_stall ? 10000000ull : kWaitLimitNs;
  CUtensorMap tsa, tsb;
  if (!sf_maps(mx, C::MX, ta, &tsa, &tsb)) return MOE_ECUDA;
  return launch<T, OutT, BN, false, B_MN, RAGGED_M, EPI, PAIR, KAT>(
      ta, tb, to, to2, ti, tsa, tsb, p, ragged_m_tiles(g, N / BN, C::TM), s);
}

// RAGGED_K GEMM: dW_e[M, N] = G_e^T . X_e with G [R, M] and X [R, N] (both act, M/N-major).
template <typename T, typename OutT, int BN, bool PAIR>
static moe_status run_k(const GemmShape& g, const void* G, int M, const void* X, int N, void* dW,
                        bool accum, const int32_t* offsets, const CUtensorMap* g_maps,
                        int* status, cudaStream_t s, const MxRefs& mx = MxRefs()) {
  using C = Cfg<T, OutT, BN, EPI_STORE, PAIR, RAGGED_K>;
  constexpr int ES = sizeof(T);
  CUtensorMap ta, tb, to;
  if constexpr (C::MX) {
    if (!make_tmap(&ta, G, ES, M, g.R, C::MNB, C::KB, Box::MNMajor)) return MOE_ECUDA;
    if (!make_tmap(&tb, X, ES, N, g.R, C::MNB, C::KB, Box::MNMajor)) return MOE_ECUDA;
  } else {
    // 16-bit / fp32: one 3-D request per operand and stage (the kernel's wgrad loads)
    if (!make_tmap_mn3(&ta, G, ES, M, g.R, C::KB, BM / C::MNB)) return MOE_ECUDA;
    if (!make_tmap_mn3(&tb, X, ES, N, g.R, C::KB, C::BNC / C::MNB)) return MOE_ECUDA;
  }
  if (!make_tmap(&to, dW, (int)sizeof(OutT), N, (uint64_t)g.E * M, 32, 32, Box::Chunk))
    return MOE_ECUDA;
  Params p{};
  p.offsets = offsets;
  p.E = g.E;
  p.R = g.R;
  p.M = M;
  p.N = N;
  p.f = g.f;
  p.out = dW;
  p.accumulate = accum ? 1 : 0;
  p.a_maps = g_maps;
  p.sfa = mx.a;
  p.sfb = mx.b;
  p.tile_pref = mx.tile_pref;
  p.status = status;
  p.stall = g.test_stall ? 1 : 0;
  p.wait_ns = g.test_stall ? 10000000ull : kWaitLimitNs;
  CUtensorMap tsa, tsb;
  if (!sf_maps(mx, C::MX, ta, &tsa, &tsb)) return MOE_ECUDA;
  const long long tiles = (long long)g.E * (M / C::TM) * (N / BN);
  return launch<T, OutT, BN, true, true, RAGGED_K, EPI_STORE, PAIR>(
      ta, tb, to, to, to, tsa, tsb, p, tiles > (1 << 30) ? (1 << 30) : (int)tiles, s);
}

#define MOE_DISPATCH_BN(bn, CALL)                             \
  do {                                                        \
    if ((bn) == 256) { constexpr int BN = 256; return CALL; } \
    if ((bn) == 128) { constexpr int BN = 128; return CALL; } \
    { constexpr int BN = 64; return CALL; }                   \
  } while (0)

// CTA pairs for the 16-bit kernels; the TF32 kernels run one CTA per tile.
template <typename T>
constexpr bool kPair = sizeof(T) == 2;
// K atoms per stage of the 16-bit pair forward and FC1-dgrad GEMMs (Cfg)
constexpr int kWideAtoms = 2;

template <typename T>
static moe_status fc1_fwd(const GemmShape& g, const void* x_perm, const void* W13,
                          const int32_t* off, void* H13, void* a, int* st, cudaStream_t s) {
  // accumulator grid: 2f columns, each tile = BN/2 gate columns + the matching BN/2 up columns
  if constexpr (kPair<T>) {
    if (g.f % 128 == 0 && g.d % 128 == 0)
      return run_m<T, false, EPI_SWIGLU_FWD, 256, true, T, kWideAtoms>(
          g, x_perm, g.d, W13, 2 * g.f, 2 * g.f, g.d, H13, 2 * g.f, a, nullptr, off, st, s);
  }
  if (g.f % 128 == 0)
    return run_m<T, false, EPI_SWIGLU_FWD, 256, kPair<T>>(g, x_perm, g.d, W13, 2 * g.f, 2 * g.f,
                                                           g.d, H13, 2 * g.f, a, nullptr, off, st,
                                                           s);
  return run_m<T, false, EPI_SWIGLU_FWD, 128, kPair<T>>(g, x_perm, g.d, W13, 2 * g.f, 2 * g.f, g.d,
                                                         H13, 2 * g.f, a, nullptr, off, st, s);
}

template <typename T, typename OutT = T>
static moe_status fc2_fwd(const GemmShape& g, const void* a, const void* W2, const int32_t* off,
                          void* y_perm, int* st, cudaStream_t s) {
  if constexpr (kPair<T> && sizeof(OutT) == 2) {   // (fp32 staging leaves room for two stages)
    if (g.d % 256 == 0 && g.f % 128 == 0)
      return run_m<T, false, EPI_STORE, 256, true, OutT, kWideAtoms>(
          g, a, g.f, W2, g.d, g.d, g.f, y_perm, g.d, nullptr, nullptr, off, st, s);
  }
  if (g.d % 256 == 0)
    return run_m<T, false, EPI_STORE, 256, kPair<T>, OutT>(g, a, g.f, W2, g.d, g.d, g.f, y_perm,
                                                            g.d, nullptr, nullptr, off, st, s);
  return run_m<T, false, EPI_STORE, 128, kPair<T>, OutT>(g, a, g.f, W2, g.d, g.d, g.f, y_perm, g.d,
                                                          nullptr, nullptr, off, st, s);
}

template <typename T>
static moe_status fc2_dgrad(const GemmShape& g, const void* dy_perm, const void* W2,
                            const void* H13, const int32_t* off, void* dH13, int* st,
                            cudaStream_t s) {
  // dA = dY . W2_e: K = d, N = f; B[n, k] = W2[e*d + k, n] (M/N-major)
  if constexpr (kPair<T>) {
    if (g.f % 256 == 0)
      return run_m<T, true, EPI_SWIGLU_BWD, 256, true>(g, dy_perm, g.d, W2, g.f, g.d, g.f, dH13,
                                                        2 * g.f, nullptr, H13, off, st, s);
  }
  if (g.f % 128 == 0)
    return run_m<T, true, EPI_SWIGLU_BWD, 128, kPair<T>>(g, dy_perm, g.d, W2, g.f, g.d, g.f, dH13,
                                                          2 * g.f, nullptr, H13, off, st, s);
  return run_m<T, true, EPI_SWIGLU_BWD, 64, false>(g, dy_perm, g.d, W2, g.f, g.d, g.f, dH13,
                                                    2 * g.f, nullptr, H13, off, st, s);
}

template <typename T, typename OutT = T>
static moe_status fc1_dgrad(const GemmShape& g, const void* dH13, const void* W13,
                            const int32_t* off, void* dx_perm, int* st, cudaStream_t s) {
  // dX = dH13 . W13_e: K = 2f, N = d; B[n, k] = W13[e*2f + k, n] (M/N-major)
  if constexpr (kPair<T> && sizeof(OutT) == 2) {
    if (g.d % 256 == 0)   // K = 2f, a multiple of 128
      return run_m<T, true, EPI_STORE, 256, true, OutT, kWideAtoms>(
          g, dH13, 2 * g.f, W13, g.d, 2 * g.f, g.d, dx_perm, g.d, nullptr, nullptr, off, st, s);
  }
  if (g.d % 256 == 0)
    return run_m<T, true, EPI_STORE, 256, kPair<T>, OutT>(g, dH13, 2 * g.f, W13, g.d, 2 * g.f, g.d,
                                                           dx_perm, g.d, nullptr, nullptr, off, st,
                                                           s);
  return run_m<T, true, EPI_STORE, 128, kPair<T>, OutT>(g, dH13, 2 * g.f, W13, g.d, 2 * g.f, g.d,
                                                         dx_perm, g.d, nullptr, nullptr, off, st, s);
}

template <typename T, typename OutT>
static moe_status wgrad_t(const GemmShape& g, const void* G, int M, const void* X, int N, void* dW,
                          bool accum, const int32_t* off, const CUtensorMap* maps, int* st,
                          cudaStream_t s) {
  // pairs need 256-row output tiles and B halves of whole 64-column blocks (BN >= 128)
  const int bn = pick_bn(N);
  if (kPair<T> && M % 256 == 0 && bn >= 128) {
    if (bn == 256)
      return run_k<T, OutT, 256, kPair<T>>(g, G, M, X, N, dW, accum, off, maps, st, s);
    return run_k<T, OutT, 128, kPair<T>>(g, G, M, X, N, dW, accum, off, maps, st, s);
  }
  MOE_DISPATCH_BN(bn, (run_k<T, OutT, BN, false>(g, G, M, X, N, dW, accum, off, maps, st, s)));
}

template <typename T>
static moe_status wgrad(const GemmShape& g, const void* G, int M, const void* X, int N, void* dW,
                        bool dw_fp32, bool accum, const int32_t* off, const CUtensorMap* maps,
                        int* st, cudaStream_t s) {
  if (dw_fp32) return wgrad_t<T, float>(g, G, M, X, N, dW, accum, off, maps, st, s);
  return wgrad_t<T, T>(g, G, M, X, N, dW, false, off, maps, st, s);
}

// Builds the per-expert maps of both wgrad G operands (dY for FC2, dH13 for FC1) into
// `maps` [2E] before either wgrad runs.
template <typename T>
static moe_status build_wgrad_maps(const GemmShape& g, const void* dy_perm, const void* dH13,
                                   const int32_t* off, CUtensorMap* maps, cudaStream_t s) {
  using C = Cfg<T, T, 128, EPI_STORE>;
  constexpr int ES = sizeof(T);
  CUtensorMap t0, t1;
  if constexpr (C::MX) {
    if (!make_tmap(&t0, dy_perm, ES, g.d, g.R, C::MNB, C::KB, Box::MNMajor)) return MOE_ECUDA;
    if (!make_tmap(&t1, dH13, ES, 2 * (uint64_t)g.f, g.R, C::MNB, C::KB, Box::MNMajor))
      return MOE_ECUDA;
  } else {
    // the 3-D maps of the kernel's A loads (BM columns, i.e. BM / MNB blocks, a request)
    if (!make_tmap_mn3(&t0, dy_perm, ES, g.d, g.R, C::KB, BM / C::MNB)) return MOE_ECUDA;
    if (!make_tmap_mn3(&t1, dH13, ES, 2 * (uint64_t)g.f, g.R, C::KB, BM / C::MNB))
      return MOE_ECUDA;
  }
  const int threads = 2 * g.E;
  return launch_pdl(expert_maps_kernel, (threads + 127) / 128, 128, 0, s, t0, t1, off, g.E, g.R,
                    maps) == cudaSuccess ? MOE_OK : MOE_ECUDA;
}

// ------------------------------------------------------------------------ MXFP8 GEMMs
// Operands are quantised (E4M3 + E8M0 per 32 along each GEMM's K) right before the GEMM
// that reads them, except a along d_ff, which FC1's SwiGLU epilogue quantises from the
// bf16 values it stores; all quantised tensors and scales live in the workspace (MxWork).
// Scales stream through shared memory into TMEM per stage.
static inline moe_status cuq(cudaError_t e) { return e == cudaSuccess ? MOE_OK : MOE_ECUDA; }
#define MOE_MX_TRY(x)              \
  do {                             \
    moe_status _r = (x);           \
    if (_r != MOE_OK) return _r;   \
  } while (0)

static Params::Sf sf_ref(const uint8_t* base, int seg_uniform, bool k_major, int W) {
  Params::Sf f;
  f.base = base;
  f.seg_uniform = seg_uniform;
  f.k_major = k_major ? 1 : 0;
  f.W = W;
  return f;
}

// Segments of the experts' rows (their prefixes are computed once per direction).
static MxSegs act_segs(const GemmShape& g, const int32_t* off, const MxWork& w) {
  MxSegs a;
  a.off = off;
  a.tile_pref = w.act_pref;
  a.blk_pref = w.act_pref + (g.E + 1);
  a.E = g.E;
  return a;
}
static MxSegs weight_segs(int E, int rows) {
  MxSegs s;
  s.E = E;
  s.rows = rows;
  return s;
}

// Scale references of an activation operand (ragged expert segments of the R rows, C
// columns) and of a weight operand (E uniform segments of `rows` rows).
static void act_sf(Params::Sf& f, int64_t& chunks, const GemmShape& g, const uint8_t* sf, int C,
                   bool k_major) {
  f = sf_ref(sf, 0, k_major, C / 128);
  chunks = static_cast<int64_t>(mx_sf_bytes(g.R, C, g.E) / 512);
}
static void weight_sf(Params::Sf& f, int64_t& chunks, const GemmShape& g, const uint8_t* sf,
                      int rows, int C, bool k_major) {
  f = sf_ref(sf, rows / 128, k_major, C / 128);
  chunks = static_cast<int64_t>(g.E) * (rows / 128) * (C / 128);
}

// MXFP8 GEMMs run 256 x 256 CTA-pair tiles where the output's N (and, for wgrad, M)
// divides by 256, else 128 x 128 single-CTA tiles.  The fused SwiGLU forward always has
// 2*d_ff % 256 == 0 (MXFP8 needs d_ff % 128 == 0).
static moe_status mx_fwd(const GemmShape& g, const void* x_perm, const void* W13, const void* W2,
                         const int32_t* off, void* H13, void* a, void* y_perm, int* st,
                         cudaStream_t s, const MxWork& w) {
  const int E = g.E, d = g.d, f = g.f;
  const MxSegs act = act_segs(g, off, w);
  MOE_MX_TRY(cuq(launch_mx_prefix(off, E, w.act_pref, w.act_pref + (E + 1), s)));
  // FC1: x_perm and W13 rowwise along d; W13's scales in the gate/up tile order
  MOE_MX_TRY(cuq(launch_mx_quant(x_perm, g.R, d, act, 0, w.xr, w.xr_sf, nullptr, nullptr, st, s)));
  // (with w_col_in_fwd also column-wise, for the backward's FC1 dgrad: one pass)
  MOE_MX_TRY(cuq(launch_mx_quant(W13, (int64_t)E * 2 * f, d, weight_segs(E, 2 * f), f, w.w13r,
                                 w.w13r_sf, w.w_col_in_fwd ? w.w13c : nullptr,
                                 w.w_col_in_fwd ? w.w13c_sf : nullptr, st, s)));
  MxRefs m1;
  act_sf(m1.a, m1.a_chunks, g, w.xr_sf, d, true);
  weight_sf(m1.b, m1.b_chunks, g, w.w13r_sf, 2 * f, d, true);
  m1.tile_pref = w.act_pref;
  m1.q_codes = w.ar;          // FC1's epilogue also writes a rowwise along d_ff (FC2's K)
  m1.q_sf = w.ar_sf;
  m1.q_ld = f;
  MOE_MX_TRY((run_m<fp8, false, EPI_SWIGLU_FWD, 256, true, bf16>(
      g, w.xr, d, w.w13r, 2 * f, 2 * f, d, H13, 2 * f, a, nullptr, off, st, s, m1)));
  // FC2: W2 rowwise along d_ff (a's codes came from FC1)
  MOE_MX_TRY(cuq(launch_mx_quant(W2, (int64_t)E * d, f, weight_segs(E, d), 0, w.w2r, w.w2r_sf,
                                 w.w_col_in_fwd ? w.w2c : nullptr,
                                 w.w_col_in_fwd ? w.w2c_sf : nullptr, st, s)));
  MxRefs m2;
  act_sf(m2.a, m2.a_chunks, g, w.ar_sf, f, true);
  weight_sf(m2.b, m2.b_chunks, g, w.w2r_sf, d, f, true);
  m2.tile_pref = w.act_pref;
  if (d % 256 == 0)
    return run_m<fp8, false, EPI_STORE, 256, true, bf16>(g, w.ar, f, w.w2r, d, d, f, y_perm, d,
                                                          nullptr, nullptr, off, st, s, m2);
  return run_m<fp8, false, EPI_STORE, 128, false, bf16>(g, w.ar, f, w.w2r, d, d, f, y_perm, d,
                                                         nullptr, nullptr, off, st, s, m2);
}

template <typename OutT>
static moe_status mx_wgrad(const GemmShape& g, const uint8_t* G, int M, const uint8_t* X, int N,
                           void* dW, bool accum, const int32_t* off, const CUtensorMap* maps,
                           int* st, cudaStream_t s, const MxRefs& m) {
  if (M % 256 == 0 && N % 256 == 0)
    return run_k<fp8, OutT, 256, true>(g, G, M, X, N, dW, accum, off, maps, st, s, m);
  return run_k<fp8, OutT, 128, false>(g, G, M, X, N, dW, accum, off, maps, st, s, m);
}

template <typename OutT>
static moe_status mx_bwd(const GemmShape& g, const void* dy_perm, const void* x_perm,
                         const void* H13, const void* a, const void* W13, const void* W2,
                         const int32_t* off, void* dH13, void* dx_perm, void* dW13, void* dW2,
                         bool accum, CUtensorMap* maps, int* st, cudaStream_t s, const MxWork& w) {
  const int E = g.E, d = g.d, f = g.f;
  const MxSegs act = act_segs(g, off, w);
  MOE_MX_TRY(cuq(launch_mx_prefix(off, E, w.act_pref, w.act_pref + (E + 1), s)));
  // dY both ways in one pass: rowwise along d (FC2 dgrad), colwise along tokens (FC2 wgrad);
  // W2 colwise along its d rows (FC2 dgrad)
  MOE_MX_TRY(cuq(launch_mx_quant(dy_perm, g.R, d, act, 0, w.dyr, w.dyr_sf, w.dyc, w.dyc_sf, st, s)));
  if (!w.w_col_ready)   // (else the forward's pass made them)
    MOE_MX_TRY(cuq(launch_mx_quant(W2, (int64_t)E * d, f, weight_segs(E, d), 0, nullptr, nullptr,
                                   w.w2c, w.w2c_sf, st, s)));
  MxRefs m1;
  act_sf(m1.a, m1.a_chunks, g, w.dyr_sf, d, true);
  weight_sf(m1.b, m1.b_chunks, g, w.w2c_sf, d, f, false);
  m1.tile_pref = w.act_pref;
  if (f % 256 == 0)
    MOE_MX_TRY((run_m<fp8, true, EPI_SWIGLU_BWD, 256, true, bf16>(
        g, w.dyr, d, w.w2c, f, d, f, dH13, 2 * f, nullptr, H13, off, st, s, m1)));
  else
    MOE_MX_TRY((run_m<fp8, true, EPI_SWIGLU_BWD, 128, false, bf16>(
        g, w.dyr, d, w.w2c, f, d, f, dH13, 2 * f, nullptr, H13, off, st, s, m1)));
  // FC2 wgrad (dW2_e = dY_e^T . a_e, K = the expert's tokens): a colwise along tokens
  MOE_MX_TRY(cuq(launch_mx_quant(a, g.R, f, act, 0, nullptr, nullptr, w.ac, w.ac_sf, st, s)));
  MOE_MX_TRY(build_wgrad_maps<fp8>(g, w.dyc, w.dhc, off, maps, s));
  MxRefs m2;
  act_sf(m2.a, m2.a_chunks, g, w.dyc_sf, d, false);
  act_sf(m2.b, m2.b_chunks, g, w.ac_sf, f, false);
  m2.tile_pref = w.act_pref;
  MOE_MX_TRY(mx_wgrad<OutT>(g, w.dyc, d, w.ac, f, dW2, accum, off, maps, st, s, m2));
  // dH13 both ways (FC1 dgrad, FC1 wgrad), W13 colwise along its 2*d_ff rows, x_perm
  // colwise along tokens.  (Quantising dH13's rows in FC2 dgrad's epilogue instead was
  // slower: that epilogue holds the single accumulator, so its MMAs wait for it.)
  MOE_MX_TRY(cuq(launch_mx_quant(dH13, g.R, 2 * f, act, 0, w.dhr, w.dhr_sf, w.dhc, w.dhc_sf, st, s)));
  if (!w.w_col_ready)
    MOE_MX_TRY(cuq(launch_mx_quant(W13, (int64_t)E * 2 * f, d, weight_segs(E, 2 * f), 0, nullptr,
                                   nullptr, w.w13c, w.w13c_sf, st, s)));
  MxRefs m3;
  act_sf(m3.a, m3.a_chunks, g, w.dhr_sf, 2 * f, true);
  weight_sf(m3.b, m3.b_chunks, g, w.w13c_sf, 2 * f, d, false);
  m3.tile_pref = w.act_pref;
  if (d % 256 == 0)
    MOE_MX_TRY((run_m<fp8, true, EPI_STORE, 256, true, bf16>(g, w.dhr, 2 * f, w.w13c, d, 2 * f, d,
                                                             dx_perm, d, nullptr, nullptr, off,
                                                             st, s, m3)));
  else
    MOE_MX_TRY((run_m<fp8, true, EPI_STORE, 128, false, bf16>(g, w.dhr, 2 * f, w.w13c, d, 2 * f,
                                                              d, dx_perm, d, nullptr, nullptr,
                                                              off, st, s, m3)));
  // FC1 wgrad (dW13_e = dH13_e^T . X_e)
  MOE_MX_TRY(cuq(launch_mx_quant(x_perm, g.R, d, act, 0, nullptr, nullptr, w.xc, w.xc_sf, st, s)));
  MxRefs m4;
  act_sf(m4.a, m4.a_chunks, g, w.dhc_sf, 2 * f, false);
  act_sf(m4.b, m4.b_chunks, g, w.xc_sf, d, false);
  m4.tile_pref = w.act_pref;
  return mx_wgrad<OutT>(g, w.dhc, 2 * f, w.xc, d, dW13, accum, off, maps + E, st, s, m4);
}

// ------------------------------------------------------------------------ router GEMMs
// The router projection and its two backward products as one-segment GEMMs (no offsets:
// all T rows form the single segment), bf16 operands, fp32 accumulation.  E % 64 == 0.
static int bn_of(int n) { return n % 256 == 0 ? 256 : n % 128 == 0 ? 128 : 64; }

static moe_status router_logits_tc(int T, int d, int E, const void* x, const void* Wr,
                                   float* logits, int* st, cudaStream_t s) {
  const GemmShape g{1, T, d, 0, false, false};
  // logits[T,E] = x[T,d] . Wr[d,E]: B = Wr read M/N-major ([K=d rows, N=E cols])
  switch (bn_of(E)) {
    case 256:
      return run_m<bf16, true, EPI_STORE, 256, true, float>(g, x, d, Wr, E, d, E, logits, E,
                                                           nullptr, nullptr, nullptr, st, s);
    case 128:
      return run_m<bf16, true, EPI_STORE, 128, true, float>(g, x, d, Wr, E, d, E, logits, E,
                                                           nullptr, nullptr, nullptr, st, s);
    default:
      return run_m<bf16, true, EPI_STORE, 64, false, float>(g, x, d, Wr, E, d, E, logits, E,
                                                           nullptr, nullptr, nullptr, st, s);
  }
}

static moe_status router_dx_tc(int T, int d, int E, const void* dl16, const void* Wr,
                               float* dx_extra, int* st, cudaStream_t s) {
  const GemmShape g{1, T, d, 0, false, false};
  // dx_extra[T,d] = d_logits[T,E] . Wr^T: B = Wr read K-major ([N=d rows, K=E cols])
  if (d % 256 == 0)
    return run_m<bf16, false, EPI_STORE, 256, true, float>(g, dl16, E, Wr, d, d, E, dx_extra, d,
                                                          nullptr, nullptr, nullptr, st, s);
  return run_m<bf16, false, EPI_STORE, 128, true, float>(g, dl16, E, Wr, d, d, E, dx_extra, d,
                                                        nullptr, nullptr, nullptr, st, s);
}

static moe_status router_dwr_tc(int T, int d, int E, const void* x, const void* dl16, void* dWr,
                                CUtensorMap* maps, int* st, cudaStream_t s) {
  const GemmShape g{1, T, d, 0, false, false};
  // dWr[d,E] = x^T . d_logits: a ragged-K GEMM over the one segment (K = T)
  using C = Cfg<bf16, bf16, 128, EPI_STORE>;
  CUtensorMap t0;
  if (!make_tmap_mn3(&t0, x, 2, d, T, C::KB, BM / C::MNB)) return MOE_ECUDA;
  if (launch_pdl(expert_maps_kernel, 1, 128, 0, s, t0, t0, (const int32_t*)nullptr, 1, T, maps) !=
      cudaSuccess)
    return MOE_ECUDA;
  const int bn = bn_of(E);
  if (d % 256 == 0 && bn >= 128) {
    if (bn == 256) return run_k<bf16, bf16, 256, true>(g, x, d, dl16, E, dWr, false, nullptr, maps, st, s);
    return run_k<bf16, bf16, 128, true>(g, x, d, dl16, E, dWr, false, nullptr, maps, st, s);
  }
  MOE_DISPATCH_BN(bn, (run_k<bf16, bf16, BN, false>(g, x, d, dl16, E, dWr, false, nullptr, maps,
                                                     st, s)));
}

// ------------------------------------------------------------------------ shared expert
// A dense SwiGLU FFN over all T tokens: the grouped GEMMs with one segment (no offsets),
// the FC2 output and the FC1 input gradient in fp32 (added into the combine / unpermute).
template <typename T>
static moe_status shared_fwd_t(const GemmShape& g1, const void* x, const void* W13s,
                               const void* W2s, void* H13s, void* as, float* ys, int* st,
                               cudaStream_t s) {
  moe_status r = fc1_fwd<T>(g1, x, W13s, nullptr, H13s, as, st, s);
  if (r != MOE_OK) return r;
  return fc2_fwd<T, float>(g1, as, W2s, nullptr, ys, st, s);
}

template <typename T>
static moe_status shared_bwd_t(const GemmShape& g1, const void* dy, const void* x,
                               const void* H13s, const void* as, const void* W13s,
                               const void* W2s, void* dH13s, float* dxs, void* dW13s, void* dW2s,
                               bool dw_fp32, bool dw_accum, CUtensorMap* maps, int* st,
                               cudaStream_t s) {
  moe_status r = build_wgrad_maps<T>(g1, dy, dH13s, nullptr, maps, s);
  if (r != MOE_OK) return r;
  r = fc2_dgrad<T>(g1, dy, W2s, H13s, nullptr, dH13s, st, s);
  if (r != MOE_OK) return r;
  r = wgrad<T>(g1, dy, g1.d, as, g1.f, dW2s, dw_fp32, dw_accum, nullptr, maps, st, s);
  if (r != MOE_OK) return r;
  r = fc1_dgrad<T, float>(g1, dH13s, W13s, nullptr, dxs, st, s);
  if (r != MOE_OK) return r;
  return wgrad<T>(g1, dH13s, 2 * g1.f, x, g1.d, dW13s, dw_fp32, dw_accum, nullptr, maps + 1, st, s);
}

}  // namespace gemm

moe_status gemm_fwd(const GemmShape& g, const void* x_perm, const void* W13, const void* W2,
                    const int32_t* offsets, void* H13, void* a, void* y_perm, int* status,
                    cudaStream_t s, const MxWork* mx) {
  if (g.mx) {
    if (!mx) return MOE_EINVAL;
    return gemm::mx_fwd(g, x_perm, W13, W2, offsets, H13, a, y_perm, status, s, *mx);
  }
  moe_status st;
  if (g.fp32) {
    st = gemm::fc1_fwd<float>(g, x_perm, W13, offsets, H13, a, status, s);
    if (st != MOE_OK) return st;
    return gemm::fc2_fwd<float>(g, a, W2, offsets, y_perm, status, s);
  }
  st = gemm::fc1_fwd<__nv_bfloat16>(g, x_perm, W13, offsets, H13, a, status, s);
  if (st != MOE_OK) return st;
  return gemm::fc2_fwd<__nv_bfloat16>(g, a, W2, offsets, y_perm, status, s);
}

template <typename T>
static moe_status gemm_bwd_t(const GemmShape& g, const void* dy_perm, const void* x_perm,
                             const void* H13, const void* a, const void* W13, const void* W2,
                             const int32_t* off, void* dH13, void* dx_perm, void* dW13, void* dW2,
                             bool dw_fp32, bool dw_accum, void* maps_ws, int* st,
                             cudaStream_t s) {
  CUtensorMap* maps = reinterpret_cast<CUtensorMap*>(maps_ws);
  moe_status r = gemm::build_wgrad_maps<T>(g, dy_perm, dH13, off, maps, s);
  if (r != MOE_OK) return r;
  r = gemm::fc2_dgrad<T>(g, dy_perm, W2, H13, off, dH13, st, s);
  if (r != MOE_OK) return r;
  r = gemm::wgrad<T>(g, dy_perm, g.d, a, g.f, dW2, dw_fp32, dw_accum, off, maps, st, s);
  if (r != MOE_OK) return r;
  r = gemm::fc1_dgrad<T>(g, dH13, W13, off, dx_perm, st, s);
  if (r != MOE_OK) return r;
  return gemm::wgrad<T>(g, dH13, 2 * g.f, x_perm, g.d, dW13, dw_fp32, dw_accum, off, maps + g.E,
                        st, s);
}

moe_status gemm_bwd(const GemmShape& g, const void* dy_perm, const void* x_perm, const void* H13,
                    const void* a, const void* W13, const void* W2, const int32_t* offsets,
                    void* dH13, void* dx_perm, void* dW13, void* dW2, bool dw_fp32,
                    bool dw_accum, void* maps_ws, int* status, cudaStream_t s,
                    const MxWork* mx) {
  if (g.mx) {
    if (!mx) return MOE_EINVAL;
    CUtensorMap* maps = reinterpret_cast<CUtensorMap*>(maps_ws);
    if (dw_fp32)
      return gemm::mx_bwd<float>(g, dy_perm, x_perm, H13, a, W13, W2, offsets, dH13, dx_perm, dW13,
                                 dW2, dw_accum, maps, status, s, *mx);
    return gemm::mx_bwd<__nv_bfloat16>(g, dy_perm, x_perm, H13, a, W13, W2, offsets, dH13,
                                       dx_perm, dW13, dW2, false, maps, status, s, *mx);
  }
  if (g.fp32)
    return gemm_bwd_t<float>(g, dy_perm, x_perm, H13, a, W13, W2, offsets, dH13, dx_perm, dW13,
                             dW2, dw_fp32, dw_accum, maps_ws, status, s);
  return gemm_bwd_t<__nv_bfloat16>(g, dy_perm, x_perm, H13, a, W13, W2, offsets, dH13, dx_perm,
                                   dW13, dW2, dw_fp32, dw_accum, maps_ws, status, s);
}

moe_status router_logits_tc(int T, int d, int E, const void* x, const void* Wr, float* logits,
                            int* status, cudaStream_t s) {
  return gemm::router_logits_tc(T, d, E, x, Wr, logits, status, s);
}
moe_status router_bwd_tc(int T, int d, int E, const void* x, const void* Wr, const void* dl16,
                         float* dx_extra, void* dWr, void* maps_ws, int* status, cudaStream_t s) {
  moe_status r = gemm::router_dx_tc(T, d, E, dl16, Wr, dx_extra, status, s);
  if (r != MOE_OK) return r;
  return gemm::router_dwr_tc(T, d, E, x, dl16, dWr, reinterpret_cast<CUtensorMap*>(maps_ws),
                             status, s);
}

moe_status shared_fwd(const GemmShape& g, const void* x, const void* W13s, const void* W2s,
                      void* H13s, void* as, float* ys, int* status, cudaStream_t s) {
  const GemmShape g1{1, g.R, g.d, g.f, g.fp32, false, g.test_stall};
  if (g.fp32) return gemm::shared_fwd_t<float>(g1, x, W13s, W2s, H13s, as, ys, status, s);
  return gemm::shared_fwd_t<__nv_bfloat16>(g1, x, W13s, W2s, H13s, as, ys, status, s);
}
moe_status shared_bwd(const GemmShape& g, const void* dy, const void* x, const void* H13s,
                      const void* as, const void* W13s, const void* W2s, void* dH13s, float* dxs,
                      void* dW13s, void* dW2s, bool dw_fp32, bool dw_accum, void* maps_ws,
                      int* status, cudaStream_t s) {
  const GemmShape g1{1, g.R, g.d, g.f, g.fp32, false, g.test_stall};
  CUtensorMap* maps = reinterpret_cast<CUtensorMap*>(maps_ws);
  if (g.fp32)
    return gemm::shared_bwd_t<float>(g1, dy, x, H13s, as, W13s, W2s, dH13s, dxs, dW13s, dW2s,
                                     dw_fp32, dw_accum, maps, status, s);
  return gemm::shared_bwd_t<__nv_bfloat16>(g1, dy, x, H13s, as, W13s, W2s, dH13s, dxs, dW13s, dW2s,
                                           dw_fp32, dw_accum, maps, status, s);
}

}  // namespace moe
