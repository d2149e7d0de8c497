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
// Kernel structure (one CTA per SM, 192 threads):
//   warp 0      TMA producer: 128-byte-swizzled operand tiles into a ring of stages
//   warp 1      tcgen05.mma issuer (one thread) + tensor-memory allocation
//   warps 2..5  epilogue: tensor memory -> registers -> fused math -> global memory
// Two fp32 accumulators of 128 x BN live in tensor memory so the epilogue of one
// tile overlaps the main loop of the next.
//
// Two groupings:
//   RAGGED_M  forward and dgrad: expert e owns rows [off_e, off_e+1) of the routed
//             activations; tiles of 128 rows start at off_e and rows past the
//             expert's end are computed but never stored.
//   RAGGED_K  wgrad: dW_e = G_e^T . X_e sums over the expert's rows; the last
//             K-block of an expert is partial and its foreign rows are zeroed in
//             shared memory before the MMA reads them.  An expert with no rows
//             writes dW_e = 0.
#include <cuda.h>
#include <cuda_runtime.h>
#include <cuda_bf16.h>

#include <mutex>

#include "common.cuh"
#include "internal.h"
#include "sm100.cuh"

namespace moe {
namespace gemm {

using bf16 = __nv_bfloat16;
using namespace moe::sm100;

enum { RAGGED_M = 0, RAGGED_K = 1 };
enum { EPI_STORE = 0, EPI_SWIGLU_FWD = 1, EPI_SWIGLU_BWD = 2 };

constexpr int BM = 128;
constexpr int kThreads = 192;

struct Params {
  const int32_t* offsets;  // [E+1]
  int E, R;
  int M;                   // RAGGED_K: rows of dW_e
  int N;                   // width of the accumulator grid (columns of the output per expert)
  int K;                   // RAGGED_M: reduction length
  int b_rows_per_expert;   // expert e's rows start at e * b_rows_per_expert in B's tensor map
  int f;                   // d_ff (SwiGLU epilogues)
  void* out;               // main output
  int64_t ldo;             // its row stride in elements (RAGGED_M)
  void* out_a;             // SwiGLU forward: a [R, f]
  const void* aux;         // SwiGLU backward: H13 [R, 2f]
  int out_fp32;            // RAGGED_K: dW element type is float
  int accumulate;          // RAGGED_K: dW += result (float dW only)
  int* status;
};

template <typename T, int BN>
struct Cfg {
  static constexpr int ES = sizeof(T);
  static constexpr int KB = 128 / ES;     // K elements per stage (one 128-byte swizzle row)
  static constexpr int MNB = 128 / ES;    // M/N elements per 128-byte block (M/N-major tiles)
  static constexpr int UK = 32 / ES;      // K of one MMA instruction
  static constexpr int A_BYTES = BM * 128;
  static constexpr int B_BYTES = BN * 128;
  static constexpr int STAGE = A_BYTES + B_BYTES;
  static constexpr int STAGES = (196 * 1024) / STAGE > 8 ? 8 : (196 * 1024) / STAGE;
  static constexpr int TMEM_COLS = 2 * BN;
  static constexpr size_t smem_bytes(int E) {
    return 1024 /*alignment slack*/ + size_t(STAGES) * STAGE + 256 /*barriers, flags*/ +
           size_t(2 * (E + 1) + 4) * sizeof(int);
  }
};

struct Tile {
  int e, n0, m0, row0, rows_end, kb, cnt;
};

template <int MODE, int BN, int KB>
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
    tl.m0 = (mtg - s_mt[lo]) * BM;
    tl.row0 = s_off[lo] + tl.m0;
    tl.rows_end = s_off[lo + 1];
    tl.n0 = nt * BN;
    tl.kb = K / KB;
    tl.cnt = 0;
  } else {
    const int per = m_tiles * n_tiles;
    tl.e = t / per;
    const int r = t - tl.e * per;
    const int mt = r / n_tiles;
    tl.m0 = mt * BM;
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
template <typename T>
__device__ __forceinline__ void load32(const T* src, float* v) {
  constexpr int PER = 16 / sizeof(T);
#pragma unroll
  for (int i = 0; i < 32; i += PER) {
    Vec16<T> pk;
    pk.raw = *reinterpret_cast<const uint4*>(src + i);
    pk.to_float(v + i);
  }
}

__device__ __forceinline__ float sigmoid_f(float z) { return 1.0f / (1.0f + __expf(-z)); }

__device__ __forceinline__ void bits_to_f32(const uint32_t* v, float* f) {
#pragma unroll
  for (int i = 0; i < 32; ++i) f[i] = __uint_as_float(v[i]);
}

template <typename T, int BN, bool A_MN, bool B_MN, int MODE, int EPI>
__global__ void __launch_bounds__(kThreads, 1)
grouped_gemm_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
                    const Params p) {
  using C = Cfg<T, BN>;
  constexpr bool kTF32 = sizeof(T) == 4;
  constexpr uint32_t IDESC = idesc_f32acc(BM, BN, kTF32 ? 2u : 1u, A_MN, B_MN);
  static_assert(BN == 64 || BN == 128 || BN == 256, "tile width");
  static_assert(MODE == RAGGED_M || (A_MN && B_MN && EPI == EPI_STORE), "wgrad layout");

  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~uintptr_t(1023));
  uint8_t* tiles = smem;
  uint64_t* full = reinterpret_cast<uint64_t*>(tiles + C::STAGES * C::STAGE);
  uint64_t* empty = full + C::STAGES;
  uint64_t* tfull = empty + C::STAGES;
  uint64_t* tempty = tfull + 2;
  uint64_t* fin = tempty + 2;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(fin + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
  int* s_total = reinterpret_cast<int*>(tmem_slot + 2);
  int* s_off = s_total + 2;
  int* s_mt = s_off + (p.E + 1);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int E = p.E;
  const int n_tiles = p.N / BN;
  const int m_tiles = MODE == RAGGED_K ? p.M / BM : 0;

  for (int i = threadIdx.x; i <= E; i += kThreads) s_off[i] = p.offsets[i];
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
        mt = c > 0 ? (c + BM - 1) / BM : 0;
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
        mbar_init(&tempty[a], 4);
      }
      mbar_init(fin, 1);
      fence_mbar_init();
    }
  }
  __syncthreads();
  const int total = s_total[0];
  if (static_cast<int>(blockIdx.x) >= total) return;   // uniform over the CTA

  if (warp == 1) tmem_alloc(tmem_slot, C::TMEM_COLS);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;

  if (warp == 0) {
    // ------------------------------------------------------------------ TMA producer
    if (lane == 0) {
      tma_prefetch_desc(&tmA);
      tma_prefetch_desc(&tmB);
      int stage = 0;
      uint32_t phase = 0;
      uint32_t armed = 0, armed_par = 0;
      bool stop = false;
      for (int t = blockIdx.x; t < total && !stop; t += gridDim.x) {
        const Tile tl = decode_tile<MODE, BN, C::KB>(t, n_tiles, m_tiles, s_off, s_mt, E, p.K);
        for (int kb = 0; kb < tl.kb; ++kb) {
          if (!mbar_wait(&empty[stage], phase ^ 1u, abort_flag, p.status)) { stop = true; break; }
          uint8_t* sA = tiles + stage * C::STAGE;
          uint8_t* sB = sA + C::A_BYTES;
          mbar_arrive_expect_tx(&full[stage], C::STAGE);
          armed |= 1u << stage;
          armed_par = (armed_par & ~(1u << stage)) | (phase << stage);
          const int k0 = kb * C::KB;
          if (MODE == RAGGED_M) {
            tma_load_2d(sA, &tmA, &full[stage], k0, tl.row0);
            const int brow = tl.e * p.b_rows_per_expert;
            if (!B_MN) {
              if (EPI == EPI_SWIGLU_FWD) {
                const int h0 = tl.n0 / 2;
                tma_load_2d(sB, &tmB, &full[stage], k0, brow + h0);
                tma_load_2d(sB + (BN / 2) * 128, &tmB, &full[stage], k0, brow + p.f + h0);
              } else {
                tma_load_2d(sB, &tmB, &full[stage], k0, brow + tl.n0);
              }
            } else {
#pragma unroll
              for (int i = 0; i < BN / C::MNB; ++i)
                tma_load_2d(sB + i * C::KB * 128, &tmB, &full[stage], tl.n0 + i * C::MNB,
                            brow + k0);
            }
          } else {
#pragma unroll
            for (int i = 0; i < BM / C::MNB; ++i)
              tma_load_2d(sA + i * C::KB * 128, &tmA, &full[stage], tl.m0 + i * C::MNB,
                          tl.row0 + k0);
#pragma unroll
            for (int i = 0; i < BN / C::MNB; ++i)
              tma_load_2d(sB + i * C::KB * 128, &tmB, &full[stage], tl.n0 + i * C::MNB,
                          tl.row0 + k0);
          }
          if (++stage == C::STAGES) { stage = 0; phase ^= 1u; }
        }
      }
      // Teardown: every armed stage's bytes must have landed before the CTA exits.
      for (int s = 0; s < C::STAGES; ++s)
        if (armed & (1u << s)) mbar_wait_teardown(&full[s], (armed_par >> s) & 1u);
    }
    __syncwarp();
  } else if (warp == 1) {
    // ------------------------------------------------------------------ MMA issuer
    int stage = 0;
    uint32_t phase = 0;
    int acc = 0;
    uint32_t acc_phase = 0;
    bool stop = false;
    for (int t = blockIdx.x; t < total && !stop; t += gridDim.x) {
      const Tile tl = decode_tile<MODE, BN, C::KB>(t, n_tiles, m_tiles, s_off, s_mt, E, p.K);
      if (!mbar_wait_warp(&tempty[acc], acc_phase ^ 1u, abort_flag, p.status)) break;
      tc_fence_after();
      const uint32_t d_tmem = tmem_base + static_cast<uint32_t>(acc * BN);
      for (int kb = 0; kb < tl.kb; ++kb) {
        if (!mbar_wait_warp(&full[stage], phase, abort_flag, p.status)) { stop = true; break; }
        tc_fence_after();
        uint8_t* sA = tiles + stage * C::STAGE;
        if (MODE == RAGGED_K && kb == tl.kb - 1) {
          const int valid = tl.cnt - kb * C::KB;
          if (valid < C::KB) {
            // Rows [valid, KB) of this K-block belong to later experts: zero them in A.
            const int rows = C::KB - valid;
            const int per_blk = rows * 8;   // 16-byte chunks per M block
            for (int i = lane; i < (BM / C::MNB) * per_blk; i += 32) {
              const int blk = i / per_blk;
              const int rem = i - blk * per_blk;
              uint8_t* dst = sA + blk * C::KB * 128 + (valid + (rem >> 3)) * 128 + (rem & 7) * 16;
              *reinterpret_cast<uint4*>(dst) = make_uint4(0u, 0u, 0u, 0u);
            }
            fence_proxy_async_smem();
          }
          __syncwarp();
        }
        if (lane == 0) {
          const uint32_t a_base = smem_u32(sA);
          const uint32_t b_base = a_base + C::A_BYTES;
          // M/N-major TF32 tiles use the 32-byte-atom swizzle (4-row K groups)
          constexpr uint32_t MN_LAYOUT = kTF32 ? kLayoutSW128Atom32 : kLayoutSW128;
          constexpr uint32_t MN_SBO = kTF32 ? 512 : 1024;
#pragma unroll
          for (int kk = 0; kk < C::KB / C::UK; ++kk) {
            const uint64_t ad =
                A_MN ? sdesc(a_base + kk * C::UK * 128, C::KB * 128, MN_SBO, MN_LAYOUT)
                     : sdesc(a_base + kk * 32, 16, 1024, kLayoutSW128);
            const uint64_t bd =
                B_MN ? sdesc(b_base + kk * C::UK * 128, C::KB * 128, MN_SBO, MN_LAYOUT)
                     : sdesc(b_base + kk * 32, 16, 1024, kLayoutSW128);
            umma<kTF32>(d_tmem, ad, bd, IDESC, (kb | kk) != 0 ? 1u : 0u);
          }
          umma_commit(&empty[stage]);
        }
        __syncwarp();
        if (++stage == C::STAGES) { stage = 0; phase ^= 1u; }
      }
      if (lane == 0) umma_commit(&tfull[acc]);
      __syncwarp();
      if (++acc == 2) { acc = 0; acc_phase ^= 1u; }
    }
    if (lane == 0) {
      umma_commit(fin);
      mbar_wait_teardown(fin, 0);
    }
    __syncwarp();
  } else {
    // ------------------------------------------------------------------ epilogue
    const int q = warp & 3;                 // tensor-memory lane quadrant of this warp
    const int r = q * 32 + lane;            // tile row
    int acc = 0;
    uint32_t acc_phase = 0;
    for (int t = blockIdx.x; t < total; t += gridDim.x) {
      const Tile tl = decode_tile<MODE, BN, C::KB>(t, n_tiles, m_tiles, s_off, s_mt, E, p.K);
      if (!mbar_wait_warp(&tfull[acc], acc_phase, abort_flag, p.status)) break;
      tc_fence_after();
      const uint32_t tb = tmem_base + (static_cast<uint32_t>(q * 32) << 16) +
                          static_cast<uint32_t>(acc * BN);
      uint32_t v[32];
      if (MODE == RAGGED_M) {
        const int64_t grow = tl.row0 + r;
        const bool valid = grow < tl.rows_end;
        if (EPI == EPI_STORE) {
          T* out = reinterpret_cast<T*>(p.out) + grow * p.ldo + tl.n0;
#pragma unroll 1
          for (int c = 0; c < BN; c += 32) {
            tmem_ld32(tb + c, v);
            tmem_ld_wait();
            reg_fence32(v);
            if (valid) {
              float fv[32];
              bits_to_f32(v, fv);
              store32<T>(out + c, fv);
            }
          }
        } else if (EPI == EPI_SWIGLU_FWD) {
          const int h0 = tl.n0 / 2;
          T* h13 = reinterpret_cast<T*>(p.out) + grow * (2 * (int64_t)p.f) + h0;
          T* aa = reinterpret_cast<T*>(p.out_a) + grow * (int64_t)p.f + h0;
          uint32_t v3[32];
#pragma unroll 1
          for (int c = 0; c < BN / 2; c += 32) {
            tmem_ld32(tb + c, v);
            tmem_ld32(tb + BN / 2 + c, v3);
            tmem_ld_wait();
            reg_fence32(v);
            reg_fence32(v3);
            if (valid) {
              float h1[32], h3[32];
              bits_to_f32(v, h1);
              bits_to_f32(v3, h3);
              store32<T>(h13 + c, h1);
              store32<T>(h13 + p.f + c, h3);
              float av[32];
#pragma unroll
              for (int i = 0; i < 32; ++i) av[i] = h1[i] * sigmoid_f(h1[i]) * h3[i];
              store32<T>(aa + c, av);
            }
          }
        } else {  // EPI_SWIGLU_BWD: accumulator = dA
          const T* h13 = reinterpret_cast<const T*>(p.aux) + grow * (2 * (int64_t)p.f) + tl.n0;
          T* dh = reinterpret_cast<T*>(p.out) + grow * (2 * (int64_t)p.f) + tl.n0;
#pragma unroll 1
          for (int c = 0; c < BN; c += 32) {
            tmem_ld32(tb + c, v);
            tmem_ld_wait();
            reg_fence32(v);
            if (valid) {
              float h1[32], h3[32], d1[32], d3[32], da[32];
              load32<T>(h13 + c, h1);
              load32<T>(h13 + p.f + c, h3);
              bits_to_f32(v, da);
#pragma unroll
              for (int i = 0; i < 32; ++i) {
                const float s = sigmoid_f(h1[i]);
                d1[i] = da[i] * h3[i] * s * (1.0f + h1[i] * (1.0f - s));
                d3[i] = da[i] * h1[i] * s;
              }
              store32<T>(dh + c, d1);
              store32<T>(dh + p.f + c, d3);
            }
          }
        }
      } else {
        // RAGGED_K: dW_e[m0 + r, n0 .. n0 + BN)
        const int64_t off = (int64_t)tl.e * p.M * p.N + (int64_t)(tl.m0 + r) * p.N + tl.n0;
        const bool has = tl.kb > 0;
#pragma unroll 1
        for (int c = 0; c < BN; c += 32) {
          if (has) {
            tmem_ld32(tb + c, v);
            tmem_ld_wait();
            reg_fence32(v);
          } else {
#pragma unroll
            for (int i = 0; i < 32; ++i) v[i] = 0u;
          }
          float fv[32];
          bits_to_f32(v, fv);
          if (p.out_fp32) {
            float* o = reinterpret_cast<float*>(p.out) + off + c;
            if (p.accumulate) {
              float old[32];
              load32<float>(o, old);
#pragma unroll
              for (int i = 0; i < 32; ++i) fv[i] += old[i];
            }
            store32<float>(o, fv);
          } else {
            store32<T>(reinterpret_cast<T*>(p.out) + off + c, fv);
          }
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&tempty[acc]);
      if (++acc == 2) { acc = 0; acc_phase ^= 1u; }
    }
  }

  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem_base, C::TMEM_COLS);
  }
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

// 2-D row-major tensor [rows, cols] with 128-byte swizzled boxes of [box_rows, box_cols].
// `mn_major` boxes of 32-bit elements use the 32-byte-atom variant of the swizzle, the
// layout the tensor core accepts for M/N-major TF32 operands.
static bool make_tmap(CUtensorMap* m, const void* base, bool fp32, uint64_t cols, uint64_t rows,
                      uint32_t box_cols, uint32_t box_rows, bool mn_major = false) {
  EncodeTiledFn enc = encode_fn();
  if (!enc) return false;
  const uint64_t es = fp32 ? 4 : 2;
  cuuint64_t dims[2] = {cols, rows};
  cuuint64_t strides[1] = {cols * es};
  cuuint32_t box[2] = {box_cols, box_rows};
  cuuint32_t estr[2] = {1, 1};
  CUresult r = enc(m, fp32 ? CU_TENSOR_MAP_DATA_TYPE_FLOAT32 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2,
                   const_cast<void*>(base), dims, strides, box, estr,
                   CU_TENSOR_MAP_INTERLEAVE_NONE,
                   (fp32 && mn_major) ? CU_TENSOR_MAP_SWIZZLE_128B_ATOM_32B
                                      : CU_TENSOR_MAP_SWIZZLE_128B,
                   CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

template <typename T, int BN, bool A_MN, bool B_MN, int MODE, int EPI>
static moe_status launch(const CUtensorMap& ta, const CUtensorMap& tb, const Params& p,
                         int max_tiles, cudaStream_t s) {
  using C = Cfg<T, BN>;
  auto kern = grouped_gemm_kernel<T, BN, A_MN, B_MN, MODE, EPI>;
  const size_t smem = C::smem_bytes(p.E);
  if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           static_cast<int>(smem)) != cudaSuccess)
    return MOE_ECUDA;
  int grid = num_sms();
  if (max_tiles < grid) grid = max_tiles;
  if (grid < 1) return MOE_OK;
  kern<<<grid, kThreads, smem, s>>>(ta, tb, p);
  return cudaGetLastError() == cudaSuccess ? MOE_OK : MOE_ECUDA;
}

static int pick_bn(int n) { return n % 256 == 0 ? 256 : n % 128 == 0 ? 128 : 64; }

// Upper bound of the ragged-M tile count: sum_e ceil(cnt_e / BM) <= R / BM + E.
static int ragged_m_tiles(const GemmShape& g, int n_tiles) {
  const long long mt = (long long)g.R / BM + g.E;
  const long long t = mt * n_tiles;
  return t > (1 << 30) ? (1 << 30) : static_cast<int>(t);
}

// RAGGED_M GEMM, A K-major [R, K] act, B K-major weights [E*N_rows, K] (B_MN = false)
// or M/N-major weights [E*K, N] (B_MN = true).
template <typename T, bool B_MN, int EPI, int BN>
static moe_status run_m(const GemmShape& g, const void* A, int K, const void* B, int N,
                        int b_rows_per_expert, int b_cols, void* out, int64_t ldo, void* out_a,
                        const void* aux, const int32_t* offsets, int* status, cudaStream_t s) {
  using C = Cfg<T, BN>;
  const bool fp32 = sizeof(T) == 4;
  CUtensorMap ta, tb;
  if (!make_tmap(&ta, A, fp32, K, g.R, C::KB, BM)) return MOE_ECUDA;
  if (!B_MN) {
    const int box_rows = EPI == EPI_SWIGLU_FWD ? BN / 2 : BN;
    if (!make_tmap(&tb, B, fp32, K, (uint64_t)g.E * b_rows_per_expert, C::KB, box_rows))
      return MOE_ECUDA;
  } else {
    if (!make_tmap(&tb, B, fp32, b_cols, (uint64_t)g.E * b_rows_per_expert, C::MNB, C::KB, true))
      return MOE_ECUDA;
  }
  Params p{};
  p.offsets = offsets;
  p.E = g.E;
  p.R = g.R;
  p.N = N;
  p.K = K;
  p.b_rows_per_expert = b_rows_per_expert;
  p.f = g.f;
  p.out = out;
  p.ldo = ldo;
  p.out_a = out_a;
  p.aux = aux;
  p.status = status;
  return launch<T, BN, false, B_MN, RAGGED_M, EPI>(ta, tb, p, ragged_m_tiles(g, N / BN), s);
}

// RAGGED_K GEMM: dW_e[M, N] = G_e^T . X_e with G [R, M] and X [R, N] (both act, M/N-major).
template <typename T, int BN>
static moe_status run_k(const GemmShape& g, const void* G, int M, const void* X, int N, void* dW,
                        bool dw_fp32, bool accum, const int32_t* offsets, int* status,
                        cudaStream_t s) {
  using C = Cfg<T, BN>;
  const bool fp32 = sizeof(T) == 4;
  CUtensorMap ta, tb;
  if (!make_tmap(&ta, G, fp32, M, g.R, C::MNB, C::KB, true)) return MOE_ECUDA;
  if (!make_tmap(&tb, X, fp32, N, g.R, C::MNB, C::KB, true)) return MOE_ECUDA;
  Params p{};
  p.offsets = offsets;
  p.E = g.E;
  p.R = g.R;
  p.M = M;
  p.N = N;
  p.f = g.f;
  p.out = dW;
  p.out_fp32 = dw_fp32 ? 1 : 0;
  p.accumulate = accum ? 1 : 0;
  p.status = status;
  const long long tiles = (long long)g.E * (M / BM) * (N / BN);
  return launch<T, BN, true, true, RAGGED_K, EPI_STORE>(
      ta, tb, p, tiles > (1 << 30) ? (1 << 30) : (int)tiles, s);
}

#define MOE_DISPATCH_BN(bn, CALL)           \
  do {                                      \
    if ((bn) == 256) { constexpr int BN = 256; return CALL; } \
    if ((bn) == 128) { constexpr int BN = 128; return CALL; } \
    { constexpr int BN = 64; return CALL; }                   \
  } while (0)

template <typename T>
static moe_status fc1_fwd(const GemmShape& g, const void* x_perm, const void* W13,
                          const int32_t* off, void* H13, void* a, int* st, cudaStream_t s) {
  // accumulator grid: 2f columns, each tile = BN/2 gate columns + the matching BN/2 up columns
  const int bn = g.f % 128 == 0 ? 256 : 128;
  if (bn == 256)
    return run_m<T, false, EPI_SWIGLU_FWD, 256>(g, x_perm, g.d, W13, 2 * g.f, 2 * g.f, g.d, H13,
                                                 2 * (int64_t)g.f, a, nullptr, off, st, s);
  return run_m<T, false, EPI_SWIGLU_FWD, 128>(g, x_perm, g.d, W13, 2 * g.f, 2 * g.f, g.d, H13,
                                               2 * (int64_t)g.f, a, nullptr, off, st, s);
}

template <typename T>
static moe_status fc2_fwd(const GemmShape& g, const void* a, const void* W2, const int32_t* off,
                          void* y_perm, int* st, cudaStream_t s) {
  if (g.d % 256 == 0)
    return run_m<T, false, EPI_STORE, 256>(g, a, g.f, W2, g.d, g.d, g.f, y_perm, g.d, nullptr,
                                            nullptr, off, st, s);
  return run_m<T, false, EPI_STORE, 128>(g, a, g.f, W2, g.d, g.d, g.f, y_perm, g.d, nullptr,
                                          nullptr, off, st, s);
}

template <typename T>
static moe_status fc2_dgrad(const GemmShape& g, const void* dy_perm, const void* W2,
                            const void* H13, const int32_t* off, void* dH13, int* st,
                            cudaStream_t s) {
  // dA = dY . W2_e: K = d, N = f; B[n, k] = W2[e*d + k, n] (M/N-major)
  MOE_DISPATCH_BN(pick_bn(g.f),
                  (run_m<T, true, EPI_SWIGLU_BWD, BN>(g, dy_perm, g.d, W2, g.f, g.d, g.f, dH13,
                                                      2 * (int64_t)g.f, nullptr, H13, off, st, s)));
}

template <typename T>
static moe_status fc1_dgrad(const GemmShape& g, const void* dH13, const void* W13,
                            const int32_t* off, void* dx_perm, int* st, cudaStream_t s) {
  // dX = dH13 . W13_e: K = 2f, N = d; B[n, k] = W13[e*2f + k, n] (M/N-major)
  if (g.d % 256 == 0)
    return run_m<T, true, EPI_STORE, 256>(g, dH13, 2 * g.f, W13, g.d, 2 * g.f, g.d, dx_perm, g.d,
                                           nullptr, nullptr, off, st, s);
  return run_m<T, true, EPI_STORE, 128>(g, dH13, 2 * g.f, W13, g.d, 2 * g.f, g.d, dx_perm, g.d,
                                         nullptr, nullptr, off, st, s);
}

template <typename T>
static moe_status wgrad(const GemmShape& g, const void* G, int M, const void* X, int N, void* dW,
                        bool dw_fp32, bool accum, const int32_t* off, int* st, cudaStream_t s) {
  MOE_DISPATCH_BN(pick_bn(N), (run_k<T, BN>(g, G, M, X, N, dW, dw_fp32, accum, off, st, s)));
}

}  // namespace gemm

moe_status gemm_fwd(const GemmShape& g, const void* x_perm, const void* W13, const void* W2,
                    const int32_t* offsets, void* H13, void* a, void* y_perm, int* status,
                    cudaStream_t s) {
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
                             bool dw_fp32, bool dw_accum, int* st, cudaStream_t s) {
  moe_status r = gemm::fc2_dgrad<T>(g, dy_perm, W2, H13, off, dH13, st, s);
  if (r != MOE_OK) return r;
  r = gemm::wgrad<T>(g, dy_perm, g.d, a, g.f, dW2, dw_fp32, dw_accum, off, st, s);
  if (r != MOE_OK) return r;
  r = gemm::fc1_dgrad<T>(g, dH13, W13, off, dx_perm, st, s);
  if (r != MOE_OK) return r;
  return gemm::wgrad<T>(g, dH13, 2 * g.f, x_perm, g.d, dW13, dw_fp32, dw_accum, off, st, s);
}

moe_status gemm_bwd(const GemmShape& g, const void* dy_perm, const void* x_perm, const void* H13,
                    const void* a, const void* W13, const void* W2, const int32_t* offsets,
                    void* dH13, void* dx_perm, void* dW13, void* dW2, bool dw_fp32,
                    bool dw_accum, int* status, cudaStream_t s) {
  if (g.fp32)
    return gemm_bwd_t<float>(g, dy_perm, x_perm, H13, a, W13, W2, offsets, dH13, dx_perm, dW13,
                             dW2, dw_fp32, dw_accum, status, s);
  return gemm_bwd_t<__nv_bfloat16>(g, dy_perm, x_perm, H13, a, W13, W2, offsets, dH13, dx_perm,
                                   dW13, dW2, dw_fp32, dw_accum, status, s);
}

}  // namespace moe
