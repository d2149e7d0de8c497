// Row-wise dispatch into the expert-contiguous buffers, the weighted combine back to
// token order, and their backward passes.
//
// Dispatch writes each selected token row straight into its expert's input buffer
// (unite.ai, "पैरालेलिज़्म, प्रिसीजन, और मेमोरी तकनीकें"; donmalab.com, "擴展與最佳化手段");
// the write-ups name expert data movement as one of the costs MXFP8 reduces
// (unite.ai, same section).  All four passes are HBM-bound row copies: one warp per
// token, 16-byte vector loads and stores, each x row read once and written k times
// (dispatch), each routed row read once (combine, unpermute-reduce).  Combine and
// unpermute are gathers summed in fp32 in a fixed order: no atomics, deterministic.
#include <algorithm>

#include <cuda_runtime.h>
#include <cuda_bf16.h>

#include "common.cuh"
#include "internal.h"

namespace moe {

namespace {

constexpr int kWarps = 8;

__device__ __forceinline__ int bcast(int v, int src) { return __shfl_sync(0xffffffffu, v, src); }
__device__ __forceinline__ float bcastf(float v, int src) {
  return __shfl_sync(0xffffffffu, v, src);
}

// x_perm[slot[t,j]] = x[t]
template <typename T>
__global__ void __launch_bounds__(kWarps * 32) dispatch_kernel(const T* __restrict__ x,
                                                               const int32_t* __restrict__ slot,
                                                               T* __restrict__ x_perm, int T_,
                                                               int d, int k, int R, int* status) {
  pdl_wait();
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int t = blockIdx.x * kWarps + warp;
  if (t >= T_) return;
  int my = -1;
  if (lane < k) {
    my = slot[(int64_t)t * k + lane];
    if (my < 0 || my >= R) {
      set_status(status, MOE_DEV_BAD_INDEX);
      my = -1;
    }
  }
  constexpr int V = 16 / sizeof(T);
  const int nvec = d / V;
  const T* src = x + (int64_t)t * d;
  constexpr int U = 4;
  // warp-uniform trip counts: the slot broadcasts below need every lane
  for (int base = 0; base < nvec; base += 32 * U) {
    uint4 buf[U];
#pragma unroll
    for (int u = 0; u < U; ++u) {
      const int v = base + u * 32 + lane;
      if (v < nvec) buf[u] = ld_stream16(src + (int64_t)v * V);
      // fp32: x_perm feeds TF32 GEMMs only (FC1, FC1 wgrad): rounded to TF32 here
      if constexpr (sizeof(T) == 4) buf[u] = tf32_round4(buf[u]);
    }
    for (int j = 0; j < k; ++j) {
      const int s = bcast(my, j);
      if (s < 0) continue;
      T* dst = x_perm + (int64_t)s * d;
#pragma unroll
      for (int u = 0; u < U; ++u) {
        const int v = base + u * 32 + lane;
        if (v < nvec) stg16(dst + (int64_t)v * V, buf[u]);
      }
    }
  }
  pdl_trigger();
}

// y[t] = sum_j w_tj * src[slot[t,j]] (+ extra[t]), w = gates or 1
template <typename T, int KMAX>
__global__ void __launch_bounds__(kWarps * 32) gather_sum_kernel(
    const T* __restrict__ src, const float* __restrict__ gates, const int32_t* __restrict__ slot,
    const float* __restrict__ extra, const float* __restrict__ extra2, T* __restrict__ y, int T_,
    int d, int k, int R, int* status) {
  pdl_wait();
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int t = blockIdx.x * kWarps + warp;
  if (t >= T_) return;
  int my_s = -1;
  float my_g = 0.f;
  if (lane < k) {
    my_s = slot[(int64_t)t * k + lane];
    my_g = gates ? gates[(int64_t)t * k + lane] : 1.0f;
    if (my_s < 0 || my_s >= R) {
      set_status(status, MOE_DEV_BAD_INDEX);
      my_s = -1;
    }
  }
  int s[KMAX];
  float g[KMAX];
#pragma unroll
  for (int j = 0; j < KMAX; ++j) {
    s[j] = bcast(my_s, j);
    g[j] = bcastf(my_g, j);
  }
  constexpr int V = 16 / sizeof(T);
  const int nvec = d / V;
  for (int v = lane; v < nvec; v += 32) {
    float acc[V];
#pragma unroll
    for (int i = 0; i < V; ++i) acc[i] = 0.f;
    if (extra) {
      const float* ex = extra + (int64_t)t * d + (int64_t)v * V;
#pragma unroll
      for (int i = 0; i < V; i += 4) {
        const float4 e4 = *reinterpret_cast<const float4*>(ex + i);
        acc[i] = e4.x; acc[i + 1] = e4.y; acc[i + 2] = e4.z; acc[i + 3] = e4.w;
      }
    }
    if (extra2) {
      const float* ex = extra2 + (int64_t)t * d + (int64_t)v * V;
#pragma unroll
      for (int i = 0; i < V; i += 4) {
        const float4 e4 = *reinterpret_cast<const float4*>(ex + i);
        acc[i] += e4.x; acc[i + 1] += e4.y; acc[i + 2] += e4.z; acc[i + 3] += e4.w;
      }
    }
    Vec16<T> in[KMAX];
#pragma unroll
    for (int j = 0; j < KMAX; ++j)
      if (j < k && s[j] >= 0) in[j].raw = ld_stream16(src + (int64_t)s[j] * d + (int64_t)v * V);
#pragma unroll
    for (int j = 0; j < KMAX; ++j) {
      if (j < k && s[j] >= 0) {
        float f[V];
        in[j].to_float(f);
#pragma unroll
        for (int i = 0; i < V; ++i) acc[i] = fmaf(g[j], f[i], acc[i]);
      }
    }
    Vec16<T> o;
    o.from_float(acc);
    stg16(y + (int64_t)t * d + (int64_t)v * V, o.raw);
  }
  pdl_trigger();
}

// dy_perm[slot] = g * dy[t]; dg = <dy[t], y_perm[slot]>; d_logits via the softmax Jacobian
template <typename T, int KMAX>
__global__ void __launch_bounds__(kWarps * 32) combine_bwd_kernel(
    const T* __restrict__ dy, const T* __restrict__ y_perm, const float* __restrict__ gates,
    const int32_t* __restrict__ topk_idx, const int32_t* __restrict__ slot, T* __restrict__ dy_perm,
    float* __restrict__ d_logits, int T_, int d, int k, int E, int R, int* status) {
  pdl_wait();
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int t = blockIdx.x * kWarps + warp;
  if (t >= T_) return;
  int my_s = -1, my_e = -1;
  float my_g = 0.f;
  if (lane < k) {
    my_s = slot[(int64_t)t * k + lane];
    my_e = topk_idx[(int64_t)t * k + lane];
    my_g = gates[(int64_t)t * k + lane];
    if (my_s < 0 || my_s >= R || my_e < 0 || my_e >= E) {
      set_status(status, MOE_DEV_BAD_INDEX);
      my_s = -1;
    }
  }
  int s[KMAX];
  float g[KMAX], dot[KMAX];
#pragma unroll
  for (int j = 0; j < KMAX; ++j) {
    s[j] = bcast(my_s, j);
    g[j] = bcastf(my_g, j);
    dot[j] = 0.f;
  }
  constexpr int V = 16 / sizeof(T);
  const int nvec = d / V;
  for (int v = lane; v < nvec; v += 32) {
    Vec16<T> gy;
    gy.raw = ld_stream16(dy + (int64_t)t * d + (int64_t)v * V);
    float fdy[V];
    gy.to_float(fdy);
    Vec16<T> yin[KMAX];
#pragma unroll
    for (int j = 0; j < KMAX; ++j)
      if (j < k && s[j] >= 0) yin[j].raw = ld_stream16(y_perm + (int64_t)s[j] * d + (int64_t)v * V);
#pragma unroll
    for (int j = 0; j < KMAX; ++j) {
      if (j < k && s[j] >= 0) {
        float fy[V], o[V];
        yin[j].to_float(fy);
#pragma unroll
        for (int i = 0; i < V; ++i) {
          dot[j] = fmaf(fdy[i], fy[i], dot[j]);
          o[i] = g[j] * fdy[i];
          // fp32: dy_perm feeds TF32 GEMMs only (FC2 dgrad, FC2 wgrad): rounded to TF32
          if constexpr (sizeof(T) == 4) o[i] = tf32_round(o[i]);
        }
        Vec16<T> pk;
        pk.from_float(o);
        stg16(dy_perm + (int64_t)s[j] * d + (int64_t)v * V, pk.raw);
      }
    }
  }
  // lane j ends with dg_j
  float my_dg = 0.f;
#pragma unroll
  for (int j = 0; j < KMAX; ++j) {
    const float tot = warp_sum(dot[j]);
    if (lane == j) my_dg = tot;
  }
  const float sgd = warp_sum(lane < k ? my_g * my_dg : 0.f);
  const float my_dl = my_g * (my_dg - sgd);
  // d_logits row: selected experts get their value, the rest 0
  float* row = d_logits + (int64_t)t * E;
  for (int e = lane; e < E; e += 32) row[e] = 0.f;
  __syncwarp();
  if (lane < k && my_e >= 0 && my_e < E) row[my_e] = my_dl;
  pdl_trigger();
}

// y[i] += extra[i] (fp32 add, one rounding to T)
template <typename T>
__global__ void add_f32_kernel(T* y, const float* __restrict__ extra, int64_t n) {
  constexpr int V = 16 / sizeof(T);
  const int64_t nv = n / V;
  for (int64_t v = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; v < nv;
       v += (int64_t)gridDim.x * blockDim.x) {
    Vec16<T> a;
    a.raw = *reinterpret_cast<const uint4*>(y + v * V);
    float f[V];
    a.to_float(f);
#pragma unroll
    for (int i = 0; i < V; ++i) f[i] += extra[v * V + i];
    a.from_float(f);
    stg16(y + v * V, a.raw);
  }
}

inline int kmax_of(int k) { return k <= 1 ? 1 : k <= 2 ? 2 : k <= 4 ? 4 : k <= 8 ? 8 : k <= 16 ? 16 : 32; }

}  // namespace

cudaError_t launch_add_f32(bool fp32, int64_t n, void* y, const float* extra, cudaStream_t s) {
  if (n == 0) return cudaSuccess;
  const int blocks = 4 * num_sms();
  if (fp32) add_f32_kernel<float><<<blocks, 256, 0, s>>>((float*)y, extra, n);
  else add_f32_kernel<__nv_bfloat16><<<blocks, 256, 0, s>>>((__nv_bfloat16*)y, extra, n);
  return cudaGetLastError();
}

// dst = src rounded to TF32 (tf32_round), n a multiple of 4: the fp32 weights (and the
// shared expert's x and dy) before the TF32 GEMMs read them.
__global__ void tf32_round_kernel(const float* __restrict__ src, float* __restrict__ dst,
                                  int64_t n) {
  const int64_t nv = n / 4;
  for (int64_t v = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; v < nv;
       v += (int64_t)gridDim.x * blockDim.x)
    reinterpret_cast<uint4*>(dst)[v] = tf32_round4(reinterpret_cast<const uint4*>(src)[v]);
}

cudaError_t launch_tf32_round(int64_t n, const float* src, float* dst, cudaStream_t s) {
  if (n == 0) return cudaSuccess;
  if (n % 4 != 0) return cudaErrorInvalidValue;
  const int64_t nv = n / 4;
  const int blocks = (int)std::min<int64_t>((nv + 255) / 256, (int64_t)num_sms() * 8);
  tf32_round_kernel<<<blocks, 256, 0, s>>>(src, dst, n);
  return cudaGetLastError();
}

// bf16 copy (round to nearest even) of a float array; n a multiple of 8.
__global__ void f32_to_bf16_kernel(const float* __restrict__ src, __nv_bfloat16* dst, int64_t n) {
  const int64_t nv = n / 8;
  for (int64_t v = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; v < nv;
       v += (int64_t)gridDim.x * blockDim.x) {
    const float4 a = reinterpret_cast<const float4*>(src)[2 * v];
    const float4 b = reinterpret_cast<const float4*>(src)[2 * v + 1];
    const float f[8] = {a.x, a.y, a.z, a.w, b.x, b.y, b.z, b.w};
    Vec16<__nv_bfloat16> o;
    o.from_float(f);
    stg16(dst + v * 8, o.raw);
  }
}

cudaError_t launch_f32_to_bf16(int64_t n, const float* src, void* dst, cudaStream_t s) {
  if (n == 0) return cudaSuccess;
  if (n % 8 != 0) return cudaErrorInvalidValue;
  const int64_t nv = n / 8;
  const int blocks = (int)std::min<int64_t>((nv + 255) / 256, (int64_t)num_sms() * 8);
  f32_to_bf16_kernel<<<blocks, 256, 0, s>>>(src, reinterpret_cast<__nv_bfloat16*>(dst), n);
  return cudaGetLastError();
}

cudaError_t launch_dispatch(bool fp32, int T, int d, int k, int R, const void* x,
                            const int32_t* slot, void* x_perm, int* status, cudaStream_t s) {
  if (T == 0) return cudaSuccess;
  const int blocks = (T + kWarps - 1) / kWarps;
  if (fp32)
    return launch_pdl(dispatch_kernel<float>, blocks, kWarps * 32, 0, s, (const float*)x, slot,
                      (float*)x_perm, T, d, k, R, status);
  return launch_pdl(dispatch_kernel<__nv_bfloat16>, blocks, kWarps * 32, 0, s,
                    (const __nv_bfloat16*)x, slot, (__nv_bfloat16*)x_perm, T, d, k, R, status);
}

template <typename T>
static cudaError_t gather_sum_t(int km, int blocks, cudaStream_t s, const void* src,
                                const float* gates, const int32_t* slot, const float* extra,
                                const float* extra2, void* y, int T_, int d, int k, int R,
                                int* status) {
#define MOE_GS(KM)                                                                             \
  return launch_pdl(gather_sum_kernel<T, KM>, blocks, kWarps * 32, 0, s, (const T*)src, gates, \
                    slot, extra, extra2, (T*)y, T_, d, k, R, status)
  switch (km) {
    case 1: MOE_GS(1);
    case 2: MOE_GS(2);
    case 4: MOE_GS(4);
    case 8: MOE_GS(8);
    case 16: MOE_GS(16);
    default: MOE_GS(32);
  }
#undef MOE_GS
}

cudaError_t launch_gather_sum(bool fp32, int T, int d, int k, int R, const void* src,
                              const float* gates, const int32_t* slot, const float* extra,
                              void* y, int* status, cudaStream_t s, const float* extra2) {
  if (T == 0) return cudaSuccess;
  const int blocks = (T + kWarps - 1) / kWarps;
  const int km = kmax_of(k);
  if (fp32)
    return gather_sum_t<float>(km, blocks, s, src, gates, slot, extra, extra2, y, T, d, k, R,
                               status);
  return gather_sum_t<__nv_bfloat16>(km, blocks, s, src, gates, slot, extra, extra2, y, T, d, k,
                                     R, status);
}

template <typename T>
static cudaError_t combine_bwd_t(int km, int blocks, cudaStream_t s, const void* dy,
                                 const void* y_perm, const float* gates, const int32_t* idx,
                                 const int32_t* slot, void* dy_perm, float* dl, int T_, int d,
                                 int k, int E, int R, int* status) {
#define MOE_CB(KM)                                                                              \
  return launch_pdl(combine_bwd_kernel<T, KM>, blocks, kWarps * 32, 0, s, (const T*)dy,         \
                    (const T*)y_perm, gates, idx, slot, (T*)dy_perm, dl, T_, d, k, E, R, status)
  switch (km) {
    case 1: MOE_CB(1);
    case 2: MOE_CB(2);
    case 4: MOE_CB(4);
    case 8: MOE_CB(8);
    case 16: MOE_CB(16);
    default: MOE_CB(32);
  }
#undef MOE_CB
}

cudaError_t launch_combine_bwd(bool fp32, int T, int d, int k, int E, int R, const void* dy,
                               const void* y_perm, const float* gates, const int32_t* topk_idx,
                               const int32_t* slot, void* dy_perm, float* d_logits, int* status,
                               cudaStream_t s) {
  if (T == 0) return cudaSuccess;
  const int blocks = (T + kWarps - 1) / kWarps;
  const int km = kmax_of(k);
  if (fp32)
    return combine_bwd_t<float>(km, blocks, s, dy, y_perm, gates, topk_idx, slot, dy_perm,
                                d_logits, T, d, k, E, R, status);
  return combine_bwd_t<__nv_bfloat16>(km, blocks, s, dy, y_perm, gates, topk_idx, slot, dy_perm,
                                      d_logits, T, d, k, E, R, status);
}

}  // namespace moe
