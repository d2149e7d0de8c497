// GPU-resident routing: top-k selection, renormalised gates, per-expert counts and
// offsets, and the expert-sorted slot of every (token, j) pair.
//
// The write-ups say the routing metadata now stays on the GPU, removing the old
// path's host round trip for the expert-group sizes, so the CPU can queue work
// without waiting for a copy back (deniz.in, "Ai2, Olmo-core 3'ü Apache 2.0 ile
// yayınladı", section "Yeni stack nasıl çalışıyor"; unite.ai, "पैरालेलिज़्म, प्रिसीजन,
// और मेमोरी तकनीकें").  Two launches (three above 256 experts, or above 32768 tokens
// when the caller gives no counter), no host sync:
//   1. topk:  one warp per token, logits in registers, k rounds of warp arg-max
//             (ties to the lower expert index); gates = softmax over the kept
//             logits; an expert histogram per 64 tokens (one CTA each, so even a
//             few thousand tokens spread over every SM).
//   2. prefix: per expert, an exclusive scan of the histogram rows gives the base of
//             every 256-token slot CTA inside the expert, the counts, and offsets =
//             exclusive scan of the counts.  Up to 512 histogram rows (32768 tokens)
//             and 256 experts, each slot CTA sums the rows it needs itself (step 3).
//             Above that, the last top-k CTA to finish runs the scan (a counter in
//             global memory, the classic fence-then-count pattern: no CTA waits for
//             another), each expert's column split over several threads; above 256
//             experts, where top-k runs 8-warp CTAs, it is a separate one-CTA launch.
//   3. slots: per warp of 32 tokens, a bitmask per expert of the lanes that chose
//             it; a token's rank inside the expert is the population count of the
//             lower lanes' bits plus the bases of earlier warps and CTAs.  So the
//             rows of an expert come out in token order.
#include <cuda_runtime.h>
#include <cuda_bf16.h>
#include <math.h>

#include "common.cuh"
#include "internal.h"

namespace moe {

namespace {

constexpr int kWarps = 8;
static_assert(kWarps * 32 == kRouteTokensPerCta, "one token per lane in the slot pass");
constexpr int kHistRowsPerCta = kRouteTokensPerCta / kRouteTokensPerHistRow;
static_assert(kHistRowsPerCta * kRouteTokensPerHistRow == kRouteTokensPerCta, "whole rows");

// Order-preserving 32-bit key of a logit: a > b as floats iff key(a) > key(b), with -0
// taken as +0 (they compare equal as floats).  Every logit's key is above 0, the key of
// "no candidate" (NaN is mapped to -inf before it gets here).
__device__ __forceinline__ uint32_t logit_key(float f) {
  const uint32_t b = __float_as_uint(f == 0.f ? 0.f : f);
  return (b & 0x80000000u) ? ~b : (b | 0x80000000u);
}
__device__ __forceinline__ float key_logit(uint32_t key) {
  return __uint_as_float((key & 0x80000000u) ? (key & 0x7fffffffu) : ~key);
}

// The scan, run by one CTA of 1024 threads.  Expert e's histogram column (nrows rows
// of 64 tokens) is cut into J = 1024 / Ep chunks of consecutive rows (Ep = E rounded up
// to 32), one thread each: a first pass sums the chunk (up to 32 rows held in
// registers, so all of a chunk's loads are in flight at once), the chunk sums give each
// thread its starting base, and a second pass writes the base at every 256-token slot
// CTA's first row.  Then offsets = exclusive scan of the experts' totals.  capacity > 0:
// the padded layout, offsets[e] = e * capacity instead.  The histogram is read with
// L1-bypassing loads: other CTAs of the same launch may have written it.
constexpr int kScanThreads = 1024;
constexpr int kScanKeep = 32;
__device__ __forceinline__ void scan_body(const int32_t* __restrict__ hist, int nrows, int E,
                                          int capacity, int32_t* __restrict__ cta_base,
                                          int32_t* __restrict__ counts,
                                          int32_t* __restrict__ offsets, int* s_part) {
  const int Ep = (E + 31) & ~31;                  // <= 1024
  const int J = kScanThreads / Ep;                // chunks per expert
  const int e = threadIdx.x % Ep, j = threadIdx.x / Ep;
  const bool live = e < E && j < J;
  const int per = (nrows + J - 1) / J;
  const int r0 = min(nrows, j * per), r1 = min(nrows, r0 + per);
  const bool keep = per <= kScanKeep;
  int vals[kScanKeep];
  int sum = 0;
  if (live) {
    if (keep) {
#pragma unroll
      for (int i = 0; i < kScanKeep; ++i) {
        const int r = r0 + i;
        vals[i] = r < r1 ? __ldcg(hist + (int64_t)r * E + e) : 0;
        sum += vals[i];
      }
    } else {
#pragma unroll 8
      for (int r = r0; r < r1; ++r) sum += __ldcg(hist + (int64_t)r * E + e);
    }
  }
  if (j < J) s_part[j * Ep + e] = sum;
  __syncthreads();
  int tot = 0;
  if (live) {
    int run = 0;
    for (int jj = 0; jj < J; ++jj) {
      const int v = s_part[jj * Ep + e];
      if (jj < j) run += v;
      tot += v;
    }
    if (keep) {
#pragma unroll
      for (int i = 0; i < kScanKeep; ++i) {
        const int r = r0 + i;
        if (r < r1 && r % kHistRowsPerCta == 0)
          cta_base[(int64_t)(r / kHistRowsPerCta) * E + e] = run;
        run += vals[i];
      }
    } else {
#pragma unroll 8
      for (int r = r0; r < r1; ++r) {
        if (r % kHistRowsPerCta == 0) cta_base[(int64_t)(r / kHistRowsPerCta) * E + e] = run;
        run += __ldcg(hist + (int64_t)r * E + e);
      }
    }
    if (j == 0) counts[e] = tot;
  }
  __syncthreads();                                // every chunk sum read
  // block-wide inclusive scan of the totals (thread i: expert i; Hillis-Steele)
  if (j == 0 && e < Ep) s_part[e] = e < E ? tot : 0;
  if (threadIdx.x >= Ep) s_part[threadIdx.x] = 0;
  __syncthreads();
  const int x = threadIdx.x;
  const int own = s_part[x];
  for (int o = 1; o < kScanThreads; o <<= 1) {
    const int add = x >= o ? s_part[x - o] : 0;
    __syncthreads();
    s_part[x] += add;
    __syncthreads();
  }
  if (x < E) offsets[x] = capacity > 0 ? x * capacity : s_part[x] - own;
  if (x == kScanThreads - 1) offsets[E] = capacity > 0 ? E * capacity : s_part[kScanThreads - 1];
}

__global__ void __launch_bounds__(kScanThreads) scan_kernel(const int32_t* __restrict__ hist,
                                                            int nrows, int E, int capacity,
                                                            int32_t* __restrict__ cta_base,
                                                            int32_t* __restrict__ counts,
                                                            int32_t* __restrict__ offsets) {
  __shared__ int s_part[kScanThreads];
  scan_body(hist, nrows, E, capacity, cta_base, counts, offsets, s_part);
}

// Top-k runs 32 warps per 64-token CTA (2 tokens a warp), two CTAs per SM.  Above 256
// experts a lane's logits need more registers than that allows: 8 warps there.
template <int NPL>
constexpr int topk_warps() { return NPL <= 8 ? 32 : 8; }
template <int NPL>
constexpr int topk_ctas_per_sm() { return NPL <= 8 ? 2 : 1; }

// Scan arguments for the top-k CTAs that finish last (fused: 32-warp CTAs, E <= 256).
struct FusedScan {
  unsigned int* done;      // CTAs finished so far (zero between launches; reset by the last)
  int capacity;
  int32_t* cta_base;
  int32_t* counts;
  int32_t* offsets;
};

// One warp per token.  Each round of the selection takes the largest remaining key of
// every lane (its lowest index on ties), the warp's largest key by one reduction and the
// lowest index holding it by a second: ties go to the lower expert index, as the
// descending stable order of the logits has it.
// FUSED: the CTA that finishes last runs the scan (compiled only where it is used: its
// register arrays do not fit the 32 registers a thread of the scan-free CTAs has).
template <int NPL, bool FUSED>   // logits per lane = ceil(E / 32)
__global__ void __launch_bounds__(topk_warps<NPL>() * 32, topk_ctas_per_sm<NPL>())
topk_kernel(const float* __restrict__ logits, int T, int E, int k, int32_t* __restrict__ topk_idx,
            float* __restrict__ gates, int32_t* __restrict__ hist, FusedScan fs) {
  extern __shared__ int s_hist[];          // [E] (fused: [max(E, kScanThreads)], then the scan's)
  pdl_wait();
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  for (int e = threadIdx.x; e < E; e += blockDim.x) s_hist[e] = 0;
  __syncthreads();

  const int t0 = blockIdx.x * kRouteTokensPerHistRow;
  // a warp's tokens: their logits are all loaded before the first selection (NPL <= 4:
  // two tokens a warp, 2 * NPL registers), so their memory latencies overlap
  constexpr int kPre = NPL <= 4 ? kRouteTokensPerHistRow / topk_warps<NPL>() : 1;
  float pre[kPre][NPL];
  if constexpr (kPre > 1) {
#pragma unroll
    for (int u = 0; u < kPre; ++u) {
      const int t = t0 + warp + u * topk_warps<NPL>();
#pragma unroll
      for (int c = 0; c < NPL; ++c) {
        const int e = c * 32 + lane;
        pre[u][c] = t < T && e < E ? logits[(int64_t)t * E + e] : 0.f;
      }
    }
  }
  for (int i = warp, u = 0; i < kRouteTokensPerHistRow; i += topk_warps<NPL>(), ++u) {
    const int t = t0 + i;
    if (t >= T) break;
    const float* row = logits + (int64_t)t * E;
    uint32_t key[NPL];
#pragma unroll
    for (int c = 0; c < NPL; ++c) {
      const int e = c * 32 + lane;
      float f = 0.f;
      if constexpr (kPre > 1) {
#pragma unroll
        for (int uu = 0; uu < kPre; ++uu)
          if (uu == u) f = pre[uu][c];
      } else {
        f = e < E ? row[e] : 0.f;
      }
      // a NaN logit ranks as -inf (it would lose every comparison, and a row of them
      // would select no expert at all)
      if (f != f) f = -INFINITY;
      key[c] = e < E ? logit_key(f) : 0u;
    }
    uint32_t my_key = 0u, top_key = 0u;
    int my_idx = 0;
    for (int j = 0; j < k; ++j) {
      uint32_t bk = 0u;
      int bc = 0;
#pragma unroll
      for (int c = 0; c < NPL; ++c) {
        if (key[c] > bk) {                 // strict: the lowest c wins a tie inside the lane
          bk = key[c];
          bc = c;
        }
      }
      const uint32_t wmax = __reduce_max_sync(0xffffffffu, bk);
      const uint32_t widx =
          __reduce_min_sync(0xffffffffu, bk == wmax ? static_cast<uint32_t>(bc * 32 + lane) : ~0u);
      if (static_cast<int>(widx & 31u) == lane) {
#pragma unroll
        for (int c = 0; c < NPL; ++c)
          if (c == static_cast<int>(widx >> 5)) key[c] = 0u;   // taken
      }
      if (j == 0) top_key = wmax;
      if (lane == j) {
        my_key = wmax;
        my_idx = static_cast<int>(widx);
      }
    }
    // gates: softmax over the kept logits, lane j holds entry j
    const float z = lane < k ? expf(key_logit(my_key) - key_logit(top_key)) : 0.f;
    const float sum = warp_sum(z);
    if (lane < k) {
      topk_idx[(int64_t)t * k + lane] = my_idx;
      gates[(int64_t)t * k + lane] = z / sum;
      if (my_idx < E) atomicAdd(&s_hist[my_idx], 1);   // always true for k <= E
    }
  }
  __syncthreads();
  for (int e = threadIdx.x; e < E; e += blockDim.x) hist[(int64_t)blockIdx.x * E + e] = s_hist[e];
  // This CTA is done: the slot kernel (a programmatic dependent, which waits for this
  // grid's completion itself) may be scheduled once every CTA got here.  Not earlier:
  // CTAs scheduled while top-k holds the SMs would crowd onto the few with room.
  pdl_trigger();
  if constexpr (FUSED && topk_warps<NPL>() * 32 == kScanThreads) {
    if (fs.done == nullptr) return;
    // the last CTA to finish scans every CTA's histogram row
    __shared__ int s_last;
    __threadfence();                     // this CTA's row, visible before it is counted
    __syncthreads();                     // (and every read of s_hist done)
    if (threadIdx.x == 0) s_last = atomicAdd(fs.done, 1u) == gridDim.x - 1;
    __syncthreads();
    if (!s_last) return;
    __threadfence();                     // every counted CTA's row is visible from here
    scan_body(hist, gridDim.x, E, fs.capacity, fs.cta_base, fs.counts, fs.offsets, s_hist);
    if (threadIdx.x == 0) *fs.done = 0u;   // ready for the next launch
  }
}

// Slots of one 256-token CTA.  NPL = 0: the expert bases of the CTA come from the scan
// (cta_base, offsets).  NPL > 0 (E <= 32 * NPL <= 256, at most kSlotScanRows histogram
// rows): the CTA sums the histogram rows itself -- its warps stride over the rows, lane L
// holds experts L + 32c -- into the rows before it (its base in each expert) and all rows
// (the counts), then scans the counts into offsets; CTA 0 writes counts and offsets.  No
// CTA waits for another and no separate scan runs: every CTA reads the histogram
// (nrows x E int32, 128 KB at 16384 tokens and 128 experts) from L2.
constexpr int kSlotScanRows = 512;
// 1024 threads: all 32 warps sum the histogram rows (a few rows each, all loads in
// flight at once), the first kWarps warps (one token a lane) place the CTA's tokens
constexpr int kSlotWarps = 32;
constexpr int kSlotThreads = kSlotWarps * 32;
static_assert(kSlotWarps >= kWarps, "the token warps are the first warps");
template <int NPL>
__global__ void __launch_bounds__(kSlotThreads) slot_kernel(
    const int32_t* __restrict__ topk_idx, const float* __restrict__ gates,
    int32_t* __restrict__ offsets, const int32_t* __restrict__ cta_base,
    const int32_t* __restrict__ hist, int nrows, int32_t* __restrict__ counts, int T, int E,
    int k, int capacity, int32_t* __restrict__ slot, int32_t* __restrict__ row_token,
    float* __restrict__ row_gate, int* status) {
  extern __shared__ unsigned s_mem[];
  unsigned* masks = s_mem;                                          // [kWarps][E]
  int* wbase = reinterpret_cast<int*>(s_mem + kWarps * E);          // [kWarps][E]
  int* s_off = wbase + kWarps * E;                                  // [E] (NPL > 0)
  int* s_pre = s_off + E;                                           // [kSlotWarps][E]
  int* s_tot = s_pre + kSlotWarps * E;                              // [kSlotWarps][E]
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  // launched as a programmatic dependent of the top-k kernel: everything it wrote is
  // visible from here on
  pdl_wait();
  int start = 0;                     // thread e: the CTA's first row in expert e
  if constexpr (NPL > 0) {
    // per-warp sums of the rows before this CTA and of all rows, into s_pre / s_tot
    const int r_cta = blockIdx.x * kHistRowsPerCta;
    int pre[NPL], tot[NPL];
#pragma unroll
    for (int c = 0; c < NPL; ++c) pre[c] = tot[c] = 0;
#pragma unroll 4
    for (int r = warp; r < nrows; r += kSlotWarps) {
#pragma unroll
      for (int c = 0; c < NPL; ++c) {
        const int e = c * 32 + lane;
        const int v = e < E ? __ldcg(hist + (int64_t)r * E + e) : 0;
        tot[c] += v;
        if (r < r_cta) pre[c] += v;
      }
    }
#pragma unroll
    for (int c = 0; c < NPL; ++c) {
      const int e = c * 32 + lane;
      if (e < E) {
        s_pre[warp * E + e] = pre[c];
        s_tot[warp * E + e] = tot[c];
      }
    }
    __syncthreads();
    // thread e: base and count of expert e; offsets = exclusive scan of the counts
    const int e = threadIdx.x;                 // E <= 256 < blockDim.x
    int base = 0, cnt = 0;
    if (e < E) {
#pragma unroll 8
      for (int w = 0; w < kSlotWarps; ++w) {
        base += s_pre[w * E + e];
        cnt += s_tot[w * E + e];
      }
    }
    int incl = cnt;                            // warp-inclusive scan, then across warps
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int v = __shfl_up_sync(0xffffffffu, incl, o);
      if (lane >= o) incl += v;
    }
    __shared__ int s_warp[kSlotWarps];
    if (lane == 31) s_warp[warp] = incl;
    __syncthreads();
    int before = 0, total = 0;
#pragma unroll 8
    for (int w = 0; w < kSlotWarps; ++w) {
      before += w < warp ? s_warp[w] : 0;
      total += s_warp[w];
    }
    const int off = capacity > 0 ? e * capacity : before + incl - cnt;
    if (e < E) {
      s_off[e] = off;
      start = off + base;
      if (blockIdx.x == 0) {
        counts[e] = cnt;
        offsets[e] = off;
      }
    }
    if (blockIdx.x == 0 && e == 0) offsets[E] = capacity > 0 ? E * capacity : total;
  }
  for (int i = threadIdx.x; i < kWarps * E; i += blockDim.x) masks[i] = 0u;
  __syncthreads();
  const int t = blockIdx.x * kRouteTokensPerCta + threadIdx.x;
  const bool live = threadIdx.x < kRouteTokensPerCta && t < T;   // warps 0 .. kWarps-1
  if (live) {
    for (int j = 0; j < k; ++j) {
      const int e = topk_idx[(int64_t)t * k + j];
      if (e >= 0 && e < E) atomicOr(&masks[warp * E + e], 1u << lane);
    }
  }
  __syncthreads();
  for (int e = threadIdx.x; e < E; e += blockDim.x) {
    int run = NPL > 0 ? start : offsets[e] + cta_base[(int64_t)blockIdx.x * E + e];
#pragma unroll
    for (int w = 0; w < kWarps; ++w) {
      wbase[w * E + e] = run;
      run += __popc(masks[w * E + e]);
    }
  }
  __syncthreads();
  if (live) {
    const unsigned lower = (1u << lane) - 1u;
    for (int j = 0; j < k; ++j) {
      const int e = topk_idx[(int64_t)t * k + j];
      if (e < 0 || e >= E) {
        set_status(status, MOE_DEV_BAD_INDEX);
        slot[(int64_t)t * k + j] = -1;
        continue;
      }
      const int s = wbase[warp * E + e] + __popc(masks[warp * E + e] & lower);
      const int off_e = NPL > 0 ? s_off[e] : offsets[e];
      if (capacity > 0 && s - off_e >= capacity) {
        // padded layout: the expert's rows are full (the capacity is below its count)
        set_status(status, MOE_DEV_BAD_INDEX);
        slot[(int64_t)t * k + j] = -1;
        continue;
      }
      slot[(int64_t)t * k + j] = s;
      row_token[s] = t;
      row_gate[s] = gates[(int64_t)t * k + j];
    }
  }
  pdl_trigger();
}

template <int NPL>
cudaError_t launch_topk(const float* logits, int T, int E, int k, int32_t* idx, float* gates,
                        int32_t* hist, const FusedScan& fs, cudaStream_t s) {
  const int ctas = route_hist_rows(T);
  // the fused scan reuses the histogram's shared memory (kScanThreads ints)
  const bool fused = fs.done != nullptr;
  const int words = fused && E < kScanThreads ? kScanThreads : E;
  if (fused)
    return launch_pdl(topk_kernel<NPL, true>, ctas, topk_warps<NPL>() * 32, words * sizeof(int),
                      s, logits, T, E, k, idx, gates, hist, fs);
  return launch_pdl(topk_kernel<NPL, false>, ctas, topk_warps<NPL>() * 32, words * sizeof(int), s,
                    logits, T, E, k, idx, gates, hist, fs);
}

// ----------------------------------------------------------------------------- router GEMM
// C[m, n] = sum_k A[m*sam + k*sak] * B[k*sbk + n*sbn], 32x32 output tile per block of
// 256 threads (4 outputs each), fp32 accumulation.
template <typename TA, typename TB, typename TC>
__global__ void __launch_bounds__(256) router_gemm_kernel(int M, int N, int K, const TA* A,
                                                          int64_t sam, int64_t sak, const TB* B,
                                                          int64_t sbk, int64_t sbn, TC* C,
                                                          int accumulate) {
  __shared__ float sA[32][33];
  __shared__ float sB[32][33];
  const int m0 = blockIdx.y * 32, n0 = blockIdx.x * 32;
  const int tx = threadIdx.x & 31, ty = threadIdx.x >> 5;   // ty in 0..7
  float acc[4] = {0.f, 0.f, 0.f, 0.f};
  for (int k0 = 0; k0 < K; k0 += 32) {
    for (int r = ty; r < 32; r += 8) {
      const int m = m0 + r, kk = k0 + tx;
      sA[r][tx] = (m < M && kk < K) ? Elem<TA>::to_f(A[m * sam + kk * sak]) : 0.f;
      const int kb = k0 + r, n = n0 + tx;
      sB[r][tx] = (kb < K && n < N) ? Elem<TB>::to_f(B[kb * sbk + n * sbn]) : 0.f;
    }
    __syncthreads();
#pragma unroll 8
    for (int kk = 0; kk < 32; ++kk) {
      const float b = sB[kk][tx];
#pragma unroll
      for (int i = 0; i < 4; ++i) acc[i] += sA[ty + 8 * i][kk] * b;
    }
    __syncthreads();
  }
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const int m = m0 + ty + 8 * i, n = n0 + tx;
    if (m < M && n < N) {
      float v = acc[i];
      if (accumulate) v += Elem<TC>::to_f(C[(int64_t)m * N + n]);
      C[(int64_t)m * N + n] = Elem<TC>::from_f(v);
    }
  }
}

// Expert load statistics: one CTA, thread e reads counts[e] (e < E <= 1024).  Sums in
// int64 (exact); the spread about the mean in double, reduced in a fixed order.
template <typename V, typename Op>
__device__ __forceinline__ V block_reduce(V v, Op op, V identity, V* scratch) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v = op(v, __shfl_xor_sync(0xffffffffu, v, o));
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (lane == 0) scratch[warp] = v;
  __syncthreads();
  const int nw = (blockDim.x + 31) >> 5;
  v = lane < nw ? scratch[lane] : identity;
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v = op(v, __shfl_xor_sync(0xffffffffu, v, o));
  __syncthreads();   // scratch free for the next reduction
  return v;
}

__global__ void __launch_bounds__(1024) load_stats_kernel(const int32_t* __restrict__ counts, int E,
                                                          moe_load_stats_t* out, int32_t* status) {
  __shared__ long long s_ll[32];
  __shared__ double s_d[32];
  const int e = threadIdx.x;
  long long c = 0;
  if (e < E) {
    c = counts[e];
    if (c < 0) {
      set_status(reinterpret_cast<int*>(status), MOE_DEV_BAD_OFFSETS);
      c = 0;
    }
  }
  auto add = [](long long a, long long b) { return a + b; };
  const long long lo = INT32_MIN, hi = INT32_MAX;
  const long long total = block_reduce(c, add, 0LL, s_ll);
  const long long mx = block_reduce(e < E ? c : lo,
                                    [](long long a, long long b) { return a > b ? a : b; }, lo, s_ll);
  const long long mn = block_reduce(e < E ? c : hi,
                                    [](long long a, long long b) { return a < b ? a : b; }, hi, s_ll);
  const long long empty = block_reduce((long long)(e < E && c == 0), add, 0LL, s_ll);
  const double mean = (double)total / (double)E;
  const double dev = e < E ? ((double)c - mean) * ((double)c - mean) : 0.0;
  const double ss = block_reduce(dev, [](double a, double b) { return a + b; }, 0.0, s_d);
  if (e == 0) {
    moe_load_stats_t r;
    r.total = total;
    r.max_count = (int32_t)mx;
    r.min_count = (int32_t)mn;
    r.num_empty = (int32_t)empty;
    r.num_experts = E;
    r.mean = mean;
    r.max_over_mean = total > 0 ? (double)mx / mean : 0.0;
    r.cv = total > 0 ? sqrt(ss / (double)E) / mean : 0.0;
    *out = r;
  }
}

}  // namespace

cudaError_t launch_route(const moe_desc& d, const float* logits, int32_t* topk_idx, float* gates,
                         int32_t* counts, int32_t* offsets, int32_t* slot, int32_t* row_token,
                         float* row_gate, int32_t* hist, int32_t* cta_base,
                         unsigned int* done_counter, int* status, cudaStream_t s) {
  const int T = d.T, E = d.E, k = d.k;
  const int ctas = route_ctas(T);
  cudaError_t err;
  const int npl = (E + 31) / 32;
  const int C = d.capacity;
  const int nrows = route_hist_rows(T);
  // up to 256 experts and kSlotScanRows histogram rows the slot CTAs sum the histogram
  // themselves; else, up to 256 experts, the last top-k CTA runs the scan (the CTAs have
  // 1024 threads); above that a one-CTA scan launch
  const bool in_slot = npl <= 8 && nrows <= kSlotScanRows;
  const bool fused = !in_slot && npl <= 8 && done_counter != nullptr;
  FusedScan fs{fused ? done_counter : nullptr, C, cta_base, counts, offsets};
  if (npl <= 1) err = launch_topk<1>(logits, T, E, k, topk_idx, gates, hist, fs, s);
  else if (npl <= 2) err = launch_topk<2>(logits, T, E, k, topk_idx, gates, hist, fs, s);
  else if (npl <= 4) err = launch_topk<4>(logits, T, E, k, topk_idx, gates, hist, fs, s);
  else if (npl <= 8) err = launch_topk<8>(logits, T, E, k, topk_idx, gates, hist, fs, s);
  else if (npl <= 16) err = launch_topk<16>(logits, T, E, k, topk_idx, gates, hist, fs, s);
  else err = launch_topk<32>(logits, T, E, k, topk_idx, gates, hist, fs, s);
  if (err != cudaSuccess) return err;
  if (!fused && !in_slot) {
    scan_kernel<<<1, kScanThreads, 0, s>>>(hist, nrows, E, C, cta_base, counts, offsets);
    if ((err = cudaGetLastError()) != cudaSuccess) return err;
  }
  const size_t smem =
      (size_t(2) * kWarps * E + (in_slot ? E + size_t(2) * kSlotWarps * E : 0)) * sizeof(int);
  if (C > 0 && T > 0) {
    // padded layout: rows no token fills are marked (token -1, gate 0)
    const size_t rows = (size_t)E * C;
    if ((err = cudaMemsetAsync(row_token, 0xff, rows * 4, s)) != cudaSuccess) return err;
    if ((err = cudaMemsetAsync(row_gate, 0, rows * 4, s)) != cudaSuccess) return err;
  }
  // The slot kernel is a programmatic dependent of the kernel before it (top-k, or the
  // scan): it may be scheduled while that one drains and waits for it in-kernel.  (The
  // padded layout's memsets come between them: then it is an ordinary launch.)
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(ctas, 1, 1);
  cfg.blockDim = dim3(kSlotThreads, 1, 1);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = s;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = C > 0 ? 0 : 1;
  auto go = [&](auto kern) {
    if (smem > 48 * 1024) {
      const cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                                 static_cast<int>(smem));
      if (e != cudaSuccess) return e;
    }
    return cudaLaunchKernelEx(&cfg, kern, (const int32_t*)topk_idx, (const float*)gates, offsets,
                              (const int32_t*)cta_base, (const int32_t*)hist, nrows, counts, T, E,
                              k, C, slot, row_token, row_gate, status);
  };
  if (!in_slot) err = go(slot_kernel<0>);
  else if (npl <= 1) err = go(slot_kernel<1>);
  else if (npl <= 2) err = go(slot_kernel<2>);
  else if (npl <= 4) err = go(slot_kernel<4>);
  else err = go(slot_kernel<8>);
  if (err != cudaSuccess) return err;
  return cudaGetLastError();
}

cudaError_t launch_load_stats(const int32_t* counts, int E, moe_load_stats_t* out, int32_t* status,
                              cudaStream_t s) {
  const int threads = (E + 31) / 32 * 32;
  load_stats_kernel<<<1, threads, 0, s>>>(counts, E, out, status);
  return cudaGetLastError();
}

cudaError_t launch_router_gemm(bool fp32_act, int M, int N, int K, const void* A, int64_t sam,
                               int64_t sak, bool a_is_act, const void* B, int64_t sbk,
                               int64_t sbn, bool b_is_act, void* C, bool c_is_act,
                               bool accumulate, cudaStream_t s) {
  dim3 grid((N + 31) / 32, (M + 31) / 32);
  using bf = __nv_bfloat16;
#define MOE_RG(TA, TB, TC)                                                                     \
  router_gemm_kernel<TA, TB, TC><<<grid, 256, 0, s>>>(M, N, K, (const TA*)A, sam, sak,           \
                                                      (const TB*)B, sbk, sbn, (TC*)C,             \
                                                      accumulate ? 1 : 0)
  if (fp32_act) {
    // every operand is float
    MOE_RG(float, float, float);
  } else if (a_is_act && b_is_act && !c_is_act) {
    MOE_RG(bf, bf, float);          // logits = x . Wr
  } else if (!a_is_act && b_is_act && !c_is_act) {
    MOE_RG(float, bf, float);       // d_logits . Wr^T into a float buffer
  } else if (a_is_act && !b_is_act && c_is_act) {
    MOE_RG(bf, float, bf);          // dWr = x^T . d_logits
  } else {
    return cudaErrorInvalidValue;
  }
#undef MOE_RG
  return cudaGetLastError();
}

}  // namespace moe
