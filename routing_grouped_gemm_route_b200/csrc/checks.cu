// Optional device checks of the routing layout (the MOE_CHECKS environment switch).
//
// The kernels always check the indices they are given (an out-of-range slot or expert
// index sets MOE_DEV_BAD_INDEX and the row is skipped; offsets that are not an exclusive
// scan ending at R set MOE_DEV_BAD_OFFSETS in the grouped GEMM).  With MOE_CHECKS set,
// the calls that produce or consume the expert-sorted layout also verify it as a whole,
// which those local checks cannot: that `slot` maps the T*k (token, expert) pairs to
// distinct rows (a device bitmap with one bit per row), that the offsets are a monotone
// scan of the counts ending at R (ragged layout) or the multiples of the capacity
// (padded layout), that every pair's row lies in its expert's range, and that
// row_token[slot[t,j]] == t.  A failure sets MOE_DEV_CHECK_FAILED; nothing else changes.
#include <cuda_runtime.h>
#include <stdint.h>

#include <algorithm>

#include "common.cuh"
#include "internal.h"

namespace moe {
namespace {

// offsets / counts: one thread per expert.
__global__ void check_offsets_kernel(const int32_t* __restrict__ offsets,
                                     const int32_t* __restrict__ counts, int E, int R, int capacity,
                                     int* status) {
  for (int e = blockIdx.x * blockDim.x + threadIdx.x; e <= E; e += gridDim.x * blockDim.x) {
    bool ok = true;
    if (e == 0) ok = offsets[0] == 0;
    if (e == E) ok = capacity > 0 ? offsets[E] == E * capacity : offsets[E] == R;
    if (e < E) {
      const int span = offsets[e + 1] - offsets[e];
      ok = span >= 0 && (capacity > 0 ? span == capacity : true);
      if (counts) ok = ok && counts[e] >= 0 && (capacity > 0 ? counts[e] <= capacity : counts[e] == span);
    }
    if (!ok) set_status(status, MOE_DEV_CHECK_FAILED);
  }
}

// slot: every pair's row in [0, R), no row taken twice (bitmap, cleared beforehand);
// with topk_idx and offsets, the row inside its expert's range; with row_token, the row's
// token is the pair's.
__global__ void check_slots_kernel(const int32_t* __restrict__ slot,
                                   const int32_t* __restrict__ topk_idx,
                                   const int32_t* __restrict__ offsets,
                                   const int32_t* __restrict__ row_token, int T, int k, int E,
                                   int R, uint32_t* __restrict__ bitmap, int* status) {
  const int64_t n = (int64_t)T * k;
  for (int64_t i = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; i < n;
       i += (int64_t)gridDim.x * blockDim.x) {
    const int s = slot[i];
    bool ok = s >= 0 && s < R;
    if (ok) {
      const uint32_t bit = 1u << (s & 31);
      ok = (atomicOr(&bitmap[s >> 5], bit) & bit) == 0;          // not taken before
      if (topk_idx && offsets) {
        const int e = topk_idx[i];
        ok = ok && e >= 0 && e < E && s >= offsets[e] && s < offsets[e + 1];
      }
      if (row_token) ok = ok && row_token[s] == static_cast<int>(i / k);
    }
    if (!ok) set_status(status, MOE_DEV_CHECK_FAILED);
  }
}

}  // namespace

bool checks_enabled() {
  const char* v = getenv("MOE_CHECKS");
  return v && v[0] && !(v[0] == '0' && v[1] == 0);
}

size_t check_scratch_bytes(int64_t R) { return (size_t)((R + 31) / 32) * 4; }

cudaError_t launch_checks(const int32_t* slot, const int32_t* topk_idx, const int32_t* offsets,
                          const int32_t* counts, const int32_t* row_token, int T, int k, int E,
                          int R, int capacity, uint32_t* bitmap, int* status, cudaStream_t s) {
  cudaError_t err;
  if (offsets) {
    check_offsets_kernel<<<(E + 256) / 256, 256, 0, s>>>(offsets, counts, E, R, capacity, status);
    if ((err = cudaGetLastError()) != cudaSuccess) return err;
  }
  if (slot && T > 0) {
    if ((err = cudaMemsetAsync(bitmap, 0, check_scratch_bytes(R), s)) != cudaSuccess) return err;
    const int64_t n = (int64_t)T * k;
    const int blocks = (int)std::min<int64_t>((n + 255) / 256, (int64_t)num_sms() * 8);
    check_slots_kernel<<<blocks, 256, 0, s>>>(slot, topk_idx, offsets, row_token, T, k, E, R,
                                             bitmap, status);
    if ((err = cudaGetLastError()) != cudaSuccess) return err;
  }
  return cudaSuccess;
}

}  // namespace moe
