// moe_route_noalloc: the routing entry point for callers that cannot hand the library a
// workspace.  Its scratch (the per-CTA expert histograms and the CTA bases inside each
// expert) lives in one file-scope device array instead of caller memory.
//
// Host code must not pass `g_route_scratch` itself to a kernel: in host code that name
// is only a host-side stand-in for the device array.  The device address is looked up
// once per device with cudaGetSymbolAddress, with that device current, and cached.
#include <cuda_runtime.h>

#include <mutex>

#include "internal.h"
#include "moe.h"

namespace moe {
namespace {

static __device__ __align__(256) unsigned char g_route_scratch[MOE_ROUTE_NOALLOC_SCRATCH_BYTES];

constexpr int kMaxDevices = 64;
std::mutex g_mutex;
void* g_scratch_ptr[kMaxDevices] = {nullptr};

// Device address of the scratch array on the current device (looked up on first use).
moe_status scratch_address(void** out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return MOE_ECUDA;
  if (dev < 0 || dev >= kMaxDevices) return MOE_EUNSUPPORTED;
  std::lock_guard<std::mutex> lock(g_mutex);
  if (!g_scratch_ptr[dev]) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_route_scratch) != cudaSuccess || !p) return MOE_ECUDA;
    g_scratch_ptr[dev] = p;
  }
  *out = g_scratch_ptr[dev];
  return MOE_OK;
}

inline bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

}  // namespace
}  // namespace moe

using namespace moe;

extern "C" moe_status moe_route_noalloc(const moe_desc* desc, const float* logits,
                                        int32_t* topk_idx, float* gates, int32_t* counts,
                                        int32_t* offsets, int32_t* slot, int32_t* row_token,
                                        float* row_gate, void* stream) {
  moe_status st = moe_check_desc(desc);
  if (st != MOE_OK) return st;
  const moe_desc& d = *desc;
  // The padded layout flags tokens beyond an expert's capacity in a status word, and
  // this call has none to report it through: refused rather than dropped silently.
  if (d.capacity > 0) return MOE_EUNSUPPORTED;
  // scratch: a 256-byte header (the routing's CTA counter), the histogram [ceil(T/64)][E],
  // then the slot-CTA bases [ceil(T/256)][E], int32 each, 256-byte aligned
  const size_t hist_bytes = size_t(route_hist_rows(d.T)) * d.E * sizeof(int32_t);
  const size_t base_bytes = size_t(route_ctas(d.T)) * d.E * sizeof(int32_t);
  const size_t part_al = (hist_bytes + 255) / 256 * 256;
  if (256 + part_al + base_bytes > size_t(MOE_ROUTE_NOALLOC_SCRATCH_BYTES)) return MOE_EWORKSPACE;
  if (!counts || !offsets) return MOE_EINVAL;
  if (!aligned16(counts) || !aligned16(offsets)) return MOE_EALIGN;
  const void* tok[] = {logits, topk_idx, gates, slot, row_token, row_gate};
  for (const void* p : tok) {
    if (d.T > 0 && !p) return MOE_EINVAL;
    if (p && !aligned16(p)) return MOE_EALIGN;
  }
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  if (d.T == 0) {
    if (cudaMemsetAsync(counts, 0, sizeof(int32_t) * d.E, s) != cudaSuccess) return MOE_ECUDA;
    return cudaMemsetAsync(offsets, 0, sizeof(int32_t) * (d.E + 1), s) == cudaSuccess ? MOE_OK
                                                                                   : MOE_ECUDA;
  }
  void* base = nullptr;
  st = scratch_address(&base);
  if (st != MOE_OK) return st;
  // The histogram and the bases are written in full before they are read; the CTA
  // counter must start at zero and is cleared here (every routing launch also leaves it
  // zero).  No status word: in the ragged layout routing writes only expert indices it
  // selected itself (always in [0, E)) and slots inside its own counts, so the kernels
  // have no error to flag.
  unsigned int* counter = static_cast<unsigned int*>(base);
  int32_t* hist = reinterpret_cast<int32_t*>(static_cast<char*>(base) + 256);
  int32_t* cta_base = reinterpret_cast<int32_t*>(static_cast<char*>(base) + 256 + part_al);
  if (cudaMemsetAsync(counter, 0, sizeof(unsigned int), s) != cudaSuccess) return MOE_ECUDA;
  return launch_route(d, logits, topk_idx, gates, counts, offsets, slot, row_token, row_gate, hist,
                      cta_base, counter, nullptr, s) == cudaSuccess
             ? MOE_OK
             : MOE_ECUDA;
}
