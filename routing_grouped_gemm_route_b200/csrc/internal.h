// Internal launchers shared by the C-ABI entry points (not part of the ABI).
#pragma once

#include <cuda_runtime.h>
#include <stddef.h>
#include <stdint.h>

#include "moe.h"

namespace moe {

int num_sms();

// Launch as a programmatic dependent of the previous kernel in the stream (the kernel
// calls pdl_wait() before it touches global memory).
template <typename... KArgs, typename... Args>
cudaError_t launch_pdl(void (*kern)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t s,
                       Args... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = s;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kern, static_cast<KArgs>(args)...);
}

// ----------------------------------------------------------------------------- routing
// Top-k CTAs take 64 tokens each and write one row of the expert histogram; the slot
// CTAs take 256 (8 warps x 32 tokens) and read the expert bases at their first token.
constexpr int kRouteTokensPerHistRow = 64;
constexpr int kRouteTokensPerCta = 256;
inline int route_hist_rows(int T) { return (T + kRouteTokensPerHistRow - 1) / kRouteTokensPerHistRow; }
inline int route_ctas(int T) { return (T + kRouteTokensPerCta - 1) / kRouteTokensPerCta; }

// hist: route_hist_rows(T) x E int32; cta_base: route_ctas(T) x E int32 (scratch);
// done_counter: one word that is zero before the launch (the routing leaves it zero), or
// null to run the scan as a launch of its own.
cudaError_t launch_route(const moe_desc& d, const float* logits, int32_t* topk_idx, float* gates,
                         int32_t* counts, int32_t* offsets, int32_t* slot, int32_t* row_token,
                         float* row_gate, int32_t* hist, int32_t* cta_base,
                         unsigned int* done_counter, int* status, cudaStream_t s);

// C[M,N] (fp32 out, or act out) = A . B with arbitrary element strides; a plain
// CUDA-core kernel for the small router projections.
cudaError_t launch_load_stats(const int32_t* counts, int E, moe_load_stats_t* out, int32_t* status,
                              cudaStream_t s);
cudaError_t launch_router_gemm(bool fp32_act, int M, int N, int K, const void* A, int64_t sam,
                               int64_t sak, bool a_is_act, const void* B, int64_t sbk,
                               int64_t sbn, bool b_is_act, void* C, bool c_is_act,
                               bool accumulate, cudaStream_t s);

// MOE_CHECKS: whole-layout verification of the routing (slot a permutation / injection
// into the experts' ranges, offsets a monotone scan), setting MOE_DEV_CHECK_FAILED.
bool checks_enabled();
size_t check_scratch_bytes(int64_t R);   // the bitmap: one bit per routed row
// null slot: offsets only; null topk_idx / offsets / counts / row_token: those parts skipped
cudaError_t launch_checks(const int32_t* slot, const int32_t* topk_idx, const int32_t* offsets,
                          const int32_t* counts, const int32_t* row_token, int T, int k, int E,
                          int R, int capacity, uint32_t* bitmap, int* status, cudaStream_t s);

// ----------------------------------------------------------------------------- permute
// R: the number of routed rows (slots must be in [0, R)): T*k, or E*capacity padded.
cudaError_t launch_dispatch(bool fp32, int T, int d, int k, int R, const void* x,
                            const int32_t* slot, void* x_perm, int* status, cudaStream_t s);
// y[t] = sum_j w_tj * src[slot[t,j]] (+ extra[t] fp32 when given); w = gates or all ones.
// y[t] = extra[t] + extra2[t] + sum_j gates[t,j] * src[slot[t,j]] (fp32 sum; null extras
// and gates = 1 when gates is null)
cudaError_t launch_gather_sum(bool fp32, int T, int d, int k, int R, const void* src,
                              const float* gates, const int32_t* slot, const float* extra,
                              void* y, int* status, cudaStream_t s, const float* extra2 = nullptr);
// y[i] += extra[i] for n elements (fp32 add, one rounding to the act type)
cudaError_t launch_add_f32(bool fp32, int64_t n, void* y, const float* extra, cudaStream_t s);
cudaError_t launch_combine_bwd(bool fp32, int T, int d, int k, int E, int R, const void* dy,
                               const void* y_perm, const float* gates, const int32_t* topk_idx,
                               const int32_t* slot, void* dy_perm, float* d_logits, int* status,
                               cudaStream_t s);

// ----------------------------------------------------------------------------- MXFP8
size_t mx_sf_bytes(int64_t R, int C, int E);
// Row segments of a quantised tensor: the experts' ragged rows (off [E+1] with tile_pref /
// blk_pref their prefixes of ceil(rows_e/128) and ceil(rows_e/32), from launch_mx_prefix),
// or, with rows > 0, E uniform segments of `rows` rows (a weight tensor [E*rows, C]).
struct MxSegs {
  const int32_t* off = nullptr;
  const int32_t* tile_pref = nullptr;
  const int32_t* blk_pref = nullptr;
  int E = 0;
  int rows = 0;
};
cudaError_t launch_mx_prefix(const int32_t* seg_off, int E, int32_t* tile_pref, int32_t* blk_pref,
                             cudaStream_t s);
// x [R, C] bf16 -> rowwise codes/scales (codes_r non-null) and/or colwise ones (codes_c
// non-null), one read of x.  perm_f > 0: SwiGLU weight order of the rowwise scales.
cudaError_t launch_mx_quant(const void* x, int64_t R, int C, const MxSegs& g, int perm_f,
                            uint8_t* codes_r, uint8_t* sf_r, uint8_t* codes_c, uint8_t* sf_c,
                            int* status, cudaStream_t s);
// The C-ABI quantiser: prefix into `scratch` (2*(E+1) int32), then one direction.
cudaError_t launch_mx_quantize(const void* x, int64_t R, int C, const int32_t* seg_off, int E,
                               bool colwise, uint8_t* codes, uint8_t* sf, int32_t* scratch,
                               int* status, cudaStream_t s);

// Device buffers of the MXFP8 grouped GEMMs (codes + 512-byte scale chunks).
struct MxWork {
  int32_t* act_pref;      // [2(E+1)]: tile prefix (then 32-row prefix) of the experts' rows
  uint8_t *xr, *xr_sf, *xc, *xc_sf;       // x_perm rowwise / colwise
  uint8_t *ar, *ar_sf, *ac, *ac_sf;       // a
  uint8_t *dyr, *dyr_sf, *dyc, *dyc_sf;   // dy_perm
  uint8_t *dhr, *dhr_sf, *dhc, *dhc_sf;   // dH13
  uint8_t *w13r, *w13r_sf, *w13c, *w13c_sf;
  uint8_t *w2r, *w2r_sf, *w2c, *w2c_sf;
  // MOE_FLAG_MX_KEEP_WEIGHT_CODES: the forward's weight passes also write the column-wise
  // codes (w13c, w2c); the backward finds them ready and skips its weight passes
  bool w_col_in_fwd = false;
  bool w_col_ready = false;
};

// ----------------------------------------------------------------------------- grouped GEMM
struct GemmShape {
  int E, R, d, f;
  bool fp32;   // fp32 storage / TF32 MMA, else bf16
  bool mx;     // bf16 storage, MXFP8 (E4M3 + E8M0 per 32) GEMM operands
  bool test_stall = false;   // MOE_FLAG_TEST_WAIT_TIMEOUT: no loads, 10 ms waits
};
// FC1 (+SwiGLU epilogue) and FC2 forward.
moe_status gemm_fwd(const GemmShape& g, const void* x_perm, const void* W13, const void* W2,
                    const int32_t* offsets, void* H13, void* a, void* y_perm, int* status,
                    cudaStream_t s, const MxWork* mx = nullptr);
// FC2 dgrad (+SwiGLU bwd), FC2 wgrad, FC1 dgrad, FC1 wgrad.  `maps_ws`: 2*E*128 bytes
// of 128-byte-aligned device scratch for the per-expert tensor maps of the wgrads.
constexpr size_t kTensorMapBytes = 128;
moe_status gemm_bwd(const GemmShape& g, const void* dy_perm, const void* x_perm, const void* H13,
                    const void* a, const void* W13, const void* W2, const int32_t* offsets,
                    void* dH13, void* dx_perm, void* dW13, void* dW2, bool dw_fp32,
                    bool dw_accum, void* maps_ws, int* status, cudaStream_t s,
                    const MxWork* mx = nullptr);

// Router GEMMs on the tensor cores (bf16 operands, fp32 accumulation; E % 64 == 0):
// logits[T,E] = x . Wr; dx_extra[T,d] = dl16 . Wr^T (float); dWr[d,E] = x^T . dl16 (bf16),
// with dl16 the bf16 copy of d_logits and maps_ws 2 tensor maps of device scratch.
moe_status router_logits_tc(int T, int d, int E, const void* x, const void* Wr, float* logits,
                            int* status, cudaStream_t s);
moe_status router_bwd_tc(int T, int d, int E, const void* x, const void* Wr, const void* dl16,
                         float* dx_extra, void* dWr, void* maps_ws, int* status, cudaStream_t s);
cudaError_t launch_f32_to_bf16(int64_t n, const float* src, void* dst, cudaStream_t s);
// dst[i] = src[i] rounded to TF32 (n a multiple of 4)
cudaError_t launch_tf32_round(int64_t n, const float* src, float* dst, cudaStream_t s);

// Shared expert (a dense SwiGLU FFN over all g.R = T rows, one segment): forward writes
// H13s, as (act) and ys [T,d] (float); backward writes dH13s (act scratch), dxs [T,d]
// (float) and dW13s / dW2s (one expert's slice).  maps_ws: 2 tensor maps of scratch.
moe_status shared_fwd(const GemmShape& g, const void* x, const void* W13s, const void* W2s,
                      void* H13s, void* as, float* ys, int* status, cudaStream_t s);
moe_status shared_bwd(const GemmShape& g, const void* dy, const void* x, const void* H13s,
                      const void* as, const void* W13s, const void* W2s, void* dH13s, float* dxs,
                      void* dW13s, void* dW2s, bool dw_fp32, bool dw_accum, void* maps_ws,
                      int* status, cudaStream_t s);

}  // namespace moe
