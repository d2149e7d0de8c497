// C-ABI entry points: argument checks on the host, workspace carving and kernel
// launches on the caller's stream.  No call allocates, frees or waits for the device
// (except moe_read_device_status, whose purpose is to wait).
#include <cuda_runtime.h>
#include <stdint.h>
#include <string.h>

#include <mutex>
#include <unordered_map>

#include "internal.h"
#include "moe.h"

namespace moe {

int num_sms() {
  static int cache[64] = {0};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return 148;
  if (cache[dev] == 0) {
    int n = 0;
    if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0)
      n = 148;
    cache[dev] = n;
  }
  return cache[dev];
}

namespace {

constexpr size_t kAlign = 256;
// The workspace's first 256 bytes (zeroed by moe_workspace_init): the status word at 0,
// the routing's CTA counter here (every routing launch leaves it zero again).
constexpr size_t kRouteCounterOffset = 128;
inline size_t up(size_t x) { return (x + kAlign - 1) / kAlign * kAlign; }
inline bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }
inline size_t act_bytes(const moe_desc& d) { return d.dtype == MOE_FP32 ? 4 : 2; }
// Routed rows: T*k, or E*capacity in the capacity-padded layout (none without tokens).
inline int64_t R_of(const moe_desc& d) {
  if (d.T == 0) return 0;
  return d.capacity > 0 ? (int64_t)d.E * d.capacity : (int64_t)d.T * d.k;
}
inline bool padded(const moe_desc& d) { return d.capacity > 0 && d.T > 0; }
inline cudaStream_t S(void* s) { return reinterpret_cast<cudaStream_t>(s); }

struct WsLayout {
  size_t status, hist, cta_base, maps, dy_perm, dH13, dx_perm, dx_router;
  size_t rc_x_perm, rc_H13, rc_a, rc_y_perm;   // MOE_FLAG_RECOMPUTE: the activations
  size_t dl16;                                  // bf16 copy of d_logits (router, bf16)
  size_t sh_f32, sh_dH13, rc_sh_H13, rc_sh_a;   // shared expert: y / dx (float), dH13, recompute
  size_t mx_ints, mx_bytes[24];   // MXFP8 operands (codes and scale chunks), see MxWork
  size_t w13_t, w2_t, x_t, dy_t;  // fp32: TF32-rounded weights (and shared expert's x, dy)
  size_t checks;                  // MOE_CHECKS bitmap
  size_t total;
};

WsLayout ws_layout(const moe_desc& d) {
  WsLayout w;
  const size_t es = act_bytes(d);
  const size_t R = (size_t)R_of(d);
  const size_t hrows = (size_t)route_hist_rows(d.T), ctas = (size_t)route_ctas(d.T);
  size_t o = 0;
  w.status = o; o += kAlign;
  w.hist = o; o = up(o + hrows * d.E * 4);
  w.cta_base = o; o = up(o + ctas * d.E * 4);
  w.maps = o; o = up(o + 2 * (size_t)d.E * kTensorMapBytes);
  w.checks = o; o = up(o + check_scratch_bytes((int64_t)R));
  w.dy_perm = o; o = up(o + R * d.d * es);
  w.dH13 = o; o = up(o + R * 2 * (size_t)d.d_ff * es);
  w.dx_perm = o; o = up(o + R * d.d * es);
  w.dx_router = o;
  if (d.flags & MOE_FLAG_ROUTER) o = up(o + (size_t)d.T * d.d * 4);
  w.dl16 = o;
  if (d.flags & MOE_FLAG_ROUTER) o = up(o + (size_t)d.T * d.E * 2);
  const bool sh = d.flags & MOE_FLAG_SHARED_EXPERT;
  const bool rc = d.flags & MOE_FLAG_RECOMPUTE;
  const size_t T = d.T;
  w.sh_f32 = o; if (sh) o = up(o + T * d.d * 4);
  w.sh_dH13 = o; if (sh) o = up(o + T * 2 * (size_t)d.d_ff * es);
  w.rc_sh_H13 = o; if (sh && rc) o = up(o + T * 2 * (size_t)d.d_ff * es);
  w.rc_sh_a = o; if (sh && rc) o = up(o + T * (size_t)d.d_ff * es);
  w.rc_x_perm = o; if (rc) o = up(o + R * d.d * es);
  w.rc_H13 = o; if (rc) o = up(o + R * 2 * (size_t)d.d_ff * es);
  w.rc_a = o; if (rc) o = up(o + R * (size_t)d.d_ff * es);
  w.rc_y_perm = o; if (rc) o = up(o + R * d.d * es);
  w.w13_t = o; w.w2_t = o; w.x_t = o; w.dy_t = o;
  if (d.dtype == MOE_FP32) {
    const size_t nw = (size_t)d.E + (sh ? 1 : 0);
    w.w13_t = o; o = up(o + nw * 2 * (size_t)d.d_ff * d.d * 4);
    w.w2_t = o; o = up(o + nw * (size_t)d.d * d.d_ff * 4);
    w.x_t = o; if (sh) o = up(o + T * d.d * 4);
    w.dy_t = o; if (sh) o = up(o + T * d.d * 4);
  }
  w.mx_ints = o;
  if (d.dtype == MOE_MXFP8) {
    const size_t E = d.E, f = d.d_ff, dm = d.d;
    o = up(o + 2 * (E + 1) * 4);
    // (rows, cols, segments) of x_perm r/c, a r/c, dy r/c, dH13 r/c, W13 r/c, W2 r/c
    const size_t rows[12] = {R, R, R, R, R, R, R, R, E * 2 * f, E * 2 * f, E * dm, E * dm};
    const size_t cols[12] = {dm, dm, f, f, dm, dm, 2 * f, 2 * f, dm, dm, f, f};
    for (int i = 0; i < 12; ++i) {
      w.mx_bytes[2 * i] = o;
      o = up(o + rows[i] * cols[i]);
      w.mx_bytes[2 * i + 1] = o;
      o = up(o + mx_sf_bytes((int64_t)rows[i], (int)cols[i], d.E));
    }
  }
  w.total = o;
  return w;
}



moe_saved_layout saved_layout(const moe_desc& d) {
  moe_saved_layout s;
  const size_t es = act_bytes(d);
  const size_t T = d.T, k = d.k, R = (size_t)R_of(d), E = d.E;
  size_t o = 0;
  s.topk_idx = o; o = up(o + T * k * 4);
  s.gates = o; o = up(o + T * k * 4);
  s.counts = o; o = up(o + E * 4);
  s.offsets = o; o = up(o + (E + 1) * 4);
  s.slot = o; o = up(o + T * k * 4);
  s.row_token = o; o = up(o + R * 4);
  s.row_gate = o; o = up(o + R * 4);
  s.logits = o;
  if (d.flags & MOE_FLAG_ROUTER) o = up(o + T * E * 4);
  const bool keep = !(d.flags & MOE_FLAG_RECOMPUTE);   // else recomputed in the backward
  s.x_perm = o; if (keep) o = up(o + R * d.d * es);
  s.H13 = o; if (keep) o = up(o + R * 2 * (size_t)d.d_ff * es);
  s.a = o; if (keep) o = up(o + R * (size_t)d.d_ff * es);
  s.y_perm = o; if (keep) o = up(o + R * d.d * es);
  // shared expert: its H13 [T,2f] and a [T,f] for the backward
  const bool sh = keep && (d.flags & MOE_FLAG_SHARED_EXPERT);
  s.H13_shared = o; if (sh) o = up(o + T * 2 * (size_t)d.d_ff * es);
  s.a_shared = o; if (sh) o = up(o + T * (size_t)d.d_ff * es);
  s.total = o;
  return s;
}

moe_status check(const moe_desc* d) {
  if (!d) return MOE_EINVAL;
  if (d->T < 0 || d->d <= 0 || d->d_ff <= 0 || d->E < 1 || d->E > 1024 || d->k < 1 ||
      d->k > 32 || d->k > d->E)
    return MOE_EINVAL;
  if (d->d % 128 != 0 || d->d_ff % 64 != 0) return MOE_EINVAL;
  if ((int64_t)d->T * d->k >= (int64_t(1) << 31)) return MOE_EINVAL;
  if ((int64_t)d->E * 2 * d->d_ff >= (int64_t(1) << 31) || (int64_t)d->E * d->d >= (int64_t(1) << 31))
    return MOE_EINVAL;
  if (d->dtype != MOE_FP32 && d->dtype != MOE_BF16 && d->dtype != MOE_MXFP8) return MOE_EINVAL;
  if (d->flags & ~(MOE_FLAG_ROUTER | MOE_FLAG_DW_FP32 | MOE_FLAG_ACCUM_DW | MOE_FLAG_RECOMPUTE |
                   MOE_FLAG_SHARED_EXPERT | MOE_FLAG_MX_KEEP_WEIGHT_CODES |
                   MOE_FLAG_TEST_WAIT_TIMEOUT))
    return MOE_EINVAL;
  if ((d->flags & MOE_FLAG_MX_KEEP_WEIGHT_CODES) && d->dtype != MOE_MXFP8) return MOE_EINVAL;
  if (d->capacity < 0 || (int64_t)d->E * d->capacity >= (int64_t(1) << 31)) return MOE_EINVAL;
  if (d->flags & MOE_FLAG_SHARED_EXPERT) {
    if (d->dtype == MOE_MXFP8) return MOE_EUNSUPPORTED;
    if ((int64_t)(d->E + 1) * 2 * d->d_ff >= (int64_t(1) << 31) ||
        (int64_t)(d->E + 1) * d->d >= (int64_t(1) << 31))
      return MOE_EINVAL;
  }
  if ((d->flags & MOE_FLAG_ACCUM_DW) && !(d->flags & MOE_FLAG_DW_FP32)) return MOE_EINVAL;
  if (d->dtype == MOE_MXFP8 && d->d_ff % 128 != 0) return MOE_EUNSUPPORTED;
  return MOE_OK;
}

// Every pointer in the list must be non-null and 16-byte aligned.
moe_status ptrs(std::initializer_list<const void*> ps) {
  for (const void* p : ps) {
    if (!p) return MOE_EINVAL;
    if (!aligned16(p)) return MOE_EALIGN;
  }
  return MOE_OK;
}
// Pointers to buffers whose size is a multiple of T: with no tokens they may be null
// (an empty tensor has no storage); otherwise as above.
moe_status tptrs(const moe_desc& d, std::initializer_list<const void*> ps) {
  if (d.T > 0) return ptrs(ps);
  for (const void* p : ps)
    if (p && !aligned16(p)) return MOE_EALIGN;
  return MOE_OK;
}

moe_status ws_ok(const moe_desc& d, const void* ws, size_t ws_bytes) {
  if (!ws) return MOE_EINVAL;
  if (!aligned16(ws)) return MOE_EALIGN;
  if (ws_bytes < ws_layout(d).total) return MOE_EWORKSPACE;
  return MOE_OK;
}

inline int* status_ptr(void* ws) { return reinterpret_cast<int*>(ws); }
template <typename P>
inline P* at(void* base, size_t off) {
  return reinterpret_cast<P*>(reinterpret_cast<char*>(base) + off);
}
template <typename P>
inline const P* at(const void* base, size_t off) {
  return reinterpret_cast<const P*>(reinterpret_cast<const char*>(base) + off);
}
inline moe_status cu(cudaError_t e) { return e == cudaSuccess ? MOE_OK : MOE_ECUDA; }

MxWork mx_work(const moe_desc& d, void* ws) {
  const WsLayout w = ws_layout(d);
  MxWork m;
  int32_t* ints = at<int32_t>(ws, w.mx_ints);
  m.act_pref = ints;
  uint8_t* b[24];
  for (int i = 0; i < 24; ++i) b[i] = at<uint8_t>(ws, w.mx_bytes[i]);
  m.xr = b[0]; m.xr_sf = b[1]; m.xc = b[2]; m.xc_sf = b[3];
  m.ar = b[4]; m.ar_sf = b[5]; m.ac = b[6]; m.ac_sf = b[7];
  m.dyr = b[8]; m.dyr_sf = b[9]; m.dyc = b[10]; m.dyc_sf = b[11];
  m.dhr = b[12]; m.dhr_sf = b[13]; m.dhc = b[14]; m.dhc_sf = b[15];
  m.w13r = b[16]; m.w13r_sf = b[17]; m.w13c = b[18]; m.w13c_sf = b[19];
  m.w2r = b[20]; m.w2r_sf = b[21]; m.w2c = b[22]; m.w2c_sf = b[23];
  return m;
}

#define MOE_TRY(expr)                  \
  do {                                 \
    moe_status _st = (expr);           \
    if (_st != MOE_OK) return _st;     \
  } while (0)

// rows < 0: the routed rows T*k; else that many rows (the shared expert's T)
GemmShape gshape(const moe_desc& d, int rows = -1) {
  GemmShape g;
  g.E = d.E;
  g.R = rows < 0 ? (int)R_of(d) : rows;
  g.d = d.d;
  g.f = d.d_ff;
  g.fp32 = d.dtype == MOE_FP32;
  g.mx = d.dtype == MOE_MXFP8;
  g.test_stall = (d.flags & MOE_FLAG_TEST_WAIT_TIMEOUT) != 0;
  return g;
}

// fp32: the TF32 GEMMs read W13 / W2 rounded to TF32 (workspace copies made here; the
// tensor core would otherwise truncate them); other dtypes read them as they are.
struct Weights {
  const void* W13;
  const void* W2;
};
moe_status tf32_weights(const moe_desc& d, const void* W13, const void* W2, void* ws,
                        cudaStream_t s, Weights* out) {
  out->W13 = W13;
  out->W2 = W2;
  if (d.dtype != MOE_FP32) return MOE_OK;
  const WsLayout w = ws_layout(d);
  const int64_t nw = (int64_t)d.E + ((d.flags & MOE_FLAG_SHARED_EXPERT) ? 1 : 0);
  float* w13 = at<float>(ws, w.w13_t);
  float* w2 = at<float>(ws, w.w2_t);
  MOE_TRY(cu(launch_tf32_round(nw * 2 * d.d_ff * d.d, static_cast<const float*>(W13), w13, s)));
  MOE_TRY(cu(launch_tf32_round(nw * d.d * d.d_ff, static_cast<const float*>(W2), w2, s)));
  out->W13 = w13;
  out->W2 = w2;
  return MOE_OK;
}
// fp32 with the shared expert: its GEMMs read x (and dy) directly, rounded here
const void* tf32_tokens(const moe_desc& d, const void* src, size_t off, void* ws, cudaStream_t s,
                        moe_status* st) {
  *st = MOE_OK;
  if (d.dtype != MOE_FP32 || d.T == 0) return src;
  float* dst = at<float>(ws, off);
  *st = cu(launch_tf32_round((int64_t)d.T * d.d, static_cast<const float*>(src), dst, s));
  return dst;
}

// ---------------------------------------------------------------------------- bodies
// Permutation steps with the layout's row bound; the padded layout first clears the
// expert buffers its rows scatter into (padding rows must be zero for the weight
// gradients, which sum over every row of an expert).
moe_status dispatch_body(const moe_desc& d, const void* x, const int32_t* slot, void* x_perm,
                         int* st, cudaStream_t s) {
  const int R = (int)R_of(d);
  if (padded(d)) MOE_TRY(cu(cudaMemsetAsync(x_perm, 0, (size_t)R * d.d * act_bytes(d), s)));
  return cu(launch_dispatch(d.dtype == MOE_FP32, d.T, d.d, d.k, R, x, slot, x_perm, st, s));
}
moe_status combine_bwd_body(const moe_desc& d, const void* dy, const void* y_perm,
                            const float* gates, const int32_t* idx, const int32_t* slot,
                            void* dy_perm, float* d_logits, int* st, cudaStream_t s) {
  const int R = (int)R_of(d);
  if (padded(d)) MOE_TRY(cu(cudaMemsetAsync(dy_perm, 0, (size_t)R * d.d * act_bytes(d), s)));
  return cu(launch_combine_bwd(d.dtype == MOE_FP32, d.T, d.d, d.k, d.E, R, dy, y_perm, gates, idx,
                               slot, dy_perm, d_logits, st, s));
}

moe_status route_body(const moe_desc& d, const float* logits, int32_t* idx, float* gates,
                      int32_t* counts, int32_t* offsets, int32_t* slot, int32_t* row_token,
                      float* row_gate, void* ws, cudaStream_t s) {
  const WsLayout w = ws_layout(d);
  if (d.T == 0) {
    MOE_TRY(cu(cudaMemsetAsync(counts, 0, sizeof(int32_t) * d.E, s)));
    return cu(cudaMemsetAsync(offsets, 0, sizeof(int32_t) * (d.E + 1), s));
  }
  MOE_TRY(cu(launch_route(d, logits, idx, gates, counts, offsets, slot, row_token, row_gate,
                          at<int32_t>(ws, w.hist), at<int32_t>(ws, w.cta_base),
                          at<unsigned int>(ws, kRouteCounterOffset), status_ptr(ws), s)));
  if (checks_enabled())
    MOE_TRY(cu(launch_checks(slot, idx, offsets, counts, row_token, d.T, d.k, d.E, (int)R_of(d),
                             d.capacity, at<uint32_t>(ws, w.checks), status_ptr(ws), s)));
  return MOE_OK;
}

// MOE_FLAG_MX_KEEP_WEIGHT_CODES: for each workspace, the weights (pointers and shape) whose
// column-wise MX codes the last forward on it left in its w13c / w2c buffers.
struct KeptCodes {
  const void* W13;
  const void* W2;
  int E, d, f;
  bool operator==(const KeptCodes& o) const {
    return W13 == o.W13 && W2 == o.W2 && E == o.E && d == o.d && f == o.f;
  }
};
std::mutex g_kept_mu;
std::unordered_map<const void*, KeptCodes> g_kept;

bool keep_codes(const moe_desc& d) {
  return d.dtype == MOE_MXFP8 && (d.flags & MOE_FLAG_MX_KEEP_WEIGHT_CODES);
}
// After an MXFP8 forward enqueued its weight passes: remember (flag) or forget.
void kept_after_fwd(const moe_desc& d, const void* ws, const void* W13, const void* W2) {
  if (d.dtype != MOE_MXFP8) return;
  std::lock_guard<std::mutex> lk(g_kept_mu);
  if (keep_codes(d)) g_kept[ws] = KeptCodes{W13, W2, d.E, d.d, d.d_ff};
  else g_kept.erase(ws);
}
bool kept_ready(const moe_desc& d, const void* ws, const void* W13, const void* W2) {
  if (!keep_codes(d)) return false;
  std::lock_guard<std::mutex> lk(g_kept_mu);
  const auto it = g_kept.find(ws);
  return it != g_kept.end() && it->second == KeptCodes{W13, W2, d.E, d.d, d.d_ff};
}
void kept_forget(const void* ws) {
  std::lock_guard<std::mutex> lk(g_kept_mu);
  g_kept.erase(ws);
}

moe_status gemm_bwd_body(const moe_desc& d, const void* dy_perm, const void* x_perm,
                         const void* H13, const void* a, const void* W13, const void* W2,
                         const int32_t* offsets, void* dH13, void* dx_perm, void* dW13, void* dW2,
                         void* ws, cudaStream_t s) {
  const bool fp32_dw = d.flags & MOE_FLAG_DW_FP32;
  const bool acc = d.flags & MOE_FLAG_ACCUM_DW;
  if (R_of(d) == 0) {
    if (acc) return MOE_OK;
    const size_t es = fp32_dw ? 4 : act_bytes(d);
    MOE_TRY(cu(cudaMemsetAsync(dW13, 0, (size_t)d.E * 2 * d.d_ff * d.d * es, s)));
    return cu(cudaMemsetAsync(dW2, 0, (size_t)d.E * d.d * d.d_ff * es, s));
  }
  MxWork mx = mx_work(d, ws);
  mx.w_col_ready = kept_ready(d, ws, W13, W2);
  Weights wt;
  MOE_TRY(tf32_weights(d, W13, W2, ws, s, &wt));
  return gemm_bwd(gshape(d), dy_perm, x_perm, H13, a, wt.W13, wt.W2, offsets, dH13, dx_perm, dW13,
                  dW2, fp32_dw, acc, at<char>(ws, ws_layout(d).maps), status_ptr(ws), s, &mx);
}

// bf16 router GEMMs run on the tensor cores when E is a multiple of 64; fp32 (and other
// E) use the CUDA-core kernel.
inline bool router_tc(const moe_desc& d) { return d.dtype != MOE_FP32 && d.E % 64 == 0; }

moe_status router_fwd_body(const moe_desc& d, const void* x, const void* Wr, float* logits,
                           int* status, cudaStream_t s) {
  if (d.T == 0) return MOE_OK;
  if (router_tc(d)) return router_logits_tc(d.T, d.d, d.E, x, Wr, logits, status, s);
  const bool f32 = d.dtype == MOE_FP32;
  // logits[T,E] = x[T,d] . Wr[d,E]
  return cu(launch_router_gemm(f32, d.T, d.E, d.d, x, d.d, 1, true, Wr, d.E, 1, true, logits,
                               false, false, s));
}

moe_status router_bwd_body(const moe_desc& d, const void* x, const void* Wr,
                           const float* d_logits, float* dx_extra, void* dx_act, void* dWr,
                           void* ws, cudaStream_t s) {
  const bool f32 = d.dtype == MOE_FP32;
  if (d.T > 0 && dx_extra && router_tc(d)) {
    // d_logits rounded once to bf16 feeds both tensor-core products
    const WsLayout w = ws_layout(d);
    void* dl16 = at<char>(ws, w.dl16);
    MOE_TRY(cu(launch_f32_to_bf16((int64_t)d.T * d.E, d_logits, dl16, s)));
    return router_bwd_tc(d.T, d.d, d.E, x, Wr, dl16, dx_extra, dWr, at<char>(ws, w.maps),
                         status_ptr(ws), s);
  }
  if (d.T > 0) {
    if (dx_extra) {
      // dx_extra[T,d] (float) = d_logits[T,E] . Wr^T
      MOE_TRY(cu(launch_router_gemm(f32, d.T, d.d, d.E, d_logits, d.E, 1, false, Wr, 1, d.E, true,
                                    dx_extra, false, false, s)));
    } else {
      // dx[T,d] (act) += d_logits . Wr^T
      if (!f32) return MOE_EUNSUPPORTED;   // bf16 in-place add goes through dx_extra
      MOE_TRY(cu(launch_router_gemm(f32, d.T, d.d, d.E, d_logits, d.E, 1, false, Wr, 1, d.E, true,
                                    dx_act, true, true, s)));
    }
  }
  // dWr[d,E] = x^T . d_logits
  if (d.T == 0) {
    return cu(cudaMemsetAsync(dWr, 0, (size_t)d.d * d.E * act_bytes(d), s));
  }
  return cu(launch_router_gemm(f32, d.d, d.E, d.T, x, 1, d.d, true, d_logits, d.E, 1, false, dWr,
                               true, false, s));
}

}  // namespace
}  // namespace moe

using namespace moe;

extern "C" {

const char* moe_status_string(int32_t st) {
  switch (st) {
    case MOE_OK: return "ok";
    case MOE_EINVAL: return "invalid argument";
    case MOE_EALIGN: return "pointer not 16-byte aligned";
    case MOE_EWORKSPACE: return "workspace or saved buffer too small";
    case MOE_EUNSUPPORTED: return "unsupported configuration";
    case MOE_ECUDA: return "CUDA error";
    case MOE_EDEVICE: return "device-side error flagged in the status word";
    default: return "unknown status";
  }
}

moe_status moe_check_desc(const moe_desc* desc) { return check(desc); }

moe_status moe_workspace_size(const moe_desc* desc, size_t* bytes) {
  MOE_TRY(check(desc));
  if (!bytes) return MOE_EINVAL;
  *bytes = ws_layout(*desc).total;
  return MOE_OK;
}

moe_status moe_saved_layout_get(const moe_desc* desc, moe_saved_layout* out) {
  MOE_TRY(check(desc));
  if (!out) return MOE_EINVAL;
  *out = saved_layout(*desc);
  return MOE_OK;
}

moe_status moe_workspace_init(void* ws, size_t ws_bytes, void* stream) {
  if (!ws) return MOE_EINVAL;
  if (!aligned16(ws)) return MOE_EALIGN;
  if (ws_bytes < 256) return MOE_EWORKSPACE;
  kept_forget(ws);
  return cu(cudaMemsetAsync(ws, 0, 256, S(stream)));
}

moe_status moe_read_device_status(const void* ws, void* stream, int32_t* bits) {
  if (!ws || !bits) return MOE_EINVAL;
  int32_t v = 0;
  if (cudaMemcpyAsync(&v, ws, sizeof(v), cudaMemcpyDeviceToHost, S(stream)) != cudaSuccess)
    return MOE_ECUDA;
  if (cudaStreamSynchronize(S(stream)) != cudaSuccess) return MOE_ECUDA;
  *bits = v;
  return v ? MOE_EDEVICE : MOE_OK;
}

moe_status moe_router_logits(const moe_desc* desc, const void* x, const void* Wr, float* logits,
                             void* stream) {
  MOE_TRY(check(desc));
  MOE_TRY(tptrs(*desc, {x, logits}));
  MOE_TRY(ptrs({Wr}));
  return router_fwd_body(*desc, x, Wr, logits, nullptr, S(stream));
}

moe_status moe_route(const moe_desc* desc, const float* logits, int32_t* topk_idx, float* gates,
                     int32_t* counts, int32_t* offsets, int32_t* slot, int32_t* row_token,
                     float* row_gate, void* ws, size_t ws_bytes, void* stream) {
  MOE_TRY(check(desc));
  MOE_TRY(tptrs(*desc, {logits, topk_idx, gates, slot, row_token, row_gate}));
  MOE_TRY(ptrs({counts, offsets}));
  MOE_TRY(ws_ok(*desc, ws, ws_bytes));
  return route_body(*desc, logits, topk_idx, gates, counts, offsets, slot, row_token, row_gate, ws,
                    S(stream));
}

moe_status moe_dispatch(const moe_desc* desc, const void* x, const int32_t* slot, void* x_perm,
                        void* x_perm_sf, void* ws, size_t ws_bytes, void* stream) {
  MOE_TRY(check(desc));
  MOE_TRY(tptrs(*desc, {x, slot, x_perm}));
  if (x_perm_sf) return MOE_EINVAL;
  MOE_TRY(ws_ok(*desc, ws, ws_bytes));
  const moe_desc& d = *desc;
  if (checks_enabled())
    MOE_TRY(cu(launch_checks(slot, nullptr, nullptr, nullptr, nullptr, d.T, d.k, d.E, (int)R_of(d),
                             d.capacity, at<uint32_t>(ws, ws_layout(d).checks), status_ptr(ws),
                             S(stream))));
  return dispatch_body(d, x, slot, x_perm, status_ptr(ws), S(stream));
}

moe_status moe_grouped_gemm_fwd(const moe_desc* desc, const void* x_perm, const void* x_perm_sf,
                                const void* W13, const void* W2, const int32_t* offsets, void* H13,
                                void* a, void* y_perm, void* ws, size_t ws_bytes, void* stream) {
  MOE_TRY(check(desc));
  MOE_TRY(tptrs(*desc, {x_perm, H13, a, y_perm}));
  MOE_TRY(ptrs({W13, W2, offsets}));
  if (x_perm_sf) return MOE_EINVAL;
  MOE_TRY(ws_ok(*desc, ws, ws_bytes));
  if (R_of(*desc) == 0) return MOE_OK;
  if (checks_enabled())
    MOE_TRY(cu(launch_checks(nullptr, nullptr, offsets, nullptr, nullptr, desc->T, desc->k,
                             desc->E, (int)R_of(*desc), desc->capacity, nullptr, status_ptr(ws),
                             S(stream))));
  MxWork mx = mx_work(*desc, ws);
  mx.w_col_in_fwd = keep_codes(*desc);
  Weights wt;
  MOE_TRY(tf32_weights(*desc, W13, W2, ws, S(stream), &wt));
  MOE_TRY(gemm_fwd(gshape(*desc), x_perm, wt.W13, wt.W2, offsets, H13, a, y_perm,
                   status_ptr(ws), S(stream), &mx));
  kept_after_fwd(*desc, ws, W13, W2);
  return MOE_OK;
}

moe_status moe_combine(const moe_desc* desc, const void* y_perm, const float* gates,
                       const int32_t* slot, void* y, void* ws, size_t ws_bytes, void* stream) {
  MOE_TRY(check(desc));
  MOE_TRY(tptrs(*desc, {y_perm, gates, slot, y}));
  MOE_TRY(ws_ok(*desc, ws, ws_bytes));
  const moe_desc& d = *desc;
  return cu(launch_gather_sum(d.dtype == MOE_FP32, d.T, d.d, d.k, (int)R_of(d), y_perm, gates,
                              slot, nullptr, y, status_ptr(ws), S(stream)));
}

moe_status moe_combine_bwd(const moe_desc* desc, const void* dy, const void* y_perm,
                           const float* gates, const int32_t* topk_idx, const int32_t* slot,
                           void* dy_perm, float* d_logits, void* ws, size_t ws_bytes,
                           void* stream) {
  MOE_TRY(check(desc));
  MOE_TRY(tptrs(*desc, {dy, y_perm, gates, topk_idx, slot, dy_perm, d_logits}));
  MOE_TRY(ws_ok(*desc, ws, ws_bytes));
  const moe_desc& d = *desc;
  return combine_bwd_body(d, dy, y_perm, gates, topk_idx, slot, dy_perm, d_logits, status_ptr(ws),
                          S(stream));
}

moe_status moe_mx_scale_bytes(int64_t rows, int32_t cols, int32_t num_segments, size_t* bytes) {
  if (!bytes || rows < 0 || cols <= 0 || cols % 128 != 0 || num_segments < 1 ||
      num_segments > 1024)
    return MOE_EINVAL;
  *bytes = mx_sf_bytes(rows, cols, num_segments);
  return MOE_OK;
}

moe_status moe_mx_quantize(const void* x, int64_t rows, int32_t cols, const int32_t* seg_offsets,
                           int32_t num_segments, int32_t colwise, uint8_t* codes, uint8_t* scales,
                           void* ws, size_t ws_bytes, void* stream) {
  if (rows < 0 || rows >= (int64_t(1) << 31) || cols <= 0 || cols % 128 != 0 ||
      num_segments < 1 || num_segments > 1024 || (colwise != 0 && colwise != 1))
    return MOE_EINVAL;
  if (rows * (int64_t)cols >= (int64_t(1) << 40)) return MOE_EINVAL;
  MOE_TRY(ptrs({seg_offsets, ws}));
  if (rows > 0) MOE_TRY(ptrs({x, codes, scales}));
  if (ws_bytes < 256 + 8 * (size_t)(num_segments + 1)) return MOE_EWORKSPACE;
  int32_t* scratch = at<int32_t>(ws, 256);
  return cu(launch_mx_quantize(x, rows, cols, seg_offsets, num_segments, colwise != 0, codes,
                               scales, scratch, status_ptr(ws), S(stream)));
}

moe_status moe_grouped_gemm_bwd(const moe_desc* desc, const void* dy_perm, const void* x_perm,
                                const void* H13, const void* a, const void* W13, const void* W2,
                                const int32_t* offsets, void* dH13, void* dx_perm, void* dW13,
                                void* dW2, void* ws, size_t ws_bytes, void* stream) {
  MOE_TRY(check(desc));
  MOE_TRY(tptrs(*desc, {dy_perm, x_perm, H13, a, dH13, dx_perm}));
  MOE_TRY(ptrs({W13, W2, offsets, dW13, dW2}));
  MOE_TRY(ws_ok(*desc, ws, ws_bytes));
  return gemm_bwd_body(*desc, dy_perm, x_perm, H13, a, W13, W2, offsets, dH13, dx_perm, dW13, dW2,
                       ws, S(stream));
}

moe_status moe_dispatch_bwd(const moe_desc* desc, const void* dx_perm, const int32_t* slot,
                            void* dx, void* ws, size_t ws_bytes, void* stream) {
  MOE_TRY(check(desc));
  MOE_TRY(tptrs(*desc, {dx_perm, slot, dx}));
  MOE_TRY(ws_ok(*desc, ws, ws_bytes));
  const moe_desc& d = *desc;
  return cu(launch_gather_sum(d.dtype == MOE_FP32, d.T, d.d, d.k, (int)R_of(d), dx_perm, nullptr,
                              slot, nullptr, dx, status_ptr(ws), S(stream)));
}

moe_status moe_router_bwd(const moe_desc* desc, const void* x, const void* Wr,
                          const float* d_logits, void* dx, void* dWr, void* ws, size_t ws_bytes,
                          void* stream) {
  MOE_TRY(check(desc));
  MOE_TRY(tptrs(*desc, {x, d_logits, dx}));
  MOE_TRY(ptrs({Wr, dWr}));
  MOE_TRY(ws_ok(*desc, ws, ws_bytes));
  const moe_desc& d = *desc;
  if (d.dtype == MOE_FP32)
    return router_bwd_body(d, x, Wr, d_logits, nullptr, dx, dWr, ws, S(stream));
  // bf16: accumulate the router term in fp32, then add it to dx with one rounding
  const WsLayout w = ws_layout(d);
  if (!(d.flags & MOE_FLAG_ROUTER)) return MOE_EINVAL;
  float* extra = at<float>(ws, w.dx_router);
  MOE_TRY(router_bwd_body(d, x, Wr, d_logits, extra, nullptr, dWr, ws, S(stream)));
  return cu(launch_add_f32(false, (int64_t)d.T * d.d, dx, extra, S(stream)));
}

struct Acts {
  void *x_perm, *H13, *a, *y_perm;
  void *H13s, *as;   // shared expert
};
Acts acts(const moe_desc& d, const void* saved, const moe_saved_layout& L, void* ws) {
  Acts r;
  if (d.flags & MOE_FLAG_RECOMPUTE) {
    const WsLayout w = ws_layout(d);
    r.x_perm = at<char>(ws, w.rc_x_perm);
    r.H13 = at<char>(ws, w.rc_H13);
    r.a = at<char>(ws, w.rc_a);
    r.y_perm = at<char>(ws, w.rc_y_perm);
    r.H13s = at<char>(ws, w.rc_sh_H13);
    r.as = at<char>(ws, w.rc_sh_a);
  } else {
    void* sv = const_cast<void*>(saved);
    r.x_perm = at<char>(sv, L.x_perm);
    r.H13 = at<char>(sv, L.H13);
    r.a = at<char>(sv, L.a);
    r.y_perm = at<char>(sv, L.y_perm);
    r.H13s = at<char>(sv, L.H13_shared);
    r.as = at<char>(sv, L.a_shared);
  }
  return r;
}
// The shared expert's slice (index E) of W13 / W2 or of their gradients.
inline const void* w13_slice(const moe_desc& d, const void* W13, size_t es) {
  return static_cast<const char*>(W13) + (size_t)d.E * 2 * d.d_ff * d.d * es;
}
inline const void* w2_slice(const moe_desc& d, const void* W2, size_t es) {
  return static_cast<const char*>(W2) + (size_t)d.E * d.d * d.d_ff * es;
}

moe_status moe_load_stats(const int32_t* counts, int32_t E, moe_load_stats_t* out,
                          int32_t* status, void* stream) {
  if (E < 1 || E > 1024) return MOE_EINVAL;
  MOE_TRY(ptrs({counts, out}));
  return cu(launch_load_stats(counts, E, out, status, S(stream)));
}

moe_status moe_layer_fwd(const moe_desc* desc, const void* x, const float* logits, const void* Wr,
                         const void* W13, const void* W2, void* y, void* saved, size_t saved_bytes,
                         void* ws, size_t ws_bytes, void* stream) {
  MOE_TRY(check(desc));
  const moe_desc& d = *desc;
  const bool router = d.flags & MOE_FLAG_ROUTER;
  MOE_TRY(tptrs(d, {x, y}));
  MOE_TRY(ptrs({W13, W2, saved}));
  if (router) MOE_TRY(ptrs({Wr}));
  else MOE_TRY(tptrs(d, {logits}));
  MOE_TRY(ws_ok(d, ws, ws_bytes));
  const moe_saved_layout L = saved_layout(d);
  if (saved_bytes < L.total) return MOE_EWORKSPACE;
  cudaStream_t s = S(stream);
  int* st = status_ptr(ws);

  const float* lg = logits;
  if (router) {
    float* out = at<float>(saved, L.logits);
    MOE_TRY(router_fwd_body(d, x, Wr, out, st, s));
    lg = out;
  }
  int32_t* idx = at<int32_t>(saved, L.topk_idx);
  float* gates = at<float>(saved, L.gates);
  int32_t* slot = at<int32_t>(saved, L.slot);
  int32_t* offsets = at<int32_t>(saved, L.offsets);
  MOE_TRY(route_body(d, lg, idx, gates, at<int32_t>(saved, L.counts), offsets, slot,
                     at<int32_t>(saved, L.row_token), at<float>(saved, L.row_gate), ws, s));
  if (d.T == 0) return MOE_OK;
  const bool f32 = d.dtype == MOE_FP32;
  // the activations the backward reads: in `saved`, or workspace scratch when the
  // backward recomputes them
  const Acts A = acts(d, saved, L, ws);
  MOE_TRY(dispatch_body(d, x, slot, A.x_perm, st, s));
  MxWork mx = mx_work(d, ws);
  mx.w_col_in_fwd = keep_codes(d);
  Weights wt;
  MOE_TRY(tf32_weights(d, W13, W2, ws, s, &wt));
  MOE_TRY(gemm_fwd(gshape(d), A.x_perm, wt.W13, wt.W2, offsets, A.H13, A.a, A.y_perm, st, s, &mx));
  kept_after_fwd(d, ws, W13, W2);
  float* ys = nullptr;
  if (d.flags & MOE_FLAG_SHARED_EXPERT) {
    // the shared expert over every token, its output in fp32 for the combine to add
    const size_t es = act_bytes(d);
    ys = at<float>(ws, ws_layout(d).sh_f32);
    moe_status r;
    const void* xs = tf32_tokens(d, x, ws_layout(d).x_t, ws, s, &r);
    MOE_TRY(r);
    MOE_TRY(shared_fwd(gshape(d, d.T), xs, w13_slice(d, wt.W13, es), w2_slice(d, wt.W2, es), A.H13s,
                       A.as, ys, st, s));
  }
  return cu(launch_gather_sum(f32, d.T, d.d, d.k, (int)R_of(d), A.y_perm, gates, slot, ys, y, st,
                              s));
}

moe_status moe_layer_bwd(const moe_desc* desc, const void* dy, const void* x, const void* saved,
                         size_t saved_bytes, const void* W13, const void* W2, const void* Wr,
                         void* dx, float* d_logits, void* dW13, void* dW2, void* dWr, void* ws,
                         size_t ws_bytes, void* stream) {
  MOE_TRY(check(desc));
  const moe_desc& d = *desc;
  const bool router = d.flags & MOE_FLAG_ROUTER;
  const bool recompute = d.flags & MOE_FLAG_RECOMPUTE;
  const bool shared = d.flags & MOE_FLAG_SHARED_EXPERT;
  const size_t es = act_bytes(d);
  MOE_TRY(tptrs(d, {dy, dx, d_logits}));
  MOE_TRY(ptrs({saved, W13, W2, dW13, dW2}));
  if (router || recompute || shared) MOE_TRY(tptrs(d, {x}));
  if (router) MOE_TRY(ptrs({Wr, dWr}));
  MOE_TRY(ws_ok(d, ws, ws_bytes));
  const moe_saved_layout L = saved_layout(d);
  if (saved_bytes < L.total) return MOE_EWORKSPACE;
  const WsLayout w = ws_layout(d);
  cudaStream_t s = S(stream);
  int* st = status_ptr(ws);
  const bool f32 = d.dtype == MOE_FP32;

  const int32_t* idx = at<int32_t>(saved, L.topk_idx);
  const float* gates = at<float>(saved, L.gates);
  const int32_t* slot = at<int32_t>(saved, L.slot);
  const int32_t* offsets = at<int32_t>(saved, L.offsets);
  void* dy_perm = at<char>(ws, w.dy_perm);
  void* dH13 = at<char>(ws, w.dH13);
  void* dx_perm = at<char>(ws, w.dx_perm);
  const Acts A = acts(d, saved, L, ws);
  // (the backward GEMMs round the weights themselves; the recomputed forward and the
  // shared expert read this copy)
  Weights wt{W13, W2};
  if (recompute || shared) MOE_TRY(tf32_weights(d, W13, W2, ws, s, &wt));
  const void* xs = x;                     // the shared expert's x and dy (fp32: TF32-rounded)
  const void* dys = dy;
  if (shared) {
    moe_status r;
    xs = tf32_tokens(d, x, w.x_t, ws, s, &r);
    MOE_TRY(r);
    dys = tf32_tokens(d, dy, w.dy_t, ws, s, &r);
    MOE_TRY(r);
  }
  if (recompute && d.T > 0) {
    // the forward's activations again, from x and the saved routing (same kernels,
    // same inputs: bit-identical to the ones the forward used)
    MOE_TRY(dispatch_body(d, x, slot, A.x_perm, st, s));
    MxWork mx = mx_work(d, ws);
    mx.w_col_in_fwd = keep_codes(d);
    MOE_TRY(gemm_fwd(gshape(d), A.x_perm, wt.W13, wt.W2, offsets, A.H13, A.a, A.y_perm, st, s, &mx));
    kept_after_fwd(d, ws, W13, W2);
    if (shared)
      MOE_TRY(shared_fwd(gshape(d, d.T), xs, w13_slice(d, wt.W13, es), w2_slice(d, wt.W2, es),
                         A.H13s, A.as, at<float>(ws, w.sh_f32), st, s));
  }

  MOE_TRY(combine_bwd_body(d, dy, A.y_perm, gates, idx, slot, dy_perm, d_logits, st, s));
  MOE_TRY(gemm_bwd_body(d, dy_perm, A.x_perm, A.H13, A.a, W13, W2, offsets, dH13, dx_perm, dW13,
                        dW2, ws, s));
  float* dxs = nullptr;
  if (shared && d.T > 0) {
    // the shared expert's backward: dy is its (unpermuted, ungated) output gradient
    const size_t dw_es = (d.flags & MOE_FLAG_DW_FP32) ? 4 : es;
    dxs = at<float>(ws, w.sh_f32);
    MOE_TRY(shared_bwd(gshape(d, d.T), dys, xs, A.H13s, A.as, w13_slice(d, wt.W13, es),
                       w2_slice(d, wt.W2, es), at<char>(ws, w.sh_dH13), dxs,
                       const_cast<void*>(w13_slice(d, dW13, dw_es)),
                       const_cast<void*>(w2_slice(d, dW2, dw_es)), d.flags & MOE_FLAG_DW_FP32,
                       d.flags & MOE_FLAG_ACCUM_DW, at<char>(ws, w.maps), st, s));
  } else if (shared && !(d.flags & MOE_FLAG_ACCUM_DW)) {
    // no tokens: the shared expert's weight gradients are zero
    const size_t dw_es = (d.flags & MOE_FLAG_DW_FP32) ? 4 : es;
    MOE_TRY(cu(cudaMemsetAsync(const_cast<void*>(w13_slice(d, dW13, dw_es)), 0,
                               (size_t)2 * d.d_ff * d.d * dw_es, s)));
    MOE_TRY(cu(cudaMemsetAsync(const_cast<void*>(w2_slice(d, dW2, dw_es)), 0,
                               (size_t)d.d * d.d_ff * dw_es, s)));
  }
  float* extra = nullptr;
  if (router) {
    extra = at<float>(ws, w.dx_router);
    MOE_TRY(router_bwd_body(d, x, Wr, d_logits, extra, nullptr, dWr, ws, s));
  }
  return cu(launch_gather_sum(f32, d.T, d.d, d.k, (int)R_of(d), dx_perm, nullptr, slot, extra, dx,
                              st, s, dxs));
}

}  // extern "C"
