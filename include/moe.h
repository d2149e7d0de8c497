/*
 * moe.h -- C ABI of the B200 (sm_100a) routed mixture-of-experts layer.
 *
 * The layer is the single-GPU MoE hot path of the Olmo-core 3 training stack as the
 * write-ups describe it:
 *   - routing metadata (expert indices, gates, per-expert counts and offsets) is
 *     produced and kept on the device, with no host round trip
 *     (deniz.in, "Ai2, Olmo-core 3'ü Apache 2.0 ile yayınladı", section
 *      "Yeni stack nasıl çalışıyor"; unite.ai, "पैरालेलिज़्म, प्रिसीजन, और मेमोरी तकनीकें");
 *   - each selected token row is written straight into its expert's contiguous input
 *     buffer (same sections; donmalab.com, "擴展與最佳化手段");
 *   - a device-scheduled grouped GEMM runs the imbalanced per-expert shapes that routing
 *     produces, instead of padding every expert to a common capacity
 *     (deniz.in, "Yeni stack nasıl çalışıyor");
 *   - top-4 routing over 8..128 experts (deniz.in, "Ai2'nin raporladığı sayılar");
 *   - MXFP8 for selected operations (bigchange.ai pt-BR, opening section).
 * The pages give no formulas.  The definitions used (softmax over the experts, top k
 * kept and renormalised, ties to the lower expert index, SwiGLU expert FFN with the
 * gate applied at the combine) are stated with each call below.
 *
 * Conventions for every call
 *   - Pointers named "device" are device memory owned by the caller.  The library
 *     never allocates, frees or synchronises; every call is asynchronous on `stream`
 *     (a cudaStream_t passed as void*; NULL is the legacy default stream).
 *   - Matrices are row-major with the last index contiguous.  Tokens are rows.
 *   - All device pointers must be 16-byte aligned (MOE_EALIGN otherwise).
 *   - Element type of activations and weights ("act"): float for MOE_FP32, bfloat16
 *     for MOE_BF16 and MOE_MXFP8 (MXFP8 quantises inside the grouped GEMM calls).
 *     Logits, gates and d_logits are always float; indices are int32.
 *   - Shapes: T >= 0 tokens, d = d_model (multiple of 128), d_ff (multiple of 64),
 *     1 <= E <= 1024 experts, 1 <= k <= min(E, 32), T*k < 2^31.  R = T*k routed rows
 *     (E*capacity in the capacity-padded layout, see moe_desc.capacity).
 *   - Argument checks run on the host before any launch and return MOE_EINVAL,
 *     MOE_EALIGN, MOE_EWORKSPACE or MOE_EUNSUPPORTED with nothing launched.  A failed
 *     launch returns MOE_ECUDA.  Data-dependent faults found on the device (an index
 *     or offset out of range, a device wait that timed out) set bits of the status
 *     word in the workspace; they are read only by moe_read_device_status, an
 *     explicit synchronisation point of the caller's choosing.
 *   - `ws` is a device workspace of at least moe_workspace_size() bytes, prepared
 *     once with moe_workspace_init.  Calls that overlap on the GPU must not share one.
 */
#ifndef MOE_B200_H
#define MOE_B200_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum moe_status {
  MOE_OK = 0,
  MOE_EINVAL = -1,        /* bad descriptor, size or null pointer */
  MOE_EALIGN = -2,        /* a pointer is not 16-byte aligned */
  MOE_EWORKSPACE = -3,    /* workspace or saved buffer too small */
  MOE_EUNSUPPORTED = -4,  /* valid but not supported by this build or device */
  MOE_ECUDA = -5,         /* a CUDA call or kernel launch failed */
  MOE_EDEVICE = -6        /* moe_read_device_status found a device-side error */
} moe_status;

typedef enum moe_dtype {
  MOE_FP32 = 0,   /* fp32 storage, TF32 tensor-core GEMMs with fp32 accumulation.  The
                     GEMM operands are rounded to the nearest TF32 value (ties away from
                     zero) where they are produced: x_perm (moe_dispatch), a (FC1's
                     epilogue), dy_perm (moe_combine_bwd) and dH13 (FC2 dgrad's epilogue)
                     are stored rounded, and the GEMM calls read workspace copies of
                     W13 / W2 rounded the same way -- instead of the tensor core dropping
                     the low 13 mantissa bits (a bias towards zero) */
  MOE_BF16 = 1,   /* bf16 storage, bf16 tensor-core GEMMs with fp32 accumulation */
  MOE_MXFP8 = 2   /* bf16 storage; the grouped GEMMs quantise their operands to E4M3 with
                     an E8M0 scale per 32 along K (moe_mx_quantize) and run block-scaled
                     tensor-core MMAs with fp32 accumulation; d_ff a multiple of 128 */
} moe_dtype;

/* moe_desc.flags */
#define MOE_FLAG_ROUTER   1  /* logits = x . Wr computed on the device (else injected) */
#define MOE_FLAG_DW_FP32  2  /* dW13 / dW2 are float (else act type) */
#define MOE_FLAG_ACCUM_DW 4  /* add into existing float dW (requires MOE_FLAG_DW_FP32) */
/* Activation recompute (deniz.in, "Açık ödünleşimler": recompute drops most activation
 * memory for part of the throughput).  moe_layer_fwd keeps only the routing metadata
 * in `saved` (x_perm, H13, a, y_perm become workspace scratch), and moe_layer_bwd
 * recomputes dispatch, FC1 + SwiGLU and FC2 from x (then required) before the backward.
 * The results are bit-identical to the run without the flag. */
#define MOE_FLAG_RECOMPUTE 8
/* One shared expert (bigchange.ai pt-BR, last section: the production rows use top-4
 * routing and one shared expert): a SwiGLU FFN of the routed experts' shape applied to
 * every token with weight 1 and added to y.  W13, W2 (and dW13, dW2) then hold E+1
 * experts, the last being the shared one; the router still chooses among the first E.
 * It runs as the grouped GEMM with one segment of all T tokens; x is required in
 * moe_layer_bwd.  Not with MOE_MXFP8 (MOE_EUNSUPPORTED). */
#define MOE_FLAG_SHARED_EXPERT 16
/* MOE_MXFP8 only: keep the weights' column-wise codes from the forward for the backward.
 * The MXFP8 GEMMs read W13 and W2 quantised along d (forward) and along their rows (the
 * dgrads); without the flag each direction is a pass over the bf16 weights of its own.
 * With it, a forward call (moe_layer_fwd, moe_grouped_gemm_fwd, the recompute inside
 * moe_layer_bwd) quantises each weight both ways in one pass and records, for its
 * workspace, the W13 / W2 pointers and the shape; a backward call on the same workspace
 * with the same pointers and shape uses those codes instead of quantising the weights
 * again (any other backward quantises them as usual).  The weights must not change
 * between the two calls, as in a training step, where only the optimizer step that
 * follows the backward changes them; the calls must be ordered on the device, like the
 * forward's other outputs that the backward reads.  Results are bit-identical to the
 * run without the flag.  moe_workspace_init and a forward without the flag forget the
 * record.  MOE_EINVAL with another dtype. */
#define MOE_FLAG_MX_KEEP_WEIGHT_CODES 32
/* Test hook, off by default; the paper has no counterpart.  Every expert grouped-GEMM
 * launch (routed and shared experts) made under a descriptor with this flag issues no
 * operand loads and gives each of its
 * device waits 10 ms instead of 2 s, so the waits run out: the call sets
 * MOE_DEV_TIMEOUT in the workspace status word, writes none of its GEMM outputs, frees
 * the tensor memory it took and returns.  It exists so the bounded-wait and teardown
 * path can be exercised without faulting a GPU; after it, clear the status word with
 * moe_workspace_init before the next call. */
#define MOE_FLAG_TEST_WAIT_TIMEOUT (1 << 30)

/* device status bits */
#define MOE_DEV_BAD_INDEX   1  /* an expert index or slot was out of range; the row was skipped */
#define MOE_DEV_BAD_OFFSETS 2  /* offsets not an exclusive scan ending at R; GEMM skipped */
#define MOE_DEV_TIMEOUT     4  /* a bounded device wait gave up; results are invalid */
/* With the environment variable MOE_CHECKS set (to anything but "" or "0", read at each
 * call): moe_route and moe_layer_fwd verify the routing they produce, and moe_dispatch
 * the slots it is given, as a whole -- slot maps the T*k (token, expert) pairs to
 * distinct rows in [0,R), inside each pair's expert range, with row_token[slot[t,j]]
 * == t; offsets are a monotone scan of the counts ending at R (or the multiples of the
 * capacity); moe_grouped_gemm_fwd checks the offsets -- and set this bit on a failure.
 * The checks add device launches and a bitmap of R bits in the workspace; off by
 * default. */
#define MOE_DEV_CHECK_FAILED 8

typedef struct moe_desc {
  int32_t T, d, d_ff, E, k;
  int32_t dtype;   /* moe_dtype */
  int32_t flags;   /* MOE_FLAG_* */
  /* 0: the ragged layout (expert e owns rows [offsets[e], offsets[e+1]), R = T*k rows).
   * C > 0: the capacity-padded layout the write-ups compare the device-scheduled grouped
   * GEMM against (deniz.in, "Yeni stack nasıl çalışıyor": padding every expert group to a
   * common capacity): expert e owns rows [e*C, (e+1)*C), R = E*C; moe_route writes
   * offsets[e] = e*C (counts stay the true counts), slot = e*C + the token's rank in e,
   * and marks rows no token fills with row_token = -1, row_gate = 0; dispatch and
   * combine-bwd zero those rows.  A token whose rank reaches C gets slot -1 and sets
   * MOE_DEV_BAD_INDEX (choose C >= the largest count; results are then bit-identical to
   * the ragged layout's).  Every R-sized buffer holds E*C rows. */
  int32_t capacity;
} moe_desc;

/* Byte offsets (from the start of the caller's `saved` buffer) of the tensors that
 * moe_layer_fwd keeps for moe_layer_bwd.  Every offset is a multiple of 256. */
typedef struct moe_saved_layout {
  size_t topk_idx;   /* int32 [T,k] */
  size_t gates;      /* float [T,k] */
  size_t counts;     /* int32 [E] */
  size_t offsets;    /* int32 [E+1] */
  size_t slot;       /* int32 [T,k] */
  size_t row_token;  /* int32 [R] */
  size_t row_gate;   /* float [R] */
  size_t logits;     /* float [T,E] (router on only; else equal to `x_perm`, unused) */
  /* the four activations below are absent (zero bytes, offsets equal to `total`) with
   * MOE_FLAG_RECOMPUTE */
  size_t x_perm;     /* act [R,d] */
  size_t H13;        /* act [R,2*d_ff] */
  size_t a;          /* act [R,d_ff] */
  size_t y_perm;     /* act [R,d] */
  /* shared expert (MOE_FLAG_SHARED_EXPERT without MOE_FLAG_RECOMPUTE; else absent) */
  size_t H13_shared; /* act [T,2*d_ff] */
  size_t a_shared;   /* act [T,d_ff] */
  size_t total;      /* bytes needed */
} moe_saved_layout;

/* Human-readable name of a status code (static string). */
const char* moe_status_string(int32_t status);

/* Checks a descriptor; MOE_OK if every call below accepts it. */
moe_status moe_check_desc(const moe_desc* desc);

/* Workspace bytes that every call below needs for this descriptor (*bytes out). */
moe_status moe_workspace_size(const moe_desc* desc, size_t* bytes);

/* Layout and size of the `saved` buffer of moe_layer_fwd / moe_layer_bwd. */
moe_status moe_saved_layout_get(const moe_desc* desc, moe_saved_layout* out);

/* Zeroes the device status word of `ws` (asynchronous on `stream`).  Call once after
 * allocating a workspace, and after handling an error reported by
 * moe_read_device_status. */
moe_status moe_workspace_init(void* ws, size_t ws_bytes, void* stream);

/* Synchronises `stream`, then copies the device status word of `ws` to *bits (host).
 * Returns MOE_OK when no bit is set, MOE_EDEVICE otherwise.  This is the only call
 * that waits for the device. */
moe_status moe_read_device_status(const void* ws, void* stream, int32_t* bits);

/* S1, router projection: logits[T,E] (float, device) = x[T,d] (act) . Wr[d,E] (act),
 * fp32 accumulation.  The pages measure their headline rows with random routing
 * (bigchange.ai pt-BR, "Três números, três denominadores"); this call is the learned
 * router's projection. */
moe_status moe_router_logits(const moe_desc* desc, const void* x, const void* Wr,
                             float* logits, void* stream);

/* S2-S4, GPU-resident routing (deniz.in, "Yeni stack nasıl çalışıyor").
 * In:  logits [T,E] float.
 * Out: topk_idx [T,k] int32: per token the k experts of largest logit in descending
 *      logit order, equal logits broken towards the lower expert index;
 *      gates [T,k] float: softmax over the k kept logits (= full softmax
 *      renormalised over the kept experts);
 *      counts [E] int32: rows per expert;  offsets [E+1] int32: exclusive scan of counts;
 *      slot [T,k] int32: row of pair (t,j) in the expert-sorted order, rows of one
 *      expert in token order: slot[t,j] = offsets[e] + #{t' < t routed to e};
 *      row_token [R] int32 and row_gate [R] float: token and gate of each sorted row.
 * Every output is fully written; counts/offsets never leave the device.  A NaN logit
 * ranks as -inf (so a token always gets k distinct experts in [0,E)); a token whose
 * kept logits are all -inf gets NaN gates. */
moe_status moe_route(const moe_desc* desc, const float* logits, int32_t* topk_idx,
                     float* gates, int32_t* counts, int32_t* offsets, int32_t* slot,
                     int32_t* row_token, float* row_gate, void* ws, size_t ws_bytes,
                     void* stream);

/* Size of the device array that moe_route_noalloc uses for its scratch (4 MiB). */
#define MOE_ROUTE_NOALLOC_SCRATCH_BYTES (4 * 1024 * 1024)

/* moe_route without a workspace.  The paper has no counterpart: this entry point is a
 * library convenience for callers that cannot give the library device memory of its
 * own -- for example a host framework or plugin that plans every device buffer ahead
 * and passes only its input and output tensors, or a latency-critical caller that
 * must not call cudaMalloc because it synchronises the device.
 * Same arguments, outputs and results as moe_route, minus ws/ws_bytes, for the
 * ragged layout only: a descriptor with capacity > 0 returns MOE_EUNSUPPORTED before
 * any launch (the padded layout reports a capacity below an expert's count through
 * the workspace status word, which this call does not have; with capacity 0 routing
 * writes only indices it produced itself, so no device-side error can arise).  Its scratch
 * (expert histograms per 64 tokens and bases per 256 tokens, (ceil(T/64) + ceil(T/256))
 * * E int32) lives in one static device array of MOE_ROUTE_NOALLOC_SCRATCH_BYTES that
 * every GPU which loads this library holds until the process exits; a descriptor that
 * needs more returns MOE_EWORKSPACE before any launch (with E = 128 that allows T up to
 * about 419k tokens, with E = 1024 about 52k).  The call allocates nothing and frees
 * nothing.
 * The first call on a device looks up the array's device address (once per device,
 * with that device current); make that first call before any stream capture.
 * All calls share the one array and it keeps the last call's contents (every call
 * overwrites what it reads, so nothing needs clearing): calls that overlap on the
 * GPU -- on different streams, or from different host threads -- race and must be
 * serialised by the caller. */
moe_status moe_route_noalloc(const moe_desc* desc, const float* logits, int32_t* topk_idx,
                             float* gates, int32_t* counts, int32_t* offsets, int32_t* slot,
                             int32_t* row_token, float* row_gate, void* stream);

/* S5, row-wise dispatch: x_perm[slot[t,j]] = x[t] for every (t,j)
 * (unite.ai, "पैरालेलिज़्म, प्रिसीजन, और मेमोरी तकनीकें").  x [T,d] act, x_perm [R,d] act
 * (bf16 also for MOE_MXFP8: the grouped GEMM quantises it).  x_perm_sf is reserved and
 * must be NULL.  A slot outside [0,R) sets MOE_DEV_BAD_INDEX and that copy is skipped. */
moe_status moe_dispatch(const moe_desc* desc, const void* x, const int32_t* slot,
                        void* x_perm, void* x_perm_sf, void* ws, size_t ws_bytes,
                        void* stream);

/* S6-S7, device-scheduled grouped GEMM forward of the SwiGLU experts
 * (deniz.in, "Yeni stack nasıl çalışıyor").  For each expert e, rows
 * [offsets[e], offsets[e+1]) of x_perm form X_e:
 *   H13_e = X_e . W13_e^T          (W13 [E, 2*d_ff, d]: rows 0..d_ff-1 gate W1, then up W3)
 *   a_e   = silu(H1_e) * H3_e      (computed in fp32 from the accumulator)
 *   Y_e   = a_e . W2_e^T           (W2 [E, d, d_ff])
 * Out: H13 [R,2*d_ff], a [R,d_ff], y_perm [R,d], all act.  The tile schedule is read
 * from `offsets` on the device.  Offsets that are not an exclusive scan ending at R
 * set MOE_DEV_BAD_OFFSETS and nothing is written. */
moe_status moe_grouped_gemm_fwd(const moe_desc* desc, const void* x_perm,
                                const void* x_perm_sf, const void* W13, const void* W2,
                                const int32_t* offsets, void* H13, void* a, void* y_perm,
                                void* ws, size_t ws_bytes, void* stream);

/* S8, weighted combine (deniz.in, "Hedeflediği kapasite sorunu": each token passes
 * through only a few of the stored experts; their outputs, weighted by the token's
 * gates, are the layer's output):
 *   y[t] = sum_j gates[t,j] * y_perm[slot[t,j]], summed in fp32.
 * y_perm [R,d] act -> y [T,d] act (device).  A gather: no atomics, deterministic.  A
 * slot outside [0,R) sets MOE_DEV_BAD_INDEX and that term is skipped. */
moe_status moe_combine(const moe_desc* desc, const void* y_perm, const float* gates,
                       const int32_t* slot, void* y, void* ws, size_t ws_bytes,
                       void* stream);

/* S9, backward (chain rule) of moe_combine and of moe_route's gate softmax; device
 * buffers:
 *   dy_perm[slot[t,j]] = gates[t,j] * dy[t]                        (act [R,d])
 *   dg[t,j] = <dy[t], y_perm[slot[t,j]]>                            (fp32)
 *   d_logits[t, topk_idx[t,j]] = g_tj * (dg_tj - sum_i g_ti dg_ti), 0 elsewhere  ([T,E] float) */
moe_status moe_combine_bwd(const moe_desc* desc, const void* dy, const void* y_perm,
                           const float* gates, const int32_t* topk_idx, const int32_t* slot,
                           void* dy_perm, float* d_logits, void* ws, size_t ws_bytes,
                           void* stream);

/* S15, MXFP8 quantisation (bigchange.ai pt-BR, opening section: MXFP8 for selected
 * operations; OCP MX v1.0 rule, since the pages give none).  x [rows, cols] bf16 (device)
 * is split into row segments [seg_offsets[e], seg_offsets[e+1]) (e < num_segments; one per
 * expert; seg_offsets[num_segments] = rows).  Per block of 32 elements -- along cols
 * (colwise = 0) or along the rows of one segment starting at its first row (colwise = 1;
 * a segment's last block may be partial) -- the shared exponent is
 * s = floor(log2(amax)) - 8 clamped to [-127, 127] (-127 for an all-zero block) and each
 * element becomes E4M3(x / 2^s), round to nearest even, saturated to +-448.
 * Out: codes [rows, cols] uint8 (device, x's layout); scales: E8M0 bytes s + 127 in
 * 512-byte chunks (moe_mx_scale_bytes), chunk (tile_pref[e] + p/128) * (cols/128) +
 * col/128 with tile_pref the prefix over segments of ceil(rows_e/128) and p the row
 * inside its segment; inside a chunk the byte of (index i, block b) is
 * 16*(i%32) + 4*((i%128)/32) + b, with i = p and b = (col%128)/32 rowwise, i = col and
 * b = (p%128)/32 colwise.  Colwise, the slots of a segment's last chunk past its last
 * block are written as 0 (scale 2^-127), so a reader of whole chunks sees finite scales;
 * other slots that no block reaches (rowwise rows past a segment's end) are left
 * untouched.  cols must be a multiple of 128.  ws: at least 256 + 8*(num_segments+1)
 * bytes of device scratch; its first 4 bytes are a device status word, read with
 * moe_read_device_status (the quantiser itself has no waits and sets no status). */
moe_status moe_mx_scale_bytes(int64_t rows, int32_t cols, int32_t num_segments, size_t* bytes);
moe_status moe_mx_quantize(const void* x, int64_t rows, int32_t cols, const int32_t* seg_offsets,
                           int32_t num_segments, int32_t colwise, uint8_t* codes, uint8_t* scales,
                           void* ws, size_t ws_bytes, void* stream);

/* S10-S13, backward (chain rule) of moe_grouped_gemm_fwd, scheduled on the device from
 * `offsets` like it (deniz.in, "Yeni stack nasıl çalışıyor"); per expert e:
 *   dA_e   = dY_e . W2_e                                   (dY_e = rows of dy_perm)
 *   dH1_e  = dA_e * H3_e * s * (1 + H1_e * (1 - s)),  s = sigmoid(H1_e)
 *   dH3_e  = dA_e * silu(H1_e)                            -> dH13 [R,2*d_ff] act
 *   dW2_e  = dY_e^T . a_e                                  -> dW2  [E,d,d_ff]
 *   dX_e   = dH13_e . W13_e                                -> dx_perm [R,d] act
 *   dW13_e = dH13_e^T . X_e                                -> dW13 [E,2*d_ff,d]
 * dW is act type, or float with MOE_FLAG_DW_FP32 (added into with MOE_FLAG_ACCUM_DW).
 * An expert with no rows gets dW_e = 0 exactly (unchanged with MOE_FLAG_ACCUM_DW). */
moe_status moe_grouped_gemm_bwd(const moe_desc* desc, const void* dy_perm, const void* x_perm,
                                const void* H13, const void* a, const void* W13,
                                const void* W2, const int32_t* offsets, void* dH13,
                                void* dx_perm, void* dW13, void* dW2, void* ws,
                                size_t ws_bytes, void* stream);

/* S14, backward of moe_dispatch (unpermute-reduce; the adjoint of the row copy):
 * dx[t] = sum_j dx_perm[slot[t,j]], fp32 sum, act out (device).  A gather: no atomics,
 * deterministic. */
moe_status moe_dispatch_bwd(const moe_desc* desc, const void* dx_perm, const int32_t* slot,
                            void* dx, void* ws, size_t ws_bytes, void* stream);

/* Router backward (MOE_FLAG_ROUTER), the chain rule of moe_router_logits:
 * dx[T,d] += d_logits . Wr^T and dWr[d,E] (act) = x^T . d_logits, fp32 accumulation
 * (device buffers). */
moe_status moe_router_bwd(const moe_desc* desc, const void* x, const void* Wr,
                          const float* d_logits, void* dx, void* dWr, void* ws,
                          size_t ws_bytes, void* stream);

/* Expert load statistics of one routing (deniz.in, "Ekibin reddettiği yaklaşımlar": the
 * experts' imbalance can grow while a balancing loss improves, "Token Gerrymandering";
 * this is its measurable side -- the pages give no loss formula and none is computed).
 * From counts [E] (device, e.g. the `counts` of moe_route or of `saved`):
 *   total = sum_e counts[e], mean = total / E, max_count, min_count,
 *   num_empty = #{e : counts[e] == 0}, max_over_mean = max_count / mean (0 if total = 0),
 *   cv = sqrt(sum_e (counts[e] - mean)^2 / E) / mean (0 if total = 0),
 * written to *out, a device pointer (16-byte aligned), by one small kernel on `stream`
 * -- no host synchronisation; copy it back when needed.  Counts must be >= 0 (a
 * negative count sets MOE_DEV_BAD_OFFSETS in the status word `status`, if non-null, and
 * is read as 0).  E in [1, 1024]. */
typedef struct moe_load_stats_t {
  int64_t total;
  int32_t max_count, min_count, num_empty, num_experts;
  double mean, max_over_mean, cv;
} moe_load_stats_t;
moe_status moe_load_stats(const int32_t* counts, int32_t E, moe_load_stats_t* out,
                          int32_t* status, void* stream);

/* Whole layer forward, the path the write-ups describe end to end (deniz.in, "Yeni
 * stack nasıl çalışıyor"): [router] -> route -> dispatch -> grouped GEMM fwd -> combine,
 * in one call with no host synchronisation.
 * logits: injected routing logits [T,E] float, or NULL with MOE_FLAG_ROUTER and Wr.
 * y [T,d] act.  `saved` (moe_saved_layout.total bytes) receives the tensors listed in
 * moe_saved_layout, which moe_layer_bwd reads. */
moe_status moe_layer_fwd(const moe_desc* desc, const void* x, const float* logits,
                         const void* Wr, const void* W13, const void* W2, void* y,
                         void* saved, size_t saved_bytes, void* ws, size_t ws_bytes,
                         void* stream);

/* Whole layer backward (the chain rule of moe_layer_fwd, same calls in reverse) for
 * upstream gradient dy [T,d] act.  Out: dx [T,d] act,
 * d_logits [T,E] float, dW13, dW2 (see moe_grouped_gemm_bwd), and dWr [d,E] act when
 * MOE_FLAG_ROUTER.  x (the forward's input) is required with MOE_FLAG_ROUTER,
 * MOE_FLAG_RECOMPUTE or MOE_FLAG_SHARED_EXPERT and may be NULL otherwise. */
moe_status moe_layer_bwd(const moe_desc* desc, const void* dy, const void* x,
                         const void* saved, size_t saved_bytes, const void* W13,
                         const void* W2, const void* Wr, void* dx, float* d_logits,
                         void* dW13, void* dW2, void* dWr, void* ws, size_t ws_bytes,
                         void* stream);

#ifdef __cplusplus
}
#endif

#endif /* MOE_B200_H */
