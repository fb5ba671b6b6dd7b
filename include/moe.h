/*
 * moe.h -- C ABI of the B200 (sm_100a) MoE layer with zero-computation experts.
 *
 * The layer is the one of "LongCat-Flash Technical Report", §2.1
 * (zero-computation experts), Eq. (1):
 *
 *     MoE(x_t) = gamma * sum_{i=1}^{N+Z} g_i E_i(x_t)
 *     g_i      = R(x_t)_i  if R(x_t)_i + b_i is among the K largest of
 *                {R(x_t)_j + b_j}, else 0              (R: softmax router)
 *     E_i(x_t) = FFN_i(x_t) for i <= N;  x_t for N < i <= N+Z
 *
 * with the expert-bias budget control of §2.1.1, Eq. (2), and the optional
 * output scale gamma of §2.3.2, Eq. (8) (1 unless the caller sets it).
 * FFN_i is a SwiGLU expert: FFN(x) = W2 (SiLU(W1 x) * (W3 x)).
 *
 * The forward pass is four calls on one stream:
 *     moe_route -> moe_permute -> moe_expert_ffn -> moe_combine
 * and moe_bias_update runs beside it once per step.  Without the x_perm copy
 * (the decode-sized batches' form):
 *     moe_route_dispatch -> moe_expert_gate_up_gather -> moe_expert_down -> moe_combine
 *
 * Conventions shared by every call
 * --------------------------------
 *  - Every pointer argument except the moe_shape pointer is a DEVICE pointer
 *    owned by the caller.  The library allocates no device memory and keeps no
 *    device state between calls; scratch space is the caller's workspace.
 *  - Calls are asynchronous on `stream` (a cudaStream_t passed as void*; NULL
 *    is the legacy default stream).  No call synchronises the host except
 *    moe_get_device_status.
 *  - Row-major layouts throughout.  Weights use the out-features x in-features
 *    layout of a linear layer: w_router [E, d], w1/w3 [N, I, d], w2 [N, d, I].
 *  - dtype MOE_F32: x, weights, x_perm, y_perm, out are float32.
 *    dtype MOE_BF16: they are bfloat16; accumulation is always float32,
 *    softmax and gates are float32, intermediates h and y_perm are rounded to
 *    bf16 with round-to-nearest-even.
 *  - Host-side validation returns an error code and never aborts; the message
 *    is available from moe_last_error() on the calling thread.
 *  - Errors found on the device (an expert index out of range, inconsistent
 *    counts, a pipeline wait that ran out of iterations) set bits in the
 *    workspace status word and never trap; moe_get_device_status reads them.
 *  - Buffers whose size depends on routing (x_perm, y_perm, h) are sized for
 *    the worst case R <= T*K rows, so no call needs a device-to-host sync.
 */
#ifndef MOE_B200_H
#define MOE_B200_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum { MOE_F32 = 0, MOE_BF16 = 1 } moe_dtype;

/* Storage order of the expert weights w1, w3, w2.
 * MOE_WEIGHTS_ROW_MAJOR: [N, rows, cols] row-major (linear-layer layout).
 * MOE_WEIGHTS_TILED: the same matrices cut into 128-row x 64-column tiles,
 *   each tile stored as 16 KiB of contiguous row-major bf16, tiles ordered
 *   (expert, row block, column block); see moe_pack_weights.  Every weight
 *   tile the expert GEMMs stream is then one contiguous block of HBM.
 *   Requires bf16, d % 128 == 0 and I % 128 == 0. */
typedef enum { MOE_WEIGHTS_ROW_MAJOR = 0, MOE_WEIGHTS_TILED = 1 } moe_weight_layout;

/* T tokens, d hidden size, N FFN experts, Z zero-computation experts,
 * K experts per token (1 <= K <= N+Z <= 1024), I expert intermediate size. */
typedef struct {
  int32_t T, d, N, Z, K, I;
  int32_t dtype;         /* moe_dtype */
  int32_t weight_layout; /* moe_weight_layout of w1, w3, w2 (w_router is always row-major) */
} moe_shape;

typedef enum {
  MOE_OK = 0,
  MOE_ERR_INVALID_ARG = 1,   /* null pointer, bad shape, misaligned pointer */
  MOE_ERR_UNSUPPORTED = 2,   /* valid but not supported (e.g. bf16 d % 64 != 0) */
  MOE_ERR_WORKSPACE = 3,     /* workspace too small */
  MOE_ERR_CUDA = 4,          /* a CUDA runtime call failed */
  MOE_ERR_DEVICE_STATUS = 5  /* moe_get_device_status found device-side errors */
} moe_status;

/* Bits of the device status word. */
#define MOE_DEV_BAD_EXPERT_INDEX 0x1u  /* topk_idx entry outside [0, N+Z) (ignored) */
#define MOE_DEV_COUNT_MISMATCH 0x2u    /* counts[] disagrees with topk_idx */
#define MOE_DEV_BAD_OFFSETS 0x4u       /* offsets not monotone or beyond T*K */
#define MOE_DEV_PIPELINE_TIMEOUT 0x8u  /* a bounded wait inside a GEMM gave up */

/* Repacks n_mats bf16 matrices [rows, cols] (row-major, contiguous) into the
 * MOE_WEIGHTS_TILED order: dst tile (m, rb, cb) = rows rb*128..+127, columns
 * cb*64..+63 of matrix m, stored at tile index (m*rows/128 + rb)*cols/64 + cb.
 * w1 and w3 are packed as N matrices [I, d], w2 as N matrices [d, I].
 * rows % 128 == 0, cols % 64 == 0; src and dst must not overlap; dtype must be
 * MOE_BF16.  Done once when the weights are loaded. */
moe_status moe_pack_weights(int32_t n_mats, int32_t rows, int32_t cols, int32_t dtype,
                            const void* src, void* dst, void* stream);

/* Bytes of device workspace the calls below need for this shape.  One
 * workspace may serve every call of a layer instance, used in stream order.
 * Returns 0 for an invalid shape. */
size_t moe_workspace_bytes(const moe_shape* shape);

/* Clears the workspace status word.  Call once after allocating it. */
moe_status moe_workspace_init(void* ws, size_t ws_bytes, void* stream);

/* Router and selection: §2.1, Eq. (1).
 *   logits[t, i] = sum_j x[t, j] w_router[i, j] (+ logit_offset[t, i])   (fp32)
 *   R[t, :]      = softmax(logits[t, :]) over all E = N+Z experts          (fp32)
 *   topk_idx[t, 0..K) = the K experts with the largest R + bias, in order of
 *                       that score descending, ties to the lower index
 *   topk_gate[t, k]   = R[t, topk_idx[t, k]]   (unbiased, not renormalised)
 *   counts[i]         = number of (t, k) with topk_idx[t, k] == i   (T_i of Eq. (2))
 *   n_ffn[t]          = number of k with topk_idx[t, k] < N
 * x [T, d] (dtype), w_router [E, d] (dtype), bias [E] fp32,
 * logit_offset [T, E] fp32 or NULL (an additive input, used by tests and
 * skewed-routing workloads), topk_idx [T, K] int32, topk_gate [T, K] fp32,
 * counts [E] int32, n_ffn [T] uint8, probs_out [T, E] fp32 or NULL,
 * prob_sum [E] fp32 or NULL: prob_sum[i] = sum_t R[t, i] (the per-expert
 * probability mass of Eq. (4), summed in a fixed order).
 * bias entries must be finite. */
moe_status moe_route(const moe_shape* shape, const void* x, const void* w_router,
                     const float* bias, const float* logit_offset, int32_t* topk_idx,
                     float* topk_gate, int32_t* counts, uint8_t* n_ffn, float* probs_out,
                     float* prob_sum, void* ws, size_t ws_bytes, void* stream);

/* Dispatch to the FFN experts only (zero-computation experts get no rows).
 *   offsets[e] = sum_{e' < e} counts[e'] over FFN experts, e in [0, N];
 *                offsets[N] = R, the number of routed FFN rows.
 *   Rows of expert e are offsets[e] .. offsets[e+1]-1, in ascending token order.
 *   row_token[r] = token of row r (r < R);  slot_pos[t, k] = row of slot (t, k),
 *   or -1 when topk_idx[t, k] >= N;  x_perm[r, :] = x[row_token[r], :].
 * topk_idx [T, K] int32, counts [E] int32 (checked against topk_idx; a mismatch
 * sets MOE_DEV_COUNT_MISMATCH and topk_idx wins), offsets [N+1] int32,
 * row_token [T*K] int32, slot_pos [T, K] int32, x_perm [T*K, d] (dtype).
 * x_perm may be NULL: the layout (offsets, row_token, slot_pos) is built and
 * no row is copied; moe_expert_gate_up_gather then reads x through row_token
 * (x itself may also be NULL in that case). */
moe_status moe_permute(const moe_shape* shape, const void* x, const int32_t* topk_idx,
                       const int32_t* counts, int32_t* offsets, int32_t* row_token,
                       int32_t* slot_pos, void* x_perm, void* ws, size_t ws_bytes,
                       void* stream);

/* Router, selection and the dispatch layout in one call: §2.1, Eq. (1), with
 * the zero-computation experts given no rows.  It computes exactly what
 * moe_route followed by moe_permute with x_perm = NULL computes.  The arguments
 * are moe_route's followed by moe_permute's layout outputs (offsets [N+1],
 * row_token [T*K], slot_pos [T, K], all int32, the same definitions).  No token
 * row is copied: moe_expert_gate_up_gather reads x through row_token.
 * When the batch takes the one-launch router (decode batches: T <= 256, and
 * N <= 481 so the layout tables fit its shared memory), the CTA that completes
 * the counts also builds the layout, so the call is one kernel launch.  Other
 * shapes run moe_route's and moe_permute's kernels in sequence.
 * Errors: those of moe_route and moe_permute. */
moe_status moe_route_dispatch(const moe_shape* shape, const void* x, const void* w_router,
                              const float* bias, const float* logit_offset, int32_t* topk_idx,
                              float* topk_gate, int32_t* counts, uint8_t* n_ffn,
                              float* probs_out, float* prob_sum, int32_t* offsets,
                              int32_t* row_token, int32_t* slot_pos, void* ws, size_t ws_bytes,
                              void* stream);

/* moe_permute without a workspace argument.  The paper has no counterpart:
 * this entry point exists for callers that cannot give the library scratch
 * memory -- operator plug-ins whose interface hands over only the input and
 * output buffers of a call, and runtimes that plan all device memory at
 * start-up and refuse allocations afterwards.  It computes exactly what
 * moe_permute computes, with the same arguments minus ws/ws_bytes, and it
 * allocates nothing.
 *
 * Scratch: one 4 MiB array in device memory owned by the library, present on
 * every device that loads it until the process exits.  Limit: a status word
 * (256 bytes) and two int32 tables of ceil(T/256) x N entries, each rounded up
 * to a multiple of 256 bytes, must fit:
 *     256 + 2 * round_up(ceil(T/256) * N * 4, 256) <= 4194304,
 * for example T <= 130816 tokens at N = 1024 (and any T <= 256).  Larger
 * shapes return MOE_ERR_UNSUPPORTED with a message and launch nothing.
 * Set-up: the first call on each device looks up the array's device address
 * (cudaGetSymbolAddress) and caches it; make that first call before any
 * stream capture.
 * Sharing: every call on a device uses the same array and leaves its contents
 * behind (each call overwrites what it reads, so nothing carries over).  Calls
 * whose kernels overlap on the GPU -- on different streams, or from different
 * host threads -- race on the array and must be serialised by the caller.
 * Device-side consistency bits (bad expert index, count mismatch) go to the
 * array's own status word and are not reported; use moe_permute with a
 * workspace and moe_get_device_status to read them. */
moe_status moe_permute_noalloc(const moe_shape* shape, const void* x, const int32_t* topk_idx,
                               const int32_t* counts, int32_t* offsets, int32_t* row_token,
                               int32_t* slot_pos, void* x_perm, void* stream);

/* First half of the SwiGLU experts on the routed rows:
 *   h[r, :] = SiLU(x_perm[r, :] W1_e^T) * (x_perm[r, :] W3_e^T)   for rows r of expert e.
 * x_perm [T*K, d], w1/w3 [N, I, d], offsets [N+1] (from moe_permute),
 * h [T*K, I] (dtype).  Rows >= offsets[N] are not written. */
moe_status moe_expert_gate_up(const moe_shape* shape, const void* x_perm, const void* w1,
                              const void* w3, const int32_t* offsets, void* h, void* ws,
                              size_t ws_bytes, void* stream);

/* moe_expert_gate_up with the dispatch copy fused in: the token rows are read
 * from x through row_token (from moe_permute) instead of from x_perm,
 *   h[r, :] = SiLU(x[row_token[r], :] W1_e^T) * (x[row_token[r], :] W3_e^T).
 * x [T, d], row_token [T*K] int32 (from moe_permute or moe_route_dispatch); the
 * other arguments as moe_expert_gate_up.  With T == 0, x, row_token and h may be
 * NULL and nothing is launched.
 * A row_token entry outside [0, T) sets MOE_DEV_BAD_OFFSETS and reads row 0.
 * The token rows are copied into shared memory by the GEMM's producer
 * (16-byte asynchronous copies), so the x_perm buffer (T*K*d elements) and
 * its write and read are not needed. */
moe_status moe_expert_gate_up_gather(const moe_shape* shape, const void* x,
                                     const int32_t* row_token, const void* w1, const void* w3,
                                     const int32_t* offsets, void* h, void* ws, size_t ws_bytes,
                                     void* stream);

/* Second half: y_perm[r, :] = h[r, :] W2_e^T.  h [T*K, I], w2 [N, d, I],
 * y_perm [T*K, d] (dtype). */
moe_status moe_expert_down(const moe_shape* shape, const void* h, const void* w2,
                           const int32_t* offsets, void* y_perm, void* ws, size_t ws_bytes,
                           void* stream);

/* Both halves with h kept in the workspace:
 *   y_perm[r, :] = FFN_e(x_perm[r, :]) for each routed row r of expert e. */
moe_status moe_expert_ffn(const moe_shape* shape, const void* x_perm, const void* w1,
                          const void* w3, const void* w2, const int32_t* offsets,
                          void* y_perm, void* ws, size_t ws_bytes, void* stream);

/* ---- MXFP8 expert path ------------------------------------------------
 * FP8 blockwise-quantised experts (the LongCat series notes: FP8 with block
 * scales at inference).  Format MXFP8: E4M3 values with one power-of-two
 * scale 2^s per 32 consecutive values of a row along the GEMM reduction
 * axis; s is the smallest integer with amax <= 448 * 2^s (no saturation),
 * stored as the byte s + 127.  The expert GEMMs use the sm_100a block-scaled
 * tensor-core instructions.  Requires dtype MOE_BF16 (x, y_perm, out stay
 * bf16), d % 256 == 0 and I % 128 == 0.  The shape's weight_layout is ignored.
 */

/* Quantises n_mats bf16 matrices [rows, cols] (row-major, reduction axis =
 * cols) to MXFP8.  dst_q: rows*cols bytes per matrix, 128 x 128 tiles of 16 KiB
 * (row-major inside a tile) at tile index (m*rows/128 + rb)*cols/128 + cb.
 * dst_sf: one 512-byte atom per tile; byte 16*(r%32) + 4*(r/32) + b is the
 * scale of tile row r, 32-column block b.  w1/w3 are quantised as N matrices
 * [I, d], w2 as N matrices [d, I].  rows % 128 == 0, cols % 128 == 0. */
moe_status moe_quantize_weights_mxfp8(int32_t n_mats, int32_t rows, int32_t cols,
                                      const void* src, void* dst_q, void* dst_sf, void* stream);

/* moe_permute whose copy quantises: x_perm_q [T*K, d] E4M3 bytes and
 * x_perm_sf [T*K, d/32] scale bytes (row-major) for every routed row; the
 * layout outputs are those of moe_permute. */
moe_status moe_permute_mxfp8(const moe_shape* shape, const void* x, const int32_t* topk_idx,
                             const int32_t* counts, int32_t* offsets, int32_t* row_token,
                             int32_t* slot_pos, void* x_perm_q, void* x_perm_sf, void* ws,
                             size_t ws_bytes, void* stream);

/* h = SiLU(x_perm W1_e^T) * (x_perm W3_e^T) on MXFP8 operands (fp32
 * accumulation), written as MXFP8: h_q [T*K, I] bytes, h_sf [T*K, I/32]. */
moe_status moe_expert_gate_up_mxfp8(const moe_shape* shape, const void* x_perm_q,
                                    const void* x_perm_sf, const void* w1_q, const void* w1_sf,
                                    const void* w3_q, const void* w3_sf, const int32_t* offsets,
                                    void* h_q, void* h_sf, void* ws, size_t ws_bytes,
                                    void* stream);

/* y_perm = h W2_e^T on MXFP8 operands, written as bf16 [T*K, d]. */
moe_status moe_expert_down_mxfp8(const moe_shape* shape, const void* h_q, const void* h_sf,
                                 const void* w2_q, const void* w2_sf, const int32_t* offsets,
                                 void* y_perm, void* ws, size_t ws_bytes, void* stream);

/* Weighted sum of Eq. (1) with the zero-computation experts folded in:
 *   out[t, :] = gamma * ( sum_{k: idx < N} gate[t,k] * y_perm[slot_pos[t,k], :]
 *                         + (sum_{k: idx >= N} gate[t,k]) * x[t, :] )
 * accumulated in fp32 in this fixed order (FFN slots in k order, then the
 * identity term).  x [T, d], y_perm [T*K, d], out [T, d] (dtype). */
moe_status moe_combine(const moe_shape* shape, const void* x, const void* y_perm,
                       const int32_t* topk_idx, const float* topk_gate,
                       const int32_t* slot_pos, float gamma, void* out, void* stream);

/* Computation-budget control: §2.1.1, Eq. (2), in place on bias [N+Z] fp32:
 *   bias[i] += mu * (K_e/K * 1/N - counts[i]/(K * T_all))   for i < N,
 *   bias[i] unchanged for the Z zero-computation experts (i >= N).
 * counts [N+Z] int32 are the global-batch counts T_i, T_all the global-batch
 * token count.  The increment is formed in fp64 and the sum rounded once to
 * fp32. */
moe_status moe_bias_update(int32_t N, int32_t Z, const int32_t* counts, int64_t T_all,
                           int32_t K, float K_e, float mu, float* bias, void* stream);

/* Device-level load-balance statistics with the zero-expert group,
 * §2.1.2, Eq. (3)-(5).  The N FFN experts form D groups of G = N/D
 * consecutive experts; the Z zero-computation experts form group D.
 *   f[j] = D/(K_e T) * (selections of group j)       j < D
 *   f[D] = 1/((K - K_e) T) * (selections of zero experts)
 *   P[j] = (1/T) * sum_{i in group j} prob_sum[i]
 *   *loss = alpha * sum_{j <= D} f[j] P[j]             (loss may be NULL)
 * A token's selections of a group are counted once per selected expert of
 * that group, so f[j] = 1 at the balance point.  counts [N+Z] and prob_sum
 * [N+Z] come from moe_route over the T tokens (sum them over ranks first for a
 * global batch); f, P [D+1] fp32.  D must divide N, 0 < K_e < K, Z >= 1. */
moe_status moe_lb_stats(int32_t N, int32_t Z, int32_t D, const int32_t* counts,
                        const float* prob_sum, int64_t T, int32_t K, float K_e, float alpha,
                        float* f, float* P, float* loss, void* stream);

/* ---- Backward pass (the training half of the same layer) ---------------
 * Gradients of Eq. (1) for an upstream gradient dout = dL/d out [T, d].  The
 * top-K selection is piecewise constant in the inputs, so it is held fixed
 * and the gradient flows through the gates g = R(x)_i of the selected
 * experts, the SwiGLU experts, the identity experts and the softmax router;
 * the expert bias b (used for selection only) receives none.  With
 * a = x W1^T, u = x W3^T, h = SiLU(a) * u, y = h W2^T per routed row:
 *   dy       = gamma g dout_t                         (FFN slot of token t)
 *   dgate    = gamma <dout_t, y>  (FFN slot),  gamma <dout_t, x_t>  (zero slot)
 *   dh       = dy W2,   da = dh u SiLU'(a),   du = dh SiLU(a)
 *   SiLU'(a) = sigma(a) (1 + a (1 - sigma(a)))
 *   dx_row   = da W1 + du W3;  dW1 = da^T x, dW3 = du^T x, dW2 = dy^T h (per expert)
 *   dlogits  = R (dR - <R, dR>),  dR = dgate scattered to the selected experts
 *   dW_r     = dlogits^T x;      dx = gamma (sum of zero gates) dout + sum_k dx_row
 *                                     + dlogits W_r
 * One backward pass is, on one stream, after moe_expert_gate_up_save was used
 * for the forward gate/up half:
 *   moe_combine_backward -> moe_route_backward -> moe_expert_ffn_backward
 *   -> moe_permute_backward
 * Every reduction runs in a fixed order, so results are bit-reproducible: the
 * token gradient is gathered per token (no atomic scatter-add).  Gradients of
 * bf16 weights are bf16 (rounded once from fp32 sums), row-major in the
 * linear-layer layout whatever the shape's weight_layout. */

/* Bytes of device workspace the backward calls need for this shape (status
 * word, router-logit gradient [T, E], SwiGLU gradient [T*K, 2I]).  Clear it
 * once with moe_workspace_init.  Returns 0 for an invalid shape. */
size_t moe_backward_workspace_bytes(const moe_shape* shape);

/* moe_expert_gate_up that also keeps what the backward pass needs: besides
 * h it writes the pre-activations au[r, 0:I] = a = x_perm[r] W1_e^T and
 * au[r, I:2I] = u = x_perm[r] W3_e^T (dtype, bf16 rounded once from the fp32
 * accumulators; h is formed from the unrounded a, u as in
 * moe_expert_gate_up).  au [T*K, 2I]; other arguments as moe_expert_gate_up
 * (forward workspace). */
moe_status moe_expert_gate_up_save(const moe_shape* shape, const void* x_perm, const void* w1,
                                   const void* w3, const int32_t* offsets, void* h, void* au,
                                   void* ws, size_t ws_bytes, void* stream);

/* Backward of moe_combine (Eq. (1) weighted sum and Eq. (8) gamma):
 *   dy_perm[slot_pos[t,k], :] = gamma * gate[t,k] * dout[t, :]   (FFN slots)
 *   dgate[t, k] = gamma * <dout[t], y_perm[slot_pos[t,k]]>       (FFN slots)
 *               = gamma * <dout[t], x[t]>                        (zero slots)
 * Dot products are fp32 sums in a fixed order.  x, dout [T, d], y_perm,
 * dy_perm [T*K, d] (dtype), dgate [T, K] fp32; the routing arrays are those
 * of the forward pass.  Rows of dy_perm >= offsets[N] are not written. */
moe_status moe_combine_backward(const moe_shape* shape, const void* x, const void* y_perm,
                                const int32_t* topk_idx, const float* topk_gate,
                                const int32_t* slot_pos, const void* dout, float gamma,
                                void* dy_perm, float* dgate, void* stream);

/* Backward of the router (Eq. (1): g_i = R_i with R = softmax of x W_r^T):
 *   dlogits[t, :] = R[t, :] * (dR[t, :] - <R[t, :], dR[t, :]>), dR[t, idx[t,k]] = dgate[t,k]
 *   dw_router     = dlogits^T x          [E, d] (dtype)
 *   dx_router     = dlogits w_router     [T, d] fp32
 * probs [T, E] fp32 are the forward probabilities (moe_route's probs_out).
 * dlogits is kept in the backward workspace (bf16 for MOE_BF16).
 * Load-balance loss (§2.1.2, Eq. (3)-(5)), optional: with lb_f [D+1] fp32 the
 * f_j of moe_lb_stats (held fixed: they count selections), lb_groups = D and
 * lb_alpha = alpha, the gradient of alpha sum_j f_j P_j is added,
 *   dR[t, i] += lb_alpha * lb_f[group(i)] / lb_tokens   for every t and i,
 * group(i) = i / (N/D) for FFN experts and D for the zero experts; lb_tokens
 * is the token count P_j averages over (T, or the global batch with token
 * data parallelism).  lb_f NULL: no load-balance term. */
moe_status moe_route_backward(const moe_shape* shape, const void* x, const void* w_router,
                              const float* probs, const int32_t* topk_idx, const float* dgate,
                              const float* lb_f, int32_t lb_groups, float lb_alpha,
                              int64_t lb_tokens, void* dw_router, float* dx_router, void* ws,
                              size_t ws_bytes, void* stream);

/* Backward of the SwiGLU experts over the routed rows (per expert segment):
 *   dh = dy_perm W2_e;  da = dh u SiLU'(a);  du = dh SiLU(a)   (kept in the
 *                                                backward workspace, dtype)
 *   dx_perm = da W1_e + du W3_e                 [T*K, d]
 *   dw1[e] = da^T x_perm,  dw3[e] = du^T x_perm [N, I, d]
 *   dw2[e] = dy_perm^T h                        [N, d, I]
 * x_perm, h, au from the forward pass (moe_permute, moe_expert_gate_up_save),
 * offsets [N+1].  An expert with no rows gets zero weight gradients.  Rows of
 * dx_perm >= offsets[N] are not written.  For MOE_BF16 the tensor-core path
 * needs d % 128 == 0 and I % 128 == 0. */
moe_status moe_expert_ffn_backward(const moe_shape* shape, const void* x_perm, const void* w1,
                                   const void* w3, const void* w2, const int32_t* offsets,
                                   const void* h, const void* au, const void* dy_perm,
                                   void* dx_perm, void* dw1, void* dw3, void* dw2, void* ws,
                                   size_t ws_bytes, void* stream);

/* Token gradient, gathered per token in a fixed order (the deterministic
 * form of the scatter-add back through the dispatch):
 *   dx[t] = sum_{k: idx < N, in k order} dx_perm[slot_pos[t,k]]
 *           + gamma * (sum_{k: idx >= N} gate[t,k]) * dout[t]  (+ dx_router[t])
 * accumulated in fp32 and rounded once.  dout, dx [T, d] (dtype), dx_perm
 * [T*K, d] (dtype), dx_router [T, d] fp32 or NULL. */
moe_status moe_permute_backward(const moe_shape* shape, const void* dout,
                                const int32_t* topk_idx, const float* topk_gate,
                                const int32_t* slot_pos, const void* dx_perm,
                                const float* dx_router, float gamma, void* dx, void* stream);

/* Synchronises `stream`, reads the workspace status word into *status_out
 * (may be NULL) and clears it.  Returns MOE_ERR_DEVICE_STATUS when it was
 * non-zero. */
moe_status moe_get_device_status(void* ws, void* stream, uint32_t* status_out);

/* Message of the last error on the calling thread ("" if none). */
const char* moe_last_error(void);

/* Number of CUDA kernels this library has launched in the calling process
 * (all devices, all threads).  Instrumentation only. */
uint64_t moe_kernel_launches(void);

/* Failure-detection settings of the tensor-core GEMMs (gate/up, down, router,
 * MXFP8 and backward GEMMs), process-wide, read at each later launch.  Not part
 * of the layer: the pages have no counterpart.
 *   wait_limit_ns: time after which one bounded pipeline wait gives up
 *     (0 restores the default of 4 s).  A wait that gives up sets
 *     MOE_DEV_PIPELINE_TIMEOUT in the workspace status word; the kernel then
 *     stops issuing work, waits (bounded) for its copies in flight, frees its
 *     tensor memory and returns, leaving the context usable.  Its output is
 *     incomplete.
 *   stall_first_fill: for tests of that path only.  Non-zero makes the
 *     bf16 GEMMs' TMA producer issue nothing, so the MMA issuer's first wait
 *     runs out after wait_limit_ns; 0 turns it off.
 * Returns MOE_ERR_INVALID_ARG for a limit above one minute. */
moe_status moe_debug_set_pipeline(uint64_t wait_limit_ns, int32_t stall_first_fill);

#ifdef __cplusplus
}
#endif

#endif /* MOE_B200_H */
