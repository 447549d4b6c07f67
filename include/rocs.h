/*
 * librocs -- the ROCS (Request-Oriented Compute Sharing) forward hot path on one NVIDIA B200.
 *
 * Sources of the operations (page title, section, equation):
 *   [REV] "ROCS：面向请求的大规模推荐计算共享" -- review of arXiv:2607.27744 (liuzhao09.github.io)
 *         §2.1 Generalized Layer Masking, §2.2 Deep Cross Attention,
 *         §2.4 In-Kernel Broadcast Optimization.
 *   [SUM] "Meta推出ROCS：推荐系统推理效率提升3倍，零质量损失" -- PaperDaily summary.
 *
 * Conventions for every call:
 *   - Every tensor argument is a caller-owned DEVICE pointer (allocated by the caller, e.g. by
 *     torch); host-side structs (descriptors, weight tables) are read during the call only.
 *     The library never allocates device memory inside these calls; calls that need scratch
 *     take a caller workspace whose size the matching *_workspace query returns.
 *   - Row-major storage, innermost dimension contiguous, leading dimension = width.
 *     Weights are [out, in] (y = W x, [REV] §2.1); biases and LayerNorm parameters are fp32.
 *   - Candidates are grouped by request where a call takes `offsets` (offsets[r] <= c <
 *     offsets[r+1] belong to request r); `req_idx` (the map m of [REV] §2.4) may be in any
 *     order for rocs_linear_ikbo.
 *   - Asynchrony: each call enqueues work on `stream` (a cudaStream_t passed as void*; NULL =
 *     the legacy default stream) and returns after launch.  Calls contain no host sync and are
 *     safe to record into a CUDA graph once the arguments are fixed.
 *   - Errors: arguments are validated on the host first; on failure the call returns a status
 *     other than ROCS_OK, launches nothing and sets a thread-local message (rocs_last_error).
 *     Conditions only the device can see (a request index out of range, counts that do not sum
 *     to B_C, an internal wait that ran out) set a sticky per-handle device status word; the
 *     kernel skips the affected rows or returns early, never traps.  Read and clear it with
 *     rocs_get_device_status.
 *   - Determinism: for fixed shapes every result is bitwise reproducible (fixed reduction
 *     order, no atomics on data, no split-K); a candidate's outputs do not depend on other
 *     candidates' inputs.
 *   - No C++ exception crosses this boundary.
 */
#ifndef ROCS_H
#define ROCS_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  ROCS_OK = 0,
  ROCS_ERR_INVALID_ARG = 1,    /* host validation failed: null pointer, bad size, misaligned */
  ROCS_ERR_UNSUPPORTED = 2,    /* valid but outside what this build implements (message says) */
  ROCS_ERR_CUDA = 3,           /* a CUDA runtime/driver call failed (message has the CUDA error) */
  ROCS_ERR_WORKSPACE = 4,      /* workspace null or smaller than the *_workspace query */
  ROCS_ERR_INDEX = 5,          /* device: a request index outside [0, B_R); rows skipped */
  ROCS_ERR_DEVICE_TIMEOUT = 6, /* device: a bounded internal wait ran out; kernel returned */
  ROCS_ERR_COUNTS = 7          /* device: counts negative or not summing to B_C */
} rocs_status;

typedef enum { ROCS_F32 = 0, ROCS_BF16 = 1 } rocs_dtype;
typedef enum { ROCS_ACT_NONE = 0, ROCS_ACT_RELU = 1, ROCS_ACT_GELU = 2, ROCS_ACT_SIGMOID = 3 } rocs_act;

typedef struct rocs_context* rocs_handle_t;

/* ------------------------------------------------------------------------------------------
 * Handle.  rocs_create binds a handle to CUDA device `device` (made current for the call),
 * allocates the 4-byte device status word and resolves the driver entry point used to encode
 * TMA descriptors.  All later calls on the handle must run with that device current.
 * rocs_destroy frees what rocs_create allocated (synchronising the device first).
 * ---------------------------------------------------------------------------------------- */
rocs_status rocs_create(rocs_handle_t* handle, int device);
rocs_status rocs_destroy(rocs_handle_t handle);

/* Thread-local text of the last error returned on this thread ("" if none). */
const char* rocs_last_error(void);

/* Synchronises `stream`, copies the sticky device status word to *code (a rocs_status value,
 * ROCS_OK if nothing was flagged) and clears it. */
rocs_status rocs_get_device_status(rocs_handle_t handle, void* stream, int32_t* code);

/* Number of streaming multiprocessors of the handle's device (used for grid sizing). */
int32_t rocs_num_sms(rocs_handle_t handle);

/* ------------------------------------------------------------------------------------------
 * a0. Segment bookkeeping ([REV] §2.4: map m, candidate i belongs to request m_i).
 *   counts  [B_R]   int32, device: candidates of each request (>= 0).
 *   offsets [B_R+1] int32, device, written: exclusive running total, offsets[B_R] = B_C.
 *   req_idx [B_C]   int32, device, written: req_idx[c] = r for offsets[r] <= c < offsets[r+1].
 *   B_C is the caller's total; if the counts disagree (or one is negative) the device status
 *   becomes ROCS_ERR_COUNTS and req_idx is written only inside [0, B_C).
 *   Limits: 1 <= B_R <= 2^24, 0 <= B_C < 2^31.
 * ---------------------------------------------------------------------------------------- */
rocs_status rocs_segments_from_counts(rocs_handle_t handle, const int32_t* counts, int32_t B_R,
                                      int32_t* offsets, int32_t* req_idx, int64_t B_C, void* stream);

/* ------------------------------------------------------------------------------------------
 * Multi-GPU sharding (host only, no handle).  Requests are independent ([REV] §1: a request's
 * inputs are constant across its candidates, and requests share only the weights), so a batch
 * shards by whole requests with no exchange step.  rocs_partition_requests assigns each request
 * of one batch to one of n_parts parts (GPUs), balancing the work cost_R + counts[r] * cost_C
 * by longest-processing-time-first greedy: requests in decreasing work (ties: lower index
 * first) each go to the part with the least work so far (ties: lower part).  The largest part is
 * then within 4/3 of the best possible.  Deterministic.
 *   counts  [B_R] int32, host: candidates of each request (>= 0).
 *   part_of [B_R] int32, host, written: the part of request r, in [0, n_parts).
 *   cost_R, cost_C >= 0 and finite, not both 0; 1 <= B_R <= 2^24; 1 <= n_parts <= 4096.
 *   Returns ROCS_ERR_INVALID_ARG (nothing written) otherwise.
 * ---------------------------------------------------------------------------------------- */
rocs_status rocs_partition_requests(const int32_t* counts, int32_t B_R, int32_t n_parts, double cost_R,
                                    double cost_C, int32_t* part_of);

/* ------------------------------------------------------------------------------------------
 * a1-a3. Two-group GLM linear with in-kernel broadcast ([REV] §2.1 two-group block matrix,
 * §2.4 equation Y_i^C = Z_{m_i} + W_CC X_i^C):
 *   Y^R = act(W_RR X^R + b^R)                    on the request batch (B_R rows), once;
 *   Z   = W_CR X^R + b^C                         on the request batch, fp32, in the workspace;
 *   Y^C = act(W_CC X^C + Z[req_idx[c]])          on the candidate batch, Z gathered in the
 *                                                epilogue of the candidate GEMM (no broadcast
 *                                                tensor is ever written).
 * d_R_out may be 0 (no request output: W_RR, b_R, Y_R ignored and may be NULL).
 * dtype_in = ROCS_F32: X, W and Y are fp32 and the path is exact-order fp32 FFMA (no TF32).
 * dtype_in = ROCS_BF16: X and W are bf16, accumulation fp32 on the tensor cores, Y in
 *   dtype_out (bf16 or fp32).
 * Alignment fix ([REV] §2.4, zero padding of decomposed dims): when an input row's byte
 *   length is not a multiple of 16 the call copies the operand into a zero-padded workspace
 *   region first (results unchanged; the workspace query accounts for it).
 * Shapes: X_R [B_R, d_R_in], X_C [B_C, d_C_in], req_idx [B_C], W_RR [d_R_out, d_R_in],
 *   W_CR [d_C_out, d_R_in], W_CC [d_C_out, d_C_in], b_R [d_R_out], b_C [d_C_out],
 *   Y_R [B_R, d_R_out], Y_C [B_C, d_C_out].  All pointers 16-byte aligned.
 * ---------------------------------------------------------------------------------------- */
typedef struct {
  int32_t B_R;
  int64_t B_C;
  int32_t d_R_in, d_C_in, d_R_out, d_C_out;
  rocs_dtype dtype_in;
  rocs_dtype dtype_out;
  rocs_act act;
} rocs_ikbo_desc;

rocs_status rocs_linear_ikbo_workspace(rocs_handle_t handle, const rocs_ikbo_desc* desc, size_t* bytes);
rocs_status rocs_linear_ikbo(rocs_handle_t handle, const rocs_ikbo_desc* desc,
                             const void* X_R, const void* X_C, const int32_t* req_idx,
                             const void* W_RR, const void* W_CR, const void* W_CC,
                             const float* b_R, const float* b_C, void* Y_R, void* Y_C,
                             void* workspace, size_t workspace_bytes, void* stream);

/* ------------------------------------------------------------------------------------------
 * FP8-weight (W8A16) IKBO linear ("Compute Only Once: UG-Separation for Efficient Large
 * Recommendation Models", §三 Stage 4 and the W8A16 table of §六: 8-bit floating-point weights,
 * bf16 activations).  Weights are E4M3 bytes ("finite" E4M3: bias 7, no infinities, largest
 * magnitude 448) with one float32 scale per output channel: the effective weight is q_oi * s_o,
 * and the scale multiplies the accumulated dot product before the bias, Z[m] and activation.
 *
 * rocs_quantize_weights_fp8: per-output-channel quantisation of W [rows, cols] (ROCS_F32 or
 *   ROCS_BF16, device): s_r = max_c |W_rc| / 448 in float32 (1 for an all-zero row), Q_rc =
 *   E4M3(W_rc / s_r) with the division in float32, rounded to nearest even and saturated.
 *   Q [rows, cols] uint8 and scale [rows] float32 written.
 *
 * rocs_linear_ikbo_w8: rocs_linear_ikbo (dtype_in = ROCS_BF16) with the three weight blocks as
 *   (Q_RR, s_RR), (Q_CR, s_CR), (Q_CC, s_CC).  Shapes as rocs_linear_ikbo; Q_* [out, in] uint8;
 *   s_* [out] float32.  By default a GEMM side with at most 64 rows streams the weights through
 *   a register-tiled kernel (each byte read once, converted to f16 operands in registers), and a
 *   larger side expands its weights to bf16 in the workspace once (exactly) and runs the tcgen05
 *   GEMM.  With rocs_set_w8_tensor_cores(handle, 1) and d_R_in, d_C_in multiples of 128, the FP8
 *   weights go to the tcgen05 tensor cores directly instead: TMA brings each weight tile into
 *   shared memory as bytes, where it is converted to f16 exactly (every E4M3 value is an f16
 *   value) and multiplied with the activations, brought to f16 once per call with a per-row
 *   power-of-two shift that the epilogue undoes; the weights then must be 16-byte aligned.  Both
 *   give the same results up to fp32 summation order.  Requires d_R_in % 8 == 0 and
 *   d_C_in % 8 == 0; weights at least 8-byte aligned.  Workspace: rocs_linear_ikbo_w8_workspace
 *   (query it after choosing the path: the two paths need different amounts).
 * ---------------------------------------------------------------------------------------- */
rocs_status rocs_quantize_weights_fp8(rocs_handle_t handle, const void* W, rocs_dtype w_dtype, int32_t rows,
                                      int32_t cols, uint8_t* Q, float* scale, void* stream);
rocs_status rocs_linear_ikbo_w8_workspace(rocs_handle_t handle, const rocs_ikbo_desc* desc, size_t* bytes);
rocs_status rocs_linear_ikbo_w8(rocs_handle_t handle, const rocs_ikbo_desc* desc, const void* X_R,
                                const void* X_C, const int32_t* req_idx, const uint8_t* Q_RR,
                                const uint8_t* Q_CR, const uint8_t* Q_CC, const float* s_RR,
                                const float* s_CR, const float* s_CC, const float* b_R, const float* b_C,
                                void* Y_R, void* Y_C, void* workspace, size_t workspace_bytes,
                                void* stream);

/* ------------------------------------------------------------------------------------------
 * rocs_linear_ikbo_noalloc: the same operation as rocs_linear_ikbo for callers that cannot
 * allocate device memory at all, not even a workspace to hand over -- for example plugin hosts
 * and serving loops that plan every device buffer up front and forbid allocation while
 * requests are in flight.  The paper has no counterpart; this is a deployment variant.
 *   - Scratch: Z = W_CR X^R + b^C lives in one built-in device array of 1,048,576 fp32 values
 *     (4 MiB) that every GPU loading the library keeps until the process exits.  Requests with
 *     B_R * d_C_out above that limit, or bf16 rows that would need the alignment fix
 *     (d_R_in or d_C_in not a multiple of 8), return ROCS_ERR_UNSUPPORTED with a message
 *     pointing to rocs_linear_ikbo.  The call never calls an allocation or free routine.
 *   - Set-up: the first call on each device (with that device current, as for every call on
 *     the handle) looks up the array's device address once and caches it.  Under lazy module
 *     loading (the CUDA 12 default) the driver loads the library's device code, and commits the
 *     4 MiB array, at that first call: make it once per device as a warm-up, before serving and
 *     before any stream capture; later calls allocate nothing.  A call from a context other than
 *     the one of the first call looks the address up again in its own context.  Resetting the
 *     device (cudaDeviceReset) while the library stays loaded is not supported: the cached
 *     address may then no longer be the array's.
 *   - Sharing: all calls on a device use the same array, and it keeps the last call's Z.
 *     Z is fully rewritten before it is read, so nothing has to be cleared, but calls whose
 *     work overlaps on the GPU (different streams, or different host threads) race on it:
 *     order them on one stream or with events.
 *   - Arguments, layouts, dtypes and results are those of rocs_linear_ikbo.
 * ---------------------------------------------------------------------------------------- */
rocs_status rocs_linear_ikbo_noalloc(rocs_handle_t handle, const rocs_ikbo_desc* desc,
                                     const void* X_R, const void* X_C, const int32_t* req_idx,
                                     const void* W_RR, const void* W_CR, const void* W_CC,
                                     const float* b_R, const float* b_C, void* Y_R, void* Y_C,
                                     void* stream);

/* ------------------------------------------------------------------------------------------
 * a6. Concat + residual + group-local LayerNorm ([SUM]: normalisation statistics per group,
 * never over the concatenation; [REV] §2.1 Figure 2(b)).  For each of `rows` rows:
 *   x = concat(X1[row, 0:w1], X2[row, 0:w2]) (+ residual[row, 0:w1+w2] if non-NULL)
 *   Y[row] = (x - mean(x)) / sqrt(var(x) + eps) * gamma + beta   (biased variance)
 * One call normalises one group; the request and candidate groups are separate calls.
 * X2 may be NULL with w2 = 0.  X1, X2, residual and Y share dtype `io` (bf16 or fp32);
 * gamma, beta fp32 [w1+w2].  Statistics in fp32.  1 <= w1 + w2 <= 8192.
 * ---------------------------------------------------------------------------------------- */
rocs_status rocs_group_layernorm(rocs_handle_t handle, const void* X1, int32_t w1, const void* X2,
                                 int32_t w2, const void* residual, int64_t rows, const float* gamma,
                                 const float* beta, float eps, void* Y, rocs_dtype io, void* stream);

/* ------------------------------------------------------------------------------------------
 * a4. Block-masked factorization machine ([REV] §2.1 FM equation, Figure 2(c)).
 *   E_R [B_R, n_R, D] bf16, E_C [B_C, n_C, D] bf16, req_idx [B_C].
 *   F_R [B_R, n_R*n_R]: F^R_r = E^R_r E^R_r^T (request x request only), row-major.
 *   F_C [B_C, n_C*(n_R+n_C)]: F^C_c = E^C_c [E^R_{m_c} ; E^C_c]^T, columns ordered
 *       [request tokens, candidate tokens].
 *   Outputs in `out` dtype (bf16 or fp32); fp32 accumulation on the tensor cores.
 *   Limits: n_R <= 64, n_C <= 32, D % 16 == 0, D <= 256.  F_R may be NULL.
 * ---------------------------------------------------------------------------------------- */
rocs_status rocs_fm_masked(rocs_handle_t handle, const void* E_R, const void* E_C,
                           const int32_t* req_idx, int32_t B_R, int64_t B_C, int32_t n_R,
                           int32_t n_C, int32_t D, void* F_R, void* F_C, rocs_dtype out, void* stream);

/* ------------------------------------------------------------------------------------------
 * a4/a8. Token-axis linear compression as a GLM linear over tokens ([REV] §2.1 masked linear
 * applied along the embedding-count axis; Wukong's LCB, Figure 1(d); the DCA query
 * generator's LCB, §2.2):
 *   L^R_r = P_RR E^R_r                       [o_R, D]
 *   L^C_c = P_CR E^R_{m_c} + P_CC E^C_c       [o_C, D]   (P_CR E^R computed once per request)
 *   P_RR [o_R, n_R], P_CR [o_C, n_R], P_CC [o_C, n_C] bf16; no bias.  o_R may be 0.
 *   Outputs L_R [B_R, o_R, D], L_C [B_C, o_C, D] in `out` dtype; row strides ld_LR / ld_LC
 *   elements (>= o*D) so results can land inside a wider token buffer.
 *   Workspace: o_C * D * B_R fp32 (see rocs_token_lcb_workspace).
 * ---------------------------------------------------------------------------------------- */
rocs_status rocs_token_lcb_workspace(rocs_handle_t handle, int32_t B_R, int32_t o_C, int32_t D, size_t* bytes);
rocs_status rocs_token_lcb(rocs_handle_t handle, const void* E_R, const void* E_C,
                           const int32_t* req_idx, int32_t B_R, int64_t B_C, int32_t n_R,
                           int32_t n_C, int32_t D, const void* P_RR, const void* P_CR,
                           const void* P_CC, int32_t o_R, int32_t o_C, void* L_R, int64_t ld_LR,
                           void* L_C, int64_t ld_LC, rocs_dtype out, void* workspace,
                           size_t workspace_bytes, void* stream);

/* ------------------------------------------------------------------------------------------
 * a9. Grouped cross-attention with shared K/V ([REV] §2.2 A_i = Attn(Q_i, S_i W_K, S_i W_V),
 * §2.4 IKBO-DCA: the kernel reads request-batch K/V and the map directly).
 *   Q [rows, H*d_h] bf16, query rows grouped by request: offsets[r] <= q < offsets[r+1]
 *     attend to request r.  offsets int32 [B_R+1], device.
 *   K, V [B_R, L, H*d_h] bf16 (each request's K/V stored once).
 *   O [rows, ld_O] in `out` dtype (bf16 or fp32), head h at columns [h*d_h, (h+1)*d_h).
 *   O_q = softmax(q k^T * scale) v per head; fp32 softmax statistics.
 *   kv_len int32 [B_R], device, or NULL: request r's keys are the first kv_len[r] of its L rows
 *     (a ragged history, 1 <= kv_len[r] <= L); later rows are padding and never attended.  A
 *     length outside [1, L] sets ROCS_ERR_COUNTS and that request's rows are not written.
 *     NULL: every request has L keys.
 *   Each (request, head)'s K/V is staged in shared memory once and shared by that request's
 *   queries (no per-candidate copy of K/V exists) when L * d_h <= 32768; longer histories are
 *   streamed through a shared-memory ring of 64-key blocks.
 *   Limits: d_h in {32, 64}; B_R * L < 2^31.
 * ---------------------------------------------------------------------------------------- */
rocs_status rocs_dca_cross_attn(rocs_handle_t handle, const void* Q, const void* K, const void* V,
                                const int32_t* offsets, int32_t B_R, int64_t rows, int32_t L,
                                int32_t H, int32_t d_h, float scale, void* O, int64_t ld_O,
                                rocs_dtype out, const int32_t* kv_len, void* stream);

/* ------------------------------------------------------------------------------------------
 * Candidates in any order ([REV] §2.4 notes that IKBO-DCA depends on how candidates are laid out
 * around their request; the segment path above takes them grouped).
 *
 * rocs_sort_by_request: stable counting sort of B_C candidates by their request index.
 *   req_idx [B_C] int32, device, any order; a value outside [0, B_R) is an error.
 *   perm    [B_C] int32, device, written: perm[k] = the candidate at position k of the grouped
 *           order.  Candidates of one request keep their relative order; candidates with a bad
 *           index come after every valid one (in their order) and set ROCS_ERR_INDEX in the
 *           device status.
 *   offsets [B_R+1] int32, device, written: offsets[r] = first position of request r in perm,
 *           offsets[B_R] = the number of candidates with a valid index.
 *   workspace: rocs_sort_by_request_workspace bytes, 16-byte aligned (an int histogram of
 *           (B_R + 1) x ceil(B_C / chunk) entries, chunk >= 512).
 *   Limits: 1 <= B_R <= 2^24, 0 <= B_C < 2^31.  Errors: ROCS_ERR_INVALID_ARG, ROCS_ERR_WORKSPACE.
 *
 * rocs_dca_cross_attn_unsorted: rocs_dca_cross_attn for query rows in any order, each with its
 *   request index req_idx [rows] instead of grouped offsets.  The call sorts the rows (as
 *   rocs_sort_by_request), gathers Q into that order, runs the segment path and writes each valid
 *   row of O at its original position; rows with a bad index are left unwritten (and the device
 *   status says ROCS_ERR_INDEX).  Results equal rocs_dca_cross_attn on the grouped rows.
 *   Q, K, V, O, L, H, d_h, scale, ld_O, out and limits: as rocs_dca_cross_attn.
 *   workspace: rocs_dca_cross_attn_unsorted_workspace bytes, 16-byte aligned (the permutation,
 *   offsets, the sort histogram, Q and O in grouped order).
 * ---------------------------------------------------------------------------------------- */
rocs_status rocs_sort_by_request_workspace(rocs_handle_t handle, int32_t B_R, int64_t B_C, size_t* bytes);
rocs_status rocs_sort_by_request(rocs_handle_t handle, const int32_t* req_idx, int32_t B_R, int64_t B_C,
                                 int32_t* perm, int32_t* offsets, void* workspace, size_t workspace_bytes,
                                 void* stream);
rocs_status rocs_dca_cross_attn_unsorted_workspace(rocs_handle_t handle, int32_t B_R, int64_t rows, int32_t H,
                                                   int32_t d_h, rocs_dtype out, size_t* bytes);
rocs_status rocs_dca_cross_attn_unsorted(rocs_handle_t handle, const void* Q, const void* K, const void* V,
                                         const int32_t* req_idx, int32_t B_R, int64_t rows, int32_t L,
                                         int32_t H, int32_t d_h, float scale, void* O, int64_t ld_O,
                                         rocs_dtype out, const int32_t* kv_len, void* workspace,
                                         size_t workspace_bytes, void* stream);

/* ------------------------------------------------------------------------------------------
 * a7. DCA shared sequence encoder and its K/V projections, request-only ([REV] §2.2:
 * S_i = Enc_i(S_{i-1}); S_i and its K/V computed once per request).
 *   Enc(S) = LN(S + MHSA(S) W_O^T), MHSA non-causal with Q = S W_Q^T, K = S W_K^T,
 *   V = S W_V^T, H heads; LN per token over d.
 *   After layer i: K^R_i = S_i W_K^R^T, V^R_i = S_i W_V^R^T, K^C_i = S_i W_K^C^T,
 *   V^C_i = S_i W_V^C^T.
 *   Hist [B_R, L, d] bf16.  S [layers, B_R, L, d] bf16 written.
 *   KV [layers, 4, B_R, L, d] bf16 written, order (K^R, V^R, K^C, V^C).
 *   lengths int32 [B_R], device, or NULL: request r's history is its first lengths[r] rows
 *     (1 <= lengths[r] <= L); the self-attention takes only those rows as keys.  Rows after them
 *     are padding: they are computed like the others (every per-row step is row-independent) and
 *     their S and K/V rows are unspecified, but they never reach a history row.  NULL: every
 *     history has L rows.  Histories longer than the staged kernels hold (L * d_h > 32768) are
 *     streamed through shared memory.
 * ---------------------------------------------------------------------------------------- */
typedef struct {
  const void *Wq, *Wk, *Wv, *Wo;       /* [d, d] bf16 */
  const float *ln_gamma, *ln_beta;     /* [d] */
  const void *WK_R, *WV_R, *WK_C, *WV_C; /* [d, d] bf16 */
} rocs_dca_layer_weights;

#define ROCS_MAX_LAYERS 8

typedef struct {
  int32_t B_R, L, d, H, layers;
} rocs_dca_desc;

rocs_status rocs_dca_encode_workspace(rocs_handle_t handle, const rocs_dca_desc* desc, size_t* bytes);
rocs_status rocs_dca_encode(rocs_handle_t handle, const rocs_dca_desc* desc, const void* Hist,
                            const int32_t* lengths /* [B_R] or NULL */,
                            const rocs_dca_layer_weights* weights /* [layers] */, void* S, void* KV,
                            void* workspace, size_t workspace_bytes, void* stream);

/* ------------------------------------------------------------------------------------------
 * a0-a11. Whole ROCS forward ([REV] §2.1 Figure 1(d) ROCSified Wukong stack, §2.2 DCA,
 * §2.4 IKBO), one call.  Which parts run is set by the descriptor:
 *   glm_layers > 0: Wukong-style GLM stack on E_R [B_R, n_R, D], E_C [B_C, n_C, D]; each layer
 *     E' = GroupLN(concat(MLP(FM(E)), LCB(E)) + E) with a two-layer GLM-MLP (GELU hidden).
 *   dca_layers > 0: DCA over history Hist [B_R, L, d]; depth i's query generator reads either
 *     the DCA's own embeddings Y_R [B_R, q_n_R, q_dim], Y_C [B_C, q_n_C, q_dim] with earlier
 *     depths' outputs appended as one token per group (dca_query_source = 0), or the GLM stack's
 *     layer i-1 output (dca_query_source = 1, q_dim = D).
 *   score_h1 > 0: candidate scoring head sigmoid(w3 ReLU(W2 ReLU(IKBO([E^R_m, A^R_m] |
 *     [E^C, A^C])) + b2) + b3).
 * Inputs/outputs are device pointers; unused ones may be NULL.  Counts are device int32 [B_R];
 * the call writes offsets / req_idx itself (outputs, device).  Inputs are bf16; outputs E_R,
 * E_C, A_R, A_C and score are fp32, S is bf16.
 * Precision: tensor-core products are bf16 x bf16 with fp32 accumulation.  Activations that feed
 * a tensor-core GEMM or the attention scores on the candidate path are kept as a bf16 hi/lo
 * pair (hi = bf16(x), lo = bf16(x - hi)), and activations no GEMM consumes (the GLM residual
 * stream, MLP and LCB outputs, attention outputs) stay fp32, so rounding of intermediates does
 * not accumulate across the stacked layers.  Split operands need widths that are multiples of
 * 64 (n_R^2, n_C(n_R+n_C), hidden, q_dim, d).
 * GLM limits (else ROCS_ERR_INVALID_ARG): n_R + n_C <= 64; D a multiple of 16, at most 256;
 * n * D <= 8192 per group; fm_out + lcb_out = n per group (the residual); 1 <= lcb_out_C <= 8.
 * With D = 128 and n_C <= 16 the candidate FM, token LCB and query token of a layer run as one
 * pass over the embeddings where its shared memory fits (always for bf16 layer-0 inputs; for the
 * fp32 stream of later layers while n_R + 16 <= 48), and as separate kernels otherwise, with the
 * same results.
 * Graph replay (a11): the handle records each distinct call (the bytes of the descriptor, the
 * weight/input/output pointer structs and the workspace pointer and size).  The first call
 * with a given record launches the kernels directly; the second captures the same launch
 * sequence into a CUDA graph (on a stream the handle owns) and launches it on `stream`; later
 * calls replay it.  The graph reads the caller's buffers at replay time, so new contents of
 * the same buffers are picked up; different pointers or sizes make a new record (the handle
 * keeps the 8 most recent).  rocs_set_graph_replay(h, 0) turns replay off (every call then
 * launches directly), as does per-launch timing while it runs.  Not callable while `stream`
 * itself is being captured by the caller when replay is on.
 * ---------------------------------------------------------------------------------------- */
typedef struct {
  const void *W_RR, *W_CR, *W_CC;  /* bf16 [out, in] */
  const float *b_R, *b_C;
} rocs_glm_linear_weights;

typedef struct {
  rocs_glm_linear_weights mlp1, mlp2;
  const void *P_RR, *P_CR, *P_CC;  /* token-axis LCB, bf16 */
  const float *lnR_gamma, *lnR_beta, *lnC_gamma, *lnC_beta;
} rocs_glm_layer_weights;

typedef struct {
  const void *p_RR, *p_CR, *p_CC;  /* token LCB to one token, bf16 [1, n] */
  rocs_glm_linear_weights mlp1, mlp2;
} rocs_qgen_weights;

typedef struct {
  rocs_glm_linear_weights s1;      /* W_RR / b_R unused (no request output) */
  const void* W2; const float* b2; /* [h2, h1] bf16, [h2] */
  const void* w3; const float* b3; /* [1, h2] bf16, [1] */
} rocs_score_weights;

typedef struct {
  rocs_glm_layer_weights glm[ROCS_MAX_LAYERS];
  rocs_dca_layer_weights dca[ROCS_MAX_LAYERS];
  rocs_qgen_weights qgen[ROCS_MAX_LAYERS];
  rocs_score_weights score;
} rocs_model_weights;

typedef struct {
  int32_t B_R;
  int64_t B_C;
  /* GLM stack */
  int32_t glm_layers, n_R, n_C, D, hidden, fm_out_R, fm_out_C, lcb_out_R, lcb_out_C;
  /* DCA */
  int32_t dca_layers, L, d, H, q_n_R, q_n_C, q_dim, dca_query_source;
  /* scoring head */
  int32_t score_h1, score_h2;
} rocs_model_desc;

typedef struct {
  const int32_t* counts;            /* [B_R] */
  const void *E_R, *E_C;            /* GLM inputs */
  const void* Hist;                 /* DCA history */
  const void *Y_R, *Y_C;            /* DCA own query embeddings (source 0) */
  const int32_t* hist_len;          /* [B_R] or NULL: request r's history is its first hist_len[r] of
                                       the L rows of Hist (1 <= hist_len[r] <= L; the rest is padding,
                                       never a key).  NULL: every history has L rows. */
} rocs_inputs;

typedef struct {
  int32_t* offsets;                 /* [B_R+1] written (NULL: kept in the workspace) */
  int32_t* req_idx;                 /* [B_C] written (NULL: kept in the workspace) */
  void *E_R, *E_C;                  /* final GLM outputs, fp32 [B_R, n_R, D] / [B_C, n_C, D] (nullable) */
  void* S;                          /* bf16 [dca_layers, B_R, L, d] (nullable) */
  void *A_R, *A_C;                  /* fp32 [dca_layers, B_R, d], [dca_layers, B_C, d] (nullable) */
  float* score;                     /* [B_C] (nullable) */
} rocs_outputs;

rocs_status rocs_forward_workspace(rocs_handle_t handle, const rocs_model_desc* model, size_t* bytes);
rocs_status rocs_forward(rocs_handle_t handle, const rocs_model_desc* model,
                         const rocs_model_weights* weights, const rocs_inputs* inputs,
                         rocs_outputs* outputs, void* workspace, size_t workspace_bytes, void* stream);
/* Turns rocs_forward's graph replay on (enable = 1, the default) or off (0) for this handle.
 * Errors: ROCS_ERR_INVALID_ARG for a NULL handle or another value of enable. */
rocs_status rocs_set_graph_replay(rocs_handle_t handle, int32_t enable);

/* Fused IKBO launch ([REV] §2.4: the request and candidate GEMMs in one persistent kernel) on
 * (enable = 1, the default) or off (0) for this handle.  It applies to the bf16 path of
 * rocs_linear_ikbo and to every IKBO linear inside rocs_forward, where the candidate GEMM has
 * K >= 1024 (a hi/lo split input counting twice) or at most 32768 candidates; other shapes keep
 * the two launches, which measured faster there.  Fused, the request GEMM's tiles
 * come first in every CTA's order and publish completion flags (kept in the workspace, zeroed by
 * each call); a candidate tile's epilogue waits (bounded) for the flags of the request tiles whose
 * Z rows it gathers, and the launch is cooperative, so every CTA is resident.  Results are
 * identical to the two-launch form.  A wait that runs out sets ROCS_ERR_DEVICE_TIMEOUT in the
 * device status and leaves the affected rows unwritten.
 * Errors: ROCS_ERR_INVALID_ARG for a NULL handle or another value of enable. */
rocs_status rocs_set_ikbo_fused(rocs_handle_t handle, int32_t enable);

/* Test hook for the failure-detection path; off by default and not for production use.  The
 * pages have no counterpart: it exists so that a test can make the fused IKBO launch's bounded
 * completion-flag wait run out on purpose, without faulting or hanging the GPU.
 * With flag_index >= 0, every later fused IKBO launch on this handle skips publishing completion
 * flag `flag_index` (the request GEMM's tile in row block b and output column tile n has index
 * b * n_tiles + n; with d_C_out <= 256 there is one column tile, so the index is the request
 * block) and bounds each completion-flag wait by wait_budget_cycles SM clock cycles (clock64)
 * instead of about 1 s.  The candidate tiles that gather Z rows from that request block then give
 * up after the budget: ROCS_ERR_DEVICE_TIMEOUT is set in the device status, those candidate rows
 * are left unwritten, and the kernel returns normally (its CTAs drain their copies and MMAs and
 * release tensor memory), so the next call on the stream runs as usual.  flag_index = -1 turns the
 * hook off and restores the default budget (wait_budget_cycles is then ignored).
 * Errors: ROCS_ERR_INVALID_ARG for a NULL handle, flag_index < -1, or, with flag_index >= 0, a
 * budget outside [1e3, 1e10] cycles. */
rocs_status rocs_test_withhold_ikbo_flag(rocs_handle_t handle, int32_t flag_index, int64_t wait_budget_cycles);

/* Measurement: the exponential throughput that bounds the DCA attention kernels (one exponential
 * per score, [REV] §2.2 grouped cross-attention and the shared encoder).  The pages give no such
 * rate.  Every thread of a grid that fills all SMs carries eight independent pairs of scores
 * through the attention softmax's per-score steps: scale and shift on the packed FMA path, 2^x,
 * packing to bf16 pairs; n_poly of every eight pairs (0..8) take the FMA-pipe polynomial, the rest
 * MUFU ex2 (the attention kernels use n_poly = 3).  Writes the best of five timed launches as
 * exponentials per second to *exp2_per_second.  Synchronises `stream`; allocates nothing.
 * Errors: ROCS_ERR_INVALID_ARG (NULL handle or output, n_poly outside [0, 8]); ROCS_ERR_CUDA. */
rocs_status rocs_probe_exp2_rate(rocs_handle_t handle, int32_t n_poly, double* exp2_per_second, void* stream);

/* FP8-weight linears on the tensor cores ([UGS] §三 Stage 4): with enable = 1, rocs_linear_ikbo_w8
 * on this handle feeds the E4M3 weights to tcgen05 MMAs through a shared-memory conversion to f16
 * (when both input widths are multiples of 128); with enable = 0, the default, it uses the
 * register-tiled weight-streaming kernel and the bf16 expansion, which measured faster on most
 * shapes.  Errors: ROCS_ERR_INVALID_ARG for a NULL handle or another value of enable. */
rocs_status rocs_set_w8_tensor_cores(rocs_handle_t handle, int32_t enable);

/* ------------------------------------------------------------------------------------------
 * Per-launch timing (tracing).  After rocs_timing_start(h, max_launches), every kernel the
 * library launches for handle h records a CUDA event before and after itself on the stream it
 * is launched on (events from a pool of 2 * max_launches, created here; launches beyond the
 * pool are counted as dropped).  rocs_timing_stop waits for those events, writes one text line
 * per launch site "<call-site>:<kernel> <launches> <total_ms>" (NUL-terminated) into `report`,
 * destroys the events and stops recording.  Not for use inside CUDA-graph capture.
 * ---------------------------------------------------------------------------------------- */
rocs_status rocs_timing_start(rocs_handle_t handle, int32_t max_launches);
rocs_status rocs_timing_stop(rocs_handle_t handle, char* report, size_t report_bytes);

#ifdef __cplusplus
}
#endif
#endif /* ROCS_H */
