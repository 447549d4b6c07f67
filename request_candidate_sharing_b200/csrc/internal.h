// Host-side internal interfaces of librocs (not part of the C ABI).
#pragma once
#include <cuda.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include <string>
#include <vector>

#include "../../include/rocs.h"

// Per-launch CUDA-event timing (see rocs_timing_start / rocs_timing_stop).
struct RocsTimer {
  bool enabled = false;
  std::vector<cudaEvent_t> pool;   // 2 events per recorded launch
  size_t next = 0;
  std::vector<std::string> labels; // label of launch i uses pool[2i], pool[2i+1]
  long long dropped = 0;           // launches beyond the pool size
};

// One recorded rocs_forward: the call's argument bytes (model, weights, inputs, outputs,
// workspace) and, from the second identical call on, its launch sequence as a CUDA graph.
struct ForwardGraph {
  std::vector<uint8_t> key;
  int calls = 0;
  cudaGraphExec_t exec = nullptr;
};

struct rocs_context {
  int device = 0;
  int num_sms = 148;
  int* d_status = nullptr;   // sticky device status word
  void* encode_fn = nullptr; // cuTensorMapEncodeTiled
  RocsTimer timer;
  int graph_replay = 1;                 // rocs_set_graph_replay
  int ikbo_fused = 1;                   // rocs_set_ikbo_fused
  int w8_tensor_cores = 0;              // rocs_set_w8_tensor_cores: FP8 operands on tcgen05 (opt-in)
  int test_withhold_flag = -1;          // rocs_test_withhold_ikbo_flag: flag never published (-1: none)
  long long test_flag_budget = 0;       // ... and the flag-wait budget in SM cycles (0: the default ~1 s)
  cudaStream_t capture_stream = nullptr;   // forward graphs are captured here (never the legacy stream)
  std::vector<ForwardGraph> graphs;     // at most kMaxForwardGraphs, most recent last
};

constexpr size_t kMaxForwardGraphs = 8;

namespace rocs {

// The handle whose API call is running on this thread, and the call-site label that prefixes
// kernel names in the timing report; set by the entry points in api.cpp.
extern thread_local rocs_context* g_ctx;
extern thread_local const char* g_site;

struct SiteLabel {
  const char* prev;
  explicit SiteLabel(const char* site) : prev(g_site) { g_site = site; }
  ~SiteLabel() { g_site = prev; }
};

// Records start/stop events around one kernel launch on `s` when timing is enabled.
struct LaunchTimer {
  rocs_context* ctx;
  cudaStream_t s;
  long long idx = -1;
  LaunchTimer(const char* kernel, cudaStream_t stream) : ctx(g_ctx), s(stream) {
    if (!ctx || !ctx->timer.enabled) return;
    RocsTimer& t = ctx->timer;
    if (2 * (t.next + 1) > t.pool.size()) {
      ++t.dropped;
      return;
    }
    idx = (long long)t.next++;
    t.labels.push_back(std::string(g_site ? g_site : "api") + ":" + kernel);
    cudaEventRecord(t.pool[2 * idx], s);
  }
  ~LaunchTimer() {
    if (idx >= 0) cudaEventRecord(ctx->timer.pool[2 * idx + 1], s);
  }
};

void set_error(const char* fmt, ...);
rocs_status cuda_check(cudaError_t e, const char* what);
// Host validation of an IKBO linear's descriptor (dims, dtypes, activation); error messages are
// prefixed with `who`, the entry point's name.
rocs_status check_ikbo_desc(const rocs_ikbo_desc* d, const char* who);

// One GEMM problem for the tcgen05 kernel:
//   out[r, c] = act( scale[c] * sum_k A[r, k] * B[c, k] + bias[c] + Z[gidx[r], c] )
// A [M, K] bf16 (row stride lda), B [N, K] bf16 (row stride ldb); bias, Z, gidx optional.
// split_a: A rows hold a hi/lo pair [hi (K) | lo (K)] of one fp32-precise activation
//   (K % 64 == 0); the kernel accumulates hi*B + lo*B.
// out_mode: 0 fp32, 1 bf16, 2 bf16 hi/lo pair (row [hi (N) | lo (N)], ldo >= 2N).
struct GemmDesc {
  const void* A = nullptr; long long lda = 0; int M = 0; int K = 0; int split_a = 0;
  const void* B = nullptr; long long ldb = 0; int N = 0;
  const float* bias = nullptr;
  const float* scale = nullptr;   // per-column factor on the accumulator, before bias and Z
  const float* Z = nullptr; long long ldz = 0; const int32_t* gidx = nullptr; int gidx_bound = 0;
  void* out = nullptr; long long ldo = 0; int out_mode = 1; int act = ROCS_ACT_NONE;
  // One launch for a request GEMM and the candidate GEMM that gathers its output (the IKBO
  // mega-kernel): flag_role 1 marks the problem writing Z (it publishes each finished tile in
  // `flags`, zeroed by the caller before the launch, ceil(M / 128) * ceil(N / BN) ints); flag_role 2
  // marks the problem reading that Z through gidx (same flags, same N).  The launch is then
  // cooperative, so every CTA is resident and the request tiles, first in every CTA's order,
  // always finish.
  int* flags = nullptr; int flag_role = 0;
};

constexpr int kMaxGemmProblems = 4;

// Launches one persistent grouped GEMM over `nprob` problems (<= kMaxGemmProblems).
// Requirements (checked): K % 8 == 0, lda/ldb % 8 == 0, A/B 16-byte aligned, M, N, K >= 1.
rocs_status launch_gemm_bf16(rocs_context* ctx, const GemmDesc* probs, int nprob, cudaStream_t s);

// fp32 SIMT GEMM with the same epilogue (exact-order FFMA, used by the fp32 IKBO path).
rocs_status launch_gemm_f32(rocs_context* ctx, const float* A, long long lda, int M, int K, const float* B,
                            long long ldb, int N, const float* bias, const float* Z, long long ldz,
                            const int32_t* gidx, int gidx_bound, float* out, long long ldo, int act,
                            cudaStream_t s);

// FP8-weight (W8A16) linears (w8.cu).  Q: E4M3 bytes [rows, cols]; scale: one float per row.
rocs_status launch_w8_quantize(const void* W, int w_bf16, int rows, int cols, uint8_t* Q, float* scale,
                               cudaStream_t s);
// E4M3 -> bf16, exact (count even)
rocs_status launch_w8_expand(const uint8_t* Q, long long count, void* out, cudaStream_t s);
bool w8_skinny_supported(int M, int K);
// FP8-weight GEMM on the tensor cores (w8_tc.cu):
//   out[r, c] = act(2^shift[r] * scale[c] * sum_k Xh[r, k] q[c, k] + bias[c] + Z[gidx[r], c])
// Xh [M, K] f16 with row shifts from launch_w8_xprep, q [N, K] E4M3 bytes (16-byte aligned),
// K % 64 == 0.  Up to three problems share one persistent launch (problem-major tile order).
struct W8GemmDesc {
  const void* Xh = nullptr; long long ldx = 0; const int* shift = nullptr; int M = 0; int K = 0;
  const uint8_t* W8 = nullptr; int N = 0;
  const float* scale = nullptr; const float* bias = nullptr;
  const float* Z = nullptr; long long ldz = 0; const int32_t* gidx = nullptr; int gidx_bound = 0;
  void* out = nullptr; long long ldo = 0; int out_bf16 = 1; int act = ROCS_ACT_NONE;
};
bool w8_tc_supported(int K, int N);
rocs_status launch_gemm_w8(rocs_context* ctx, const W8GemmDesc* probs, int nprob, cudaStream_t s);
// X [M, K] bf16 (row stride ldx) -> Xh [M, K] f16 times 2^-shift[m], the operand of launch_w8_skinny;
// two activation sets in one launch (M1 may be 0)
rocs_status launch_w8_xprep(const void* X0, long long ldx0, int M0, int K0, void* Xh0, int* sh0, const void* X1,
                            long long ldx1, int M1, int K1, void* Xh1, int* sh1, cudaStream_t s);
// out[r, c] = act(scale[c] * sum_k X[r, k] q[c, k] + bias[c] + Z[gidx[r], c]) for M <= 64 rows, from
// the prepared Xh and shift
rocs_status launch_w8_skinny(rocs_context* ctx, const void* Xh, const int* shift, int M, int K, const uint8_t* W8,
                             int N, const float* scale, const float* bias, const float* Z, long long ldz,
                             const int32_t* gidx, int gidx_bound, void* out, long long ldo, int out_bf16, int act,
                             cudaStream_t s);

// Stable counting sort of candidates by request index (sort.cu).  perm[k] = the candidate at
// sorted position k; offsets[r] = first position of request r, offsets[B_R] = valid candidates
// (an index outside [0, B_R) sorts last and sets ROCS_ERR_INDEX).  H: plan_sort(...).h_ints ints.
struct SortPlan {
  int chunk = 0, nchunks = 0;
  long long h_ints = 0;
};
SortPlan plan_sort(int B_R, long long B_C);
rocs_status launch_sort_by_request(rocs_context* ctx, const int32_t* req_idx, int B_R, long long B_C, int32_t* perm,
                                   int32_t* offsets, int32_t* H, cudaStream_t s);
// order[k] = the request of rank k by descending query count offsets[r+1] - offsets[r] (ties by
// index), for B_R <= kRequestOrderMax.  Launching a request-per-CTA kernel in this order puts the
// longest CTAs first, so the shortest ones fill the last wave.
constexpr int kRequestOrderMax = 2048;
rocs_status launch_request_order(const int32_t* offsets, int B_R, int32_t* order, cudaStream_t s);
// dst[k] = src[perm[k]] for k < n (rows of row_bytes, a multiple of 16; 16-byte aligned rows)
rocs_status launch_gather_rows(const void* src, long long ld_src_bytes, const int32_t* perm, long long n,
                               int row_bytes, void* dst, long long ld_dst_bytes, cudaStream_t s);
// dst[perm[k]] = src[k] for k < min(n, *count) (rows of row_bytes, a multiple of 4)
rocs_status launch_scatter_rows(const void* src, long long ld_src_bytes, const int32_t* perm, const int32_t* count,
                                long long n, int row_bytes, void* dst, long long ld_dst_bytes, cudaStream_t s);

rocs_status launch_segments(rocs_context* ctx, const int32_t* counts, int B_R, int32_t* offsets,
                            int32_t* req_idx, long long B_C, cudaStream_t s);

rocs_status launch_iota(int32_t* out, int n, int step, cudaStream_t s);

// Copies a [rows, cols] matrix (row stride ld_src elements, 2 or 4 bytes each) into a
// zero-padded [rows, ld_dst] buffer.
rocs_status launch_pad_rows(const void* src, long long ld_src, void* dst, long long ld_dst, long long rows,
                            int cols, int elem_bytes, cudaStream_t s);

// in_f32: X1, X2 are fp32 (else bf16); res_f32: the residual is fp32 (else bf16).  Y is fp32 or
// bf16 (y_bf16); Y2 (optional) gets a second, bf16 copy of the output with row stride ldy2.
rocs_status launch_layernorm(rocs_context* ctx, const void* X1, int w1, long long ld1, const void* X2, int w2,
                             long long ld2, const void* res, long long ldr, long long rows, const float* gamma,
                             const float* beta, float eps, void* Y, long long ldy, int in_f32, int res_f32,
                             int y_bf16, void* Y2, long long ldy2, cudaStream_t s);

rocs_status launch_convert_bf16_f32(const void* src, long long ld_src, float* dst, long long ld_dst, long long rows,
                                    int cols, cudaStream_t s);

// Output modes shared by the FM / token-LCB / LN kernels: 0 fp32, 1 bf16, 2 bf16 hi/lo pair.
rocs_status launch_fm(rocs_context* ctx, const void* E_R, const void* E_C, const int32_t* req_idx, int B_R,
                      long long B_C, int n_R, int n_C, int D, void* F_R, void* F_C, int in_f32, int out_mode,
                      cudaStream_t s);

// One pass over the candidates' embeddings (D = 128): masked-FM products as bf16 hi/lo pairs, the
// token LCB output L_C (fp32, o_C tokens, Z^L from the request side) and, if tC is non-NULL, the
// one-token query-generator LCB (hi/lo pairs, Z^Q from the request side).
// Whether the fused pass takes this layer (D 128, n_C <= 16, 1 <= o_C <= 8, and its shared
// memory, which grows with n_R and with fp32 embeddings, fits).
bool glm_cand_fused_fits(int D, int n_R, int n_C, int o_C, int in_f32);
rocs_status launch_glm_cand_fused(rocs_context* ctx, const void* E_R, const void* E_C, const int32_t* req_idx,
                                  int B_R, long long B_C, int n_R, int n_C, int in_f32, void* F_C, const void* P_CC,
                                  int o_C, const float* ZL, float* L_C, const void* q_pCC, const float* ZQ, void* tC,
                                  cudaStream_t s);

rocs_status launch_token_lcb(rocs_context* ctx, const void* E_R, long long ld_ER, const void* E_C,
                             long long ld_EC, const int32_t* req_idx, int B_R, long long B_C, int n_R, int n_C,
                             int D, const void* P_RR, const void* P_CR, const void* P_CC, int o_R, int o_C,
                             void* L_R, long long ld_LR, void* L_C, long long ld_LC, int in_f32, int out_mode,
                             long long lo_R, long long lo_C, float* ws_Z, cudaStream_t s);

// q_split: Q rows hold [hi (H*d_h) | lo (H*d_h)] (ldq covers both).  O in fp32 or bf16 (out_bf16);
// O2 (optional) receives a bf16 copy with row stride ldo2.
rocs_status launch_attention(rocs_context* ctx, const void* Q, long long ldq, int q_split, const void* K,
                             const void* V, long long ldkv, long long kv_req_stride, const int32_t* offsets, int B_R,
                             long long rows, int L, int H, int d_h, float scale, void* O, long long ldo,
                             int out_bf16, void* O2, long long ldo2, cudaStream_t s, const int32_t* kv_len = nullptr,
                             int q_by_kv = 0);

// Same contract as launch_attention.  _stream: K/V streamed through a small shared-memory ring
// (any number of query rows per request); _single: one query row per request (a few at most),
// K/V read straight from HBM (L <= 1024).
rocs_status launch_attention_stream(rocs_context* ctx, const void* Q, long long ldq, int q_split, const void* K,
                                    const void* V, long long ldkv, long long kv_req_stride, const int32_t* offsets,
                                    int B_R, long long rows, int L, int H, int d_h, float scale, void* O,
                                    long long ldo, int out_bf16, void* O2, long long ldo2, cudaStream_t s,
                                    const int32_t* kv_len = nullptr, int q_by_kv = 0);
rocs_status launch_attention_single(rocs_context* ctx, const void* Q, long long ldq, int q_split, const void* K,
                                    const void* V, long long ldkv, long long kv_req_stride, const int32_t* offsets,
                                    int B_R, long long rows, int L, int H, int d_h, float scale, void* O,
                                    long long ldo, int out_bf16, void* O2, long long ldo2, cudaStream_t s,
                                    const int32_t* kv_len = nullptr);

// tcgen05/TMEM attention (one CTA per (request, head), K/V resident in shared memory): d_h 32
// (L <= 1024) or 64 (L <= 256 with hi/lo queries, 512 without).  kv_rows = rows of K/V (B_R * L).
// Returns ROCS_ERR_UNSUPPORTED, launching nothing, for shapes outside that range.
// Request query's cross-attention with K^R = S W_K^R and V^R = S W_V^R absorbed into the query and
// the output (one query per request; Q rows are bf16 hi/lo pairs [hi (d) | lo (d)]).
bool attention_req_absorbed_supported(int d, int H, int L);
rocs_status launch_attention_req_absorbed(rocs_context* ctx, const void* Q, long long ldq, const void* S,
                                          const void* WK, const void* WV, int B_R, int L, int d, int H, float scale,
                                          float* O, long long ldo, void* O2, long long ldo2, cudaStream_t s,
                                          const int32_t* kv_len, void* scratch);
// bytes of device scratch (256-byte aligned) the absorbed request attention needs for B_R requests
// of up to L history rows: the k' pairs and the per-split softmax states
size_t attention_req_absorbed_scratch(int B_R, int L);
rocs_status launch_attention_tc(rocs_context* ctx, const void* Q, long long ldq, int q_split, const void* K,
                                const void* V, long long ldkv, long long kv_rows, const int32_t* offsets, int B_R,
                                long long rows, int L, int H, int d_h, float scale, void* O, long long ldo,
                                int out_bf16, void* O2, long long ldo2, cudaStream_t s,
                                const int32_t* out_rows = nullptr, const int32_t* kv_len = nullptr,
                                int q_by_kv = 0, const int32_t* order = nullptr);

// Exponentials per second of the attention softmax's per-score steps with n_poly of every eight
// pairs on the FMA-pipe polynomial (probe.cu); synchronises s.
rocs_status probe_exp2_rate(rocs_context* ctx, int n_poly, double* rate, cudaStream_t s);

rocs_status launch_score_head(const void* X, long long ldx, long long rows, int K, const void* w,
                              const float* b, float* out, cudaStream_t s);

}  // namespace rocs
