// librocs C ABI: argument validation, workspace planning and launch sequencing.  Every
// arithmetic step runs in the CUDA kernels of this directory; this file only checks arguments,
// carves the caller's workspace and enqueues launches on the caller's stream.
#include <cuda_runtime.h>

#include <algorithm>
#include <cmath>
#include <cstdarg>
#include <cstdio>
#include <cstring>
#include <queue>
#include <string>
#include <vector>

#include "internal.h"

namespace rocs {

static thread_local std::string g_last_error;
thread_local rocs_context* g_ctx = nullptr;
thread_local const char* g_site = nullptr;

struct CtxGuard {
  rocs_context* prev;
  explicit CtxGuard(rocs_context* h) : prev(g_ctx) { g_ctx = h; }
  ~CtxGuard() { g_ctx = prev; }
};

void set_error(const char* fmt, ...) {
  char buf[512];
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(buf, sizeof(buf), fmt, ap);
  va_end(ap);
  g_last_error = buf;
}

rocs_status cuda_check(cudaError_t e, const char* what) {
  if (e == cudaSuccess) return ROCS_OK;
  set_error("%s: %s", what, cudaGetErrorString(e));
  return ROCS_ERR_CUDA;
}

namespace {

#define ROCS_TRY(x)                     \
  do {                                  \
    rocs_status _st = (x);              \
    if (_st != ROCS_OK) return _st;     \
  } while (0)

#define ROCS_REQUIRE(cond, ...)             \
  do {                                      \
    if (!(cond)) {                          \
      set_error(__VA_ARGS__);               \
      return ROCS_ERR_INVALID_ARG;          \
    }                                       \
  } while (0)

inline bool aligned16(const void* p) { return ((uintptr_t)p & 15) == 0; }
inline long long round_up(long long x, long long a) { return (x + a - 1) / a * a; }

// Bump allocator over the caller's workspace; with base == nullptr it only measures.
struct Carver {
  char* base;
  size_t used = 0;
  explicit Carver(void* b) : base((char*)b) {}
  void* take(size_t bytes) {
    used = (size_t)round_up((long long)used, 256);
    void* p = base ? base + used : nullptr;
    used += bytes;
    return p;
  }
};

// ------------------------------------------------------------------------------------------
// IKBO linear, bf16 tensor-core path (two launches: request GEMM, candidate GEMM + gather).
// ------------------------------------------------------------------------------------------
struct IkboArgs {
  int B_R; long long B_C; int dRi, dCi, dRo, dCo;
  const void* X_R; long long ldxr;
  const void* X_C; long long ldxc;
  const int32_t* req_idx;
  const void *W_RR, *W_CR, *W_CC;
  const float *b_R, *b_C;
  void* Y_R; long long ldyr;
  void* Y_C; long long ldyc;
  int out_mode; int act;     // 0 fp32, 1 bf16, 2 bf16 hi/lo pair
  int split_in = 0;          // X_R / X_C rows hold [hi (d_in) | lo (d_in)]
  float* Z;   // [B_R, dCo] fp32 scratch
  int* flags = nullptr;      // ikbo_flag_ints(B_R, dCo) ints: request and candidate GEMMs in one launch
  const float *s_RR = nullptr, *s_CR = nullptr, *s_CC = nullptr;   // per-output-channel accumulator scales
};

// Completion flags of one fused IKBO launch: one int per (128-request block, 32-column block), an
// upper bound on the request GEMM's tiles for any tile width.
long long ikbo_flag_ints(long long B_R, long long dCo) { return ((B_R + 127) / 128) * ((dCo + 31) / 32); }

rocs_status ikbo_bf16(rocs_context* ctx, const IkboArgs& a, cudaStream_t s) {
  GemmDesc req[3];
  int nreq = 0;
  if (a.dRo > 0) {
    GemmDesc& g = req[nreq++];
    g.A = a.X_R; g.lda = a.ldxr; g.M = a.B_R; g.K = a.dRi; g.split_a = a.split_in;
    g.B = a.W_RR; g.ldb = a.dRi; g.N = a.dRo;
    g.bias = a.b_R; g.scale = a.s_RR; g.out = a.Y_R; g.ldo = a.ldyr; g.out_mode = a.out_mode; g.act = a.act;
  }
  {
    GemmDesc& g = req[nreq++];
    g.A = a.X_R; g.lda = a.ldxr; g.M = a.B_R; g.K = a.dRi; g.split_a = a.split_in;
    g.B = a.W_CR; g.ldb = a.dRi; g.N = a.dCo;
    g.bias = a.b_C; g.scale = a.s_CR; g.out = a.Z; g.ldo = a.dCo; g.out_mode = 0; g.act = ROCS_ACT_NONE;
  }
  // [REV] §2.4's single launch where it pays: the candidate GEMM's tiles are long (K >= 1024, a
  // split operand counting twice), or there are few of them (a separate request launch is then a
  // large share).  At short K with many candidates the candidate epilogue is the bottleneck, and
  // the fused form's wait for the first Z tiles costs more than the launch it saves.
  const long long keff = (long long)a.dCi * (a.split_in ? 2 : 1);
  const bool fuse = a.B_C > 0 && a.flags != nullptr && ctx->ikbo_fused && (keff >= 1024 || a.B_C <= 32768);
  if (fuse) {
    // request GEMMs' tiles first, then the candidate tiles, whose epilogues wait for the Z tiles
    // they gather (completion flags, zeroed here)
    GemmDesc& z = req[nreq - 1];
    z.flags = a.flags; z.flag_role = 1;
    GemmDesc& g = req[nreq++];
    g.A = a.X_C; g.lda = a.ldxc; g.M = (int)a.B_C; g.K = a.dCi; g.split_a = a.split_in;
    g.B = a.W_CC; g.ldb = a.dCi; g.N = a.dCo;
    g.Z = a.Z; g.ldz = a.dCo; g.gidx = a.req_idx; g.gidx_bound = a.B_R; g.scale = a.s_CC;
    g.out = a.Y_C; g.ldo = a.ldyc; g.out_mode = a.out_mode; g.act = a.act;
    g.flags = a.flags; g.flag_role = 2;
    std::string site = std::string(g_site ? g_site : "ikbo") + ".ikbo";
    SiteLabel sl(site.c_str());
    ROCS_TRY(cuda_check(cudaMemsetAsync(a.flags, 0, (size_t)ikbo_flag_ints(a.B_R, a.dCo) * 4, s), "zero IKBO flags"));
    return launch_gemm_bf16(ctx, req, nreq, s);
  }
  {
    std::string site = std::string(g_site ? g_site : "ikbo") + ".req";
    SiteLabel sl(site.c_str());
    ROCS_TRY(launch_gemm_bf16(ctx, req, nreq, s));
  }
  if (a.B_C > 0) {
    std::string site = std::string(g_site ? g_site : "ikbo") + ".cand";
    SiteLabel sl(site.c_str());
    GemmDesc g;
    g.A = a.X_C; g.lda = a.ldxc; g.M = (int)a.B_C; g.K = a.dCi; g.split_a = a.split_in;
    g.B = a.W_CC; g.ldb = a.dCi; g.N = a.dCo;
    g.Z = a.Z; g.ldz = a.dCo; g.gidx = a.req_idx; g.gidx_bound = a.B_R; g.scale = a.s_CC;
    g.out = a.Y_C; g.ldo = a.ldyc; g.out_mode = a.out_mode; g.act = a.act;
    ROCS_TRY(launch_gemm_bf16(ctx, &g, 1, s));
  }
  return ROCS_OK;
}

// Plain candidate-side GEMM (no request group): out = act(X W^T + b).
rocs_status linear_bf16(rocs_context* ctx, const void* X, long long ldx, long long M, int K, const void* W, int N,
                        const float* b, void* out, long long ldo, int out_mode, int act, cudaStream_t s) {
  if (M == 0) return ROCS_OK;
  GemmDesc g;
  g.A = X; g.lda = ldx; g.M = (int)M; g.K = K;
  g.B = W; g.ldb = K; g.N = N;
  g.bias = b; g.out = out; g.ldo = ldo; g.out_mode = out_mode; g.act = act;
  return launch_gemm_bf16(ctx, &g, 1, s);
}

// Attention against per-request K/V: the tcgen05 kernel where its shared memory holds the
// request's K/V, else the streaming (cross) or resident (self) mma.sync kernels.
// kv_len (nullable): request r's keys are the first kv_len[r] of its L rows (a ragged history);
// q_by_kv: its query rows too (a self-attention over the ragged history).  Histories too long to
// stage in shared memory take the streaming kernel.
rocs_status attention_best(rocs_context* ctx, bool streaming_fallback, const void* Q, long long ldq, int q_split,
                           const void* K, const void* V, long long ldkv, const int32_t* offsets, int B_R,
                           long long rows, int L, int H, int d_h, float scale, void* O, long long ldo, int out_bf16,
                           void* O2, long long ldo2, cudaStream_t s, const int32_t* kv_len = nullptr,
                           int q_by_kv = 0, const int32_t* order = nullptr) {
  rocs_status st = launch_attention_tc(ctx, Q, ldq, q_split, K, V, ldkv, (long long)B_R * L, offsets, B_R, rows, L, H,
                                       d_h, scale, O, ldo, out_bf16, O2, ldo2, s, nullptr, kv_len, q_by_kv, order);
  if (st != ROCS_ERR_UNSUPPORTED) return st;
  if (!streaming_fallback) {
    st = launch_attention(ctx, Q, ldq, q_split, K, V, ldkv, (long long)L * ldkv, offsets, B_R, rows, L, H, d_h, scale,
                          O, ldo, out_bf16, O2, ldo2, s, kv_len, q_by_kv);
    if (st != ROCS_ERR_UNSUPPORTED) return st;
  }
  return launch_attention_stream(ctx, Q, ldq, q_split, K, V, ldkv, (long long)L * ldkv, offsets, B_R, rows, L, H,
                                 d_h, scale, O, ldo, out_bf16, O2, ldo2, s, kv_len, q_by_kv);
}

// Workspace of rocs_linear_ikbo: Z, then (only if a row is not 16-B aligned) padded operands.
struct IkboPlan {
  float* Z = nullptr;
  int* flags = nullptr;
  void *XR = nullptr, *XC = nullptr, *WRR = nullptr, *WCR = nullptr, *WCC = nullptr;
  int kR = 0, kC = 0;   // padded K
  bool padR = false, padC = false;
  size_t bytes = 0;
};

IkboPlan plan_ikbo(const rocs_ikbo_desc* d, void* ws) {
  IkboPlan p;
  Carver c(ws);
  p.Z = (float*)c.take((size_t)d->B_R * d->d_C_out * 4);
  if (d->dtype_in == ROCS_BF16 && d->B_C > 0) p.flags = (int*)c.take((size_t)ikbo_flag_ints(d->B_R, d->d_C_out) * 4);
  if (d->dtype_in == ROCS_BF16) {
    p.padR = (d->d_R_in % 8) != 0;
    p.padC = (d->d_C_in % 8) != 0;
    p.kR = (int)round_up(d->d_R_in, 8);
    p.kC = (int)round_up(d->d_C_in, 8);
    if (p.padR) {
      p.XR = c.take((size_t)d->B_R * p.kR * 2);
      if (d->d_R_out > 0) p.WRR = c.take((size_t)d->d_R_out * p.kR * 2);
      p.WCR = c.take((size_t)d->d_C_out * p.kR * 2);
    }
    if (p.padC) {
      p.XC = c.take((size_t)d->B_C * p.kC * 2);
      p.WCC = c.take((size_t)d->d_C_out * p.kC * 2);
    }
  }
  p.bytes = c.used;
  return p;
}

rocs_status check_ikbo_desc(const rocs_ikbo_desc* d) { return rocs::check_ikbo_desc(d, "rocs_linear_ikbo"); }

}  // namespace

rocs_status check_ikbo_desc(const rocs_ikbo_desc* d, const char* who) {
  ROCS_REQUIRE(d != nullptr, "%s: desc is NULL", who);
  ROCS_REQUIRE(d->B_R >= 1, "%s: B_R=%d must be >= 1", who, d->B_R);
  ROCS_REQUIRE(d->B_C >= 0 && d->B_C < 2147483647LL, "%s: B_C=%lld out of range", who, (long long)d->B_C);
  ROCS_REQUIRE(d->d_R_in >= 1 && d->d_C_in >= 1 && d->d_C_out >= 1 && d->d_R_out >= 0,
               "%s: dims must be positive (d_R_out may be 0)", who);
  ROCS_REQUIRE(d->dtype_in == ROCS_F32 || d->dtype_in == ROCS_BF16, "%s: bad dtype_in", who);
  ROCS_REQUIRE(d->dtype_out == ROCS_F32 || d->dtype_out == ROCS_BF16, "%s: bad dtype_out", who);
  ROCS_REQUIRE(!(d->dtype_in == ROCS_F32 && d->dtype_out != ROCS_F32), "%s: the fp32 path writes fp32 outputs", who);
  ROCS_REQUIRE(d->act >= ROCS_ACT_NONE && d->act <= ROCS_ACT_SIGMOID, "%s: bad act", who);
  return ROCS_OK;
}

}  // namespace rocs

using namespace rocs;

// =============================================================================================
// handle
// =============================================================================================
extern "C" rocs_status rocs_create(rocs_handle_t* handle, int device) {
  ROCS_REQUIRE(handle != nullptr, "rocs_create: handle is NULL");
  *handle = nullptr;
  int prev = 0;
  ROCS_TRY(cuda_check(cudaGetDevice(&prev), "cudaGetDevice"));
  ROCS_TRY(cuda_check(cudaSetDevice(device), "cudaSetDevice"));
  rocs_context* ctx = new (std::nothrow) rocs_context();
  if (!ctx) {
    set_error("rocs_create: out of host memory");
    cudaSetDevice(prev);
    return ROCS_ERR_CUDA;
  }
  ctx->device = device;
  rocs_status st = ROCS_OK;
  cudaDeviceProp prop;
  st = cuda_check(cudaGetDeviceProperties(&prop, device), "cudaGetDeviceProperties");
  if (st == ROCS_OK && prop.major < 10) {
    set_error("rocs_create: device %d is sm_%d%d; librocs is built for sm_100a", device, prop.major, prop.minor);
    st = ROCS_ERR_UNSUPPORTED;
  }
  if (st == ROCS_OK) {
    ctx->num_sms = prop.multiProcessorCount;
    st = cuda_check(cudaMalloc(&ctx->d_status, sizeof(int)), "cudaMalloc(status)");
  }
  if (st == ROCS_OK) st = cuda_check(cudaMemset(ctx->d_status, 0, sizeof(int)), "cudaMemset(status)");
  if (st == ROCS_OK) {
    cudaDriverEntryPointQueryResult q;
    st = cuda_check(cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ctx->encode_fn, cudaEnableDefault, &q),
                    "cudaGetDriverEntryPoint(cuTensorMapEncodeTiled)");
    if (st == ROCS_OK && (q != cudaDriverEntryPointSuccess || !ctx->encode_fn)) {
      set_error("rocs_create: cuTensorMapEncodeTiled not available");
      st = ROCS_ERR_UNSUPPORTED;
    }
  }
  cudaSetDevice(prev);
  if (st != ROCS_OK) {
    if (ctx->d_status) cudaFree(ctx->d_status);
    delete ctx;
    return st;
  }
  *handle = ctx;
  return ROCS_OK;
}

extern "C" rocs_status rocs_destroy(rocs_handle_t h) {
  if (!h) return ROCS_OK;
  cudaDeviceSynchronize();
  for (ForwardGraph& g : h->graphs)
    if (g.exec) cudaGraphExecDestroy(g.exec);
  if (h->capture_stream) cudaStreamDestroy(h->capture_stream);
  if (h->d_status) cudaFree(h->d_status);
  delete h;
  return ROCS_OK;
}

extern "C" const char* rocs_last_error(void) { return g_last_error.c_str(); }

extern "C" int32_t rocs_num_sms(rocs_handle_t h) { return h ? h->num_sms : 0; }

extern "C" rocs_status rocs_get_device_status(rocs_handle_t h, void* stream, int32_t* code) {
  ROCS_REQUIRE(h && code, "rocs_get_device_status: NULL argument");
  ROCS_TRY(cuda_check(cudaStreamSynchronize((cudaStream_t)stream), "cudaStreamSynchronize"));
  int v = 0;
  ROCS_TRY(cuda_check(cudaMemcpy(&v, h->d_status, sizeof(int), cudaMemcpyDeviceToHost), "read status"));
  ROCS_TRY(cuda_check(cudaMemset(h->d_status, 0, sizeof(int)), "clear status"));
  *code = v;
  return ROCS_OK;
}

// =============================================================================================
// Multi-GPU sharding: whole requests per part, longest processing time first
// =============================================================================================
extern "C" rocs_status rocs_partition_requests(const int32_t* counts, int32_t B_R, int32_t n_parts, double cost_R,
                                               double cost_C, int32_t* part_of) {
  ROCS_REQUIRE(counts && part_of, "rocs_partition_requests: NULL argument");
  ROCS_REQUIRE(B_R >= 1 && B_R <= (1 << 24), "rocs_partition_requests: B_R out of range");
  ROCS_REQUIRE(n_parts >= 1 && n_parts <= 4096, "rocs_partition_requests: n_parts out of range");
  ROCS_REQUIRE(std::isfinite(cost_R) && std::isfinite(cost_C) && cost_R >= 0 && cost_C >= 0 &&
                   (cost_R > 0 || cost_C > 0),
               "rocs_partition_requests: costs must be finite, >= 0 and not both 0");
  for (int32_t r = 0; r < B_R; ++r) ROCS_REQUIRE(counts[r] >= 0, "rocs_partition_requests: negative count");
  std::vector<int32_t> idx(B_R);
  for (int32_t r = 0; r < B_R; ++r) idx[r] = r;
  // decreasing work; equal work keeps index order
  std::stable_sort(idx.begin(), idx.end(), [&](int32_t a, int32_t b) { return counts[a] > counts[b]; });
  // least-loaded part first, ties to the lower part
  using Slot = std::pair<double, int32_t>;
  std::priority_queue<Slot, std::vector<Slot>, std::greater<Slot>> parts;
  for (int32_t p = 0; p < n_parts; ++p) parts.push({0.0, p});
  for (int32_t r : idx) {
    Slot s = parts.top();
    parts.pop();
    part_of[r] = s.second;
    s.first += cost_R + cost_C * (double)counts[r];
    parts.push(s);
  }
  return ROCS_OK;
}

// =============================================================================================
// a0
// =============================================================================================
extern "C" rocs_status rocs_segments_from_counts(rocs_handle_t h, const int32_t* counts, int32_t B_R,
                                                 int32_t* offsets, int32_t* req_idx, int64_t B_C, void* stream) {
  CtxGuard ctx_guard_(h);
  ROCS_REQUIRE(h, "rocs_segments_from_counts: handle is NULL");
  ROCS_REQUIRE(counts && offsets, "rocs_segments_from_counts: counts/offsets NULL");
  ROCS_REQUIRE(B_R >= 1 && B_R <= (1 << 24), "rocs_segments_from_counts: B_R=%d out of range", B_R);
  ROCS_REQUIRE(B_C >= 0 && B_C < 2147483647LL, "rocs_segments_from_counts: B_C out of range");
  ROCS_REQUIRE(B_C == 0 || req_idx, "rocs_segments_from_counts: req_idx NULL");
  return launch_segments(h, counts, B_R, offsets, req_idx, B_C, (cudaStream_t)stream);
}

// =============================================================================================
// a1-a3
// =============================================================================================
extern "C" rocs_status rocs_linear_ikbo_workspace(rocs_handle_t h, const rocs_ikbo_desc* d, size_t* bytes) {
  ROCS_REQUIRE(h && bytes, "rocs_linear_ikbo_workspace: NULL argument");
  ROCS_TRY(check_ikbo_desc(d));
  *bytes = plan_ikbo(d, nullptr).bytes;
  return ROCS_OK;
}

extern "C" rocs_status rocs_linear_ikbo(rocs_handle_t h, const rocs_ikbo_desc* d, const void* X_R, const void* X_C,
                                        const int32_t* req_idx, const void* W_RR, const void* W_CR,
                                        const void* W_CC, const float* b_R, const float* b_C, void* Y_R, void* Y_C,
                                        void* ws, size_t ws_bytes, void* stream) {
  CtxGuard ctx_guard_(h);
  ROCS_REQUIRE(h, "rocs_linear_ikbo: handle is NULL");
  ROCS_TRY(check_ikbo_desc(d));
  ROCS_REQUIRE(X_R && W_CR && b_C, "rocs_linear_ikbo: X_R, W_CR, b_C must be non-NULL");
  ROCS_REQUIRE(d->d_R_out == 0 || (W_RR && b_R && Y_R), "rocs_linear_ikbo: W_RR, b_R, Y_R needed when d_R_out > 0");
  ROCS_REQUIRE(d->B_C == 0 || (X_C && W_CC && req_idx && Y_C), "rocs_linear_ikbo: candidate pointers NULL");
  const void* ptrs[] = {X_R, X_C, W_RR, W_CR, W_CC, b_R, b_C, Y_R, Y_C, ws};
  for (const void* p : ptrs) ROCS_REQUIRE(aligned16(p), "rocs_linear_ikbo: pointers must be 16-byte aligned");
  IkboPlan need = plan_ikbo(d, nullptr);
  if (ws == nullptr || ws_bytes < need.bytes) {
    set_error("rocs_linear_ikbo: workspace %zu B < required %zu B", ws_bytes, need.bytes);
    return ROCS_ERR_WORKSPACE;
  }
  IkboPlan p = plan_ikbo(d, ws);
  cudaStream_t s = (cudaStream_t)stream;
  if (d->dtype_in == ROCS_F32) {
    if (d->d_R_out > 0)
      ROCS_TRY(launch_gemm_f32(h, (const float*)X_R, d->d_R_in, d->B_R, d->d_R_in, (const float*)W_RR, d->d_R_in,
                               d->d_R_out, b_R, nullptr, 0, nullptr, 0, (float*)Y_R, d->d_R_out, d->act, s));
    ROCS_TRY(launch_gemm_f32(h, (const float*)X_R, d->d_R_in, d->B_R, d->d_R_in, (const float*)W_CR, d->d_R_in,
                             d->d_C_out, b_C, nullptr, 0, nullptr, 0, p.Z, d->d_C_out, ROCS_ACT_NONE, s));
    if (d->B_C > 0)
      ROCS_TRY(launch_gemm_f32(h, (const float*)X_C, d->d_C_in, (int)d->B_C, d->d_C_in, (const float*)W_CC,
                               d->d_C_in, d->d_C_out, nullptr, p.Z, d->d_C_out, req_idx, d->B_R, (float*)Y_C,
                               d->d_C_out, d->act, s));
    return ROCS_OK;
  }
  IkboArgs a;
  a.B_R = d->B_R; a.B_C = d->B_C; a.dRi = d->d_R_in; a.dCi = d->d_C_in; a.dRo = d->d_R_out; a.dCo = d->d_C_out;
  a.X_R = X_R; a.ldxr = d->d_R_in; a.X_C = X_C; a.ldxc = d->d_C_in; a.req_idx = req_idx;
  a.W_RR = W_RR; a.W_CR = W_CR; a.W_CC = W_CC; a.b_R = b_R; a.b_C = b_C;
  a.Y_R = Y_R; a.ldyr = d->d_R_out; a.Y_C = Y_C; a.ldyc = d->d_C_out;
  a.out_mode = d->dtype_out == ROCS_BF16 ? 1 : 0; a.act = d->act; a.Z = p.Z; a.flags = p.flags;
  // a1: alignment fix -- zero-pad K of any operand pair whose rows are not 16-byte multiples.
  if (p.padR) {
    ROCS_TRY(launch_pad_rows(X_R, d->d_R_in, p.XR, p.kR, d->B_R, d->d_R_in, 2, s));
    if (d->d_R_out > 0) ROCS_TRY(launch_pad_rows(W_RR, d->d_R_in, p.WRR, p.kR, d->d_R_out, d->d_R_in, 2, s));
    ROCS_TRY(launch_pad_rows(W_CR, d->d_R_in, p.WCR, p.kR, d->d_C_out, d->d_R_in, 2, s));
    a.X_R = p.XR; a.ldxr = p.kR; a.W_RR = p.WRR; a.W_CR = p.WCR; a.dRi = p.kR;
  }
  if (p.padC && d->B_C > 0) {
    ROCS_TRY(launch_pad_rows(X_C, d->d_C_in, p.XC, p.kC, d->B_C, d->d_C_in, 2, s));
    ROCS_TRY(launch_pad_rows(W_CC, d->d_C_in, p.WCC, p.kC, d->d_C_out, d->d_C_in, 2, s));
    a.X_C = p.XC; a.ldxc = p.kC; a.W_CC = p.WCC; a.dCi = p.kC;
  }
  return ikbo_bf16(h, a, s);
}

// =============================================================================================
// FP8-weight (W8A16) IKBO linear
// =============================================================================================
namespace rocs {
namespace {

struct W8Plan {
  float* Z = nullptr;
  int* flags = nullptr;
  void *WRR = nullptr, *WCR = nullptr, *WCC = nullptr;   // bf16 expansions (large-M paths only)
  void *XhR = nullptr, *XhC = nullptr;                    // f16 activations (weight-streaming paths only)
  int *shR = nullptr, *shC = nullptr;
  bool req_skinny = false, cand_skinny = false;
  bool tc = false;   // the FP8-weight tcgen05 GEMM on both sides (input widths multiples of 64)
  size_t bytes = 0;
};

W8Plan plan_w8(const rocs_context* h, const rocs_ikbo_desc* d, void* ws) {
  W8Plan p;
  Carver c(ws);
  p.tc = h->w8_tensor_cores && w8_tc_supported(d->d_R_in, d->d_C_out) && w8_tc_supported(d->d_C_in, d->d_C_out);
  if (p.tc) {
    p.Z = (float*)c.take((size_t)d->B_R * d->d_C_out * 4);
    p.XhR = c.take((size_t)d->B_R * d->d_R_in * 2);
    p.shR = (int*)c.take((size_t)d->B_R * 4);
    if (d->B_C > 0) {
      p.XhC = c.take((size_t)d->B_C * d->d_C_in * 2);
      p.shC = (int*)c.take((size_t)d->B_C * 4);
    }
    p.bytes = c.used;
    return p;
  }
  p.req_skinny = w8_skinny_supported(d->B_R, d->d_R_in);
  p.cand_skinny = d->B_C == 0 || w8_skinny_supported((int)d->B_C, d->d_C_in);
  p.Z = (float*)c.take((size_t)d->B_R * d->d_C_out * 4);
  if (!p.cand_skinny) p.flags = (int*)c.take((size_t)ikbo_flag_ints(d->B_R, d->d_C_out) * 4);
  if (!p.req_skinny) {
    if (d->d_R_out > 0) p.WRR = c.take((size_t)d->d_R_out * d->d_R_in * 2);
    p.WCR = c.take((size_t)d->d_C_out * d->d_R_in * 2);
  }
  if (!p.cand_skinny) p.WCC = c.take((size_t)d->d_C_out * d->d_C_in * 2);
  if (p.req_skinny) {
    p.XhR = c.take((size_t)d->B_R * d->d_R_in * 2);
    p.shR = (int*)c.take((size_t)d->B_R * 4);
  }
  if (p.cand_skinny && d->B_C > 0) {
    p.XhC = c.take((size_t)d->B_C * d->d_C_in * 2);
    p.shC = (int*)c.take((size_t)d->B_C * 4);
  }
  p.bytes = c.used;
  return p;
}

rocs_status check_w8_desc(const rocs_ikbo_desc* d) {
  ROCS_TRY(check_ikbo_desc(d));
  ROCS_REQUIRE(d->dtype_in == ROCS_BF16, "rocs_linear_ikbo_w8: activations must be bf16");
  ROCS_REQUIRE(d->d_R_in % 8 == 0 && d->d_C_in % 8 == 0, "rocs_linear_ikbo_w8: d_R_in and d_C_in must be multiples of 8");
  return ROCS_OK;
}

}  // namespace
}  // namespace rocs

extern "C" rocs_status rocs_quantize_weights_fp8(rocs_handle_t h, const void* W, rocs_dtype w_dtype, int32_t rows,
                                                 int32_t cols, uint8_t* Q, float* scale, void* stream) {
  CtxGuard ctx_guard_(h);
  ROCS_REQUIRE(h, "rocs_quantize_weights_fp8: handle is NULL");
  ROCS_REQUIRE(rows >= 0 && cols >= 0, "rocs_quantize_weights_fp8: negative size");
  ROCS_REQUIRE(w_dtype == ROCS_F32 || w_dtype == ROCS_BF16, "rocs_quantize_weights_fp8: bad dtype");
  ROCS_REQUIRE(rows == 0 || cols == 0 || (W && Q && scale), "rocs_quantize_weights_fp8: NULL argument");
  return launch_w8_quantize(W, w_dtype == ROCS_BF16, rows, cols, Q, scale, (cudaStream_t)stream);
}

extern "C" rocs_status rocs_linear_ikbo_w8_workspace(rocs_handle_t h, const rocs_ikbo_desc* d, size_t* bytes) {
  ROCS_REQUIRE(h && bytes, "rocs_linear_ikbo_w8_workspace: NULL argument");
  ROCS_TRY(check_w8_desc(d));
  *bytes = plan_w8(h, d, nullptr).bytes;
  return ROCS_OK;
}

extern "C" rocs_status rocs_linear_ikbo_w8(rocs_handle_t h, const rocs_ikbo_desc* d, const void* X_R,
                                           const void* X_C, const int32_t* req_idx, const uint8_t* Q_RR,
                                           const uint8_t* Q_CR, const uint8_t* Q_CC, const float* s_RR,
                                           const float* s_CR, const float* s_CC, const float* b_R, const float* b_C,
                                           void* Y_R, void* Y_C, void* ws, size_t ws_bytes, void* stream) {
  CtxGuard ctx_guard_(h);
  ROCS_REQUIRE(h, "rocs_linear_ikbo_w8: handle is NULL");
  ROCS_TRY(check_w8_desc(d));
  ROCS_REQUIRE(X_R && Q_CR && s_CR && b_C, "rocs_linear_ikbo_w8: X_R, Q_CR, s_CR, b_C must be non-NULL");
  ROCS_REQUIRE(d->d_R_out == 0 || (Q_RR && s_RR && b_R && Y_R),
               "rocs_linear_ikbo_w8: Q_RR, s_RR, b_R, Y_R needed when d_R_out > 0");
  ROCS_REQUIRE(d->B_C == 0 || (X_C && Q_CC && s_CC && req_idx && Y_C), "rocs_linear_ikbo_w8: candidate pointers NULL");
  const void* ptrs[] = {X_R, X_C, Y_R, Y_C, ws};
  for (const void* p : ptrs) ROCS_REQUIRE(aligned16(p), "rocs_linear_ikbo_w8: X, Y and workspace must be 16-byte aligned");
  const void* wq[] = {Q_RR, Q_CR, Q_CC};
  for (const void* p : wq) ROCS_REQUIRE(((uintptr_t)p & 7) == 0, "rocs_linear_ikbo_w8: weights must be 8-byte aligned");
  const W8Plan need = plan_w8(h, d, nullptr);
  if (ws_bytes < need.bytes) {
    set_error("rocs_linear_ikbo_w8: workspace %zu B < required %zu B", ws_bytes, need.bytes);
    return ROCS_ERR_WORKSPACE;
  }
  const W8Plan p = plan_w8(h, d, ws);
  cudaStream_t s = (cudaStream_t)stream;
  const int out_bf16 = d->dtype_out == ROCS_BF16;
  if (p.tc) {
    // FP8 weights straight to the tensor cores: activations to f16 once (both sides, one launch),
    // then [Y^R | Z] in one launch and the candidate GEMM with the Z[m] gather in a second
    for (const void* q : wq)
      ROCS_REQUIRE(((uintptr_t)q & 15) == 0, "rocs_linear_ikbo_w8: weights must be 16-byte aligned");
    {
      SiteLabel sl("ikbo_w8");
      ROCS_TRY(launch_w8_xprep(X_R, d->d_R_in, d->B_R, d->d_R_in, p.XhR, p.shR, X_C, d->d_C_in, (int)d->B_C,
                               d->d_C_in, p.XhC, p.shC, s));
    }
    W8GemmDesc req[2];
    int nreq = 0;
    if (d->d_R_out > 0) {
      W8GemmDesc& g = req[nreq++];
      g.Xh = p.XhR; g.ldx = d->d_R_in; g.shift = p.shR; g.M = d->B_R; g.K = d->d_R_in;
      g.W8 = Q_RR; g.N = d->d_R_out; g.scale = s_RR; g.bias = b_R;
      g.out = Y_R; g.ldo = d->d_R_out; g.out_bf16 = out_bf16; g.act = d->act;
    }
    {
      W8GemmDesc& g = req[nreq++];
      g.Xh = p.XhR; g.ldx = d->d_R_in; g.shift = p.shR; g.M = d->B_R; g.K = d->d_R_in;
      g.W8 = Q_CR; g.N = d->d_C_out; g.scale = s_CR; g.bias = b_C;
      g.out = p.Z; g.ldo = d->d_C_out; g.out_bf16 = 0; g.act = ROCS_ACT_NONE;
    }
    {
      SiteLabel sl("ikbo_w8.req");
      ROCS_TRY(launch_gemm_w8(h, req, nreq, s));
    }
    if (d->B_C == 0) return ROCS_OK;
    W8GemmDesc g;
    g.Xh = p.XhC; g.ldx = d->d_C_in; g.shift = p.shC; g.M = (int)d->B_C; g.K = d->d_C_in;
    g.W8 = Q_CC; g.N = d->d_C_out; g.scale = s_CC;
    g.Z = p.Z; g.ldz = d->d_C_out; g.gidx = req_idx; g.gidx_bound = d->B_R;
    g.out = Y_C; g.ldo = d->d_C_out; g.out_bf16 = out_bf16; g.act = d->act;
    SiteLabel sl("ikbo_w8.cand");
    return launch_gemm_w8(h, &g, 1, s);
  }
  // request side: weight-streaming kernel at small B_R, else the bf16 expansion and the tcgen05
  // GEMM (both with the channel scales on the accumulator)
  IkboArgs a;
  a.B_R = d->B_R; a.B_C = d->B_C; a.dRi = d->d_R_in; a.dCi = d->d_C_in; a.dRo = d->d_R_out; a.dCo = d->d_C_out;
  a.X_R = X_R; a.ldxr = d->d_R_in; a.X_C = X_C; a.ldxc = d->d_C_in; a.req_idx = req_idx;
  a.b_R = b_R; a.b_C = b_C; a.Y_R = Y_R; a.ldyr = d->d_R_out; a.Y_C = Y_C; a.ldyc = d->d_C_out;
  a.out_mode = out_bf16 ? 1 : 0; a.act = d->act; a.Z = p.Z; a.flags = p.flags;
  a.s_RR = s_RR; a.s_CR = s_CR; a.s_CC = s_CC;
  {
    // both sides' activations as f16 operands of the weight-streaming kernel, in one launch
    const bool prepR = p.req_skinny, prepC = p.cand_skinny && d->B_C > 0;
    SiteLabel sl("ikbo_w8");
    if (prepR && prepC)
      ROCS_TRY(launch_w8_xprep(X_R, d->d_R_in, d->B_R, d->d_R_in, p.XhR, p.shR, X_C, d->d_C_in, (int)d->B_C,
                               d->d_C_in, p.XhC, p.shC, s));
    else if (prepR)
      ROCS_TRY(launch_w8_xprep(X_R, d->d_R_in, d->B_R, d->d_R_in, p.XhR, p.shR, nullptr, 0, 0, 0, nullptr, nullptr, s));
    else if (prepC)
      ROCS_TRY(launch_w8_xprep(X_C, d->d_C_in, (int)d->B_C, d->d_C_in, p.XhC, p.shC, nullptr, 0, 0, 0, nullptr, nullptr,
                               s));
  }
  if (p.req_skinny) {
    SiteLabel sl("ikbo_w8.req");
    if (d->d_R_out > 0)
      ROCS_TRY(launch_w8_skinny(h, p.XhR, p.shR, d->B_R, d->d_R_in, Q_RR, d->d_R_out, s_RR, b_R, nullptr, 0, nullptr,
                                0, Y_R, d->d_R_out, out_bf16, d->act, s));
    ROCS_TRY(launch_w8_skinny(h, p.XhR, p.shR, d->B_R, d->d_R_in, Q_CR, d->d_C_out, s_CR, b_C, nullptr, 0, nullptr, 0,
                              p.Z, d->d_C_out, 0, ROCS_ACT_NONE, s));
  } else {
    if (d->d_R_out > 0) ROCS_TRY(launch_w8_expand(Q_RR, (long long)d->d_R_out * d->d_R_in, p.WRR, s));
    ROCS_TRY(launch_w8_expand(Q_CR, (long long)d->d_C_out * d->d_R_in, p.WCR, s));
  }
  if (d->B_C > 0 && p.cand_skinny) {
    if (!p.req_skinny) {   // the request GEMMs alone (the candidate side does not run on tcgen05)
      IkboArgs r = a;
      r.B_C = 0; r.W_RR = p.WRR; r.W_CR = p.WCR;
      SiteLabel sl("ikbo_w8");
      ROCS_TRY(ikbo_bf16(h, r, s));
    }
    SiteLabel sl("ikbo_w8.cand");
    return launch_w8_skinny(h, p.XhC, p.shC, (int)d->B_C, d->d_C_in, Q_CC, d->d_C_out, s_CC, nullptr, p.Z,
                            d->d_C_out, req_idx, d->B_R, Y_C, d->d_C_out, out_bf16, d->act, s);
  }
  if (d->B_C > 0) ROCS_TRY(launch_w8_expand(Q_CC, (long long)d->d_C_out * d->d_C_in, p.WCC, s));
  if (p.req_skinny) {
    if (d->B_C == 0) return ROCS_OK;
    // request outputs exist; the candidate GEMM alone on tcgen05 (no request problems in it)
    GemmDesc g;
    g.A = X_C; g.lda = d->d_C_in; g.M = (int)d->B_C; g.K = d->d_C_in;
    g.B = p.WCC; g.ldb = d->d_C_in; g.N = d->d_C_out;
    g.Z = p.Z; g.ldz = d->d_C_out; g.gidx = req_idx; g.gidx_bound = d->B_R; g.scale = s_CC;
    g.out = Y_C; g.ldo = d->d_C_out; g.out_mode = out_bf16 ? 1 : 0; g.act = d->act;
    SiteLabel sl("ikbo_w8.cand");
    return launch_gemm_bf16(h, &g, 1, s);
  }
  a.W_RR = p.WRR; a.W_CR = p.WCR; a.W_CC = p.WCC;
  SiteLabel sl("ikbo_w8");
  return ikbo_bf16(h, a, s);
}

// =============================================================================================
// a6
// =============================================================================================
extern "C" rocs_status rocs_group_layernorm(rocs_handle_t h, const void* X1, int32_t w1, const void* X2, int32_t w2,
                                            const void* residual, int64_t rows, const float* gamma, const float* beta,
                                            float eps, void* Y, rocs_dtype io, void* stream) {
  CtxGuard ctx_guard_(h);
  ROCS_REQUIRE(h, "rocs_group_layernorm: handle is NULL");
  ROCS_REQUIRE(X1 && gamma && beta && Y, "rocs_group_layernorm: NULL argument");
  ROCS_REQUIRE(w1 >= 1 && w2 >= 0 && w1 + w2 <= 8192, "rocs_group_layernorm: widths w1=%d w2=%d unsupported", w1, w2);
  ROCS_REQUIRE(w2 == 0 || X2, "rocs_group_layernorm: X2 NULL with w2 > 0");
  ROCS_REQUIRE(rows >= 0, "rocs_group_layernorm: rows < 0");
  ROCS_REQUIRE(io == ROCS_F32 || io == ROCS_BF16, "rocs_group_layernorm: bad dtype");
  ROCS_REQUIRE(eps > 0.f, "rocs_group_layernorm: eps must be > 0");
  const int f32 = io == ROCS_F32;
  return launch_layernorm(h, X1, w1, w1, w2 ? X2 : nullptr, w2, w2, residual, w1 + w2, rows, gamma, beta, eps, Y,
                          w1 + w2, f32, f32, !f32, nullptr, 0, (cudaStream_t)stream);
}

// =============================================================================================
// a4
// =============================================================================================
extern "C" rocs_status rocs_fm_masked(rocs_handle_t h, const void* E_R, const void* E_C, const int32_t* req_idx,
                                      int32_t B_R, int64_t B_C, int32_t n_R, int32_t n_C, int32_t D, void* F_R,
                                      void* F_C, rocs_dtype out, void* stream) {
  CtxGuard ctx_guard_(h);
  ROCS_REQUIRE(h, "rocs_fm_masked: handle is NULL");
  ROCS_REQUIRE(E_R && (B_C == 0 || (E_C && req_idx && F_C)), "rocs_fm_masked: NULL argument");
  ROCS_REQUIRE(B_R >= 1 && B_C >= 0 && B_C < 2147483647LL, "rocs_fm_masked: bad batch sizes");
  ROCS_REQUIRE(n_R >= 1 && n_C >= 1 && n_R + n_C <= 64, "rocs_fm_masked: n_R + n_C must be <= 64");
  ROCS_REQUIRE(D >= 16 && D <= 256 && D % 16 == 0, "rocs_fm_masked: D=%d must be a multiple of 16 in [16, 256]", D);
  ROCS_REQUIRE(aligned16(E_R) && aligned16(E_C), "rocs_fm_masked: inputs must be 16-byte aligned");
  ROCS_REQUIRE(out == ROCS_F32 || out == ROCS_BF16, "rocs_fm_masked: bad dtype");
  return launch_fm(h, E_R, E_C, req_idx, B_R, B_C, n_R, n_C, D, F_R, F_C, 0, out == ROCS_BF16 ? 1 : 0,
                   (cudaStream_t)stream);
}

extern "C" rocs_status rocs_token_lcb_workspace(rocs_handle_t h, int32_t B_R, int32_t o_C, int32_t D, size_t* bytes) {
  ROCS_REQUIRE(h && bytes, "rocs_token_lcb_workspace: NULL argument");
  *bytes = (size_t)B_R * o_C * D * 4;
  return ROCS_OK;
}

extern "C" rocs_status rocs_token_lcb(rocs_handle_t h, const void* E_R, const void* E_C, const int32_t* req_idx,
                                      int32_t B_R, int64_t B_C, int32_t n_R, int32_t n_C, int32_t D,
                                      const void* P_RR, const void* P_CR, const void* P_CC, int32_t o_R, int32_t o_C,
                                      void* L_R, int64_t ld_LR, void* L_C, int64_t ld_LC, rocs_dtype out, void* ws,
                                      size_t ws_bytes, void* stream) {
  CtxGuard ctx_guard_(h);
  ROCS_REQUIRE(h, "rocs_token_lcb: handle is NULL");
  ROCS_REQUIRE(B_R >= 1 && B_C >= 0 && n_R >= 1 && n_C >= 1 && D >= 1 && D <= 256, "rocs_token_lcb: bad sizes");
  ROCS_REQUIRE(o_R >= 0 && o_C >= 1 && o_C <= 8 && n_C <= 64, "rocs_token_lcb: need 1 <= o_C <= 8, n_C <= 64");
  ROCS_REQUIRE(E_R && P_CR && P_CC && (o_R == 0 || (P_RR && L_R)) && (B_C == 0 || (E_C && req_idx && L_C)),
               "rocs_token_lcb: NULL argument");
  ROCS_REQUIRE(ld_LR >= (int64_t)o_R * D && ld_LC >= (int64_t)o_C * D, "rocs_token_lcb: output strides too small");
  ROCS_REQUIRE(out == ROCS_F32 || out == ROCS_BF16, "rocs_token_lcb: bad dtype");
  const size_t need = (size_t)B_R * o_C * D * 4;
  if (!ws || ws_bytes < need) {
    set_error("rocs_token_lcb: workspace %zu B < required %zu B", ws_bytes, need);
    return ROCS_ERR_WORKSPACE;
  }
  return launch_token_lcb(h, E_R, (long long)n_R * D, E_C, (long long)n_C * D, req_idx, B_R, B_C, n_R, n_C, D, P_RR,
                          P_CR, P_CC, o_R, o_C, L_R, ld_LR, L_C, ld_LC, 0, out == ROCS_BF16 ? 1 : 0, 0, 0, (float*)ws,
                          (cudaStream_t)stream);
}

// =============================================================================================
// a9
// =============================================================================================
extern "C" rocs_status rocs_dca_cross_attn(rocs_handle_t h, const void* Q, const void* K, const void* V,
                                           const int32_t* offsets, int32_t B_R, int64_t rows, int32_t L, int32_t H,
                                           int32_t d_h, float scale, void* O, int64_t ld_O, rocs_dtype out,
                                           const int32_t* kv_len, void* stream) {
  CtxGuard ctx_guard_(h);
  ROCS_REQUIRE(h, "rocs_dca_cross_attn: handle is NULL");
  ROCS_REQUIRE(Q && K && V && offsets && O, "rocs_dca_cross_attn: NULL argument");
  ROCS_REQUIRE(B_R >= 1 && rows >= 0 && L >= 1 && H >= 1, "rocs_dca_cross_attn: bad sizes");
  ROCS_REQUIRE(d_h == 32 || d_h == 64, "rocs_dca_cross_attn: d_h=%d (32 or 64 supported)", d_h);
  ROCS_REQUIRE((long long)B_R * L < 2147483647LL, "rocs_dca_cross_attn: B_R*L too large");
  ROCS_REQUIRE(ld_O >= (int64_t)H * d_h && ld_O % 2 == 0, "rocs_dca_cross_attn: ld_O too small or odd");
  ROCS_REQUIRE(aligned16(Q) && aligned16(K) && aligned16(V) && aligned16(O), "rocs_dca_cross_attn: misaligned");
  ROCS_REQUIRE(out == ROCS_F32 || out == ROCS_BF16, "rocs_dca_cross_attn: bad dtype");
  ROCS_REQUIRE(std::isfinite(scale), "rocs_dca_cross_attn: scale not finite");
  const long long dm = (long long)H * d_h;
  return attention_best(h, true, Q, dm, 0, K, V, dm, offsets, B_R, rows, L, H, d_h, scale, O, ld_O, out == ROCS_BF16,
                        nullptr, 0, (cudaStream_t)stream, kv_len);
}

// =============================================================================================
// candidates in any order: stable sort by request, and the cross-attention over it
// =============================================================================================
namespace rocs {
namespace {

struct UnsortedPlan {
  int32_t *perm = nullptr, *offsets = nullptr, *H = nullptr, *order = nullptr;
  void *Qs = nullptr, *Os = nullptr;
  size_t bytes = 0;
};

UnsortedPlan plan_unsorted(int B_R, long long rows, long long qrow_bytes, long long orow_bytes, void* ws) {
  UnsortedPlan p;
  Carver c(ws);
  p.perm = (int32_t*)c.take((size_t)rows * 4 + 4);
  p.offsets = (int32_t*)c.take((size_t)(B_R + 1) * 4);
  p.H = (int32_t*)c.take((size_t)plan_sort(B_R, rows).h_ints * 4 + 4);
  if (B_R <= kRequestOrderMax) p.order = (int32_t*)c.take((size_t)B_R * 4);
  if (qrow_bytes > 0) {
    p.Qs = c.take((size_t)(rows * qrow_bytes) + 16);
    p.Os = c.take((size_t)(rows * orow_bytes) + 16);
  }
  p.bytes = c.used;
  return p;
}

}  // namespace
}  // namespace rocs

extern "C" rocs_status rocs_sort_by_request_workspace(rocs_handle_t h, int32_t B_R, int64_t B_C, size_t* bytes) {
  ROCS_REQUIRE(h && bytes, "rocs_sort_by_request_workspace: NULL argument");
  ROCS_REQUIRE(B_R >= 1 && B_R <= (1 << 24) && B_C >= 0 && B_C < 2147483647LL,
               "rocs_sort_by_request_workspace: B_R=%d B_C=%lld out of range", B_R, (long long)B_C);
  Carver c(nullptr);
  c.take((size_t)plan_sort(B_R, B_C).h_ints * 4 + 4);
  *bytes = c.used;
  return ROCS_OK;
}

extern "C" rocs_status rocs_sort_by_request(rocs_handle_t h, const int32_t* req_idx, int32_t B_R, int64_t B_C,
                                            int32_t* perm, int32_t* offsets, void* ws, size_t ws_bytes,
                                            void* stream) {
  CtxGuard ctx_guard_(h);
  ROCS_REQUIRE(h, "rocs_sort_by_request: handle is NULL");
  ROCS_REQUIRE(B_R >= 1 && B_R <= (1 << 24) && B_C >= 0 && B_C < 2147483647LL,
               "rocs_sort_by_request: B_R=%d B_C=%lld out of range", B_R, (long long)B_C);
  ROCS_REQUIRE(offsets && (B_C == 0 || (req_idx && perm && ws)), "rocs_sort_by_request: NULL argument");
  size_t need = 0;
  ROCS_TRY(rocs_sort_by_request_workspace(h, B_R, B_C, &need));
  if (B_C > 0 && ws_bytes < need) {
    set_error("rocs_sort_by_request: workspace %zu B < required %zu B", ws_bytes, need);
    return ROCS_ERR_WORKSPACE;
  }
  return launch_sort_by_request(h, req_idx, B_R, B_C, perm, offsets, (int32_t*)ws, (cudaStream_t)stream);
}

extern "C" rocs_status rocs_dca_cross_attn_unsorted_workspace(rocs_handle_t h, int32_t B_R, int64_t rows, int32_t H,
                                                              int32_t d_h, rocs_dtype out, size_t* bytes) {
  ROCS_REQUIRE(h && bytes, "rocs_dca_cross_attn_unsorted_workspace: NULL argument");
  ROCS_REQUIRE(B_R >= 1 && B_R <= (1 << 24) && rows >= 0 && rows < 2147483647LL && H >= 1 && d_h >= 1,
               "rocs_dca_cross_attn_unsorted_workspace: bad sizes");
  ROCS_REQUIRE(out == ROCS_F32 || out == ROCS_BF16, "rocs_dca_cross_attn_unsorted_workspace: bad dtype");
  const long long dm = (long long)H * d_h;
  *bytes = plan_unsorted(B_R, rows, dm * 2, dm * (out == ROCS_BF16 ? 2 : 4), nullptr).bytes;
  return ROCS_OK;
}

extern "C" rocs_status rocs_dca_cross_attn_unsorted(rocs_handle_t h, const void* Q, const void* K, const void* V,
                                                    const int32_t* req_idx, int32_t B_R, int64_t rows, int32_t L,
                                                    int32_t H, int32_t d_h, float scale, void* O, int64_t ld_O,
                                                    rocs_dtype out, const int32_t* kv_len, void* ws, size_t ws_bytes,
                                                    void* stream) {
  CtxGuard ctx_guard_(h);
  ROCS_REQUIRE(h, "rocs_dca_cross_attn_unsorted: handle is NULL");
  ROCS_REQUIRE(Q && K && V && O && (rows == 0 || (req_idx && ws)), "rocs_dca_cross_attn_unsorted: NULL argument");
  ROCS_REQUIRE(B_R >= 1 && B_R <= (1 << 24) && rows >= 0 && rows < 2147483647LL && L >= 1 && H >= 1,
               "rocs_dca_cross_attn_unsorted: bad sizes");
  ROCS_REQUIRE(d_h == 32 || d_h == 64, "rocs_dca_cross_attn_unsorted: d_h=%d (32 or 64 supported)", d_h);
  ROCS_REQUIRE((long long)B_R * L < 2147483647LL, "rocs_dca_cross_attn_unsorted: B_R*L too large");
  ROCS_REQUIRE(ld_O >= (int64_t)H * d_h && ld_O % 2 == 0, "rocs_dca_cross_attn_unsorted: ld_O too small or odd");
  ROCS_REQUIRE(aligned16(Q) && aligned16(K) && aligned16(V) && aligned16(O) && aligned16(ws),
               "rocs_dca_cross_attn_unsorted: misaligned");
  ROCS_REQUIRE(out == ROCS_F32 || out == ROCS_BF16, "rocs_dca_cross_attn_unsorted: bad dtype");
  ROCS_REQUIRE(std::isfinite(scale), "rocs_dca_cross_attn_unsorted: scale not finite");
  if (rows == 0) return ROCS_OK;
  const long long dm = (long long)H * d_h;
  const int es = out == ROCS_BF16 ? 2 : 4;
  const UnsortedPlan need = plan_unsorted(B_R, rows, dm * 2, dm * es, nullptr);
  if (ws_bytes < need.bytes) {
    set_error("rocs_dca_cross_attn_unsorted: workspace %zu B < required %zu B", ws_bytes, need.bytes);
    return ROCS_ERR_WORKSPACE;
  }
  const UnsortedPlan p = plan_unsorted(B_R, rows, dm * 2, dm * es, ws);
  cudaStream_t s = (cudaStream_t)stream;
  // sort by request (stable), gather the query rows into that order, attend on the segment path,
  // and write every valid row at the caller's position
  ROCS_TRY(launch_sort_by_request(h, req_idx, B_R, rows, p.perm, p.offsets, p.H, s));
  if (p.order != nullptr) ROCS_TRY(launch_request_order(p.offsets, B_R, p.order, s));
  ROCS_TRY(launch_gather_rows(Q, dm * 2, p.perm, rows, (int)(dm * 2), p.Qs, dm * 2, s));
  // the tcgen05 kernel writes each row straight to its caller position (out_rows = perm); the
  // other kernels write the grouped order, which is then scattered
  const rocs_status st = launch_attention_tc(h, p.Qs, dm, 0, K, V, dm, (long long)B_R * L, p.offsets, B_R, rows, L,
                                             H, d_h, scale, O, ld_O, out == ROCS_BF16, nullptr, 0, s, p.perm, kv_len, 0,
                                             p.order);
  if (st != ROCS_ERR_UNSUPPORTED) return st;
  ROCS_TRY(attention_best(h, true, p.Qs, dm, 0, K, V, dm, p.offsets, B_R, rows, L, H, d_h, scale, p.Os, dm,
                          out == ROCS_BF16, nullptr, 0, s, kv_len, 0, p.order));
  return launch_scatter_rows(p.Os, dm * es, p.perm, p.offsets + B_R, rows, (int)(dm * es), O, ld_O * es, s);
}

// =============================================================================================
// a7
// =============================================================================================
namespace rocs {
namespace {

struct EncScratch {
  void *q, *k, *v, *att, *tmp;
  int32_t* self_off;
};

EncScratch carve_encoder(Carver& c, long long rowsL, int d, int B_R) {
  EncScratch e;
  const size_t b = (size_t)rowsL * d * 2;
  e.q = c.take(b);
  e.k = c.take(b);
  e.v = c.take(b);
  e.att = c.take(b);
  e.tmp = c.take(b);
  e.self_off = (int32_t*)c.take((size_t)(B_R + 1) * 4);
  return e;
}

// One encoder layer S_out = LN(S_in + MHSA(S_in) W_O^T) and the four K/V projections of S_out.
// lengths (nullable): request r's history is its first lengths[r] rows; the rows after them are
// padding, computed like any row by the row-wise steps (each row's LayerNorm and projections are
// independent) but neither keys nor queries of the self-attention, so nothing in them reaches a
// history row.  Their attention output is left as the workspace holds it.
rocs_status encoder_layer(rocs_context* ctx, const EncScratch& e, int B_R, int L, int d, int H,
                          const rocs_dca_layer_weights& w, const void* S_in, void* S_out, void* KR, void* VR, void* KC,
                          void* VC, cudaStream_t s, const int32_t* lengths = nullptr) {
  const long long M = (long long)B_R * L;
  GemmDesc g[4];
  const void* Ws[3] = {w.Wq, w.Wk, w.Wv};
  void* outs[3] = {e.q, e.k, e.v};
  for (int i = 0; i < 3; ++i) {
    g[i] = GemmDesc();
    g[i].A = S_in; g[i].lda = d; g[i].M = (int)M; g[i].K = d;
    g[i].B = Ws[i]; g[i].ldb = d; g[i].N = d;
    g[i].out = outs[i]; g[i].ldo = d; g[i].out_mode = 1;
  }
  SiteLabel sl0("enc.qkv");
  ROCS_TRY(launch_gemm_bf16(ctx, g, 3, s));
  SiteLabel sl1("enc.attn");
  ROCS_TRY(attention_best(ctx, false, e.q, d, 0, e.k, e.v, d, e.self_off, B_R, M, L, H, d / H,
                          1.0f / std::sqrt((float)(d / H)), e.att, d, 1, nullptr, 0, s, lengths, 1));
  SiteLabel sl2("enc.wo");
  ROCS_TRY(linear_bf16(ctx, e.att, d, M, d, w.Wo, d, nullptr, e.tmp, d, 1, ROCS_ACT_NONE, s));
  SiteLabel sl3("enc.ln");
  ROCS_TRY(launch_layernorm(ctx, e.tmp, d, d, nullptr, 0, 0, S_in, d, M, w.ln_gamma, w.ln_beta, 1e-5f, S_out, d, 0, 0,
                            1, nullptr, 0, s));
  SiteLabel sl4("enc.kv");
  // KR/VR NULL: only the candidate group's K/V (the request query's attention absorbs its
  // projections, see attn_req.cu)
  const bool req_kv = KR != nullptr && VR != nullptr;
  const void* Wk[4] = {w.WK_C, w.WV_C, w.WK_R, w.WV_R};
  void* kv[4] = {KC, VC, KR, VR};
  const int nkv = req_kv ? 4 : 2;
  for (int i = 0; i < nkv; ++i) {
    g[i] = GemmDesc();
    g[i].A = S_out; g[i].lda = d; g[i].M = (int)M; g[i].K = d;
    g[i].B = Wk[i]; g[i].ldb = d; g[i].N = d;
    g[i].out = kv[i]; g[i].ldo = d; g[i].out_mode = 1;
  }
  return launch_gemm_bf16(ctx, g, nkv, s);
}

rocs_status check_dca_desc(const rocs_dca_desc* d) {
  ROCS_REQUIRE(d, "dca: desc NULL");
  ROCS_REQUIRE(d->B_R >= 1 && d->L >= 1 && d->d >= 16 && d->H >= 1 && d->d % d->H == 0,
               "dca: bad sizes B_R=%d L=%d d=%d H=%d", d->B_R, d->L, d->d, d->H);
  ROCS_REQUIRE(d->layers >= 1 && d->layers <= ROCS_MAX_LAYERS, "dca: layers=%d out of range", d->layers);
  const int dh = d->d / d->H;
  ROCS_REQUIRE(dh == 32 || dh == 64, "dca: head width %d (32 or 64 supported)", dh);
  ROCS_REQUIRE(d->d % 8 == 0 && d->d <= 8192, "dca: d must be a multiple of 8");
  ROCS_REQUIRE((long long)d->B_R * d->L < 2147483647LL, "dca: B_R*L too large");
  return ROCS_OK;
}

}  // namespace
}  // namespace rocs

extern "C" rocs_status rocs_dca_encode_workspace(rocs_handle_t h, const rocs_dca_desc* d, size_t* bytes) {
  ROCS_REQUIRE(h && bytes, "rocs_dca_encode_workspace: NULL argument");
  ROCS_TRY(check_dca_desc(d));
  Carver c(nullptr);
  carve_encoder(c, (long long)d->B_R * d->L, d->d, d->B_R);
  *bytes = c.used;
  return ROCS_OK;
}

extern "C" rocs_status rocs_dca_encode(rocs_handle_t h, const rocs_dca_desc* d, const void* Hist,
                                       const int32_t* lengths, const rocs_dca_layer_weights* w, void* S, void* KV,
                                       void* ws, size_t ws_bytes, void* stream) {
  CtxGuard ctx_guard_(h);
  ROCS_REQUIRE(h, "rocs_dca_encode: handle is NULL");
  ROCS_TRY(check_dca_desc(d));
  ROCS_REQUIRE(Hist && w && S && KV, "rocs_dca_encode: NULL argument");
  for (int l = 0; l < d->layers; ++l) {
    const rocs_dca_layer_weights& x = w[l];
    ROCS_REQUIRE(x.Wq && x.Wk && x.Wv && x.Wo && x.ln_gamma && x.ln_beta && x.WK_R && x.WV_R && x.WK_C && x.WV_C,
                 "rocs_dca_encode: layer %d has a NULL weight", l);
  }
  Carver need(nullptr);
  carve_encoder(need, (long long)d->B_R * d->L, d->d, d->B_R);
  if (!ws || ws_bytes < need.used) {
    set_error("rocs_dca_encode: workspace %zu B < required %zu B", ws_bytes, need.used);
    return ROCS_ERR_WORKSPACE;
  }
  Carver c(ws);
  EncScratch e = carve_encoder(c, (long long)d->B_R * d->L, d->d, d->B_R);
  cudaStream_t s = (cudaStream_t)stream;
  ROCS_TRY(launch_iota(e.self_off, d->B_R + 1, d->L, s));
  const size_t per = (size_t)d->B_R * d->L * d->d * 2;
  const void* cur = Hist;
  for (int l = 0; l < d->layers; ++l) {
    char* Sl = (char*)S + per * l;
    char* kv = (char*)KV + per * 4 * l;
    ROCS_TRY(encoder_layer(h, e, d->B_R, d->L, d->d, d->H, w[l], cur, Sl, kv, kv + per, kv + 2 * per, kv + 3 * per, s,
                           lengths));
    cur = Sl;
  }
  return ROCS_OK;
}

// =============================================================================================
// a0-a11: whole forward
// =============================================================================================
namespace rocs {
namespace {

// Precision layout of the forward (bf16 tensor-core arithmetic, fp32 accumulation):
//   * activations that feed a tensor-core GEMM or the attention scores on the candidate path
//     (FM output F, MLP hidden h, query-generator t and hidden, queries Q) are stored as a bf16
//     hi/lo pair, row = [hi | lo], so the activation itself carries ~16 mantissa bits;
//   * activations no GEMM consumes (MLP output o, LCB output L, the GLM residual stream E, DCA
//     outputs A and the own-query token stream Y) are fp32;
//   * the encoder stream S, its Q/K/V and the scoring head stay plain bf16.
struct FwdPlan {
  int32_t *offsets, *req_idx, *iota1;
  // GLM (E stream fp32)
  float *ER[2], *EC[2];
  void *FR, *FC, *hR, *hC;   // hi/lo pairs
  float *oR, *oC, *LR, *LC;
  float *Z1, *Z2, *ZL;
  // DCA
  EncScratch enc;
  void *S[2], *KR = nullptr, *VR = nullptr, *KC, *VC;   // KR/VR only when the request attention is not absorbed
  void* ar_scratch = nullptr;                             // the absorbed request attention's k' and split states
  float *YR, *YC;            // own-query token streams (fp32)
  void *tR, *tC, *qhR, *qhC, *QR, *QC;   // hi/lo pairs
  float *AR, *AC;            // attention outputs when no caller buffer takes them
  float *Zq1, *Zq2, *ZqL;
  // scoring
  void *xR, *xC, *h1, *h2;
  float* Zs;
  int* ikbo_flags;   // completion flags of the fused IKBO launches (reused, zeroed by each)
  int32_t* order = nullptr;   // requests by descending candidate count (the candidate attention's CTA order)
  size_t bytes;
};

FwdPlan plan_forward(const rocs_model_desc* m, void* ws, bool own_offsets, bool own_req) {
  FwdPlan p{};
  Carver c(ws);
  const long long BR = m->B_R, BC = m->B_C;
  p.offsets = own_offsets ? (int32_t*)c.take((BR + 1) * 4) : nullptr;
  p.req_idx = own_req ? (int32_t*)c.take((size_t)BC * 4 + 4) : nullptr;
  p.iota1 = (int32_t*)c.take((BR + 1) * 4);
  {
    long long maxN = std::max<long long>({(long long)m->hidden, (long long)m->fm_out_C * m->D, (long long)m->d,
                                          (long long)m->score_h1, 1LL});
    p.ikbo_flags = (int*)c.take((size_t)ikbo_flag_ints(BR, maxN) * 4);
  }
  if (m->glm_layers > 0) {
    const long long wr = (long long)m->n_R * m->D, wc = (long long)m->n_C * m->D;
    for (int i = 0; i < 2; ++i) {
      p.ER[i] = (float*)c.take(BR * wr * 4);
      p.EC[i] = (float*)c.take(BC * wc * 4);
    }
    p.FR = c.take(BR * m->n_R * m->n_R * 2 * 2);
    p.FC = c.take(BC * (long long)m->n_C * (m->n_R + m->n_C) * 2 * 2);
    p.hR = c.take(BR * m->hidden * 2 * 2);
    p.hC = c.take(BC * m->hidden * 2 * 2);
    p.oR = (float*)c.take(BR * (long long)m->fm_out_R * m->D * 4);
    p.oC = (float*)c.take(BC * (long long)m->fm_out_C * m->D * 4);
    p.LR = (float*)c.take(BR * (long long)m->lcb_out_R * m->D * 4);
    p.LC = (float*)c.take(BC * (long long)m->lcb_out_C * m->D * 4);
    p.Z1 = (float*)c.take(BR * m->hidden * 4);
    p.Z2 = (float*)c.take(BR * (long long)m->fm_out_C * m->D * 4);
    p.ZL = (float*)c.take(BR * (long long)m->lcb_out_C * m->D * 4);
  }
  if (m->dca_layers > 0) {
    const long long rowsL = BR * m->L;
    p.enc = carve_encoder(c, rowsL, m->d, m->B_R);
    p.S[0] = c.take(rowsL * m->d * 2);
    p.S[1] = c.take(rowsL * m->d * 2);
    if (!attention_req_absorbed_supported(m->d, m->H, m->L)) {
      p.KR = c.take(rowsL * m->d * 2);
      p.VR = c.take(rowsL * m->d * 2);
    } else {
      p.ar_scratch = c.take(attention_req_absorbed_scratch(m->B_R, m->L));
    }
    if (m->B_R <= kRequestOrderMax) p.order = (int32_t*)c.take((size_t)m->B_R * 4);
    p.KC = c.take(rowsL * m->d * 2);
    p.VC = c.take(rowsL * m->d * 2);
    if (m->dca_query_source == 0) {
      p.YR = (float*)c.take(BR * (long long)(m->q_n_R + m->dca_layers) * m->q_dim * 4);
      p.YC = (float*)c.take(BC * (long long)(m->q_n_C + m->dca_layers) * m->q_dim * 4);
    }
    p.tR = c.take(BR * m->q_dim * 2 * 2);
    p.tC = c.take(BC * m->q_dim * 2 * 2);
    p.qhR = c.take(BR * m->d * 2 * 2);
    p.qhC = c.take(BC * m->d * 2 * 2);
    p.QR = c.take(BR * m->d * 2 * 2);
    p.QC = c.take(BC * m->d * 2 * 2);
    p.AR = (float*)c.take(BR * m->d * 4);
    p.AC = (float*)c.take(BC * m->d * 4);
    p.Zq1 = (float*)c.take(BR * m->d * 4);
    p.Zq2 = (float*)c.take(BR * m->d * 4);
    p.ZqL = (float*)c.take(BR * m->q_dim * 4);
  }
  if (m->score_h1 > 0) {
    const long long xr = (long long)m->n_R * m->D + (long long)m->dca_layers * m->d;
    const long long xc = (long long)m->n_C * m->D + (long long)m->dca_layers * m->d;
    p.xR = c.take(BR * xr * 2);
    p.xC = c.take(BC * xc * 2);
    p.h1 = c.take(BC * m->score_h1 * 2);
    p.h2 = c.take(BC * m->score_h2 * 2);
    p.Zs = (float*)c.take(BR * m->score_h1 * 4);
  }
  p.bytes = c.used;
  return p;
}

rocs_status check_model(const rocs_model_desc* m) {
  ROCS_REQUIRE(m, "rocs_forward: model NULL");
  ROCS_REQUIRE(m->B_R >= 1 && m->B_C >= 0 && m->B_C < 2147483647LL, "rocs_forward: bad batch sizes");
  ROCS_REQUIRE(m->glm_layers >= 0 && m->glm_layers <= ROCS_MAX_LAYERS && m->dca_layers >= 0 &&
                   m->dca_layers <= ROCS_MAX_LAYERS,
               "rocs_forward: layer counts out of range");
  ROCS_REQUIRE(m->glm_layers > 0 || m->dca_layers > 0, "rocs_forward: nothing to run");
  if (m->glm_layers > 0) {
    ROCS_REQUIRE(m->n_R >= 1 && m->n_C >= 1 && m->n_R + m->n_C <= 64, "rocs_forward: n_R + n_C must be <= 64");
    ROCS_REQUIRE(m->D % 16 == 0 && m->D >= 16 && m->D <= 256, "rocs_forward: D must be a multiple of 16 <= 256");
    ROCS_REQUIRE(m->hidden % 64 == 0 && m->hidden >= 64, "rocs_forward: hidden must be a multiple of 64");
    ROCS_REQUIRE((m->n_R * m->n_R) % 64 == 0 && (m->n_C * (m->n_R + m->n_C)) % 64 == 0,
                 "rocs_forward: FM widths n_R^2 and n_C(n_R+n_C) must be multiples of 64");
    ROCS_REQUIRE(m->fm_out_R + m->lcb_out_R == m->n_R && m->fm_out_C + m->lcb_out_C == m->n_C,
                 "rocs_forward: concat(FM-MLP tokens, LCB tokens) must give n_R | n_C tokens (residual)");
    ROCS_REQUIRE(m->lcb_out_C >= 1 && m->lcb_out_C <= 8 && m->fm_out_R >= 1 && m->fm_out_C >= 1,
                 "rocs_forward: token counts out of range");
    ROCS_REQUIRE((long long)m->n_R * m->D <= 8192 && (long long)m->n_C * m->D <= 8192,
                 "rocs_forward: group width exceeds 8192");
  }
  if (m->dca_layers > 0) {
    rocs_dca_desc dd = {m->B_R, m->L, m->d, m->H, m->dca_layers};
    ROCS_TRY(check_dca_desc(&dd));
    ROCS_REQUIRE(m->dca_query_source == 0 || m->dca_query_source == 1, "rocs_forward: bad dca_query_source");
    if (m->dca_query_source == 1) {
      ROCS_REQUIRE(m->glm_layers >= m->dca_layers - 1, "rocs_forward: DCA depth i needs GLM layer i-1");
      ROCS_REQUIRE(m->q_dim == m->D, "rocs_forward: q_dim must equal D when queries come from the GLM stack");
    } else {
      ROCS_REQUIRE(m->q_dim == m->d, "rocs_forward: own-query wiring appends attention tokens, q_dim must equal d");
      ROCS_REQUIRE(m->q_n_R >= 1 && m->q_n_C >= 1 && m->q_n_C + m->dca_layers <= 64,
                   "rocs_forward: query token counts out of range");
    }
    ROCS_REQUIRE(m->q_dim % 64 == 0 && m->q_dim <= 256, "rocs_forward: q_dim must be a multiple of 64 <= 256");
    ROCS_REQUIRE(m->d % 64 == 0, "rocs_forward: d must be a multiple of 64");
  }
  if (m->score_h1 > 0) {
    ROCS_REQUIRE(m->glm_layers > 0 && m->dca_layers > 0, "rocs_forward: scoring head needs GLM and DCA outputs");
    ROCS_REQUIRE(m->score_h1 % 8 == 0 && m->score_h2 % 8 == 0 && m->score_h2 >= 8,
                 "rocs_forward: scoring widths must be multiples of 8");
  }
  return ROCS_OK;
}

}  // namespace
}  // namespace rocs

extern "C" rocs_status rocs_forward_workspace(rocs_handle_t h, const rocs_model_desc* m, size_t* bytes) {
  ROCS_REQUIRE(h && bytes, "rocs_forward_workspace: NULL argument");
  ROCS_TRY(check_model(m));
  *bytes = plan_forward(m, nullptr, true, true).bytes;
  return ROCS_OK;
}

namespace {

// The forward's launch sequence (a0 .. a10) on stream s, after validation and planning.
rocs_status forward_launches(rocs_handle_t h, const rocs_model_desc* m, const rocs_model_weights* W,
                             const rocs_inputs* in, rocs_outputs* out, const FwdPlan& p, bool own_off, bool own_req,
                             cudaStream_t s) {
  const int BR = m->B_R;
  const long long BC = m->B_C;
  int32_t* offsets = own_off ? p.offsets : out->offsets;
  int32_t* req_idx = own_req ? p.req_idx : out->req_idx;

  // a0: segment bookkeeping
  SiteLabel site_fwd("fwd");
  ROCS_TRY(launch_segments(h, in->counts, BR, offsets, req_idx, BC, s));
  if (p.order != nullptr) ROCS_TRY(launch_request_order(offsets, BR, p.order, s));
  ROCS_TRY(launch_iota(p.iota1, BR + 1, 1, s));

  const long long wr = (long long)m->n_R * m->D, wc = (long long)m->n_C * m->D;
  const long long xr = m->score_h1 > 0 ? wr + (long long)m->dca_layers * m->d : 0;
  const long long xc = m->score_h1 > 0 ? wc + (long long)m->dca_layers * m->d : 0;
  // GLM residual stream: layer 0 reads the bf16 inputs, later layers the fp32 stream
  const void* ER = in->E_R;
  const void* EC = in->E_C;
  int e_f32 = 0;
  // own-query token streams (fp32): the inputs fill the first q_n tokens
  const long long yr_ld = (long long)(m->q_n_R + m->dca_layers) * m->q_dim;
  const long long yc_ld = (long long)(m->q_n_C + m->dca_layers) * m->q_dim;
  if (m->dca_layers > 0 && m->dca_query_source == 0) {
    SiteLabel sl("fwd.ytokens");
    ROCS_TRY(launch_convert_bf16_f32(in->Y_R, (long long)m->q_n_R * m->q_dim, p.YR, yr_ld, BR, m->q_n_R * m->q_dim, s));
    ROCS_TRY(launch_convert_bf16_f32(in->Y_C, (long long)m->q_n_C * m->q_dim, p.YC, yc_ld, BC, m->q_n_C * m->q_dim, s));
  }
  if (m->dca_layers > 0) ROCS_TRY(launch_iota(p.enc.self_off, BR + 1, m->L, s));

  const size_t S_plane = (size_t)BR * m->L * m->d * 2;
  const void* S_prev = in->Hist;
  const int steps = m->glm_layers > m->dca_layers ? m->glm_layers : m->dca_layers;
  const long long d2 = 2LL * m->d, q2 = 2LL * m->q_dim;

  for (int l = 0; l < steps; ++l) {
    const bool glm_l = l < m->glm_layers;
    const bool dca_l = l < m->dca_layers;
    const bool q_from_glm = dca_l && m->dca_query_source == 1;
    const int fR = m->n_R * m->n_R, fC = m->n_C * (m->n_R + m->n_C);
    const int lRw = m->lcb_out_R * m->D, lCw = m->lcb_out_C * m->D;
    bool t_done = false;
    // ---------------- a4: one pass over this layer's embeddings ----------------
    if (glm_l) {
      const rocs_glm_layer_weights& gw = W->glm[l];
      const rocs_qgen_weights* qw = q_from_glm ? &W->qgen[l] : nullptr;
      SiteLabel s_fm("glm.fm");
      // request side: F^R (hi/lo), L^R and Z^L, and the query generator's token for depth l
      ROCS_TRY(launch_fm(h, ER, EC, req_idx, BR, 0, m->n_R, m->n_C, m->D, p.FR, nullptr, e_f32, 2, s));
      ROCS_TRY(launch_token_lcb(h, ER, wr, EC, wc, req_idx, BR, 0, m->n_R, m->n_C, m->D, gw.P_RR, gw.P_CR, gw.P_CC,
                                m->lcb_out_R, m->lcb_out_C, p.LR, lRw, p.LC, lCw, e_f32, 0, 0, 0, p.ZL, s));
      if (qw)
        ROCS_TRY(launch_token_lcb(h, ER, wr, EC, wc, req_idx, BR, 0, m->n_R, m->n_C, m->D, qw->p_RR, qw->p_CR,
                                  qw->p_CC, 1, 1, p.tR, q2, p.tC, q2, e_f32, 2, m->q_dim, m->q_dim, p.ZqL, s));
      if (glm_cand_fused_fits(m->D, m->n_R, m->n_C, m->lcb_out_C, e_f32)) {
        // candidate side in one kernel: F^C (hi/lo), L^C and the depth-l query token t^C
        ROCS_TRY(launch_glm_cand_fused(h, ER, EC, req_idx, BR, BC, m->n_R, m->n_C, e_f32, p.FC, gw.P_CC, m->lcb_out_C,
                                       p.ZL, p.LC, qw ? qw->p_CC : nullptr, p.ZqL, qw ? p.tC : nullptr, s));
        t_done = qw != nullptr;
      } else {
        ROCS_TRY(launch_fm(h, ER, EC, req_idx, BR, BC, m->n_R, m->n_C, m->D, nullptr, p.FC, e_f32, 2, s));
        SiteLabel s_lcb("glm.lcb");
        ROCS_TRY(launch_token_lcb(h, ER, wr, EC, wc, req_idx, BR, BC, m->n_R, m->n_C, m->D, gw.P_RR, gw.P_CR,
                                  gw.P_CC, m->lcb_out_R, m->lcb_out_C, p.LR, lRw, p.LC, lCw, e_f32, 0, 0, 0, p.ZL, s));
      }
    }
    // ---------------- DCA depth l ----------------
    if (dca_l) {
      const rocs_dca_layer_weights& dw = W->dca[l];
      void* S_l = out->S ? (void*)((char*)out->S + S_plane * l) : p.S[l & 1];
      ROCS_TRY(encoder_layer(h, p.enc, BR, m->L, m->d, m->H, dw, S_prev, S_l, p.KR, p.VR, p.KC, p.VC, s,
                             in->hist_len));
      S_prev = S_l;
      // query generator: token LCB to one token per group (hi/lo), then the GLM-MLP
      const rocs_qgen_weights& qw = W->qgen[l];
      if (!t_done) {
        const void *qER, *qEC;
        long long qldR, qldC;
        int qnR, qnC, qf32;
        if (m->dca_query_source == 0) {
          qER = p.YR; qEC = p.YC; qldR = yr_ld; qldC = yc_ld; qnR = m->q_n_R + l; qnC = m->q_n_C + l; qf32 = 1;
        } else {
          qER = ER; qEC = EC; qldR = wr; qldC = wc; qnR = m->n_R; qnC = m->n_C; qf32 = e_f32;
        }
        SiteLabel s_qlcb("qgen.lcb");
        ROCS_TRY(launch_token_lcb(h, qER, qldR, qEC, qldC, req_idx, BR, BC, qnR, qnC, m->q_dim, qw.p_RR, qw.p_CR,
                                  qw.p_CC, 1, 1, p.tR, q2, p.tC, q2, qf32, 2, m->q_dim, m->q_dim, p.ZqL, s));
      }
      IkboArgs a1;
      a1.B_R = BR; a1.B_C = BC; a1.dRi = m->q_dim; a1.dCi = m->q_dim; a1.dRo = m->d; a1.dCo = m->d;
      a1.X_R = p.tR; a1.ldxr = q2; a1.X_C = p.tC; a1.ldxc = q2; a1.req_idx = req_idx; a1.split_in = 1;
      a1.W_RR = qw.mlp1.W_RR; a1.W_CR = qw.mlp1.W_CR; a1.W_CC = qw.mlp1.W_CC; a1.b_R = qw.mlp1.b_R; a1.b_C = qw.mlp1.b_C;
      a1.Y_R = p.qhR; a1.ldyr = d2; a1.Y_C = p.qhC; a1.ldyc = d2; a1.out_mode = 2; a1.act = ROCS_ACT_GELU;
      a1.Z = p.Zq1; a1.flags = p.ikbo_flags;
      {
        SiteLabel sl("qgen.mlp1");
        ROCS_TRY(ikbo_bf16(h, a1, s));
      }
      IkboArgs a2 = a1;
      a2.dRi = m->d; a2.dCi = m->d;
      a2.X_R = p.qhR; a2.ldxr = d2; a2.X_C = p.qhC; a2.ldxc = d2;
      a2.W_RR = qw.mlp2.W_RR; a2.W_CR = qw.mlp2.W_CR; a2.W_CC = qw.mlp2.W_CC; a2.b_R = qw.mlp2.b_R; a2.b_C = qw.mlp2.b_C;
      a2.Y_R = p.QR; a2.Y_C = p.QC; a2.act = ROCS_ACT_NONE; a2.Z = p.Zq2;
      {
        SiteLabel sl("qgen.mlp2");
        ROCS_TRY(ikbo_bf16(h, a2, s));
      }
      // grouped cross-attention (fp32 results): request queries vs request K/V, candidate
      // queries vs the request's shared K/V
      float *dR, *dC;
      long long ldR, ldC;
      if (m->dca_query_source == 0) {
        dR = p.YR + (m->q_n_R + l) * (long long)m->q_dim; ldR = yr_ld;
        dC = p.YC + (m->q_n_C + l) * (long long)m->q_dim; ldC = yc_ld;
      } else {
        dR = out->A_R ? (float*)out->A_R + (size_t)BR * m->d * l : p.AR; ldR = m->d;
        dC = out->A_C ? (float*)out->A_C + (size_t)BC * m->d * l : p.AC; ldC = m->d;
      }
      void* xR2 = m->score_h1 > 0 ? (char*)p.xR + (size_t)(wr + (long long)l * m->d) * 2 : nullptr;
      void* xC2 = m->score_h1 > 0 ? (char*)p.xC + (size_t)(wc + (long long)l * m->d) * 2 : nullptr;
      const int dh = m->d / m->H;
      const float scale = 1.0f / std::sqrt((float)dh);
      {
        SiteLabel s_xa("xattn.req");
        if (p.KR == nullptr)
          ROCS_TRY(launch_attention_req_absorbed(h, p.QR, d2, S_l, dw.WK_R, dw.WV_R, BR, m->L, m->d, m->H, scale, dR,
                                                 ldR, xR2, xr, s, in->hist_len, p.ar_scratch));
        else
          ROCS_TRY(launch_attention_single(h, p.QR, d2, 1, p.KR, p.VR, m->d, (long long)m->L * m->d, p.iota1, BR, BR,
                                           m->L, m->H, dh, scale, dR, ldR, 0, xR2, xr, s, in->hist_len));
      }
      {
        SiteLabel s_xc("xattn.cand");
        ROCS_TRY(attention_best(h, true, p.QC, d2, 1, p.KC, p.VC, m->d, offsets, BR, BC, m->L, m->H, dh, scale, dC,
                                ldC, 0, xC2, xc, s, in->hist_len, 0, p.order));
      }
      if (m->dca_query_source == 0) {
        if (out->A_R)
          ROCS_TRY(cuda_check(cudaMemcpy2DAsync((float*)out->A_R + (size_t)BR * m->d * l, (size_t)m->d * 4, dR, ldR * 4,
                                                (size_t)m->d * 4, BR, cudaMemcpyDeviceToDevice, s),
                              "copy A_R"));
        if (out->A_C && BC > 0)
          ROCS_TRY(cuda_check(cudaMemcpy2DAsync((float*)out->A_C + (size_t)BC * m->d * l, (size_t)m->d * 4, dC, ldC * 4,
                                                (size_t)m->d * 4, BC, cudaMemcpyDeviceToDevice, s),
                              "copy A_C"));
      }
    }
    // ---------------- GLM layer l: MLP and LayerNorm ----------------
    if (glm_l) {
      const rocs_glm_layer_weights& gw = W->glm[l];
      // a5: GLM-MLP as two IKBO linears; h as hi/lo pairs, o in fp32
      IkboArgs a;
      a.B_R = BR; a.B_C = BC; a.dRi = fR; a.dCi = fC; a.dRo = m->hidden; a.dCo = m->hidden;
      a.X_R = p.FR; a.ldxr = 2LL * fR; a.X_C = p.FC; a.ldxc = 2LL * fC; a.req_idx = req_idx; a.split_in = 1;
      a.W_RR = gw.mlp1.W_RR; a.W_CR = gw.mlp1.W_CR; a.W_CC = gw.mlp1.W_CC; a.b_R = gw.mlp1.b_R; a.b_C = gw.mlp1.b_C;
      a.Y_R = p.hR; a.ldyr = 2LL * m->hidden; a.Y_C = p.hC; a.ldyc = 2LL * m->hidden; a.out_mode = 2;
      a.act = ROCS_ACT_GELU; a.Z = p.Z1; a.flags = p.ikbo_flags;
      {
        SiteLabel sl("glm.mlp1");
        ROCS_TRY(ikbo_bf16(h, a, s));
      }
      const int oRw = m->fm_out_R * m->D, oCw = m->fm_out_C * m->D;
      IkboArgs b = a;
      b.dRi = m->hidden; b.dCi = m->hidden; b.dRo = oRw; b.dCo = oCw;
      b.X_R = p.hR; b.ldxr = 2LL * m->hidden; b.X_C = p.hC; b.ldxc = 2LL * m->hidden;
      b.W_RR = gw.mlp2.W_RR; b.W_CR = gw.mlp2.W_CR; b.W_CC = gw.mlp2.W_CC; b.b_R = gw.mlp2.b_R; b.b_C = gw.mlp2.b_C;
      b.Y_R = p.oR; b.ldyr = oRw; b.Y_C = p.oC; b.ldyc = oCw; b.out_mode = 0; b.act = ROCS_ACT_NONE; b.Z = p.Z2;
      {
        SiteLabel sl("glm.mlp2");
        ROCS_TRY(ikbo_bf16(h, b, s));
      }
      // a6: concat + residual + group-local LN -> next fp32 stream (plus the scoring input copy)
      const bool last = (l == m->glm_layers - 1);
      float* dR = (last && out->E_R) ? (float*)out->E_R : p.ER[(l + 1) & 1];
      float* dC = (last && out->E_C) ? (float*)out->E_C : p.EC[(l + 1) & 1];
      void* xR2 = (last && m->score_h1 > 0) ? p.xR : nullptr;
      void* xC2 = (last && m->score_h1 > 0) ? p.xC : nullptr;
      {
        SiteLabel s_ln("glm.lnR");
        ROCS_TRY(launch_layernorm(h, p.oR, oRw, oRw, p.LR, lRw, lRw, ER, wr, BR, gw.lnR_gamma, gw.lnR_beta, 1e-5f, dR,
                                  wr, 1, e_f32, 0, xR2, xr, s));
      }
      if (BC > 0) {
        SiteLabel s_lnc("glm.lnC");
        ROCS_TRY(launch_layernorm(h, p.oC, oCw, oCw, p.LC, lCw, lCw, EC, wc, BC, gw.lnC_gamma, gw.lnC_beta, 1e-5f, dC,
                                  wc, 1, e_f32, 0, xC2, xc, s));
      }
      ER = dR;
      EC = dC;
      e_f32 = 1;
    }
  }

  // ---------------- a10: scoring head ----------------
  if (m->score_h1 > 0 && BC > 0) {
    const rocs_score_weights& sw = W->score;
    IkboArgs a;
    a.B_R = BR; a.B_C = BC; a.dRi = (int)xr; a.dCi = (int)xc; a.dRo = 0; a.dCo = m->score_h1;
    a.X_R = p.xR; a.ldxr = xr; a.X_C = p.xC; a.ldxc = xc; a.req_idx = req_idx;
    a.W_RR = nullptr; a.W_CR = sw.s1.W_CR; a.W_CC = sw.s1.W_CC; a.b_R = nullptr; a.b_C = sw.s1.b_C;
    a.Y_R = nullptr; a.ldyr = 0; a.Y_C = p.h1; a.ldyc = m->score_h1; a.out_mode = 1; a.act = ROCS_ACT_RELU;
    a.Z = p.Zs; a.flags = p.ikbo_flags;
    {
      SiteLabel sl("score.l1");
      ROCS_TRY(ikbo_bf16(h, a, s));
    }
    SiteLabel s_l2("score.l2");
    ROCS_TRY(linear_bf16(h, p.h1, m->score_h1, BC, m->score_h1, sw.W2, m->score_h2, sw.b2, p.h2, m->score_h2, 1,
                         ROCS_ACT_RELU, s));
    SiteLabel s_l3("score.l3");
    if (out->score) ROCS_TRY(launch_score_head(p.h2, m->score_h2, BC, m->score_h2, sw.w3, sw.b3, out->score, s));
  }
  return ROCS_OK;
}

// Key of one rocs_forward call: every byte that the launch sequence depends on.
std::vector<uint8_t> forward_key(const rocs_model_desc* m, const rocs_model_weights* W, const rocs_inputs* in,
                                 const rocs_outputs* out, const void* ws, size_t ws_bytes) {
  std::vector<uint8_t> k;
  auto put = [&](const void* p, size_t n) {
    const uint8_t* b = static_cast<const uint8_t*>(p);
    k.insert(k.end(), b, b + n);
  };
  put(m, sizeof(*m));
  put(W, sizeof(*W));
  put(in, sizeof(*in));
  put(out, sizeof(*out));
  put(&ws, sizeof(ws));
  put(&ws_bytes, sizeof(ws_bytes));
  return k;
}

}  // namespace

extern "C" rocs_status rocs_forward(rocs_handle_t h, const rocs_model_desc* m, const rocs_model_weights* W,
                                    const rocs_inputs* in, rocs_outputs* out, void* ws, size_t ws_bytes,
                                    void* stream) {
  CtxGuard ctx_guard_(h);
  ROCS_REQUIRE(h, "rocs_forward: handle is NULL");
  ROCS_TRY(check_model(m));
  ROCS_REQUIRE(W && in && out && in->counts, "rocs_forward: NULL argument");
  if (m->glm_layers > 0) ROCS_REQUIRE(in->E_R && (m->B_C == 0 || in->E_C), "rocs_forward: GLM inputs NULL");
  if (m->dca_layers > 0) {
    ROCS_REQUIRE(in->Hist, "rocs_forward: Hist NULL");
    if (m->dca_query_source == 0) ROCS_REQUIRE(in->Y_R && (m->B_C == 0 || in->Y_C), "rocs_forward: Y_R/Y_C NULL");
  }
  for (int l = 0; l < m->glm_layers; ++l) {
    const rocs_glm_layer_weights& g = W->glm[l];
    ROCS_REQUIRE(g.mlp1.W_RR && g.mlp1.W_CR && g.mlp1.W_CC && g.mlp1.b_R && g.mlp1.b_C && g.mlp2.W_RR &&
                     g.mlp2.W_CR && g.mlp2.W_CC && g.mlp2.b_R && g.mlp2.b_C && g.P_RR && g.P_CR && g.P_CC &&
                     g.lnR_gamma && g.lnR_beta && g.lnC_gamma && g.lnC_beta,
                 "rocs_forward: GLM layer %d has a NULL weight", l);
  }
  for (int l = 0; l < m->dca_layers; ++l) {
    const rocs_dca_layer_weights& x = W->dca[l];
    const rocs_qgen_weights& q = W->qgen[l];
    ROCS_REQUIRE(x.Wq && x.Wk && x.Wv && x.Wo && x.ln_gamma && x.ln_beta && x.WK_R && x.WV_R && x.WK_C && x.WV_C &&
                     q.p_RR && q.p_CR && q.p_CC && q.mlp1.W_RR && q.mlp1.W_CR && q.mlp1.W_CC && q.mlp1.b_R &&
                     q.mlp1.b_C && q.mlp2.W_RR && q.mlp2.W_CR && q.mlp2.W_CC && q.mlp2.b_R && q.mlp2.b_C,
                 "rocs_forward: DCA layer %d has a NULL weight", l);
  }
  if (m->score_h1 > 0) {
    const rocs_score_weights& sc = W->score;
    ROCS_REQUIRE(sc.s1.W_CR && sc.s1.W_CC && sc.s1.b_C && sc.W2 && sc.b2 && sc.w3 && sc.b3,
                 "rocs_forward: scoring head has a NULL weight");
  }
  const bool own_off = out->offsets == nullptr, own_req = out->req_idx == nullptr;
  FwdPlan need = plan_forward(m, nullptr, own_off, own_req);
  if (!ws || ws_bytes < need.bytes) {
    set_error("rocs_forward: workspace %zu B < required %zu B", ws_bytes, need.bytes);
    return ROCS_ERR_WORKSPACE;
  }
  ROCS_REQUIRE(aligned16(ws), "rocs_forward: workspace must be 16-byte aligned");
  FwdPlan p = plan_forward(m, ws, own_off, own_req);
  cudaStream_t s = (cudaStream_t)stream;
  // a11: the launch sequence is replayed as a CUDA graph once the same call has been seen
  // before (the first call runs it eagerly); per-launch timing always runs eagerly
  if (!h->graph_replay || h->timer.enabled) return forward_launches(h, m, W, in, out, p, own_off, own_req, s);
  std::vector<uint8_t> key = forward_key(m, W, in, out, ws, ws_bytes);
  ForwardGraph* fg = nullptr;
  for (ForwardGraph& g : h->graphs)
    if (g.key == key) fg = &g;
  if (fg == nullptr) {
    if (h->graphs.size() >= kMaxForwardGraphs) {
      if (h->graphs.front().exec) cudaGraphExecDestroy(h->graphs.front().exec);
      h->graphs.erase(h->graphs.begin());
    }
    h->graphs.push_back(ForwardGraph());
    fg = &h->graphs.back();
    fg->key = std::move(key);
  }
  if (fg->exec == nullptr && fg->calls++ == 0) return forward_launches(h, m, W, in, out, p, own_off, own_req, s);
  if (fg->exec == nullptr) {
    if (h->capture_stream == nullptr)
      ROCS_TRY(cuda_check(cudaStreamCreateWithFlags(&h->capture_stream, cudaStreamNonBlocking), "cudaStreamCreate"));
    ROCS_TRY(cuda_check(cudaStreamBeginCapture(h->capture_stream, cudaStreamCaptureModeThreadLocal),
                        "cudaStreamBeginCapture"));
    const rocs_status st = forward_launches(h, m, W, in, out, p, own_off, own_req, h->capture_stream);
    cudaGraph_t graph = nullptr;
    const cudaError_t ce = cudaStreamEndCapture(h->capture_stream, &graph);
    if (st != ROCS_OK || ce != cudaSuccess) {
      if (graph) cudaGraphDestroy(graph);
      if (st != ROCS_OK) return st;
      return cuda_check(ce, "cudaStreamEndCapture");
    }
    const cudaError_t ie = cudaGraphInstantiate(&fg->exec, graph, 0);
    cudaGraphDestroy(graph);
    if (ie != cudaSuccess) {
      fg->exec = nullptr;
      return cuda_check(ie, "cudaGraphInstantiate");
    }
  }
  return cuda_check(cudaGraphLaunch(fg->exec, s), "cudaGraphLaunch");
}

extern "C" rocs_status rocs_set_ikbo_fused(rocs_handle_t h, int32_t enable) {
  ROCS_REQUIRE(h, "rocs_set_ikbo_fused: handle is NULL");
  ROCS_REQUIRE(enable == 0 || enable == 1, "rocs_set_ikbo_fused: enable must be 0 or 1");
  h->ikbo_fused = enable;
  return ROCS_OK;
}

extern "C" rocs_status rocs_set_w8_tensor_cores(rocs_handle_t h, int32_t enable) {
  ROCS_REQUIRE(h, "rocs_set_w8_tensor_cores: handle is NULL");
  ROCS_REQUIRE(enable == 0 || enable == 1, "rocs_set_w8_tensor_cores: enable must be 0 or 1");
  h->w8_tensor_cores = enable;
  return ROCS_OK;
}

extern "C" rocs_status rocs_probe_exp2_rate(rocs_handle_t h, int32_t n_poly, double* exp2_per_second, void* stream) {
  CtxGuard ctx_guard_(h);
  ROCS_REQUIRE(h, "rocs_probe_exp2_rate: handle is NULL");
  ROCS_REQUIRE(exp2_per_second, "rocs_probe_exp2_rate: exp2_per_second is NULL");
  ROCS_REQUIRE(n_poly >= 0 && n_poly <= 8, "rocs_probe_exp2_rate: n_poly=%d outside [0, 8]", n_poly);
  return probe_exp2_rate(h, n_poly, exp2_per_second, (cudaStream_t)stream);
}

extern "C" rocs_status rocs_test_withhold_ikbo_flag(rocs_handle_t h, int32_t flag_index, int64_t wait_budget_cycles) {
  ROCS_REQUIRE(h, "rocs_test_withhold_ikbo_flag: handle is NULL");
  ROCS_REQUIRE(flag_index >= -1, "rocs_test_withhold_ikbo_flag: flag_index=%d must be >= -1", flag_index);
  if (flag_index < 0) {
    h->test_withhold_flag = -1;
    h->test_flag_budget = 0;
    return ROCS_OK;
  }
  ROCS_REQUIRE(wait_budget_cycles >= 1000 && wait_budget_cycles <= 10000000000LL,
               "rocs_test_withhold_ikbo_flag: wait_budget_cycles=%lld outside [1e3, 1e10]",
               (long long)wait_budget_cycles);
  h->test_withhold_flag = flag_index;
  h->test_flag_budget = wait_budget_cycles;
  return ROCS_OK;
}

// =============================================================================================
// per-launch timing
// =============================================================================================
extern "C" rocs_status rocs_set_graph_replay(rocs_handle_t h, int32_t enable) {
  ROCS_REQUIRE(h, "rocs_set_graph_replay: handle is NULL");
  ROCS_REQUIRE(enable == 0 || enable == 1, "rocs_set_graph_replay: enable must be 0 or 1");
  h->graph_replay = enable;
  return ROCS_OK;
}

extern "C" rocs_status rocs_timing_start(rocs_handle_t h, int32_t max_launches) {
  ROCS_REQUIRE(h, "rocs_timing_start: handle is NULL");
  ROCS_REQUIRE(max_launches >= 1 && max_launches <= (1 << 20), "rocs_timing_start: max_launches out of range");
  RocsTimer& t = h->timer;
  ROCS_REQUIRE(!t.enabled, "rocs_timing_start: timing already running");
  int prev = 0;
  ROCS_TRY(cuda_check(cudaGetDevice(&prev), "cudaGetDevice"));
  ROCS_TRY(cuda_check(cudaSetDevice(h->device), "cudaSetDevice"));
  t.pool.assign((size_t)max_launches * 2, nullptr);
  rocs_status st = ROCS_OK;
  for (auto& e : t.pool) {
    st = cuda_check(cudaEventCreate(&e), "cudaEventCreate");
    if (st != ROCS_OK) break;
  }
  cudaSetDevice(prev);
  if (st != ROCS_OK) {
    for (auto& e : t.pool)
      if (e) cudaEventDestroy(e);
    t.pool.clear();
    return st;
  }
  t.next = 0;
  t.labels.clear();
  t.dropped = 0;
  t.enabled = true;
  return ROCS_OK;
}

extern "C" rocs_status rocs_timing_stop(rocs_handle_t h, char* report, size_t report_bytes) {
  ROCS_REQUIRE(h, "rocs_timing_stop: handle is NULL");
  RocsTimer& t = h->timer;
  ROCS_REQUIRE(t.enabled, "rocs_timing_stop: timing not running");
  t.enabled = false;
  rocs_status st = ROCS_OK;
  std::vector<std::string> names;
  std::vector<long long> counts;
  std::vector<double> totals;
  for (size_t i = 0; i < t.next && st == ROCS_OK; ++i) {
    st = cuda_check(cudaEventSynchronize(t.pool[2 * i + 1]), "cudaEventSynchronize");
    if (st != ROCS_OK) break;
    float ms = 0.f;
    st = cuda_check(cudaEventElapsedTime(&ms, t.pool[2 * i], t.pool[2 * i + 1]), "cudaEventElapsedTime");
    if (st != ROCS_OK) break;
    size_t k = 0;
    while (k < names.size() && names[k] != t.labels[i]) ++k;
    if (k == names.size()) {
      names.push_back(t.labels[i]);
      counts.push_back(0);
      totals.push_back(0.0);
    }
    counts[k] += 1;
    totals[k] += ms;
  }
  for (auto& e : t.pool) cudaEventDestroy(e);
  t.pool.clear();
  if (st != ROCS_OK) return st;
  std::string out;
  char line[256];
  for (size_t k = 0; k < names.size(); ++k) {
    snprintf(line, sizeof(line), "%s %lld %.6f\n", names[k].c_str(), counts[k], totals[k]);
    out += line;
  }
  if (t.dropped) {
    snprintf(line, sizeof(line), "dropped %lld 0\n", t.dropped);
    out += line;
  }
  if (report && report_bytes) {
    const size_t n = out.size() < report_bytes - 1 ? out.size() : report_bytes - 1;
    memcpy(report, out.data(), n);
    report[n] = 0;
    if (out.size() >= report_bytes) {
      set_error("rocs_timing_stop: report truncated (%zu bytes needed)", out.size() + 1);
      return ROCS_ERR_INVALID_ARG;
    }
  }
  return ROCS_OK;
}
