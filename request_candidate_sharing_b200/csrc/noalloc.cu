// rocs_linear_ikbo_noalloc: the two-group IKBO linear for callers that cannot allocate device
// memory at all -- neither through the library nor by handing it a workspace.  Typical cases are
// plugin hosts and serving loops that plan every device buffer up front and forbid allocation
// while requests are in flight (cudaMalloc can synchronise the device, fail under
// fragmentation, or simply not be reachable from inside the host's own memory manager).
//
// The only scratch the operation needs is the request-side contribution Z = W_CR X^R + b^C
// ([B_R, d_C_out] fp32).  Here it lives in one file-scope device array of fixed size that every
// GPU loading the library holds until the process exits; nothing is allocated or freed per call.
//
// Host code must not pass the array's name to a kernel: on the host that name is only a
// stand-in for the symbol, not a device address.  The first call on each device (with that
// device current) asks the runtime for the real address with cudaGetSymbolAddress and caches
// it, with the context it belongs to; kernels then receive that pointer.  Under lazy module
// loading (the CUDA 12 default) that first call is also when the driver loads this module and
// commits the array's 4 MiB.
#include <mutex>

#include "common.cuh"
#include "internal.h"

namespace rocs {
namespace {

// 4 MiB: Z for up to 1,048,576 fp32 values, e.g. 256 requests x 4096 outputs.
constexpr long long kNoAllocScratchFloats = 1 << 20;

static __device__ __align__(256) float g_noalloc_scratch[kNoAllocScratchFloats];

constexpr int kMaxDevices = 64;
std::mutex g_setup_mutex;
// Per device: the address of the scratch array and the CUDA context it was looked up in.  The
// array belongs to the module loaded into that context; a call from another context (a context
// the caller created, not the device's primary one) looks the address up again in its own.
float* g_scratch_addr[kMaxDevices] = {nullptr};
CUcontext g_scratch_ctx[kMaxDevices] = {nullptr};

typedef CUresult (*CtxGetCurrentFn)(CUcontext*);
CtxGetCurrentFn g_ctx_get_current = nullptr;

// Resolves the device address of the scratch array for the current device and context: once per
// (device, context), on the first call there.
rocs_status scratch_address(int device, float** out) {
  if (device < 0 || device >= kMaxDevices) {
    set_error("rocs_linear_ikbo_noalloc: device %d out of range", device);
    return ROCS_ERR_UNSUPPORTED;
  }
  std::lock_guard<std::mutex> lock(g_setup_mutex);
  if (g_ctx_get_current == nullptr) {
    void* fn = nullptr;
    cudaDriverEntryPointQueryResult q;
    cudaError_t e = cudaGetDriverEntryPoint("cuCtxGetCurrent", &fn, cudaEnableDefault, &q);
    if (e != cudaSuccess || q != cudaDriverEntryPointSuccess || fn == nullptr) {
      set_error("rocs_linear_ikbo_noalloc: cuCtxGetCurrent not available");
      return ROCS_ERR_CUDA;
    }
    g_ctx_get_current = reinterpret_cast<CtxGetCurrentFn>(fn);
  }
  CUcontext cur = nullptr;
  if (g_ctx_get_current(&cur) != CUDA_SUCCESS || cur == nullptr) {
    set_error("rocs_linear_ikbo_noalloc: no current CUDA context");
    return ROCS_ERR_CUDA;
  }
  if (g_scratch_addr[device] == nullptr || g_scratch_ctx[device] != cur) {
    void* p = nullptr;
    cudaError_t e = cudaGetSymbolAddress(&p, g_noalloc_scratch);
    if (e != cudaSuccess || p == nullptr) {
      set_error("rocs_linear_ikbo_noalloc: cudaGetSymbolAddress failed: %s", cudaGetErrorString(e));
      return ROCS_ERR_CUDA;
    }
    g_scratch_addr[device] = static_cast<float*>(p);
    g_scratch_ctx[device] = cur;
  }
  *out = g_scratch_addr[device];
  return ROCS_OK;
}

}  // namespace
}  // namespace rocs

using namespace rocs;

extern "C" rocs_status rocs_linear_ikbo_noalloc(rocs_handle_t h, const rocs_ikbo_desc* d, const void* X_R,
                                                const void* X_C, const int32_t* req_idx, const void* W_RR,
                                                const void* W_CR, const void* W_CC, const float* b_R,
                                                const float* b_C, void* Y_R, void* Y_C, void* stream) {
  if (h == nullptr) {
    set_error("rocs_linear_ikbo_noalloc: handle is NULL");
    return ROCS_ERR_INVALID_ARG;
  }
  rocs_status st = check_ikbo_desc(d, "rocs_linear_ikbo_noalloc");
  if (st != ROCS_OK) return st;
  const long long need = (long long)d->B_R * d->d_C_out;
  if (need > kNoAllocScratchFloats) {
    set_error("rocs_linear_ikbo_noalloc: B_R * d_C_out = %lld exceeds the built-in scratch of %lld floats; "
              "use rocs_linear_ikbo with a workspace",
              need, kNoAllocScratchFloats);
    return ROCS_ERR_UNSUPPORTED;
  }
  if (d->dtype_in == ROCS_BF16 && (d->d_R_in % 8 != 0 || d->d_C_in % 8 != 0)) {
    set_error("rocs_linear_ikbo_noalloc: bf16 rows must be multiples of 8 elements (no room to pad); "
              "use rocs_linear_ikbo with a workspace");
    return ROCS_ERR_UNSUPPORTED;
  }
  if (!X_R || !W_CR || !b_C || (d->d_R_out > 0 && (!W_RR || !b_R || !Y_R)) ||
      (d->B_C > 0 && (!X_C || !W_CC || !req_idx || !Y_C))) {
    set_error("rocs_linear_ikbo_noalloc: required pointer is NULL");
    return ROCS_ERR_INVALID_ARG;
  }
  const void* ptrs[] = {X_R, X_C, W_RR, W_CR, W_CC, b_R, b_C, Y_R, Y_C};
  for (const void* p : ptrs)
    if (((uintptr_t)p & 15) != 0) {
      set_error("rocs_linear_ikbo_noalloc: pointers must be 16-byte aligned");
      return ROCS_ERR_INVALID_ARG;
    }
  int cur = -1;
  st = cuda_check(cudaGetDevice(&cur), "cudaGetDevice");
  if (st != ROCS_OK) return st;
  if (cur != h->device) {
    set_error("rocs_linear_ikbo_noalloc: device %d is current but the handle is bound to device %d", cur, h->device);
    return ROCS_ERR_INVALID_ARG;
  }
  float* Z = nullptr;
  st = scratch_address(h->device, &Z);
  if (st != ROCS_OK) return st;

  rocs_context* prev_ctx = g_ctx;
  g_ctx = h;
  cudaStream_t s = (cudaStream_t)stream;
  // Z is written in full by the request-side launch before the candidate launch reads it, so
  // no part of the shared array has to start at zero.
  if (d->dtype_in == ROCS_F32) {
    if (d->d_R_out > 0)
      st = launch_gemm_f32(h, (const float*)X_R, d->d_R_in, d->B_R, d->d_R_in, (const float*)W_RR, d->d_R_in,
                           d->d_R_out, b_R, nullptr, 0, nullptr, 0, (float*)Y_R, d->d_R_out, d->act, s);
    if (st == ROCS_OK)
      st = launch_gemm_f32(h, (const float*)X_R, d->d_R_in, d->B_R, d->d_R_in, (const float*)W_CR, d->d_R_in,
                           d->d_C_out, b_C, nullptr, 0, nullptr, 0, Z, d->d_C_out, ROCS_ACT_NONE, s);
    if (st == ROCS_OK && d->B_C > 0)
      st = launch_gemm_f32(h, (const float*)X_C, d->d_C_in, (int)d->B_C, d->d_C_in, (const float*)W_CC, d->d_C_in,
                           d->d_C_out, nullptr, Z, d->d_C_out, req_idx, d->B_R, (float*)Y_C, d->d_C_out, d->act, s);
  } else {
    const int out_mode = d->dtype_out == ROCS_BF16 ? 1 : 0;
    GemmDesc req[2];
    int nreq = 0;
    if (d->d_R_out > 0) {
      GemmDesc& g = req[nreq++];
      g.A = X_R; g.lda = d->d_R_in; g.M = d->B_R; g.K = d->d_R_in;
      g.B = W_RR; g.ldb = d->d_R_in; g.N = d->d_R_out;
      g.bias = b_R; g.out = Y_R; g.ldo = d->d_R_out; g.out_mode = out_mode; g.act = d->act;
    }
    GemmDesc& gz = req[nreq++];
    gz.A = X_R; gz.lda = d->d_R_in; gz.M = d->B_R; gz.K = d->d_R_in;
    gz.B = W_CR; gz.ldb = d->d_R_in; gz.N = d->d_C_out;
    gz.bias = b_C; gz.out = Z; gz.ldo = d->d_C_out; gz.out_mode = 0; gz.act = ROCS_ACT_NONE;
    st = launch_gemm_bf16(h, req, nreq, s);
    if (st == ROCS_OK && d->B_C > 0) {
      GemmDesc g;
      g.A = X_C; g.lda = d->d_C_in; g.M = (int)d->B_C; g.K = d->d_C_in;
      g.B = W_CC; g.ldb = d->d_C_in; g.N = d->d_C_out;
      g.Z = Z; g.ldz = d->d_C_out; g.gidx = req_idx; g.gidx_bound = d->B_R;
      g.out = Y_C; g.ldo = d->d_C_out; g.out_mode = out_mode; g.act = d->act;
      st = launch_gemm_bf16(h, &g, 1, s);
    }
  }
  g_ctx = prev_ctx;
  return st;
}
