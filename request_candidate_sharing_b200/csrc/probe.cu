// Throughput probe of the attention softmax's exponentials.  No page gives this rate, and it
// bounds every DCA attention kernel here (one exponential per score), so the attention roofline
// is taken against this measurement on the GPU at hand.
//
// Each thread carries eight independent pairs of scores through the softmax's per-score steps:
// x = s * scale - m on the packed FMA path (ffma2), 2^x (MUFU ex2.approx, or the FMA-pipe
// polynomial exp2_poly2 for n_poly of the eight pairs, the split the attention kernel uses for
// n_poly = 3), and the bf16 pair packing of P.  The next iteration's score is derived from the
// exponential, so nothing can be hoisted out of the loop, and it stays in the softmax's range
// [-8, 0].  One XOR-reduced word per thread goes to a file-scope sink so the work is live.
#include <algorithm>

#include "common.cuh"
#include "internal.h"
#include "softmax_math.cuh"

namespace rocs {
namespace {

constexpr int PROBE_THREADS = 256;
constexpr int PROBE_PAIRS = 8;
constexpr int PROBE_CTAS_PER_SM = 8;   // 2048 threads per SM: every warp slot filled

__device__ uint32_t g_probe_sink;

template <int NPOLY>
__global__ void __launch_bounds__(PROBE_THREADS) exp2_probe_kernel(int iters, float seed) {
  float a[PROBE_PAIRS], b[PROBE_PAIRS];
  const float t = (float)(threadIdx.x & 63) * (1.0f / 64.0f);
#pragma unroll
  for (int c = 0; c < PROBE_PAIRS; ++c) {
    a[c] = -t - 0.1f * c - seed;
    b[c] = -t - 0.05f * c;
  }
  uint32_t acc = 0;
  for (int it = 0; it < iters; ++it) {
#pragma unroll
    for (int c = 0; c < PROBE_PAIRS; ++c) {
      float x0, x1, p0, p1;
      ffma2(a[c], b[c], 1.4426950408889634f, -0.25f, x0, x1);
      if (c >= PROBE_PAIRS - NPOLY) {
        exp2_poly2(x0, x1, p0, p1);
      } else {
        p0 = ex2_approx(x0);
        p1 = ex2_approx(x1);
      }
      acc ^= pack_bf16x2(p0, p1);
      // next scores in [-8, 0): depend on this exponential
      a[c] = fmaf(p1, -7.5f, -0.25f);
      b[c] = fmaf(p0, -7.5f, -0.25f);
    }
  }
  atomicXor(&g_probe_sink, acc);
}

template <int NPOLY>
cudaError_t launch_probe(int grid, int iters, cudaStream_t s) {
  exp2_probe_kernel<NPOLY><<<grid, PROBE_THREADS, 0, s>>>(iters, 0.0f);
  return cudaGetLastError();
}

cudaError_t launch_probe_n(int n_poly, int grid, int iters, cudaStream_t s) {
  switch (n_poly) {
    case 0: return launch_probe<0>(grid, iters, s);
    case 1: return launch_probe<1>(grid, iters, s);
    case 2: return launch_probe<2>(grid, iters, s);
    case 3: return launch_probe<3>(grid, iters, s);
    case 4: return launch_probe<4>(grid, iters, s);
    case 5: return launch_probe<5>(grid, iters, s);
    case 6: return launch_probe<6>(grid, iters, s);
    case 7: return launch_probe<7>(grid, iters, s);
    default: return launch_probe<8>(grid, iters, s);
  }
}

}  // namespace

rocs_status probe_exp2_rate(rocs_context* ctx, int n_poly, double* rate, cudaStream_t s) {
  const int grid = ctx->num_sms * PROBE_CTAS_PER_SM;
  const int iters = 4096;
  cudaEvent_t e0 = nullptr, e1 = nullptr;
  rocs_status st = cuda_check(cudaEventCreate(&e0), "cudaEventCreate");
  if (st == ROCS_OK) st = cuda_check(cudaEventCreate(&e1), "cudaEventCreate");
  if (st == ROCS_OK) st = cuda_check(launch_probe_n(n_poly, grid, iters, s), "exp2 probe warm-up launch");
  float best = 0.f;
  for (int rep = 0; rep < 5 && st == ROCS_OK; ++rep) {
    st = cuda_check(cudaEventRecord(e0, s), "cudaEventRecord");
    if (st == ROCS_OK) st = cuda_check(launch_probe_n(n_poly, grid, iters, s), "exp2 probe launch");
    if (st == ROCS_OK) st = cuda_check(cudaEventRecord(e1, s), "cudaEventRecord");
    if (st == ROCS_OK) st = cuda_check(cudaEventSynchronize(e1), "cudaEventSynchronize");
    float ms = 0.f;
    if (st == ROCS_OK) st = cuda_check(cudaEventElapsedTime(&ms, e0, e1), "cudaEventElapsedTime");
    if (st == ROCS_OK && ms > 0.f && (best == 0.f || ms < best)) best = ms;
  }
  if (e0) cudaEventDestroy(e0);
  if (e1) cudaEventDestroy(e1);
  if (st != ROCS_OK) return st;
  const double exps = (double)grid * PROBE_THREADS * iters * PROBE_PAIRS * 2.0;
  *rate = best > 0.f ? exps / (best * 1e-3) : 0.0;
  return ROCS_OK;
}

}  // namespace rocs
