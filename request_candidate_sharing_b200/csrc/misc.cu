// Small kernels of the ROCS path: segment bookkeeping, the exact-order fp32 IKBO GEMM, the
// alignment fix (zero padding), and the scoring head's final dot product + sigmoid.
#include <algorithm>

#include "common.cuh"
#include "internal.h"

namespace rocs {
namespace {

// ------------------------------------------------------------------------------------------
// a0: counts -> offsets (exclusive running total) in one CTA, then offsets -> request map.
// ([REV] §2.4: candidate i belongs to request m_i.)
// ------------------------------------------------------------------------------------------
constexpr int SCAN_THREADS = 1024;

__global__ void __launch_bounds__(SCAN_THREADS) scan_counts_kernel(const int32_t* __restrict__ counts, int B_R,
                                                                    int32_t* __restrict__ offsets, long long B_C,
                                                                    int* status) {
  __shared__ long long warp_tot[32];
  __shared__ long long carry_s;
  __shared__ int bad_s;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  if (tid == 0) { carry_s = 0; bad_s = 0; }
  __syncthreads();
  for (int base = 0; base < B_R; base += SCAN_THREADS) {
    const int r = base + tid;
    long long v = 0;
    if (r < B_R) {
      const int c = counts[r];
      if (c < 0) bad_s = 1;
      v = c < 0 ? 0 : c;
    }
    long long incl = v;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      long long n = __shfl_up_sync(0xffffffffu, incl, o);
      if (lane >= o) incl += n;
    }
    if (lane == 31) warp_tot[warp] = incl;
    __syncthreads();
    if (warp == 0) {
      long long w = warp_tot[lane];
      long long wi = w;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        long long n = __shfl_up_sync(0xffffffffu, wi, o);
        if (lane >= o) wi += n;
      }
      warp_tot[lane] = wi - w;   // exclusive prefix of warp totals
    }
    __syncthreads();
    const long long excl = carry_s + warp_tot[warp] + incl - v;
    if (r < B_R) offsets[r] = (int32_t)min(excl, (long long)INT32_MAX);
    __syncthreads();
    if (tid == SCAN_THREADS - 1) carry_s = excl + v;
    __syncthreads();
  }
  if (tid == 0) {
    offsets[B_R] = (int32_t)min(carry_s, (long long)INT32_MAX);
    if (bad_s || carry_s != B_C) set_status(status, ROCS_ERR_COUNTS);
  }
}

// One warp per request writes its candidate slots; writes outside [0, B_C) are dropped.
__global__ void expand_kernel(const int32_t* __restrict__ offsets, int B_R, int32_t* __restrict__ req_idx,
                              long long B_C) {
  const long long gw = ((long long)blockIdx.x * blockDim.x + threadIdx.x) >> 5;
  const int lane = threadIdx.x & 31;
  if (gw >= B_R) return;
  const int r = (int)gw;
  const long long lo = max(0, offsets[r]);
  const long long hi = min((long long)offsets[r + 1], B_C);
  for (long long c = lo + lane; c < hi; c += 32) req_idx[c] = r;
}

__global__ void iota_kernel(int32_t* out, int n, int step) {
  const int i = blockIdx.x * blockDim.x + threadIdx.x;
  if (i < n) out[i] = i * step;
}

// ------------------------------------------------------------------------------------------
// a1: alignment fix -- copy rows into a zero-padded buffer whose row length is 16-B aligned.
// ------------------------------------------------------------------------------------------
template <typename T>
__global__ void pad_rows_kernel(const T* __restrict__ src, long long ld_src, T* __restrict__ dst, long long ld_dst,
                                long long rows, int cols) {
  const long long total = rows * ld_dst;
  for (long long i = (long long)blockIdx.x * blockDim.x + threadIdx.x; i < total;
       i += (long long)gridDim.x * blockDim.x) {
    const long long r = i / ld_dst;
    const int c = (int)(i - r * ld_dst);
    dst[i] = c < cols ? src[r * ld_src + c] : T(0);
  }
}

// ------------------------------------------------------------------------------------------
// Exact-order fp32 GEMM with the IKBO epilogue: out[r, c] = act(sum_k A[r,k] B[c,k] + bias[c]
// + Z[gidx[r], c]).  Each output accumulates k = 0..K-1 in order with FFMA (no TF32), so the
// result does not depend on the tiling.  64x64 output tile, 256 threads, 4x4 per thread.
// ------------------------------------------------------------------------------------------
constexpr int FT = 64, FK = 16;

__global__ void __launch_bounds__(256) gemm_f32_kernel(const float* __restrict__ A, long long lda, int M, int K,
                                                       const float* __restrict__ B, long long ldb, int N,
                                                       const float* __restrict__ bias, const float* __restrict__ Z,
                                                       long long ldz, const int32_t* __restrict__ gidx,
                                                       int gidx_bound, float* __restrict__ out, long long ldo,
                                                       int act, int* status) {
  __shared__ float sA[FK][FT + 1];
  __shared__ float sB[FK][FT + 1];
  const int tx = threadIdx.x & 15, ty = threadIdx.x >> 4;
  const long long m0 = (long long)blockIdx.y * FT;
  const int n0 = blockIdx.x * FT;
  float acc[4][4];
#pragma unroll
  for (int i = 0; i < 4; ++i)
#pragma unroll
    for (int j = 0; j < 4; ++j) acc[i][j] = 0.f;
  for (int k0 = 0; k0 < K; k0 += FK) {
    for (int i = threadIdx.x; i < FK * FT; i += 256) {
      const int kk = i % FK, rr = i / FK;
      const long long ar = m0 + rr;
      const int br = n0 + rr;
      sA[kk][rr] = (ar < M && k0 + kk < K) ? A[ar * lda + k0 + kk] : 0.f;
      sB[kk][rr] = (br < N && k0 + kk < K) ? B[(long long)br * ldb + k0 + kk] : 0.f;
    }
    __syncthreads();
    const int kmax = min(FK, K - k0);
    for (int kk = 0; kk < kmax; ++kk) {
      float a[4], b[4];
#pragma unroll
      for (int i = 0; i < 4; ++i) a[i] = sA[kk][ty * 4 + i];
#pragma unroll
      for (int j = 0; j < 4; ++j) b[j] = sB[kk][tx * 4 + j];
#pragma unroll
      for (int i = 0; i < 4; ++i)
#pragma unroll
        for (int j = 0; j < 4; ++j) acc[i][j] = fmaf(a[i], b[j], acc[i][j]);
    }
    __syncthreads();
  }
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const long long r = m0 + ty * 4 + i;
    if (r >= M) continue;
    const float* zrow = nullptr;
    if (Z != nullptr) {
      const int zi = gidx[r];
      if (zi < 0 || zi >= gidx_bound) { set_status(status, ROCS_ERR_INDEX); continue; }
      zrow = Z + (long long)zi * ldz;
    }
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const int c = n0 + tx * 4 + j;
      if (c >= N) continue;
      float v = acc[i][j];
      if (bias) v += bias[c];
      if (zrow) v += zrow[c];
      out[r * ldo + c] = act_apply(v, act);
    }
  }
}

// ------------------------------------------------------------------------------------------
// Scoring head output: s[r] = sigmoid(sum_k X[r,k] w[k] + b), one warp per row, bf16 inputs.
// ------------------------------------------------------------------------------------------
__global__ void score_head_kernel(const __nv_bfloat16* __restrict__ X, long long ldx, long long rows, int K,
                                  const __nv_bfloat16* __restrict__ w, const float* __restrict__ b,
                                  float* __restrict__ out) {
  const long long row = ((long long)blockIdx.x * blockDim.x + threadIdx.x) >> 5;
  const int lane = threadIdx.x & 31;
  if (row >= rows) return;
  const __nv_bfloat16* x = X + row * ldx;
  float acc = 0.f;
  for (int k = lane; k < K; k += 32) acc = fmaf(__bfloat162float(x[k]), __bfloat162float(w[k]), acc);
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, o);
  if (lane == 0) out[row] = 1.0f / (1.0f + expf(-(acc + b[0])));
}

}  // namespace

rocs_status launch_segments(rocs_context* ctx, const int32_t* counts, int B_R, int32_t* offsets, int32_t* req_idx,
                            long long B_C, cudaStream_t s) {
  {
  LaunchTimer lt_("scan_counts", s);
  scan_counts_kernel<<<1, SCAN_THREADS, 0, s>>>(counts, B_R, offsets, B_C, ctx->d_status);
  }
  rocs_status st = cuda_check(cudaGetLastError(), "scan_counts_kernel");
  if (st != ROCS_OK || req_idx == nullptr || B_C == 0) return st;
  const long long threads = (long long)B_R * 32;
  LaunchTimer lt_("expand", s);
  expand_kernel<<<(unsigned)((threads + 255) / 256), 256, 0, s>>>(offsets, B_R, req_idx, B_C);
  return cuda_check(cudaGetLastError(), "expand_kernel");
}

rocs_status launch_iota(int32_t* out, int n, int step, cudaStream_t s) {
  LaunchTimer lt_("iota", s);
  iota_kernel<<<(n + 255) / 256, 256, 0, s>>>(out, n, step);
  return cuda_check(cudaGetLastError(), "iota_kernel");
}

rocs_status launch_pad_rows(const void* src, long long ld_src, void* dst, long long ld_dst, long long rows, int cols,
                            int elem_bytes, cudaStream_t s) {
  const long long total = rows * ld_dst;
  const int blocks = (int)std::min<long long>((total + 255) / 256, 148 * 16);
  if (total == 0) return ROCS_OK;
  LaunchTimer lt_("pad_rows", s);
  if (elem_bytes == 2)
    pad_rows_kernel<uint16_t><<<blocks, 256, 0, s>>>((const uint16_t*)src, ld_src, (uint16_t*)dst, ld_dst, rows, cols);
  else
    pad_rows_kernel<float><<<blocks, 256, 0, s>>>((const float*)src, ld_src, (float*)dst, ld_dst, rows, cols);
  return cuda_check(cudaGetLastError(), "pad_rows_kernel");
}

rocs_status launch_gemm_f32(rocs_context* ctx, const float* A, long long lda, int M, int K, const float* B,
                            long long ldb, int N, const float* bias, const float* Z, long long ldz,
                            const int32_t* gidx, int gidx_bound, float* out, long long ldo, int act, cudaStream_t s) {
  if (M == 0 || N == 0) return ROCS_OK;
  dim3 grid((N + FT - 1) / FT, (M + FT - 1) / FT);
  if (grid.y > 65535) {
    set_error("fp32 gemm: M=%d too large", M);
    return ROCS_ERR_UNSUPPORTED;
  }
  LaunchTimer lt_("gemm_f32", s);
  gemm_f32_kernel<<<grid, 256, 0, s>>>(A, lda, M, K, B, ldb, N, bias, Z, ldz, gidx, gidx_bound, out, ldo, act,
                                       ctx->d_status);
  return cuda_check(cudaGetLastError(), "gemm_f32_kernel");
}

rocs_status launch_score_head(const void* X, long long ldx, long long rows, int K, const void* w, const float* b,
                              float* out, cudaStream_t s) {
  if (rows == 0) return ROCS_OK;
  const long long threads = rows * 32;
  LaunchTimer lt_("score_head", s);
  score_head_kernel<<<(unsigned)((threads + 255) / 256), 256, 0, s>>>((const __nv_bfloat16*)X, ldx, rows, K,
                                                                       (const __nv_bfloat16*)w, b, out);
  return cuda_check(cudaGetLastError(), "score_head_kernel");
}

}  // namespace rocs
