// a6: concat + residual + group-local LayerNorm in one pass over HBM
// ([SUM]: normalisation statistics are computed inside each group, never over the
// concatenation; [REV] §2.1 Figure 2(b)).
//
// TPR threads own one row; each thread holds NV vectors of VEC elements in registers, so the
// sources (two concatenated segments and the residual) are read exactly once and the output
// written once.  Statistics in fp32: mean first, then the centred sum of squares from the
// register copy (two-pass accuracy without a second read).  128-bit loads/stores on the
// vector path; warp-shuffle + shared-memory reduction across the row's threads.
#include <algorithm>

#include "common.cuh"
#include "internal.h"

namespace rocs {
namespace {

template <typename T, int VEC>
__device__ __forceinline__ void load_vec(const T* p, float (&v)[VEC]);

template <>
__device__ __forceinline__ void load_vec<__nv_bfloat16, 8>(const __nv_bfloat16* p, float (&v)[8]) {
  const uint4 u = *reinterpret_cast<const uint4*>(p);
  v[0] = bf16_lo(u.x); v[1] = bf16_hi(u.x); v[2] = bf16_lo(u.y); v[3] = bf16_hi(u.y);
  v[4] = bf16_lo(u.z); v[5] = bf16_hi(u.z); v[6] = bf16_lo(u.w); v[7] = bf16_hi(u.w);
}
template <>
__device__ __forceinline__ void load_vec<float, 8>(const float* p, float (&v)[8]) {
  const float4 a = reinterpret_cast<const float4*>(p)[0];
  const float4 b = reinterpret_cast<const float4*>(p)[1];
  v[0] = a.x; v[1] = a.y; v[2] = a.z; v[3] = a.w; v[4] = b.x; v[5] = b.y; v[6] = b.z; v[7] = b.w;
}
template <>
__device__ __forceinline__ void load_vec<float, 4>(const float* p, float (&v)[4]) {
  const float4 a = *reinterpret_cast<const float4*>(p);
  v[0] = a.x; v[1] = a.y; v[2] = a.z; v[3] = a.w;
}
template <>
__device__ __forceinline__ void load_vec<__nv_bfloat16, 4>(const __nv_bfloat16* p, float (&v)[4]) {
  const uint2 u = *reinterpret_cast<const uint2*>(p);
  v[0] = bf16_lo(u.x); v[1] = bf16_hi(u.x); v[2] = bf16_lo(u.y); v[3] = bf16_hi(u.y);
}
template <>
__device__ __forceinline__ void load_vec<__nv_bfloat16, 1>(const __nv_bfloat16* p, float (&v)[1]) {
  v[0] = __bfloat162float(*p);
}
template <>
__device__ __forceinline__ void load_vec<float, 1>(const float* p, float (&v)[1]) {
  v[0] = *p;
}

template <typename T, int VEC>
__device__ __forceinline__ void store_vec(T* p, const float (&v)[VEC]);

template <>
__device__ __forceinline__ void store_vec<__nv_bfloat16, 8>(__nv_bfloat16* p, const float (&v)[8]) {
  uint4 u;
  u.x = pack_bf16x2(v[0], v[1]); u.y = pack_bf16x2(v[2], v[3]);
  u.z = pack_bf16x2(v[4], v[5]); u.w = pack_bf16x2(v[6], v[7]);
  *reinterpret_cast<uint4*>(p) = u;
}
template <>
__device__ __forceinline__ void store_vec<float, 8>(float* p, const float (&v)[8]) {
  reinterpret_cast<float4*>(p)[0] = make_float4(v[0], v[1], v[2], v[3]);
  reinterpret_cast<float4*>(p)[1] = make_float4(v[4], v[5], v[6], v[7]);
}
template <>
__device__ __forceinline__ void store_vec<float, 4>(float* p, const float (&v)[4]) {
  *reinterpret_cast<float4*>(p) = make_float4(v[0], v[1], v[2], v[3]);
}
template <>
__device__ __forceinline__ void store_vec<__nv_bfloat16, 4>(__nv_bfloat16* p, const float (&v)[4]) {
  *reinterpret_cast<uint2*>(p) = make_uint2(pack_bf16x2(v[0], v[1]), pack_bf16x2(v[2], v[3]));
}
template <>
__device__ __forceinline__ void store_vec<__nv_bfloat16, 1>(__nv_bfloat16* p, const float (&v)[1]) {
  *p = __float2bfloat16_rn(v[0]);
}
template <>
__device__ __forceinline__ void store_vec<float, 1>(float* p, const float (&v)[1]) {
  *p = v[0];
}

template <int TPR>
__device__ __forceinline__ float row_sum(float x, float* red) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) x += __shfl_xor_sync(0xffffffffu, x, o);
  if (TPR == 32) return x;
  // TPR/32 warps per row; one block holds exactly one row when TPR > 32.
  const int w = threadIdx.x >> 5, lane = threadIdx.x & 31;
  __syncthreads();
  if (lane == 0) red[w] = x;
  __syncthreads();
  float t = 0.f;
#pragma unroll
  for (int i = 0; i < TPR / 32; ++i) t += red[i];
  return t;
}

template <typename TIN, typename TRES, typename TOUT, int VEC, int NV, int TPR>
__global__ void __launch_bounds__(TPR == 32 ? 256 : TPR) layernorm_kernel(
    const TIN* __restrict__ X1, int w1, long long ld1, const TIN* __restrict__ X2, long long ld2,
    const TRES* __restrict__ R, long long ldr, long long rows, int width, const float* __restrict__ gamma,
    const float* __restrict__ beta, float eps, TOUT* __restrict__ Y, long long ldy, __nv_bfloat16* __restrict__ Y2,
    long long ldy2) {
  __shared__ float red[32];
  long long row;
  int t;
  if (TPR == 32) {
    row = (long long)blockIdx.x * (blockDim.x / 32) + (threadIdx.x >> 5);
    t = threadIdx.x & 31;
  } else {
    row = blockIdx.x;
    t = threadIdx.x;
  }
  const bool live = row < rows;   // uniform across a row's threads
  if (TPR == 32 && !live) return;
  float v[NV][VEC];
  float s = 0.f;
#pragma unroll
  for (int i = 0; i < NV; ++i) {
    const int c = (i * TPR + t) * VEC;
    if (live && c < width) {
      if (c < w1) load_vec<TIN, VEC>(X1 + row * ld1 + c, v[i]);
      else load_vec<TIN, VEC>(X2 + row * ld2 + (c - w1), v[i]);
      if (R != nullptr) {
        float r[VEC];
        load_vec<TRES, VEC>(R + row * ldr + c, r);
#pragma unroll
        for (int j = 0; j < VEC; ++j) v[i][j] += r[j];
      }
#pragma unroll
      for (int j = 0; j < VEC; ++j) s += v[i][j];
    } else {
#pragma unroll
      for (int j = 0; j < VEC; ++j) v[i][j] = 0.f;
    }
  }
  const float mean = row_sum<TPR>(s, red) / (float)width;
  float q = 0.f;
#pragma unroll
  for (int i = 0; i < NV; ++i) {
    const int c = (i * TPR + t) * VEC;
    if (c < width) {
#pragma unroll
      for (int j = 0; j < VEC; ++j) {
        const float d = v[i][j] - mean;
        q += d * d;
      }
    }
  }
  const float var = row_sum<TPR>(q, red) / (float)width;
  const float rstd = rsqrtf(var + eps);
  if (!live) return;
#pragma unroll
  for (int i = 0; i < NV; ++i) {
    const int c = (i * TPR + t) * VEC;
    if (c < width) {
      float o[VEC];
#pragma unroll
      for (int j = 0; j < VEC; ++j) o[j] = (v[i][j] - mean) * rstd * __ldg(gamma + c + j) + __ldg(beta + c + j);
      store_vec<TOUT, VEC>(Y + row * ldy + c, o);
      if (Y2 != nullptr) store_vec<__nv_bfloat16, VEC>(Y2 + row * ldy2 + c, o);
    }
  }
}

template <typename TIN, typename TRES, typename TOUT, int VEC, int NV, int TPR>
rocs_status run(const void* X1, int w1, long long ld1, const void* X2, long long ld2, const void* R, long long ldr,
                long long rows, int width, const float* g, const float* b, float eps, void* Y, long long ldy, void* Y2,
                long long ldy2, cudaStream_t s) {
  long long blocks;
  int threads;
  if (TPR == 32) {
    threads = 256;
    blocks = (rows + 7) / 8;
  } else {
    threads = TPR;
    blocks = rows;
  }
  if (blocks > 2147483647LL) {
    set_error("layernorm: too many rows");
    return ROCS_ERR_UNSUPPORTED;
  }
  LaunchTimer lt_("layernorm", s);
  layernorm_kernel<TIN, TRES, TOUT, VEC, NV, TPR><<<(unsigned)blocks, threads, 0, s>>>(
      (const TIN*)X1, w1, ld1, (const TIN*)X2, ld2, (const TRES*)R, ldr, rows, width, g, b, eps, (TOUT*)Y, ldy,
      (__nv_bfloat16*)Y2, ldy2);
  return cuda_check(cudaGetLastError(), "layernorm_kernel");
}

template <typename TIN, typename TRES, typename TOUT>
rocs_status dispatch(const void* X1, int w1, long long ld1, const void* X2, long long ld2, const void* R,
                     long long ldr, long long rows, int width, const float* g, const float* b, float eps, void* Y,
                     long long ldy, void* Y2, long long ldy2, bool vec, cudaStream_t s) {
#define ROCS_LN(VEC, NV, TPR) \
  return run<TIN, TRES, TOUT, VEC, NV, TPR>(X1, w1, ld1, X2, ld2, R, ldr, rows, width, g, b, eps, Y, ldy, Y2, ldy2, s)
  if (vec && sizeof(TIN) == 4) {
    // fp32 rows: one float4 per lane per vector, so each warp-wide load is 512 contiguous bytes;
    // one warp per row (registers only, no block barrier) up to 2048 values, a block beyond
    if (width <= 128) ROCS_LN(4, 1, 32);
    if (width <= 256) ROCS_LN(4, 2, 32);
    if (width <= 512) ROCS_LN(4, 4, 32);
    if (width <= 1024) ROCS_LN(4, 8, 32);
    if (width <= 2048) ROCS_LN(4, 16, 32);
    if (width <= 4096) ROCS_LN(4, 8, 128);
    ROCS_LN(4, 16, 128);
  }
  if (vec) {
    // bf16 rows: 16 bytes (8 values) per lane per vector
    if (width <= 256) ROCS_LN(8, 1, 32);
    if (width <= 512) ROCS_LN(8, 2, 32);
    if (width <= 1024) ROCS_LN(8, 4, 32);
    if (width <= 2048) ROCS_LN(8, 8, 32);
    if (width <= 4096) ROCS_LN(8, 4, 128);
    ROCS_LN(8, 8, 128);
  }
  if (width <= 1024) ROCS_LN(1, 8, 128);
  if (width <= 4096) ROCS_LN(1, 32, 128);
  ROCS_LN(1, 64, 128);
#undef ROCS_LN
}

__global__ void convert_kernel(const __nv_bfloat16* __restrict__ src, long long ld_src, float* __restrict__ dst,
                               long long ld_dst, long long rows, int cols) {
  const long long total = rows * cols;
  for (long long i = (long long)blockIdx.x * blockDim.x + threadIdx.x; i < total;
       i += (long long)gridDim.x * blockDim.x) {
    const long long r = i / cols;
    const int c = (int)(i - r * cols);
    dst[r * ld_dst + c] = __bfloat162float(src[r * ld_src + c]);
  }
}

}  // namespace

rocs_status launch_layernorm(rocs_context* ctx, const void* X1, int w1, long long ld1, const void* X2, int w2,
                             long long ld2, const void* res, long long ldr, long long rows, const float* gamma,
                             const float* beta, float eps, void* Y, long long ldy, int in_f32, int res_f32,
                             int y_bf16, void* Y2, long long ldy2, cudaStream_t s) {
  (void)ctx;
  if (rows == 0) return ROCS_OK;
  const int width = w1 + w2;
  auto al = [](const void* p) { return p == nullptr || ((uintptr_t)p & 15) == 0; };
  const bool vec = (w1 % 8 == 0) && (width % 8 == 0) && ld1 % 8 == 0 && (X2 == nullptr || ld2 % 8 == 0) &&
                   (res == nullptr || ldr % 8 == 0) && ldy % 8 == 0 && (Y2 == nullptr || ldy2 % 8 == 0) && al(X1) &&
                   al(X2) && al(res) && al(Y) && al(Y2);
  if (in_f32 && y_bf16) {
    set_error("layernorm: fp32 inputs with a bf16 primary output are not instantiated");
    return ROCS_ERR_UNSUPPORTED;
  }
  if (in_f32) {
    if (res_f32 || res == nullptr)
      return dispatch<float, float, float>(X1, w1, ld1, X2, ld2, res, ldr, rows, width, gamma, beta, eps, Y, ldy, Y2,
                                           ldy2, vec, s);
    return dispatch<float, __nv_bfloat16, float>(X1, w1, ld1, X2, ld2, res, ldr, rows, width, gamma, beta, eps, Y, ldy,
                                                 Y2, ldy2, vec, s);
  }
  if (!y_bf16 || (res != nullptr && res_f32)) {
    set_error("layernorm: bf16 inputs need a bf16 residual and output");
    return ROCS_ERR_UNSUPPORTED;
  }
  return dispatch<__nv_bfloat16, __nv_bfloat16, __nv_bfloat16>(X1, w1, ld1, X2, ld2, res, ldr, rows, width, gamma,
                                                               beta, eps, Y, ldy, Y2, ldy2, vec, s);
}

rocs_status launch_convert_bf16_f32(const void* src, long long ld_src, float* dst, long long ld_dst, long long rows,
                                    int cols, cudaStream_t s) {
  const long long total = rows * cols;
  if (total == 0) return ROCS_OK;
  const int blocks = (int)std::min<long long>((total + 255) / 256, 148 * 32);
  LaunchTimer lt_("convert", s);
  convert_kernel<<<blocks, 256, 0, s>>>((const __nv_bfloat16*)src, ld_src, dst, ld_dst, rows, cols);
  return cuda_check(cudaGetLastError(), "convert_kernel");
}

}  // namespace rocs
