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

// ---------------------------------------------------------------------------------------------
// Streaming variant for long row counts with contiguous rows (ld == width of every operand):
// one CTA per SM walks a contiguous row range; one thread bulk-copies blocks of RB rows of the two
// segments and the residual into a ring of shared-memory stages, LnRing<NV>::DEPTH warps normalise
// them (one row at a time per warp, lane j holding the float4 groups j, j + 32, ...) and write the
// outputs straight from registers.  gamma/beta live in shared memory.
// ---------------------------------------------------------------------------------------------
// Ring depth = consumer warps = stages.  Consumer warp w takes blocks w, w + DEPTH, ...; with as
// many stages as consumers every one of them lands in stage w, so each warp waits on every phase of
// its own stage's barrier in order and the phase parity is never ambiguous.  Narrow rows (width
// <= 256: 16 encoder rows per stage) run 12 deep, wide rows (a candidate row per stage) 8 deep:
// 12 measured 16% faster for the former and 3% slower for the latter.
template <int NV>
struct LnRing {
  static constexpr int DEPTH = NV <= 2 ? 12 : 8;
};
constexpr int LN_STAGE_BYTES = 16384;

template <typename T>
__device__ __forceinline__ void ld4(const T* p, float (&v)[4]);
template <>
__device__ __forceinline__ void ld4<float>(const float* p, float (&v)[4]) {
  const float4 a = *reinterpret_cast<const float4*>(p);
  v[0] = a.x; v[1] = a.y; v[2] = a.z; v[3] = a.w;
}
template <>
__device__ __forceinline__ void ld4<__nv_bfloat16>(const __nv_bfloat16* p, float (&v)[4]) {
  const uint2 u = *reinterpret_cast<const uint2*>(p);
  v[0] = bf16_lo(u.x); v[1] = bf16_hi(u.x); v[2] = bf16_lo(u.y); v[3] = bf16_hi(u.y);
}

template <typename TIN, typename TRES, typename TOUT, int NV>
__global__ void __launch_bounds__(32 * (1 + LnRing<NV>::DEPTH), 1) layernorm_ring_kernel(
    const TIN* __restrict__ X1, int w1, const TIN* __restrict__ X2, const TRES* __restrict__ R, long long rows,
    long long rows_per_block, int RB, const float* __restrict__ gamma, const float* __restrict__ beta, float eps,
    TOUT* __restrict__ Y, __nv_bfloat16* __restrict__ Y2, long long ldy2, int* status) {
  constexpr int width = NV * 128;
  const int w2 = width - w1;
  extern __shared__ __align__(128) uint8_t ln_smem[];
  float* s_gamma = reinterpret_cast<float*>(ln_smem);
  float* s_beta = s_gamma + width;
  uint8_t* ring = ln_smem + 2 * width * sizeof(float);
  __shared__ __align__(8) uint64_t full[LnRing<NV>::DEPTH], empty[LnRing<NV>::DEPTH];
  __shared__ int abort_flag_s;
  volatile int* abort_flag = &abort_flag_s;

  const long long r0 = (long long)blockIdx.x * rows_per_block;
  const long long r1 = r0 + rows_per_block < rows ? r0 + rows_per_block : rows;
  if (r0 >= r1) return;
  const int nblk = (int)((r1 - r0 + RB - 1) / RB);
  // stage layout: RB rows of X1 | RB rows of X2 | RB rows of R
  const int off2 = RB * w1 * (int)sizeof(TIN);
  const int offr = off2 + RB * w2 * (int)sizeof(TIN);

  for (int i = threadIdx.x; i < width; i += blockDim.x) {
    s_gamma[i] = gamma[i];
    s_beta[i] = beta[i];
  }
  if (threadIdx.x == 0) {
    for (int k = 0; k < LnRing<NV>::DEPTH; ++k) {
      mbar_init(&full[k], 1);
      mbar_init(&empty[k], 32);
    }
    abort_flag_s = 0;
    fence_barrier_init();
  }
  __syncthreads();
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  if (warp == 0) {
    if (lane == 0) {
      int issued = 0;
      for (int b = 0; b < nblk; ++b) {
        const int st = b % LnRing<NV>::DEPTH, use = b / LnRing<NV>::DEPTH;
        if (use > 0 && !mbar_wait(&empty[st], (use - 1) & 1, status, abort_flag)) break;
        const long long row = r0 + (long long)b * RB;
        const int nr = (int)(r1 - row < RB ? r1 - row : RB);
        uint8_t* sb = ring + st * LN_STAGE_BYTES;
        const uint32_t b1 = (uint32_t)(nr * w1 * sizeof(TIN)), b2 = (uint32_t)(nr * w2 * sizeof(TIN)),
                       br = R != nullptr ? (uint32_t)(nr * width * sizeof(TRES)) : 0u;
        mbar_arrive_expect_tx(&full[st], b1 + b2 + br);
        bulk_load(sb, X1 + row * w1, b1, &full[st]);
        if (b2) bulk_load(sb + off2, X2 + row * w2, b2, &full[st]);
        if (br) bulk_load(sb + offr, R + row * width, br, &full[st]);
        issued = b + 1;
      }
      for (int b = issued - LnRing<NV>::DEPTH < 0 ? 0 : issued - LnRing<NV>::DEPTH; b < issued; ++b)
        mbar_wait(&full[b % LnRing<NV>::DEPTH], (b / LnRing<NV>::DEPTH) & 1, status, nullptr);
    }
    return;
  }

  const int cw = warp - 1;
  for (int b = cw; b < nblk; b += LnRing<NV>::DEPTH) {
    const int st = b % LnRing<NV>::DEPTH;
    if (!__all_sync(0xffffffffu, mbar_wait(&full[st], (b / LnRing<NV>::DEPTH) & 1, status, abort_flag))) break;
    const uint8_t* sb = ring + st * LN_STAGE_BYTES;
    const long long row0 = r0 + (long long)b * RB;
    const int nr = (int)(r1 - row0 < RB ? r1 - row0 : RB);
    // narrow rows: MR rows at a time, so their reductions overlap
    constexpr int MR = NV <= 4 ? 4 : 1;
    for (int k0 = 0; k0 < nr; k0 += MR) {
      float v[MR][NV][4];
      float s[MR];
#pragma unroll
      for (int m = 0; m < MR; ++m) {
        s[m] = 0.f;
        const int k = k0 + m;
#pragma unroll
        for (int i = 0; i < NV; ++i) {
          const int col = (i * 32 + lane) * 4;
          if (k < nr) {
            if (col < w1) ld4<TIN>(reinterpret_cast<const TIN*>(sb) + k * w1 + col, v[m][i]);
            else ld4<TIN>(reinterpret_cast<const TIN*>(sb + off2) + k * w2 + (col - w1), v[m][i]);
            if (R != nullptr) {
              float rr[4];
              ld4<TRES>(reinterpret_cast<const TRES*>(sb + offr) + k * width + col, rr);
#pragma unroll
              for (int j = 0; j < 4; ++j) v[m][i][j] += rr[j];
            }
          } else {
#pragma unroll
            for (int j = 0; j < 4; ++j) v[m][i][j] = 0.f;
          }
#pragma unroll
          for (int j = 0; j < 4; ++j) s[m] += v[m][i][j];
        }
      }
      if (k0 + MR >= nr) mbar_arrive(&empty[st]);   // every read of this stage is done
#pragma unroll
      for (int o = 16; o > 0; o >>= 1)
#pragma unroll
        for (int m = 0; m < MR; ++m) s[m] += __shfl_xor_sync(0xffffffffu, s[m], o);
      float mean[MR], q[MR];
#pragma unroll
      for (int m = 0; m < MR; ++m) {
        mean[m] = s[m] * (1.0f / (float)width);
        q[m] = 0.f;
#pragma unroll
        for (int i = 0; i < NV; ++i)
#pragma unroll
          for (int j = 0; j < 4; ++j) {
            const float d = v[m][i][j] - mean[m];
            q[m] += d * d;
          }
      }
#pragma unroll
      for (int o = 16; o > 0; o >>= 1)
#pragma unroll
        for (int m = 0; m < MR; ++m) q[m] += __shfl_xor_sync(0xffffffffu, q[m], o);
#pragma unroll
      for (int m = 0; m < MR; ++m) {
        if (k0 + m >= nr) break;
        const float rstd = rsqrtf(q[m] * (1.0f / (float)width) + eps);
        const long long row = row0 + k0 + m;
#pragma unroll
        for (int i = 0; i < NV; ++i) {
          const int col = (i * 32 + lane) * 4;
          const float4 gm = *reinterpret_cast<const float4*>(s_gamma + col);
          const float4 bt = *reinterpret_cast<const float4*>(s_beta + col);
          float o[4] = {(v[m][i][0] - mean[m]) * rstd * gm.x + bt.x, (v[m][i][1] - mean[m]) * rstd * gm.y + bt.y,
                        (v[m][i][2] - mean[m]) * rstd * gm.z + bt.z, (v[m][i][3] - mean[m]) * rstd * gm.w + bt.w};
          store_vec<TOUT, 4>(Y + row * width + col, o);
          if (Y2 != nullptr) store_vec<__nv_bfloat16, 4>(Y2 + row * ldy2 + col, o);
        }
      }
    }
  }
}

template <typename TIN, typename TRES, typename TOUT, int NV>
rocs_status run_ring(rocs_context* ctx, const void* X1, int w1, const void* X2, const void* R, long long rows,
                     const float* g, const float* b, float eps, void* Y, void* Y2, long long ldy2, cudaStream_t s) {
  constexpr int width = NV * 128;
  const int row_bytes = (int)(width * sizeof(TIN) + (R != nullptr ? width * sizeof(TRES) : 0));
  const int RB = LN_STAGE_BYTES / row_bytes;
  const size_t smem = 2 * width * sizeof(float) + (size_t)LnRing<NV>::DEPTH * LN_STAGE_BYTES;
  static bool attr[64] = {false};
  if (ctx->device < 64 && !attr[ctx->device]) {
    rocs_status st = cuda_check(cudaFuncSetAttribute(layernorm_ring_kernel<TIN, TRES, TOUT, NV>,
                                                     cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem),
                                "cudaFuncSetAttribute(layernorm_ring)");
    if (st != ROCS_OK) return st;
    attr[ctx->device] = true;
  }
  const long long blocks = ctx->num_sms;
  long long per_block = (rows + blocks - 1) / blocks;
  per_block = (per_block + RB - 1) / RB * RB;
  LaunchTimer lt_("layernorm", s);
  layernorm_ring_kernel<TIN, TRES, TOUT, NV><<<(unsigned)blocks, 32 * (1 + LnRing<NV>::DEPTH), smem, s>>>(
      (const TIN*)X1, w1, (const TIN*)X2, (const TRES*)R, rows, per_block, RB, g, b, eps, (TOUT*)Y,
      (__nv_bfloat16*)Y2, ldy2, ctx->d_status);
  return cuda_check(cudaGetLastError(), "layernorm_ring_kernel");
}

template <typename TIN, typename TRES, typename TOUT>
rocs_status dispatch_ring(rocs_context* ctx, const void* X1, int w1, const void* X2, const void* R, long long rows,
                          int width, const float* g, const float* b, float eps, void* Y, void* Y2, long long ldy2,
                          cudaStream_t s) {
  switch (width) {
    case 256: return run_ring<TIN, TRES, TOUT, 2>(ctx, X1, w1, X2, R, rows, g, b, eps, Y, Y2, ldy2, s);
    case 512: return run_ring<TIN, TRES, TOUT, 4>(ctx, X1, w1, X2, R, rows, g, b, eps, Y, Y2, ldy2, s);
    case 1024: return run_ring<TIN, TRES, TOUT, 8>(ctx, X1, w1, X2, R, rows, g, b, eps, Y, Y2, ldy2, s);
    case 2048: return run_ring<TIN, TRES, TOUT, 16>(ctx, X1, w1, X2, R, rows, g, b, eps, Y, Y2, ldy2, s);
    default: return ROCS_ERR_UNSUPPORTED;
  }
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
  if (rows == 0) return ROCS_OK;
  const int width = w1 + w2;
  auto al = [](const void* p) { return p == nullptr || ((uintptr_t)p & 15) == 0; };
  const bool vec = (w1 % 8 == 0) && (width % 8 == 0) && ld1 % 8 == 0 && (X2 == nullptr || ld2 % 8 == 0) &&
                   (res == nullptr || ldr % 8 == 0) && ldy % 8 == 0 && (Y2 == nullptr || ldy2 % 8 == 0) && al(X1) &&
                   al(X2) && al(res) && al(Y) && al(Y2);
  // long runs of contiguous rows: the streaming (bulk-copy ring) variant
  const bool ring = vec && ctx != nullptr && rows >= 16384 && w1 % 128 == 0 && ld1 == w1 &&
                    (X2 == nullptr ? w2 == 0 : ld2 == w2) && (res == nullptr || ldr == width) && ldy == width;
  if (ring) {
    rocs_status st = ROCS_ERR_UNSUPPORTED;
    if (in_f32 && !y_bf16 && (res_f32 || res == nullptr))
      st = dispatch_ring<float, float, float>(ctx, X1, w1, X2, res, rows, width, gamma, beta, eps, Y, Y2, ldy2, s);
    else if (in_f32 && !y_bf16)
      st = dispatch_ring<float, __nv_bfloat16, float>(ctx, X1, w1, X2, res, rows, width, gamma, beta, eps, Y, Y2,
                                                      ldy2, s);
    else if (!in_f32 && y_bf16 && !(res != nullptr && res_f32))
      st = dispatch_ring<__nv_bfloat16, __nv_bfloat16, __nv_bfloat16>(ctx, X1, w1, X2, res, rows, width, gamma, beta,
                                                                      eps, Y, Y2, ldy2, s);
    if (st != ROCS_ERR_UNSUPPORTED) return st;
  }
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
