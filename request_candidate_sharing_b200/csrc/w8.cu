// FP8-weight (W8A16) linears ("Compute Only Once: UG-Separation ...", §三 Stage 4 and the W8A16
// table of §六: 8-bit floating-point weights, bf16 activations, dequantisation cost negligible).
//
// Weights are E4M3 bytes [out, in] with one float32 scale per output channel; the linear is
// y_o = act(s_o * sum_i q_oi x_i + b_o (+ Z[m]_o)), the scale applied to the fp32 accumulator.
//
//   w8_quantize_kernel  one warp per weight row: s = max|w| / 448 (1 for a zero row), q = E4M3(w / s)
//                       rounded to nearest even and saturated (cvt.rn.satfinite).
//   w8_expand_kernel    E4M3 -> bf16, exactly (every E4M3 value is a bf16 value); the large-M path
//                       feeds the result to the tcgen05 GEMM, which applies the scales.
//   w8_skinny_kernel    M <= 64 rows: the weight-bound regime the pages report on.  Each CTA owns 8
//                       output channels, its 8 warps split K; a lane reads 8 consecutive weight bytes
//                       of one channel and turns them into the bf16 B fragments of two m16n8k16 MMAs
//                       (the MMA's k slots are permuted so that those 8 bytes are the lane's own:
//                       slot 2t+{0,1,8,9} of the first MMA and of the second hold k0 + 8t + {0..3}
//                       and {4..7}; the X fragments use the same order).  Every weight byte is read
//                       from HBM once; the warps' partial sums meet in shared memory, where the
//                       scale, bias, Z[m] and activation are applied.
#include <algorithm>

#include "common.cuh"
#include "internal.h"
#include "mma_frag.cuh"

namespace rocs {
namespace {

constexpr float kE4M3Max = 448.0f;
constexpr int SK_WARPS = 8;
constexpr int SK_COLS = 8;
constexpr int SK_MAX_MT = 4;   // 64 rows

__device__ __forceinline__ uint32_t e4m3x2_to_bf16x2(uint16_t v) {
  uint32_t h;
  asm("cvt.rn.f16x2.e4m3x2 %0, %1;" : "=r"(h) : "h"(v));
  const float lo = __half2float(__ushort_as_half((unsigned short)(h & 0xFFFFu)));
  const float hi = __half2float(__ushort_as_half((unsigned short)(h >> 16)));
  uint32_t r;
  asm("cvt.rn.bf16x2.f32 %0, %1, %2;" : "=r"(r) : "f"(hi), "f"(lo));
  return r;
}

__device__ __forceinline__ uint8_t f32_to_e4m3(float x) {
  uint16_t d;
  const float zero = 0.f;
  asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;" : "=h"(d) : "f"(zero), "f"(x));
  return (uint8_t)(d & 0xFFu);
}

template <typename T>
__device__ __forceinline__ float load_w(const T* p);
template <>
__device__ __forceinline__ float load_w<float>(const float* p) { return *p; }
template <>
__device__ __forceinline__ float load_w<__nv_bfloat16>(const __nv_bfloat16* p) { return __bfloat162float(*p); }

template <typename T>
__global__ void w8_quantize_kernel(const T* __restrict__ W, int rows, int cols, uint8_t* __restrict__ Q,
                                   float* __restrict__ scale) {
  const long long r = ((long long)blockIdx.x * blockDim.x + threadIdx.x) >> 5;
  const int lane = threadIdx.x & 31;
  if (r >= rows) return;
  const T* w = W + r * cols;
  float amax = 0.f;
  for (int i = lane; i < cols; i += 32) amax = fmaxf(amax, fabsf(load_w(w + i)));
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, o));
  const float s = amax > 0.f ? amax / kE4M3Max : 1.0f;
  if (lane == 0) scale[r] = s;
  uint8_t* q = Q + r * cols;
  for (int i = lane; i < cols; i += 32) q[i] = f32_to_e4m3(load_w(w + i) / s);
}

__global__ void w8_expand_kernel(const uint16_t* __restrict__ Q2, long long pairs, uint32_t* __restrict__ out) {
  for (long long i = (long long)blockIdx.x * blockDim.x + threadIdx.x; i < pairs; i += (long long)gridDim.x * blockDim.x)
    out[i] = e4m3x2_to_bf16x2(Q2[i]);
}

struct SkinnyArgs {
  const __nv_bfloat16* X;
  long long ldx;
  int M, K, N;
  const uint8_t* W8;   // [N, K]
  const float* scale;
  const float* bias;
  const float* Z;
  long long ldz;
  const int32_t* gidx;
  int gidx_bound;
  void* out;
  long long ldo;
  int out_bf16, act;
  int* status;
};

template <int MT>
__global__ void __launch_bounds__(SK_WARPS * 32) w8_skinny_kernel(const SkinnyArgs a) {
  __shared__ float red[SK_WARPS][MT][32][4];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int g = lane >> 2, t = lane & 3;
  const int n0 = blockIdx.x * SK_COLS;
  const int n = n0 + g;
  // k range of this warp: K split in 32-wide steps, as evenly as possible
  const int steps = a.K / 32;
  const int s0 = steps * warp / SK_WARPS, s1 = steps * (warp + 1) / SK_WARPS;
  float acc[MT][4];
#pragma unroll
  for (int mt = 0; mt < MT; ++mt) acc[mt][0] = acc[mt][1] = acc[mt][2] = acc[mt][3] = 0.f;
  const uint8_t* wrow = a.W8 + (long long)(n < a.N ? n : 0) * a.K;
#pragma unroll 2
  for (int st = s0; st < s1; ++st) {
    const int k0 = st * 32;
    uint2 wq = make_uint2(0u, 0u);
    if (n < a.N) wq = __ldg(reinterpret_cast<const uint2*>(wrow + k0 + 8 * t));
    const uint32_t b0 = e4m3x2_to_bf16x2((uint16_t)(wq.x & 0xFFFFu));
    const uint32_t b1 = e4m3x2_to_bf16x2((uint16_t)(wq.x >> 16));
    const uint32_t c0 = e4m3x2_to_bf16x2((uint16_t)(wq.y & 0xFFFFu));
    const uint32_t c1 = e4m3x2_to_bf16x2((uint16_t)(wq.y >> 16));
#pragma unroll
    for (int mt = 0; mt < MT; ++mt) {
      const int r0 = mt * 16 + g, r1 = r0 + 8;
      uint4 xa = make_uint4(0u, 0u, 0u, 0u), xb = make_uint4(0u, 0u, 0u, 0u);
      if (r0 < a.M) xa = __ldg(reinterpret_cast<const uint4*>(a.X + r0 * a.ldx + k0 + 8 * t));
      if (r1 < a.M) xb = __ldg(reinterpret_cast<const uint4*>(a.X + r1 * a.ldx + k0 + 8 * t));
      const uint32_t fa[4] = {xa.x, xb.x, xa.y, xb.y};
      const uint32_t fb[4] = {xa.z, xb.z, xa.w, xb.w};
      mma_bf16_16816(acc[mt], fa, b0, b1);
      mma_bf16_16816(acc[mt], fb, c0, c1);
    }
  }
#pragma unroll
  for (int mt = 0; mt < MT; ++mt)
#pragma unroll
    for (int e = 0; e < 4; ++e) red[warp][mt][lane][e] = acc[mt][e];
  __syncthreads();
  // every thread finishes output elements: (mt, lane, e) -> row mt*16 + g + 8 (e >> 1), col 2t + (e & 1)
  for (int idx = threadIdx.x; idx < MT * 32 * 4; idx += SK_WARPS * 32) {
    const int mt = idx / 128, ln = (idx >> 2) & 31, e = idx & 3;
    const int row = mt * 16 + (ln >> 2) + 8 * (e >> 1);
    const int col = n0 + 2 * (ln & 3) + (e & 1);
    if (row >= a.M || col >= a.N) continue;
    float v = 0.f;
#pragma unroll
    for (int w = 0; w < SK_WARPS; ++w) v += red[w][mt][ln][e];
    v *= a.scale[col];
    if (a.bias != nullptr) v += a.bias[col];
    if (a.Z != nullptr) {
      const int zi = a.gidx[row];
      if (zi < 0 || zi >= a.gidx_bound) {
        set_status(a.status, ROCS_ERR_INDEX);
        continue;
      }
      v += a.Z[(long long)zi * a.ldz + col];
    }
    switch (a.act) {
      case ROCS_ACT_RELU: v = fmaxf(v, 0.f); break;
      case ROCS_ACT_GELU: v = gelu_erf(v); break;
      case ROCS_ACT_SIGMOID: v = sigmoid_fast(v); break;
      default: break;
    }
    if (a.out_bf16) reinterpret_cast<__nv_bfloat16*>(a.out)[row * a.ldo + col] = __float2bfloat16_rn(v);
    else reinterpret_cast<float*>(a.out)[row * a.ldo + col] = v;
  }
}

}  // namespace

rocs_status launch_w8_quantize(const void* W, int w_bf16, int rows, int cols, uint8_t* Q, float* scale, cudaStream_t s) {
  if (rows == 0 || cols == 0) return ROCS_OK;
  const long long threads = (long long)rows * 32;
  LaunchTimer lt_("w8_quantize", s);
  if (w_bf16)
    w8_quantize_kernel<__nv_bfloat16><<<(unsigned)((threads + 255) / 256), 256, 0, s>>>(
        (const __nv_bfloat16*)W, rows, cols, Q, scale);
  else
    w8_quantize_kernel<float><<<(unsigned)((threads + 255) / 256), 256, 0, s>>>((const float*)W, rows, cols, Q,
                                                                               scale);
  return cuda_check(cudaGetLastError(), "w8_quantize_kernel");
}

rocs_status launch_w8_expand(const uint8_t* Q, long long count, void* out, cudaStream_t s) {
  if (count == 0) return ROCS_OK;
  const long long pairs = count / 2;   // count is even (rows of an even width)
  LaunchTimer lt_("w8_expand", s);
  const unsigned blocks = (unsigned)std::min<long long>((pairs + 255) / 256, 148LL * 16);
  w8_expand_kernel<<<blocks, 256, 0, s>>>((const uint16_t*)Q, pairs, (uint32_t*)out);
  return cuda_check(cudaGetLastError(), "w8_expand_kernel");
}

bool w8_skinny_supported(int M, int K) { return M >= 1 && M <= 16 * SK_MAX_MT && K % 32 == 0 && K >= 32; }

rocs_status launch_w8_skinny(rocs_context* ctx, const void* X, long long ldx, int M, int K, const uint8_t* W8, int N,
                             const float* scale, const float* bias, const float* Z, long long ldz,
                             const int32_t* gidx, int gidx_bound, void* out, long long ldo, int out_bf16, int act,
                             cudaStream_t s) {
  if (M == 0 || N == 0) return ROCS_OK;
  if (!w8_skinny_supported(M, K) || ((uintptr_t)X & 15) || ldx % 8 || ((uintptr_t)W8 & 7)) {
    set_error("w8 skinny GEMM: unsupported M=%d K=%d or alignment", M, K);
    return ROCS_ERR_UNSUPPORTED;
  }
  SkinnyArgs a;
  a.X = (const __nv_bfloat16*)X; a.ldx = ldx; a.M = M; a.K = K; a.N = N; a.W8 = W8; a.scale = scale; a.bias = bias;
  a.Z = Z; a.ldz = ldz; a.gidx = gidx; a.gidx_bound = gidx_bound; a.out = out; a.ldo = ldo; a.out_bf16 = out_bf16;
  a.act = act; a.status = ctx->d_status;
  const unsigned grid = (unsigned)((N + SK_COLS - 1) / SK_COLS);
  LaunchTimer lt_("w8_skinny", s);
  const int mt = (M + 15) / 16;
  switch (mt) {
    case 1: w8_skinny_kernel<1><<<grid, SK_WARPS * 32, 0, s>>>(a); break;
    case 2: w8_skinny_kernel<2><<<grid, SK_WARPS * 32, 0, s>>>(a); break;
    case 3: w8_skinny_kernel<3><<<grid, SK_WARPS * 32, 0, s>>>(a); break;
    default: w8_skinny_kernel<4><<<grid, SK_WARPS * 32, 0, s>>>(a); break;
  }
  return cuda_check(cudaGetLastError(), "w8_skinny_kernel");
}

}  // namespace rocs
