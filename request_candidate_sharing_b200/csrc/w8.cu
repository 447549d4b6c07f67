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
//   w8_skinny_kernel    M <= 64 rows: the weight-bound regime the pages report on.  Each CTA owns NT
//                       tiles of 8 output channels and its 8 warps split K.  The tensor-core operands
//                       are f16: one cvt.rn.f16x2.e4m3x2 per weight pair gives the B fragment
//                       exactly, so the weight stream costs one conversion per two bytes.  X is
//                       brought to f16 once, per row with a power-of-two shift that puts the row's
//                       largest magnitude in [2^14, 2^15) (w8_xprep_kernel: exact for every bf16
//                       value within 2^24 of that maximum, no overflow); the epilogue undoes it.  A lane reads 8 consecutive
//                       weight bytes of one channel for eight m16n8k16 MMAs (the MMA's k slots are
//                       permuted so that those 32 bytes are the lane's own: slots 2t+{0,1,8,9} of
//                       MMA j hold k0 + 32t + 4j + {0..3}; the X fragments use the same order), so a
//                       warp step reads whole 128-byte lines of 8 weight rows; each step's X
//                       fragments serve all NT tiles.  Every
//                       weight byte is read from HBM once; the warps' partial sums meet in shared
//                       memory, where the shift, scale, bias, Z[m] and activation are applied.
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
  const __half* Xh;    // [M, K] f16, row m times 2^-shift[m]
  const int* shift;
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

// X [M, K] bf16 -> Xh [M, K] f16 times 2^-shift[m]: shift[m] puts the row's largest magnitude in
// [2^14, 2^15), clamped so that 2^-shift and 2^shift are normal floats.  One CTA per row, two
// activation sets in one launch (rows [0, M0) of set 0, then set 1); K % 8 == 0.
struct XprepSet {
  const __nv_bfloat16* X;
  long long ldx;
  int M, K;
  __half* Xh;
  int* shift;
};

__global__ void __launch_bounds__(256) w8_xprep_kernel(const XprepSet s0, const XprepSet s1) {
  __shared__ float red[8];
  const bool second = (int)blockIdx.x >= s0.M;
  const XprepSet& S = second ? s1 : s0;
  const int r = second ? (int)blockIdx.x - s0.M : (int)blockIdx.x;
  const uint4* x = reinterpret_cast<const uint4*>(S.X + r * S.ldx);
  const int nv = S.K / 8;
  float mx = 0.f;
  for (int i = threadIdx.x; i < nv; i += 256) {
    const uint4 v = __ldg(x + i);
    const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
    for (int j = 0; j < 4; ++j)
      mx = fmaxf(mx, fmaxf(fabsf(__uint_as_float(w[j] << 16)), fabsf(__uint_as_float(w[j] & 0xFFFF0000u))));
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
  if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = mx;
  __syncthreads();
  mx = red[0];
#pragma unroll
  for (int i = 1; i < 8; ++i) mx = fmaxf(mx, red[i]);
  const int sh = mx > 0.f ? min(126, max(-126, (int)((__float_as_uint(mx) >> 23) & 0xFF) - 127 - 14)) : 0;
  if (threadIdx.x == 0) S.shift[r] = sh;
  const float mul = __uint_as_float((uint32_t)(127 - sh) << 23);
  uint4* xh = reinterpret_cast<uint4*>(S.Xh + (long long)r * S.K);
  for (int i = threadIdx.x; i < nv; i += 256) {
    const uint4 v = __ldg(x + i);
    const uint32_t w[4] = {v.x, v.y, v.z, v.w};
    uint32_t o[4];
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const float lo = __uint_as_float(w[j] << 16) * mul, hi = __uint_as_float(w[j] & 0xFFFF0000u) * mul;
      asm("cvt.rn.f16x2.f32 %0, %1, %2;" : "=r"(o[j]) : "f"(hi), "f"(lo));
    }
    xh[i] = make_uint4(o[0], o[1], o[2], o[3]);
  }
}

__device__ __forceinline__ uint32_t e4m3x2_to_f16x2(uint16_t v) {
  uint32_t h;
  asm("cvt.rn.f16x2.e4m3x2 %0, %1;" : "=r"(h) : "h"(v));
  return h;
}

template <int MT, int NT>
__global__ void __launch_bounds__(SK_WARPS * 32) w8_skinny_kernel(const SkinnyArgs a) {
  __shared__ float red[SK_WARPS][MT * NT][32][4];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int g = lane >> 2, t = lane & 3;
  const int n0 = blockIdx.x * (SK_COLS * NT);
  // k range of this warp: K split in 128-wide steps (a 128-byte line of every weight row), as
  // evenly as possible; a lane owns bytes [32t, 32t + 32) of the step, i.e. four MMAs' worth of
  // its slots: MMA j (0..7) takes k = k0 + 32t + 4j + {0, 1, 2, 3} in slots 2t + {0, 1, 8, 9}
  const int steps = a.K / 128;
  const int s0 = steps * warp / SK_WARPS, s1 = steps * (warp + 1) / SK_WARPS;
  float acc[MT][NT][4];
#pragma unroll
  for (int mt = 0; mt < MT; ++mt)
#pragma unroll
    for (int nt = 0; nt < NT; ++nt) acc[mt][nt][0] = acc[mt][nt][1] = acc[mt][nt][2] = acc[mt][nt][3] = 0.f;
  // weights of the next step are loaded before this step's MMAs (two register sets)
  uint4 wcur[NT][2], wnxt[NT][2];
  auto load_w = [&](int st, uint4 (&w)[NT][2]) {
#pragma unroll
    for (int nt = 0; nt < NT; ++nt) {
      const int n = n0 + nt * SK_COLS + g;
      w[nt][0] = w[nt][1] = make_uint4(0u, 0u, 0u, 0u);
      if (n < a.N && st < s1) {
        const uint4* wp = reinterpret_cast<const uint4*>(a.W8 + (long long)n * a.K + st * 128 + 32 * t);
        w[nt][0] = __ldg(wp);
        w[nt][1] = __ldg(wp + 1);
      }
    }
  };
  load_w(s0, wcur);
  for (int st = s0; st < s1; ++st) {
    const int k0 = st * 128 + 32 * t;
    load_w(st + 1, wnxt);
    // X fragments of this lane's 32 k for every m tile (f16 pairs), reused by all NT column tiles
    uint32_t xr[MT][2][16];
#pragma unroll
    for (int mt = 0; mt < MT; ++mt)
#pragma unroll
      for (int h = 0; h < 2; ++h) {
        const int r = mt * 16 + g + 8 * h;
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          uint4 v = make_uint4(0u, 0u, 0u, 0u);
          if (r < a.M) v = __ldg(reinterpret_cast<const uint4*>(a.Xh + (long long)r * a.K + k0 + 8 * q));
          xr[mt][h][4 * q] = v.x; xr[mt][h][4 * q + 1] = v.y; xr[mt][h][4 * q + 2] = v.z; xr[mt][h][4 * q + 3] = v.w;
        }
      }
#pragma unroll
    for (int nt = 0; nt < NT; ++nt) {
      const uint4 w0 = wcur[nt][0], w1 = wcur[nt][1];
      const uint32_t wb[8] = {w0.x, w0.y, w0.z, w0.w, w1.x, w1.y, w1.z, w1.w};
#pragma unroll
      for (int j = 0; j < 8; ++j) {
        // MMA j: k = k0 + 4j + {0,1} in slots 2t, 2t+1 (b0 / a0, a1) and + {2,3} in slots 2t+8, 2t+9
        const uint32_t b0 = e4m3x2_to_f16x2((uint16_t)(wb[j] & 0xFFFFu));
        const uint32_t b1 = e4m3x2_to_f16x2((uint16_t)(wb[j] >> 16));
#pragma unroll
        for (int mt = 0; mt < MT; ++mt) {
          const uint32_t fa[4] = {xr[mt][0][2 * j], xr[mt][1][2 * j], xr[mt][0][2 * j + 1], xr[mt][1][2 * j + 1]};
          mma_f16_16816(acc[mt][nt], fa, b0, b1);
        }
      }
    }
#pragma unroll
    for (int nt = 0; nt < NT; ++nt) {
      wcur[nt][0] = wnxt[nt][0];
      wcur[nt][1] = wnxt[nt][1];
    }
  }
#pragma unroll
  for (int mt = 0; mt < MT; ++mt)
#pragma unroll
    for (int nt = 0; nt < NT; ++nt)
#pragma unroll
      for (int e = 0; e < 4; ++e) red[warp][mt * NT + nt][lane][e] = acc[mt][nt][e];
  __syncthreads();
  // every thread finishes output elements: (tile, lane, e) -> row mt*16 + g + 8 (e >> 1),
  // column n0 + nt*8 + 2t + (e & 1)
  for (int idx = threadIdx.x; idx < MT * NT * 32 * 4; idx += SK_WARPS * 32) {
    const int tile = idx / 128, ln = (idx >> 2) & 31, e = idx & 3;
    const int mt = tile / NT, nt = tile - mt * NT;
    const int row = mt * 16 + (ln >> 2) + 8 * (e >> 1);
    const int col = n0 + nt * SK_COLS + 2 * (ln & 3) + (e & 1);
    if (row >= a.M || col >= a.N) continue;
    float v = 0.f;
#pragma unroll
    for (int w = 0; w < SK_WARPS; ++w) v += red[w][tile][ln][e];
    v = v * __uint_as_float((uint32_t)(127 + a.shift[row]) << 23) * a.scale[col];
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

template <int MT>
void launch_skinny_mt(const SkinnyArgs& a, int num_sms, cudaStream_t s) {
  // column tiles per CTA: as many as keep the grid at one CTA per SM or more (X fragments are
  // loaded once per k step and reused by every column tile), at most 8 / MT (registers)
  constexpr int NT_MAX = MT == 1 ? 8 : MT == 2 ? 4 : 2;
  int nt = NT_MAX;
  while (nt > 1 && (a.N + SK_COLS * nt - 1) / (SK_COLS * nt) < num_sms) nt >>= 1;
  const unsigned grid = (unsigned)((a.N + SK_COLS * nt - 1) / (SK_COLS * nt));
  switch (nt) {
    case 8: w8_skinny_kernel<MT, (NT_MAX >= 8 ? 8 : 1)><<<grid, SK_WARPS * 32, 0, s>>>(a); break;
    case 4: w8_skinny_kernel<MT, (NT_MAX >= 4 ? 4 : 1)><<<grid, SK_WARPS * 32, 0, s>>>(a); break;
    case 2: w8_skinny_kernel<MT, 2><<<grid, SK_WARPS * 32, 0, s>>>(a); break;
    default: w8_skinny_kernel<MT, 1><<<grid, SK_WARPS * 32, 0, s>>>(a); break;
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

bool w8_skinny_supported(int M, int K) { return M >= 1 && M <= 16 * SK_MAX_MT && K % 128 == 0 && K >= 128; }

rocs_status launch_w8_xprep(const void* X0, long long ldx0, int M0, int K0, void* Xh0, int* sh0, const void* X1,
                            long long ldx1, int M1, int K1, void* Xh1, int* sh1, cudaStream_t s) {
  if (M0 + M1 == 0) return ROCS_OK;
  if (((uintptr_t)X0 & 15) || ldx0 % 8 || K0 % 8 || (M1 > 0 && (((uintptr_t)X1 & 15) || ldx1 % 8 || K1 % 8))) {
    set_error("w8 activation prep: rows must be 16-byte aligned multiples of 8 values");
    return ROCS_ERR_UNSUPPORTED;
  }
  XprepSet a{(const __nv_bfloat16*)X0, ldx0, M0, K0, (__half*)Xh0, sh0};
  XprepSet b{(const __nv_bfloat16*)X1, ldx1, M1, K1, (__half*)Xh1, sh1};
  LaunchTimer lt_("w8_xprep", s);
  w8_xprep_kernel<<<(unsigned)(M0 + M1), 256, 0, s>>>(a, b);
  return cuda_check(cudaGetLastError(), "w8_xprep_kernel");
}

rocs_status launch_w8_skinny(rocs_context* ctx, const void* Xh, const int* shift, int M, int K, const uint8_t* W8,
                             int N, const float* scale, const float* bias, const float* Z, long long ldz,
                             const int32_t* gidx, int gidx_bound, void* out, long long ldo, int out_bf16, int act,
                             cudaStream_t s) {
  if (M == 0 || N == 0) return ROCS_OK;
  if (!w8_skinny_supported(M, K) || ((uintptr_t)Xh & 15) || ((uintptr_t)W8 & 7)) {
    set_error("w8 skinny GEMM: unsupported M=%d K=%d or alignment", M, K);
    return ROCS_ERR_UNSUPPORTED;
  }
  SkinnyArgs a;
  a.Xh = (const __half*)Xh; a.shift = shift; a.M = M; a.K = K; a.N = N; a.W8 = W8; a.scale = scale; a.bias = bias;
  a.Z = Z; a.ldz = ldz; a.gidx = gidx; a.gidx_bound = gidx_bound; a.out = out; a.ldo = ldo; a.out_bf16 = out_bf16;
  a.act = act; a.status = ctx->d_status;
  LaunchTimer lt_("w8_skinny", s);
  const int mt = (M + 15) / 16;
  switch (mt) {
    case 1: launch_skinny_mt<1>(a, ctx->num_sms, s); break;
    case 2: launch_skinny_mt<2>(a, ctx->num_sms, s); break;
    case 3: launch_skinny_mt<3>(a, ctx->num_sms, s); break;
    default: launch_skinny_mt<4>(a, ctx->num_sms, s); break;
  }
  return cuda_check(cudaGetLastError(), "w8_skinny_kernel");
}

}  // namespace rocs
