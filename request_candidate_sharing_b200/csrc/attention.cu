// a9 (and the encoder's self-attention in a7): grouped attention against per-request shared K/V.
//
// [REV] §2.2: A^C_i = Attn(Q^C_i, S_i W^C_K, S_i W^C_V) -- every candidate of a request reads the
// same K/V; [REV] §2.4 (IKBO-DCA): the kernel consumes request-batch K/V plus the map directly,
// so candidates of one request hit the same physical K/V instead of a per-candidate copy.
//
// B200 design: one CTA per (request, head[, split of its query rows]).  The CTA copies that
// request/head's K and V (L x d_h bf16 each) into shared memory ONCE (cp.async, zero-padded to a
// multiple of 64 keys) and then its 16 warps sweep all of the request's query rows in 16-row
// tiles: S = Q K^T and O += P V on m16n8k16 tensor-core fragments, online softmax in fp32 with
// exp2 on the MUFU unit.  K/V are read from HBM once per (request, head) no matter how many
// candidates the request has -- the reuse the pages' kernel obtains from L2 locality.
#include <algorithm>

#include "common.cuh"
#include "internal.h"
#include "mma_frag.cuh"

namespace rocs {
namespace {

constexpr int ATT_WARPS = 16;
constexpr int ATT_THREADS = ATT_WARPS * 32;
constexpr int KB = 64;   // keys per inner block

__device__ __forceinline__ float ex2(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

__device__ __forceinline__ void cp_async16(uint32_t saddr, const void* g) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(saddr), "l"(g) : "memory");
}
__device__ __forceinline__ void cp_async_wait_all() { asm volatile("cp.async.wait_all;" ::: "memory"); }

// QSPLIT: each query row holds [hi (H*DH) | lo (H*DH)]; scores use hi*K + lo*K.
template <int DH, bool QSPLIT>
__global__ void __launch_bounds__(ATT_THREADS, 1) attn_kernel(
    const __nv_bfloat16* __restrict__ Q, long long ldq, const __nv_bfloat16* __restrict__ K,
    const __nv_bfloat16* __restrict__ V, long long ldkv, long long kv_req_stride, const int32_t* __restrict__ offsets,
    int B_R, long long rows, int L_all, int H, float scale_log2, void* O, long long ldo, int out_bf16,
    __nv_bfloat16* __restrict__ O2, long long ldo2, int splits, const int32_t* __restrict__ kv_len, int q_by_kv,
    int* status) {
  extern __shared__ __align__(16) uint8_t att_smem[];
  constexpr int PITCH = DH * 2 + 16;
  const int Ls = (L_all + KB - 1) / KB * KB;
  uint8_t* sK = att_smem;
  uint8_t* sV = att_smem + Ls * PITCH;

  const int per_r = H * splits;
  const int r = blockIdx.x / per_r;
  const int rem = blockIdx.x - r * per_r;
  const int h = rem / splits;
  const int sp = rem - h * splits;
  if (r >= B_R) return;
  const long long q0 = offsets[r];
  long long q1 = offsets[r + 1];
  if (q0 < 0 || q1 < q0 || q1 > rows) {
    if (threadIdx.x == 0) set_status(status, ROCS_ERR_INDEX);
    return;
  }
  // this request's keys: the first L of its L_all K/V rows (a ragged history), L in [1, L_all]
  const int L = kv_len != nullptr ? kv_len[r] : L_all;
  if (L < 1 || L > L_all) {
    if (threadIdx.x == 0) set_status(status, ROCS_ERR_COUNTS);
    return;
  }
  if (kv_len != nullptr && q_by_kv) q1 = min(q1, q0 + L);   // ragged self-attention: padding rows ask nothing
  const long long ntiles = (q1 - q0 + 15) / 16;
  const long long t_begin = ntiles * sp / splits, t_end = ntiles * (sp + 1) / splits;
  if (t_begin >= t_end) return;

  // ---- stage K and V of (r, h) once ----
  {
    constexpr int VPR = DH * 2 / 16;   // 16-byte vectors per row
    const __nv_bfloat16* Kb = K + (long long)r * kv_req_stride + h * DH;
    const __nv_bfloat16* Vb = V + (long long)r * kv_req_stride + h * DH;
    const uint32_t sKa = smem_u32(sK), sVa = smem_u32(sV);
    for (int i = threadIdx.x; i < Ls * VPR; i += ATT_THREADS) {
      const int l = i / VPR, v = i - l * VPR;
      const uint32_t off = l * PITCH + v * 16;
      if (l < L) {
        cp_async16(sKa + off, Kb + (long long)l * ldkv + v * 8);
        cp_async16(sVa + off, Vb + (long long)l * ldkv + v * 8);
      } else {
        *reinterpret_cast<uint4*>(sK + off) = make_uint4(0, 0, 0, 0);
        *reinterpret_cast<uint4*>(sV + off) = make_uint4(0, 0, 0, 0);
      }
    }
    cp_async_wait_all();
    __syncthreads();
  }

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int g = lane >> 2, t = lane & 3;
  const uint32_t sKa = smem_u32(sK), sVa = smem_u32(sV);

  for (long long tile = t_begin + warp; tile < t_end; tile += ATT_WARPS) {
    const long long qr0 = q0 + tile * 16;
    const long long ra = qr0 + g, rb = qr0 + g + 8;
    const bool va = ra < q1, vb = rb < q1;
    // Q fragments straight from global (each query row is read once).
    uint32_t qa[DH / 16][4];
    uint32_t ql[QSPLIT ? DH / 16 : 1][4];
    const long long lo_off = (long long)H * DH;
#pragma unroll
    for (int ks = 0; ks < DH / 16; ++ks) {
      const int c0 = h * DH + ks * 16 + 2 * t;
      const uint32_t* pa = reinterpret_cast<const uint32_t*>(Q + ra * ldq + c0);
      const uint32_t* pb = reinterpret_cast<const uint32_t*>(Q + rb * ldq + c0);
      qa[ks][0] = va ? __ldg(pa) : 0u;
      qa[ks][1] = vb ? __ldg(pb) : 0u;
      qa[ks][2] = va ? __ldg(pa + 4) : 0u;
      qa[ks][3] = vb ? __ldg(pb + 4) : 0u;
      if (QSPLIT) {
        const uint32_t* la = reinterpret_cast<const uint32_t*>(Q + ra * ldq + lo_off + c0);
        const uint32_t* lb = reinterpret_cast<const uint32_t*>(Q + rb * ldq + lo_off + c0);
        ql[ks][0] = va ? __ldg(la) : 0u;
        ql[ks][1] = vb ? __ldg(lb) : 0u;
        ql[ks][2] = va ? __ldg(la + 4) : 0u;
        ql[ks][3] = vb ? __ldg(lb + 4) : 0u;
      }
    }
    float o[DH / 8][4];
#pragma unroll
    for (int i = 0; i < DH / 8; ++i)
#pragma unroll
      for (int j = 0; j < 4; ++j) o[i][j] = 0.f;
    float m_a = -INFINITY, m_b = -INFINITY, l_a = 0.f, l_b = 0.f;

    for (int k0 = 0; k0 < Ls; k0 += KB) {
      float s[KB / 8][4];
#pragma unroll
      for (int i = 0; i < KB / 8; ++i)
#pragma unroll
        for (int j = 0; j < 4; ++j) s[i][j] = 0.f;
#pragma unroll
      for (int ks = 0; ks < DH / 16; ++ks) {
#pragma unroll
        for (int np = 0; np < KB / 16; ++np) {
          uint32_t b[4];
          load_b_frag_nmajor_x2(sKa, PITCH, k0 + np * 16, ks * 16, b);
          mma_bf16_16816(s[2 * np], qa[ks], b[0], b[1]);
          mma_bf16_16816(s[2 * np + 1], qa[ks], b[2], b[3]);
          if (QSPLIT) {
            mma_bf16_16816(s[2 * np], ql[ks], b[0], b[1]);
            mma_bf16_16816(s[2 * np + 1], ql[ks], b[2], b[3]);
          }
        }
      }
      // scale into the log2 domain, mask keys >= L, running max
      float mx_a = -INFINITY, mx_b = -INFINITY;
#pragma unroll
      for (int nt = 0; nt < KB / 8; ++nt) {
        const int key = k0 + nt * 8 + 2 * t;
        const bool k0ok = key < L, k1ok = key + 1 < L;
        s[nt][0] = k0ok ? s[nt][0] * scale_log2 : -INFINITY;
        s[nt][1] = k1ok ? s[nt][1] * scale_log2 : -INFINITY;
        s[nt][2] = k0ok ? s[nt][2] * scale_log2 : -INFINITY;
        s[nt][3] = k1ok ? s[nt][3] * scale_log2 : -INFINITY;
        mx_a = fmaxf(mx_a, fmaxf(s[nt][0], s[nt][1]));
        mx_b = fmaxf(mx_b, fmaxf(s[nt][2], s[nt][3]));
      }
      mx_a = fmaxf(mx_a, __shfl_xor_sync(0xffffffffu, mx_a, 1));
      mx_a = fmaxf(mx_a, __shfl_xor_sync(0xffffffffu, mx_a, 2));
      mx_b = fmaxf(mx_b, __shfl_xor_sync(0xffffffffu, mx_b, 1));
      mx_b = fmaxf(mx_b, __shfl_xor_sync(0xffffffffu, mx_b, 2));
      const float mn_a = fmaxf(m_a, mx_a), mn_b = fmaxf(m_b, mx_b);
      const float corr_a = ex2(m_a - mn_a), corr_b = ex2(m_b - mn_b);
      m_a = mn_a;
      m_b = mn_b;
      float rs_a = 0.f, rs_b = 0.f;
      uint32_t pa[KB / 16][4];
#pragma unroll
      for (int nt = 0; nt < KB / 8; ++nt) {
        const float p0 = ex2(s[nt][0] - mn_a), p1 = ex2(s[nt][1] - mn_a);
        const float p2 = ex2(s[nt][2] - mn_b), p3 = ex2(s[nt][3] - mn_b);
        rs_a += p0 + p1;
        rs_b += p2 + p3;
        const int j = nt >> 1;
        if ((nt & 1) == 0) {
          pa[j][0] = pack_bf16x2(p0, p1);
          pa[j][1] = pack_bf16x2(p2, p3);
        } else {
          pa[j][2] = pack_bf16x2(p0, p1);
          pa[j][3] = pack_bf16x2(p2, p3);
        }
      }
      l_a = l_a * corr_a + rs_a;
      l_b = l_b * corr_b + rs_b;
#pragma unroll
      for (int i = 0; i < DH / 8; ++i) {
        o[i][0] *= corr_a; o[i][1] *= corr_a;
        o[i][2] *= corr_b; o[i][3] *= corr_b;
      }
#pragma unroll
      for (int j = 0; j < KB / 16; ++j) {
#pragma unroll
        for (int dp = 0; dp < DH / 16; ++dp) {
          uint32_t b[4];
          load_b_frag_kmajor_x2(sVa, PITCH, k0 + j * 16, dp * 16, b);
          mma_bf16_16816(o[2 * dp], pa[j], b[0], b[1]);
          mma_bf16_16816(o[2 * dp + 1], pa[j], b[2], b[3]);
        }
      }
    }
    l_a += __shfl_xor_sync(0xffffffffu, l_a, 1);
    l_a += __shfl_xor_sync(0xffffffffu, l_a, 2);
    l_b += __shfl_xor_sync(0xffffffffu, l_b, 1);
    l_b += __shfl_xor_sync(0xffffffffu, l_b, 2);
    const float ia = 1.0f / l_a, ib = 1.0f / l_b;
#pragma unroll
    for (int i = 0; i < DH / 8; ++i) {
      const int col = h * DH + i * 8 + 2 * t;
      if (out_bf16) {
        __nv_bfloat16* Ob = reinterpret_cast<__nv_bfloat16*>(O);
        if (va) *reinterpret_cast<uint32_t*>(Ob + ra * ldo + col) = pack_bf16x2(o[i][0] * ia, o[i][1] * ia);
        if (vb) *reinterpret_cast<uint32_t*>(Ob + rb * ldo + col) = pack_bf16x2(o[i][2] * ib, o[i][3] * ib);
      } else {
        float* Of = reinterpret_cast<float*>(O);
        if (va) *reinterpret_cast<float2*>(Of + ra * ldo + col) = make_float2(o[i][0] * ia, o[i][1] * ia);
        if (vb) *reinterpret_cast<float2*>(Of + rb * ldo + col) = make_float2(o[i][2] * ib, o[i][3] * ib);
      }
      if (O2 != nullptr) {
        if (va) *reinterpret_cast<uint32_t*>(O2 + ra * ldo2 + col) = pack_bf16x2(o[i][0] * ia, o[i][1] * ia);
        if (vb) *reinterpret_cast<uint32_t*>(O2 + rb * ldo2 + col) = pack_bf16x2(o[i][2] * ib, o[i][3] * ib);
      }
    }
  }
}

}  // namespace

rocs_status launch_attention(rocs_context* ctx, const void* Q, long long ldq, int q_split, const void* K,
                             const void* V, long long ldkv, long long kv_req_stride, const int32_t* offsets, int B_R,
                             long long rows, int L, int H, int d_h, float scale, void* O, long long ldo, int out_bf16,
                             void* O2, long long ldo2, cudaStream_t s, const int32_t* kv_len, int q_by_kv) {
  if (B_R == 0 || rows == 0) return ROCS_OK;
  const int Ls = (L + KB - 1) / KB * KB;
  const int pitch = d_h * 2 + 16;
  const int smem = 2 * Ls * pitch;
  if (smem > 227 * 1024) {
    set_error("attention: L=%d d_h=%d needs %d B of shared memory", L, d_h, smem);
    return ROCS_ERR_UNSUPPORTED;
  }
  static bool attr[64][4] = {{false}};
  const int which = (d_h == 32 ? 0 : 2) + (q_split ? 1 : 0);
  if (ctx->device < 64 && !attr[ctx->device][which]) {
    cudaError_t e;
    switch (which) {
      case 0: e = cudaFuncSetAttribute(attn_kernel<32, false>, cudaFuncAttributeMaxDynamicSharedMemorySize, 227 * 1024); break;
      case 1: e = cudaFuncSetAttribute(attn_kernel<32, true>, cudaFuncAttributeMaxDynamicSharedMemorySize, 227 * 1024); break;
      case 2: e = cudaFuncSetAttribute(attn_kernel<64, false>, cudaFuncAttributeMaxDynamicSharedMemorySize, 227 * 1024); break;
      default: e = cudaFuncSetAttribute(attn_kernel<64, true>, cudaFuncAttributeMaxDynamicSharedMemorySize, 227 * 1024); break;
    }
    rocs_status st = cuda_check(e, "cudaFuncSetAttribute(attention)");
    if (st != ROCS_OK) return st;
    attr[ctx->device][which] = true;
  }
  const long long groups = (long long)B_R * H;
  int splits = (int)std::max<long long>(1, (2LL * ctx->num_sms + groups - 1) / groups);
  splits = std::min(splits, 64);
  const long long grid = groups * splits;
  if (grid > 2147483647LL) {
    set_error("attention: grid too large");
    return ROCS_ERR_UNSUPPORTED;
  }
  const float scale_log2 = scale * 1.4426950408889634f;
#define ROCS_ATT(DH, SPLIT)                                                                                         \
  attn_kernel<DH, SPLIT><<<(unsigned)grid, ATT_THREADS, smem, s>>>(                                                 \
      (const __nv_bfloat16*)Q, ldq, (const __nv_bfloat16*)K, (const __nv_bfloat16*)V, ldkv, kv_req_stride, offsets, \
      B_R, rows, L, H, scale_log2, O, ldo, out_bf16, (__nv_bfloat16*)O2, ldo2, splits, kv_len, q_by_kv,         \
      ctx->d_status)
  LaunchTimer lt_("attn", s);
  switch (which) {
    case 0: ROCS_ATT(32, false); break;
    case 1: ROCS_ATT(32, true); break;
    case 2: ROCS_ATT(64, false); break;
    default: ROCS_ATT(64, true); break;
  }
#undef ROCS_ATT
  return cuda_check(cudaGetLastError(), "attn_kernel");
}

}  // namespace rocs
