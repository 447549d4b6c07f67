// a9: candidate and request cross-attention against per-request shared K/V, two variants used by
// the forward ([REV] §2.2 grouped cross-attention; §2.4 IKBO-DCA: the kernel reads request-batch
// K/V plus the map, candidates of one request share the physical K/V).
//
// attn_stream_kernel (candidate queries): a CTA takes 128-query chunks of one (request, head)
// (chunks s, s + S, s + 2S, ... of that request) and streams the request's K/V through a
// double-buffered 64-key ring in shared memory (cp.async), so several CTAs share an SM and the
// copy of one key block overlaps the math of the previous one.  Each warp carries two 16-row
// query tiles, so every K/V fragment read from shared memory serves 32 queries.  S = Q K^T and
// O += P V on m16n8k16 tensor-core fragments, online softmax in fp32 with exp2 on the MUFU unit.
//
// attn_q1_kernel (one query row per request, the request-side cross-attention): a CTA per
// (request, head) reads that head's K/V straight from HBM once, one key per thread; the scores,
// the softmax and the weighted V sum are block reductions in fp32.
#include <algorithm>

#include "common.cuh"
#include "internal.h"
#include "mma_frag.cuh"

namespace rocs {
namespace {

constexpr int KB = 64;   // keys per block
constexpr int ST_WARPS = 4;
constexpr int ST_TPW = 2;
constexpr int ST_ROWS = ST_WARPS * ST_TPW * 16;

__device__ __forceinline__ void cp_async16(uint32_t saddr, const void* g) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(saddr), "l"(g) : "memory");
}

template <int DH, bool QSPLIT>
__global__ void __launch_bounds__(ST_WARPS * 32, 3) attn_stream_kernel(
    const __nv_bfloat16* __restrict__ Q, long long ldq, const __nv_bfloat16* __restrict__ K,
    const __nv_bfloat16* __restrict__ V, long long ldkv, long long kv_req_stride, const int32_t* __restrict__ offsets,
    int B_R, long long rows, int L_all, int H, float scale_log2, void* O, long long ldo, int out_bf16,
    __nv_bfloat16* __restrict__ O2, long long ldo2, int S, const int32_t* __restrict__ kv_len, int q_by_kv,
    int* status) {
  constexpr int PITCH = DH * 2 + 16;
  constexpr int KV_BYTES = KB * PITCH;   // one 64-key block of K (or V)
  constexpr int VPR = DH * 2 / 16;
  __shared__ __align__(16) uint8_t ring[2][2][KV_BYTES];
  const int per_r = H * S;
  const int r = blockIdx.x / per_r;
  const int rem = blockIdx.x - r * per_r;
  const int h = rem / S;
  const int sidx = rem - h * S;
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
  const long long nch = (q1 - q0 + ST_ROWS - 1) / ST_ROWS;
  if (sidx >= nch) return;
  const int nkb = (L + KB - 1) / KB;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int g = lane >> 2, t = lane & 3;
  const __nv_bfloat16* Kb = K + (long long)r * kv_req_stride + h * DH;
  const __nv_bfloat16* Vb = V + (long long)r * kv_req_stride + h * DH;
  const long long lo_off = (long long)H * DH;

  auto issue = [&](int kb, int st) {
    const uint32_t sK = smem_u32(ring[st][0]), sV = smem_u32(ring[st][1]);
    for (int i = threadIdx.x; i < KB * VPR; i += ST_WARPS * 32) {
      const int lr = i / VPR, v = i - lr * VPR;
      const int l = kb * KB + lr;
      const uint32_t off = lr * PITCH + v * 16;
      if (l < L) {
        cp_async16(sK + off, Kb + (long long)l * ldkv + v * 8);
        cp_async16(sV + off, Vb + (long long)l * ldkv + v * 8);
      } else {
        *reinterpret_cast<uint4*>(ring[st][0] + off) = make_uint4(0, 0, 0, 0);
        *reinterpret_cast<uint4*>(ring[st][1] + off) = make_uint4(0, 0, 0, 0);
      }
    }
    asm volatile("cp.async.commit_group;" ::: "memory");
  };

  for (long long ch = sidx; ch < nch; ch += S) {
    long long ra[ST_TPW], rb[ST_TPW];
    bool va[ST_TPW], vb[ST_TPW];
    uint32_t qa[ST_TPW][DH / 16][4];
    uint32_t ql[ST_TPW][QSPLIT ? DH / 16 : 1][4];
    float o[ST_TPW][DH / 8][4];
    float m_a[ST_TPW], m_b[ST_TPW], l_a[ST_TPW], l_b[ST_TPW];
#pragma unroll
    for (int tt = 0; tt < ST_TPW; ++tt) {
      const long long qr0 = q0 + ch * ST_ROWS + (warp * ST_TPW + tt) * 16;
      ra[tt] = qr0 + g;
      rb[tt] = qr0 + g + 8;
      va[tt] = ra[tt] < q1;
      vb[tt] = rb[tt] < q1;
#pragma unroll
      for (int ks = 0; ks < DH / 16; ++ks) {
        const int c0 = h * DH + ks * 16 + 2 * t;
        const uint32_t* pa = reinterpret_cast<const uint32_t*>(Q + ra[tt] * ldq + c0);
        const uint32_t* pb = reinterpret_cast<const uint32_t*>(Q + rb[tt] * ldq + c0);
        qa[tt][ks][0] = va[tt] ? __ldg(pa) : 0u;
        qa[tt][ks][1] = vb[tt] ? __ldg(pb) : 0u;
        qa[tt][ks][2] = va[tt] ? __ldg(pa + 4) : 0u;
        qa[tt][ks][3] = vb[tt] ? __ldg(pb + 4) : 0u;
        if (QSPLIT) {
          const uint32_t* la = reinterpret_cast<const uint32_t*>(Q + ra[tt] * ldq + lo_off + c0);
          const uint32_t* lb = reinterpret_cast<const uint32_t*>(Q + rb[tt] * ldq + lo_off + c0);
          ql[tt][ks][0] = va[tt] ? __ldg(la) : 0u;
          ql[tt][ks][1] = vb[tt] ? __ldg(lb) : 0u;
          ql[tt][ks][2] = va[tt] ? __ldg(la + 4) : 0u;
          ql[tt][ks][3] = vb[tt] ? __ldg(lb + 4) : 0u;
        }
      }
#pragma unroll
      for (int i = 0; i < DH / 8; ++i)
#pragma unroll
        for (int j = 0; j < 4; ++j) o[tt][i][j] = 0.f;
      m_a[tt] = m_b[tt] = -INFINITY;
      l_a[tt] = l_b[tt] = 0.f;
    }
    // warp-uniform: rows fill the chunk in order, so a warp whose first row (lane-independent) is
    // past the request's last query has no valid rows.  Every lane of a live warp runs the
    // warp-collective mma.sync / shuffles below; invalid rows only skip their stores.
    const bool warp_live = q0 + ch * ST_ROWS + (long long)warp * ST_TPW * 16 < q1;

    __syncthreads();   // the ring is free (previous chunk finished)
    issue(0, 0);
    for (int kb = 0; kb < nkb; ++kb) {
      if (kb + 1 < nkb) {
        issue(kb + 1, (kb + 1) & 1);
        asm volatile("cp.async.wait_group 1;" ::: "memory");
      } else {
        asm volatile("cp.async.wait_group 0;" ::: "memory");
      }
      __syncthreads();
      if (warp_live) {
        const uint32_t sK = smem_u32(ring[kb & 1][0]), sV = smem_u32(ring[kb & 1][1]);
        const int k0 = kb * KB;
        const bool full = k0 + KB <= L;
        float s[ST_TPW][KB / 8][4];
#pragma unroll
        for (int tt = 0; tt < ST_TPW; ++tt)
#pragma unroll
          for (int i = 0; i < KB / 8; ++i)
#pragma unroll
            for (int j = 0; j < 4; ++j) s[tt][i][j] = 0.f;
#pragma unroll
        for (int ks = 0; ks < DH / 16; ++ks) {
#pragma unroll
          for (int np = 0; np < KB / 16; ++np) {
            uint32_t b[4];
            load_b_frag_nmajor_x2(sK, PITCH, np * 16, ks * 16, b);
#pragma unroll
            for (int tt = 0; tt < ST_TPW; ++tt) {
              mma_bf16_16816(s[tt][2 * np], qa[tt][ks], b[0], b[1]);
              mma_bf16_16816(s[tt][2 * np + 1], qa[tt][ks], b[2], b[3]);
              if (QSPLIT) {
                mma_bf16_16816(s[tt][2 * np], ql[tt][ks], b[0], b[1]);
                mma_bf16_16816(s[tt][2 * np + 1], ql[tt][ks], b[2], b[3]);
              }
            }
          }
        }
        uint32_t pa[ST_TPW][KB / 16][4];
#pragma unroll
        for (int tt = 0; tt < ST_TPW; ++tt) {
          float mx_a = -INFINITY, mx_b = -INFINITY;
#pragma unroll
          for (int nt = 0; nt < KB / 8; ++nt) {
            if (!full) {
              const int key = k0 + nt * 8 + 2 * t;
              if (key >= L) { s[tt][nt][0] = -INFINITY; s[tt][nt][2] = -INFINITY; }
              if (key + 1 >= L) { s[tt][nt][1] = -INFINITY; s[tt][nt][3] = -INFINITY; }
            }
            mx_a = fmaxf(mx_a, fmaxf(s[tt][nt][0], s[tt][nt][1]));
            mx_b = fmaxf(mx_b, fmaxf(s[tt][nt][2], s[tt][nt][3]));
          }
          mx_a = fmaxf(mx_a, __shfl_xor_sync(0xffffffffu, mx_a, 1));
          mx_a = fmaxf(mx_a, __shfl_xor_sync(0xffffffffu, mx_a, 2));
          mx_b = fmaxf(mx_b, __shfl_xor_sync(0xffffffffu, mx_b, 1));
          mx_b = fmaxf(mx_b, __shfl_xor_sync(0xffffffffu, mx_b, 2));
          // running maxima kept in the scaled (log2) domain
          const float mn_a = fmaxf(m_a[tt], mx_a * scale_log2), mn_b = fmaxf(m_b[tt], mx_b * scale_log2);
          const float corr_a = ex2_approx(m_a[tt] - mn_a), corr_b = ex2_approx(m_b[tt] - mn_b);
          m_a[tt] = mn_a;
          m_b[tt] = mn_b;
          float rs_a = 0.f, rs_b = 0.f;
#pragma unroll
          for (int nt = 0; nt < KB / 8; ++nt) {
            const float p0 = ex2_approx(fmaf(s[tt][nt][0], scale_log2, -mn_a));
            const float p1 = ex2_approx(fmaf(s[tt][nt][1], scale_log2, -mn_a));
            const float p2 = ex2_approx(fmaf(s[tt][nt][2], scale_log2, -mn_b));
            const float p3 = ex2_approx(fmaf(s[tt][nt][3], scale_log2, -mn_b));
            rs_a += p0 + p1;
            rs_b += p2 + p3;
            const int j = nt >> 1;
            if ((nt & 1) == 0) {
              pa[tt][j][0] = pack_bf16x2(p0, p1);
              pa[tt][j][1] = pack_bf16x2(p2, p3);
            } else {
              pa[tt][j][2] = pack_bf16x2(p0, p1);
              pa[tt][j][3] = pack_bf16x2(p2, p3);
            }
          }
          l_a[tt] = l_a[tt] * corr_a + rs_a;
          l_b[tt] = l_b[tt] * corr_b + rs_b;
#pragma unroll
          for (int i = 0; i < DH / 8; ++i) {
            o[tt][i][0] *= corr_a; o[tt][i][1] *= corr_a;
            o[tt][i][2] *= corr_b; o[tt][i][3] *= corr_b;
          }
        }
#pragma unroll
        for (int j = 0; j < KB / 16; ++j) {
#pragma unroll
          for (int dp = 0; dp < DH / 16; ++dp) {
            uint32_t b[4];
            load_b_frag_kmajor_x2(sV, PITCH, j * 16, dp * 16, b);
#pragma unroll
            for (int tt = 0; tt < ST_TPW; ++tt) {
              mma_bf16_16816(o[tt][2 * dp], pa[tt][j], b[0], b[1]);
              mma_bf16_16816(o[tt][2 * dp + 1], pa[tt][j], b[2], b[3]);
            }
          }
        }
      }
      __syncthreads();   // everyone is done with this stage before it is refilled
    }
    if (warp_live) {
#pragma unroll
      for (int tt = 0; tt < ST_TPW; ++tt) {
        float la = l_a[tt], lb = l_b[tt];
        la += __shfl_xor_sync(0xffffffffu, la, 1);
        la += __shfl_xor_sync(0xffffffffu, la, 2);
        lb += __shfl_xor_sync(0xffffffffu, lb, 1);
        lb += __shfl_xor_sync(0xffffffffu, lb, 2);
        const float ia = 1.0f / la, ib = 1.0f / lb;
#pragma unroll
        for (int i = 0; i < DH / 8; ++i) {
          const int col = h * DH + i * 8 + 2 * t;
          const float a0 = o[tt][i][0] * ia, a1 = o[tt][i][1] * ia, b0 = o[tt][i][2] * ib, b1 = o[tt][i][3] * ib;
          if (out_bf16) {
            __nv_bfloat16* Ob = reinterpret_cast<__nv_bfloat16*>(O);
            if (va[tt]) *reinterpret_cast<uint32_t*>(Ob + ra[tt] * ldo + col) = pack_bf16x2(a0, a1);
            if (vb[tt]) *reinterpret_cast<uint32_t*>(Ob + rb[tt] * ldo + col) = pack_bf16x2(b0, b1);
          } else {
            float* Of = reinterpret_cast<float*>(O);
            if (va[tt]) *reinterpret_cast<float2*>(Of + ra[tt] * ldo + col) = make_float2(a0, a1);
            if (vb[tt]) *reinterpret_cast<float2*>(Of + rb[tt] * ldo + col) = make_float2(b0, b1);
          }
          if (O2 != nullptr) {
            if (va[tt]) *reinterpret_cast<uint32_t*>(O2 + ra[tt] * ldo2 + col) = pack_bf16x2(a0, a1);
            if (vb[tt]) *reinterpret_cast<uint32_t*>(O2 + rb[tt] * ldo2 + col) = pack_bf16x2(b0, b1);
          }
        }
      }
    }
  }
}

constexpr int Q1_THREADS = 128;
constexpr int Q1_KPT = 8;   // keys per thread: L <= 1024

template <int DH, bool QSPLIT>
__global__ void __launch_bounds__(Q1_THREADS) attn_q1_kernel(
    const __nv_bfloat16* __restrict__ Q, long long ldq, const __nv_bfloat16* __restrict__ K,
    const __nv_bfloat16* __restrict__ V, long long ldkv, long long kv_req_stride, const int32_t* __restrict__ offsets,
    int B_R, long long rows, int L_all, int H, float scale_log2, void* O, long long ldo, int out_bf16,
    __nv_bfloat16* __restrict__ O2, long long ldo2, const int32_t* __restrict__ kv_len, int* status) {
  __shared__ float sq[DH];
  __shared__ float red[Q1_THREADS / 32][DH];
  __shared__ float rmax[Q1_THREADS / 32], rsum[Q1_THREADS / 32];
  const int r = blockIdx.x / H;
  const int h = blockIdx.x - r * H;
  if (r >= B_R) return;
  const long long q0 = offsets[r], q1 = offsets[r + 1];
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
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const __nv_bfloat16* Kb = K + (long long)r * kv_req_stride + h * DH;
  const __nv_bfloat16* Vb = V + (long long)r * kv_req_stride + h * DH;
  for (long long q = q0; q < q1; ++q) {
    __syncthreads();
    if (tid < DH) {
      float v = __bfloat162float(Q[q * ldq + h * DH + tid]);
      if (QSPLIT) v += __bfloat162float(Q[q * ldq + (long long)H * DH + h * DH + tid]);
      sq[tid] = v;
    }
    __syncthreads();
    float sc[Q1_KPT];
    float mx = -INFINITY;
#pragma unroll
    for (int i = 0; i < Q1_KPT; ++i) {
      const int l = tid + i * Q1_THREADS;
      sc[i] = -INFINITY;
      if (l < L) {
        const uint4* kp = reinterpret_cast<const uint4*>(Kb + (long long)l * ldkv);
        float acc = 0.f;
#pragma unroll
        for (int v = 0; v < DH / 8; ++v) {
          const uint4 u = __ldg(kp + v);
          acc = fmaf(sq[8 * v + 0], bf16_lo(u.x), acc); acc = fmaf(sq[8 * v + 1], bf16_hi(u.x), acc);
          acc = fmaf(sq[8 * v + 2], bf16_lo(u.y), acc); acc = fmaf(sq[8 * v + 3], bf16_hi(u.y), acc);
          acc = fmaf(sq[8 * v + 4], bf16_lo(u.z), acc); acc = fmaf(sq[8 * v + 5], bf16_hi(u.z), acc);
          acc = fmaf(sq[8 * v + 6], bf16_lo(u.w), acc); acc = fmaf(sq[8 * v + 7], bf16_hi(u.w), acc);
        }
        sc[i] = acc * scale_log2;
        mx = fmaxf(mx, sc[i]);
      }
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
    if (lane == 0) rmax[warp] = mx;
    __syncthreads();
    mx = rmax[0];
#pragma unroll
    for (int w = 1; w < Q1_THREADS / 32; ++w) mx = fmaxf(mx, rmax[w]);
    float acc[DH];
#pragma unroll
    for (int e = 0; e < DH; ++e) acc[e] = 0.f;
    float sum = 0.f;
#pragma unroll
    for (int i = 0; i < Q1_KPT; ++i) {
      const int l = tid + i * Q1_THREADS;
      if (l < L) {
        const float p = ex2_approx(sc[i] - mx);
        sum += p;
        const uint4* vp = reinterpret_cast<const uint4*>(Vb + (long long)l * ldkv);
#pragma unroll
        for (int v = 0; v < DH / 8; ++v) {
          const uint4 u = __ldg(vp + v);
          acc[8 * v + 0] = fmaf(p, bf16_lo(u.x), acc[8 * v + 0]); acc[8 * v + 1] = fmaf(p, bf16_hi(u.x), acc[8 * v + 1]);
          acc[8 * v + 2] = fmaf(p, bf16_lo(u.y), acc[8 * v + 2]); acc[8 * v + 3] = fmaf(p, bf16_hi(u.y), acc[8 * v + 3]);
          acc[8 * v + 4] = fmaf(p, bf16_lo(u.z), acc[8 * v + 4]); acc[8 * v + 5] = fmaf(p, bf16_hi(u.z), acc[8 * v + 5]);
          acc[8 * v + 6] = fmaf(p, bf16_lo(u.w), acc[8 * v + 6]); acc[8 * v + 7] = fmaf(p, bf16_hi(u.w), acc[8 * v + 7]);
        }
      }
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) sum += __shfl_xor_sync(0xffffffffu, sum, o);
#pragma unroll
    for (int e = 0; e < DH; ++e) {
      float v = acc[e];
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
      if (lane == 0) red[warp][e] = v;
    }
    if (lane == 0) rsum[warp] = sum;
    __syncthreads();
    if (tid < DH) {
      float v = 0.f, tot = 0.f;
#pragma unroll
      for (int w = 0; w < Q1_THREADS / 32; ++w) {
        v += red[w][tid];
        tot += rsum[w];
      }
      const float out = v / tot;
      const long long off = q * ldo + h * DH + tid;
      if (out_bf16) reinterpret_cast<__nv_bfloat16*>(O)[off] = __float2bfloat16_rn(out);
      else reinterpret_cast<float*>(O)[off] = out;
      if (O2 != nullptr) O2[q * ldo2 + h * DH + tid] = __float2bfloat16_rn(out);
    }
  }
}

}  // namespace

rocs_status launch_attention_stream(rocs_context* ctx, const void* Q, long long ldq, int q_split, const void* K,
                                    const void* V, long long ldkv, long long kv_req_stride, const int32_t* offsets,
                                    int B_R, long long rows, int L, int H, int d_h, float scale, void* O,
                                    long long ldo, int out_bf16, void* O2, long long ldo2, cudaStream_t s,
                                    const int32_t* kv_len, int q_by_kv) {
  if (B_R == 0 || rows == 0) return ROCS_OK;
  // chunks of one request spread over S CTAs: about twice the mean number of chunks per request
  const long long mean_chunks = (rows + (long long)B_R * ST_ROWS - 1) / ((long long)B_R * ST_ROWS);
  const int S = (int)std::min<long long>(64, std::max<long long>(1, 2 * mean_chunks));
  const long long grid = (long long)B_R * H * S;
  if (grid > 2147483647LL) {
    set_error("attention: grid too large");
    return ROCS_ERR_UNSUPPORTED;
  }
  const float scale_log2 = scale * 1.4426950408889634f;
  LaunchTimer lt_("attn_stream", s);
#define ROCS_ST(DH, SPLIT)                                                                                         \
  attn_stream_kernel<DH, SPLIT><<<(unsigned)grid, ST_WARPS * 32, 0, s>>>(                                          \
      (const __nv_bfloat16*)Q, ldq, (const __nv_bfloat16*)K, (const __nv_bfloat16*)V, ldkv, kv_req_stride, offsets, \
      B_R, rows, L, H, scale_log2, O, ldo, out_bf16, (__nv_bfloat16*)O2, ldo2, S, kv_len, q_by_kv, ctx->d_status)
  if (d_h == 32) {
    if (q_split) ROCS_ST(32, true); else ROCS_ST(32, false);
  } else {
    if (q_split) ROCS_ST(64, true); else ROCS_ST(64, false);
  }
#undef ROCS_ST
  return cuda_check(cudaGetLastError(), "attn_stream_kernel");
}

rocs_status launch_attention_single(rocs_context* ctx, const void* Q, long long ldq, int q_split, const void* K,
                                    const void* V, long long ldkv, long long kv_req_stride, const int32_t* offsets,
                                    int B_R, long long rows, int L, int H, int d_h, float scale, void* O,
                                    long long ldo, int out_bf16, void* O2, long long ldo2, cudaStream_t s,
                                    const int32_t* kv_len) {
  if (B_R == 0 || rows == 0) return ROCS_OK;
  if (L > Q1_KPT * Q1_THREADS) {
    set_error("attention (single query): L=%d above %d", L, Q1_KPT * Q1_THREADS);
    return ROCS_ERR_UNSUPPORTED;
  }
  const long long grid = (long long)B_R * H;
  const float scale_log2 = scale * 1.4426950408889634f;
  LaunchTimer lt_("attn_q1", s);
#define ROCS_Q1(DH, SPLIT)                                                                                         \
  attn_q1_kernel<DH, SPLIT><<<(unsigned)grid, Q1_THREADS, 0, s>>>(                                                 \
      (const __nv_bfloat16*)Q, ldq, (const __nv_bfloat16*)K, (const __nv_bfloat16*)V, ldkv, kv_req_stride, offsets, \
      B_R, rows, L, H, scale_log2, O, ldo, out_bf16, (__nv_bfloat16*)O2, ldo2, kv_len, ctx->d_status)
  if (d_h == 32) {
    if (q_split) ROCS_Q1(32, true); else ROCS_Q1(32, false);
  } else {
    if (q_split) ROCS_Q1(64, true); else ROCS_Q1(64, false);
  }
#undef ROCS_Q1
  return cuda_check(cudaGetLastError(), "attn_q1_kernel");
}

}  // namespace rocs
