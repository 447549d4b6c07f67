// a9, request side: the request query's cross-attention with the projections absorbed.
//
// [REV] §2.2 (DCA): A^R_i = MHA(Q^R_i; K^R_i, V^R_i) with K^R_i = S_i W_K^R and V^R_i = S_i W_V^R,
// one query per request and head.  Reassociating the same sums per head h (slice [h d_h, (h+1) d_h)
// of the d output features):
//   score_t = q_h . K^R_t,h = S_t . k'_h,        k'_h = (W_K^R)_h^T q_h          (a d-vector)
//   A^R_h   = sum_t p_t V^R_t,h = (W_V^R)_h s_h,   s_h = sum_t p_t S_t             (a d-vector)
// so K^R and V^R (2 x B_R x L x d) are never written or read: the kernel reads S once and the two
// weights from L2.  Same function; the scores and outputs are fp32 sums of exact bf16 x bf16
// products (K^R and V^R are not rounded to bf16 on the way).
//
// One CTA per request, 8 warps, d = 256; each warp takes 16-row chunks of S in turn:
//   1. q = hi + lo of the request's query; k'_h (scale and log2(e) folded in) into shared memory.
//   2. per warp, 16-row chunks of S double-buffered in shared memory (cp.async; rows padded to
//      528 bytes): scores (16 rows x 8 heads) = S_chunk . k' and the weighted sums
//      s^T += S_chunk^T P run as m16n8k16 MMAs (k' as a bf16 hi/lo pair, P in bf16), with a
//      per-head online softmax (running max m, sum l) between them.
//   3. the eight warps' (m, l, s) states are merged in shared memory.
//   4. A[o] = sum_i W_V^R[o][i] s_h(o)[i] / l_h(o), written fp32 (and optionally bf16).
#include "common.cuh"
#include "internal.h"
#include "mma_frag.cuh"

namespace rocs {
namespace {

constexpr int AR_D = 256;
constexpr int AR_MAX_H = 8;
constexpr int AR_WARPS = 8;

__device__ __forceinline__ void unpack8(const uint4& u, float (&v)[8]) {
  v[0] = bf16_lo(u.x); v[1] = bf16_hi(u.x); v[2] = bf16_lo(u.y); v[3] = bf16_hi(u.y);
  v[4] = bf16_lo(u.z); v[5] = bf16_hi(u.z); v[6] = bf16_lo(u.w); v[7] = bf16_hi(u.w);
}

constexpr int AR_PITCH = AR_D * 2 + 16;   // bytes per staged row
constexpr int AR_KPITCH = AR_D + 8;        // bf16 elements per k' row (16-byte padded)

__global__ void __launch_bounds__(AR_WARPS * 32) attn_req_absorbed_kernel(
    const __nv_bfloat16* __restrict__ Q, long long ldq, const __nv_bfloat16* __restrict__ S,
    const __nv_bfloat16* __restrict__ WK, const __nv_bfloat16* __restrict__ WV, int L_all, int H, float scale_log2,
    float* __restrict__ O, long long ldo, __nv_bfloat16* __restrict__ O2, long long ldo2,
    const int32_t* __restrict__ kv_len, int* status) {
  constexpr int D = AR_D;
  __shared__ float q[D];
  __shared__ __align__(16) float kp[AR_MAX_H][D];
  __shared__ __align__(16) uint32_t pbuf[AR_WARPS][16][AR_MAX_H / 2];   // P as bf16 pairs [row][head pair]
  __shared__ __align__(16) __nv_bfloat16 kbh[AR_MAX_H * AR_KPITCH], kbl[AR_MAX_H * AR_KPITCH];
  __shared__ float wm[AR_WARPS][AR_MAX_H], wl[AR_WARPS][AR_MAX_H];
  __shared__ float inv_l[AR_MAX_H];
  // dynamic: the warps' row tiles [AR_WARPS][2 buffers][16][AR_PITCH]; after the pass, the warps' weighted
  // row sums [AR_WARPS][AR_MAX_H][D] fp32 (merged into warp 0's slot)
  extern __shared__ __align__(16) uint8_t ar_dyn[];
  auto ws = reinterpret_cast<float (*)[AR_MAX_H][D]>(ar_dyn);
  const int r = blockIdx.x;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int dh = D / H;
  const __nv_bfloat16* Sr = S + (long long)r * L_all * D;
  // this request's rows: the first L of its L_all (a ragged history), L in [1, L_all]
  const int L = kv_len != nullptr ? kv_len[r] : L_all;
  if (L < 1 || L > L_all) {
    if (tid == 0) set_status(status, ROCS_ERR_COUNTS);
    return;
  }
  uint8_t* tile = ar_dyn + warp * 32 * AR_PITCH;

  // 1. query (hi + lo) and k'_h[i] = sum_j q[h dh + j] W_K^R[h dh + j][i]
  q[tid] = __bfloat162float(Q[r * ldq + tid]) + __bfloat162float(Q[r * ldq + D + tid]);
  __syncthreads();
  // (dh is a multiple of 16: sixteen independent row loads in flight per step)
  for (int h = 0; h < H; ++h) {
    float acc = 0.f;
    for (int j0 = 0; j0 < dh; j0 += 16) {
      float w[16];
#pragma unroll
      for (int u = 0; u < 16; ++u) w[u] = __bfloat162float(WK[(long long)(h * dh + j0 + u) * D + tid]);
#pragma unroll
      for (int u = 0; u < 16; ++u) acc = fmaf(q[h * dh + j0 + u], w[u], acc);
    }
    kp[h][tid] = acc * scale_log2;
  }
  __syncthreads();

  // k' as bf16 hi / lo rows [8 heads][D] (heads >= H zero), the B operand of the score MMAs
  for (int h = 0; h < AR_MAX_H; ++h) {
    const float v = h < H ? kp[h][tid] : 0.f;
    const __nv_bfloat16 hi = __float2bfloat16_rn(v);
    kbh[h * AR_KPITCH + tid] = hi;
    kbl[h * AR_KPITCH + tid] = __float2bfloat16_rn(v - __bfloat162float(hi));
  }
  // zero the row tiles once: rows past L in a last chunk then hold finite values (times p = 0)
  for (int k = tid; k < AR_WARPS * 32 * AR_PITCH / 16; k += blockDim.x)
    reinterpret_cast<uint4*>(ar_dyn)[k] = make_uint4(0, 0, 0, 0);
  __syncthreads();

  // 2. 16-row chunks on the tensor cores (m16n8k16, fp32 accumulate) with a per-head online softmax:
  //    scores (16 rows x 8 heads) = S_chunk (16 x D) . k' (D x 8, hi + lo);
  //    s^T (D x 8 heads) += S_chunk^T (D x 16) . P (16 x 8, bf16).
  //    Lane (g, t) holds heads 2t, 2t+1 in both fragments, so each head's rescale stays in-lane.
  const int g8 = lane >> 2, t4 = lane & 3;
  uint32_t bh[D / 16][2], bl[D / 16][2];
  {
    const int j = lane >> 3, rr = lane & 7;
#pragma unroll
    for (int ks = 0; ks < D / 16; ks += 2) {
      const uint32_t off = (uint32_t)(rr * AR_KPITCH * 2 + (16 * ks + 8 * j) * 2);
      ldsm_x4(smem_u32(kbh) + off, bh[ks][0], bh[ks][1], bh[ks + 1][0], bh[ks + 1][1]);
      ldsm_x4(smem_u32(kbl) + off, bl[ks][0], bl[ks][1], bl[ks + 1][0], bl[ks + 1][1]);
    }
  }
  float m[2] = {-INFINITY, -INFINITY}, l[2] = {0.f, 0.f};
  float accO[D / 16][4];
#pragma unroll
  for (int mt = 0; mt < D / 16; ++mt) accO[mt][0] = accO[mt][1] = accO[mt][2] = accO[mt][3] = 0.f;
  const uint32_t pbase = smem_u32(&pbuf[warp][0][0]);
  // 16-row chunks, double-buffered per warp: chunk c + 1 streams in (cp.async) while chunk c runs
  auto issue_chunk = [&](int t0, int buf) {
    const int nrows = L - t0 < 16 ? L - t0 : 16;
    const uint32_t dst = smem_u32(tile + buf * 16 * AR_PITCH) + lane * 16;
#pragma unroll
    for (int k = 0; k < 16; ++k)
      if (k < nrows)
        asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(dst + k * AR_PITCH),
                     "l"(Sr + (long long)(t0 + k) * D + lane * 8)
                     : "memory");
    asm volatile("cp.async.commit_group;" ::: "memory");
  };
  const int stride = AR_WARPS * 16;
  int buf = 0;
  if (warp * 16 < L) issue_chunk(warp * 16, 0);
  for (int t0 = warp * 16; t0 < L; t0 += stride, buf ^= 1) {
    const int nrows = L - t0 < 16 ? L - t0 : 16;
    if (t0 + stride < L) {
      issue_chunk(t0 + stride, buf ^ 1);
      asm volatile("cp.async.wait_group 1;" ::: "memory");
    } else {
      asm volatile("cp.async.wait_group 0;" ::: "memory");
    }
    __syncwarp();
    const uint32_t tbase = smem_u32(tile + buf * 16 * AR_PITCH);
    // scores (16 rows x 8 heads)
    float sc[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
    for (int ks = 0; ks < D / 16; ++ks) {
      uint32_t a4[4];
      load_a_frag(tbase, AR_PITCH, 0, ks * 16, a4);
      mma_bf16_16816(sc, a4, bh[ks][0], bh[ks][1]);
      mma_bf16_16816(sc, a4, bl[ks][0], bl[ks][1]);
    }
    // rows past the chunk's end do not exist
    if (g8 >= nrows) sc[0] = sc[1] = -INFINITY;
    if (g8 + 8 >= nrows) sc[2] = sc[3] = -INFINITY;
    // online softmax for heads 2t (c = 0) and 2t + 1 (c = 1)
    float corr[2];
#pragma unroll
    for (int c = 0; c < 2; ++c) {
      float mx = fmaxf(sc[c], sc[c + 2]);
      mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 4));
      mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 8));
      mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 16));
      const float m_new = fmaxf(m[c], mx);
      corr[c] = m[c] == -INFINITY ? 0.f : exp2f(m[c] - m_new);
      sc[c] = exp2f(sc[c] - m_new);
      sc[c + 2] = exp2f(sc[c + 2] - m_new);
      float sum = sc[c] + sc[c + 2];
      sum += __shfl_xor_sync(0xffffffffu, sum, 4);
      sum += __shfl_xor_sync(0xffffffffu, sum, 8);
      sum += __shfl_xor_sync(0xffffffffu, sum, 16);
      l[c] = fmaf(l[c], corr[c], sum);
      m[c] = m_new;
    }
    // P (16 rows x 8 heads, bf16) through the warp's buffer, back as the B fragment
    pbuf[warp][g8][t4] = pack_bf16x2(sc[0], sc[1]);
    pbuf[warp][g8 + 8][t4] = pack_bf16x2(sc[2], sc[3]);
    __syncwarp();
    uint32_t pb0, pb1;
    asm volatile("ldmatrix.sync.aligned.m8n8.x2.trans.shared.b16 {%0,%1}, [%2];"
                 : "=r"(pb0), "=r"(pb1)
                 : "r"(pbase + (lane & 15) * 16));
    // s^T += S_chunk^T P, after the rescale of the old sums
#pragma unroll
    for (int mt = 0; mt < D / 16; ++mt) {
      accO[mt][0] *= corr[0];
      accO[mt][1] *= corr[1];
      accO[mt][2] *= corr[0];
      accO[mt][3] *= corr[1];
      uint32_t a4[4];
      const int j = lane >> 3;
      const uint32_t addr = tbase + (uint32_t)((((j >> 1) << 3) + (lane & 7)) * AR_PITCH + (mt * 16 + ((j & 1) << 3)) * 2);
      ldsm_x4_trans(addr, a4[0], a4[1], a4[2], a4[3]);
      mma_bf16_16816(accO[mt], a4, pb0, pb1);
    }
    __syncwarp();   // this buffer is read before the chunk after next streams into it
  }
  __syncthreads();   // every warp is done with its tile: the region now holds the weighted sums

  // 3. merge the warps' states (fragment layout: columns mt*16 + g8 (+8), heads 2t4, 2t4 + 1)
#pragma unroll
  for (int mt = 0; mt < D / 16; ++mt) {
    ws[warp][2 * t4][mt * 16 + g8] = accO[mt][0];
    ws[warp][2 * t4 + 1][mt * 16 + g8] = accO[mt][1];
    ws[warp][2 * t4][mt * 16 + g8 + 8] = accO[mt][2];
    ws[warp][2 * t4 + 1][mt * 16 + g8 + 8] = accO[mt][3];
  }
  if (g8 == 0) {
    wm[warp][2 * t4] = m[0];
    wm[warp][2 * t4 + 1] = m[1];
    wl[warp][2 * t4] = l[0];
    wl[warp][2 * t4 + 1] = l[1];
  }
  __syncthreads();
  for (int h = 0; h < H; ++h) {
    float M = -INFINITY;
#pragma unroll
    for (int w = 0; w < AR_WARPS; ++w) M = fmaxf(M, wm[w][h]);
    float sum = 0.f, lsum = 0.f;
#pragma unroll
    for (int w = 0; w < AR_WARPS; ++w) {
      const float f = wm[w][h] == -INFINITY ? 0.f : exp2f(wm[w][h] - M);   // a warp with no rows adds nothing
      sum = fmaf(f, ws[w][h][tid], sum);
      lsum = fmaf(f, wl[w][h], lsum);
    }
    __syncthreads();   // every thread has read ws[*][h][tid] before ws[0][h] is overwritten
    ws[0][h][tid] = sum;
    if (tid == 0) inv_l[h] = 1.0f / lsum;
  }
  __syncthreads();

  // 4. A[o] = W_V^R[o] . s_h(o) / l_h(o): warp w takes outputs 32w .. 32w+31, its lanes split each
  //    weight row (coalesced 512-byte rows, all rows' loads in flight) and reduce by shuffles
  {
    uint4 wr[32];
#pragma unroll
    for (int k = 0; k < 32; ++k) wr[k] = __ldg(reinterpret_cast<const uint4*>(WV + (long long)(warp * 32 + k) * D) + lane);
    float mine = 0.f;
#pragma unroll
    for (int k = 0; k < 32; ++k) {
      const int o = warp * 32 + k, h = o / dh;
      float w[8];
      unpack8(wr[k], w);
      const float4 s0 = *reinterpret_cast<const float4*>(&ws[0][h][8 * lane]);
      const float4 s1 = *reinterpret_cast<const float4*>(&ws[0][h][8 * lane + 4]);
      float a = w[0] * s0.x;
      a = fmaf(w[1], s0.y, a); a = fmaf(w[2], s0.z, a); a = fmaf(w[3], s0.w, a);
      a = fmaf(w[4], s1.x, a); a = fmaf(w[5], s1.y, a); a = fmaf(w[6], s1.z, a); a = fmaf(w[7], s1.w, a);
#pragma unroll
      for (int off = 16; off > 0; off >>= 1) a += __shfl_xor_sync(0xffffffffu, a, off);
      if (lane == k) mine = a * inv_l[h];
    }
    const int o = warp * 32 + lane;
    O[r * ldo + o] = mine;
    if (O2 != nullptr) O2[r * ldo2 + o] = __float2bfloat16_rn(mine);
  }
}

}  // namespace

bool attention_req_absorbed_supported(int d, int H, int L) {
  return d == AR_D && H >= 1 && H <= AR_MAX_H && d % H == 0 && (d / H) % 16 == 0 && L >= 1;
}

rocs_status launch_attention_req_absorbed(rocs_context* ctx, const void* Q, long long ldq, const void* S,
                                          const void* WK, const void* WV, int B_R, int L, int d, int H, float scale,
                                          float* O, long long ldo, void* O2, long long ldo2, cudaStream_t s,
                                          const int32_t* kv_len) {
  if (B_R == 0) return ROCS_OK;
  if (!attention_req_absorbed_supported(d, H, L) || ((uintptr_t)S & 15) || ((uintptr_t)WV & 15)) {
    set_error("request attention: unsupported d=%d H=%d L=%d", d, H, L);
    return ROCS_ERR_UNSUPPORTED;
  }
  constexpr int tiles = AR_WARPS * 32 * AR_PITCH, sums = AR_WARPS * AR_MAX_H * AR_D * (int)sizeof(float);
  const int smem = tiles > sums ? tiles : sums;
  static bool attr[64] = {false};
  if (ctx->device < 64 && !attr[ctx->device]) {
    rocs_status st = cuda_check(
        cudaFuncSetAttribute(attn_req_absorbed_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, smem),
        "cudaFuncSetAttribute(attn_req)");
    if (st != ROCS_OK) return st;
    attr[ctx->device] = true;
  }
  LaunchTimer lt_("attn_req", s);
  attn_req_absorbed_kernel<<<B_R, AR_WARPS * 32, smem, s>>>((const __nv_bfloat16*)Q, ldq, (const __nv_bfloat16*)S,
                                                         (const __nv_bfloat16*)WK, (const __nv_bfloat16*)WV, L, H,
                                                         scale * 1.4426950408889634f, O, ldo, (__nv_bfloat16*)O2, ldo2,
                                                         kv_len, ctx->d_status);
  return cuda_check(cudaGetLastError(), "attn_req_absorbed_kernel");
}

}  // namespace rocs
