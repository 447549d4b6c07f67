// a9, request side: the request query's cross-attention with the projections absorbed.
//
// [REV] §2.2 (DCA): A^R_i = MHA(Q^R_i; K^R_i, V^R_i) with K^R_i = S_i W_K^R and V^R_i = S_i W_V^R,
// one query per request and head.  Reassociating the same sums per head h (slice [h d_h, (h+1) d_h)
// of the d output features):
//   score_t = q_h . K^R_t,h = S_t . k'_h,        k'_h = (W_K^R)_h^T q_h          (a d-vector)
//   A^R_h   = sum_t p_t V^R_t,h = (W_V^R)_h s_h,   s_h = sum_t p_t S_t             (a d-vector)
// so K^R and V^R (2 x B_R x L x d) are never written or read: the path reads S once and the two
// weights from L2.  Same function; the scores and outputs are fp32 sums of exact bf16 x bf16
// products (K^R and V^R are not rounded to bf16 on the way).
//
// Three launches, d = 256:
//   1. attn_req_kq_kernel: k'_h for every request (scale and log2(e) folded in), written as a bf16
//      hi/lo pair [B_R][2][8 heads][d].  One CTA per (16 requests, head): each W_K^R slice is read
//      once per 16 requests.
//   2. attn_req_kernel: one CTA per (request, row split), 4 warps, two CTAs per SM.  Each warp
//      streams 16-row chunks of its split of S through a 3-stage cp.async ring in shared memory
//      (rows padded to 528 bytes): scores (16 rows x 8 heads) = S_chunk . k' and the weighted sums
//      s^T += S_chunk^T P run as m16n8k16 MMAs (k' hi + lo, P in bf16), with a per-head online
//      softmax (running max m, sum l) between them.  The four warps' states are merged in shared
//      memory and the split's (m, l, s) written out in fp32.
//   3. attn_req_combine_kernel: one CTA per (request, head) merges the P states (flash-decoding
//      style rescale by 2^(m_p - max m)) and projects A[o] = W_V^R[o] . s_h / l_h for the head's
//      d_h outputs, written fp32 (and optionally bf16).
#include "common.cuh"
#include "internal.h"
#include "mma_frag.cuh"

namespace rocs {
namespace {

constexpr int AR_D = 256;
constexpr int AR_MAX_H = 8;
constexpr int AR_WARPS = 4;                      // warps of the streaming kernel
constexpr int AR_STAGES = 3;                     // 16-row chunks in flight per warp
constexpr int AR_PITCH = AR_D * 2 + 16;          // bytes per staged row
constexpr int AR_KPITCH = AR_D + 8;              // bf16 elements per k' row (16-byte padded)
constexpr int AR_KQ_REQ = 16;                    // requests per k' CTA
constexpr int AR_MAX_SPLIT = 16;
constexpr int AR_CMB_THREADS = 128;              // combine kernel: thread t owns s columns 2t, 2t + 1
// one split's state: s [8 heads][d], m [8], l [8] (fp32)
constexpr int AR_PART = AR_MAX_H * AR_D + 2 * AR_MAX_H;
constexpr int AR_KQ_ELEMS = 2 * AR_MAX_H * AR_D;   // bf16 per request: hi [8][d], lo [8][d]

constexpr int AR_TILE_BYTES = AR_WARPS * AR_STAGES * 16 * AR_PITCH;
constexpr int AR_SMEM = AR_TILE_BYTES + 2 * AR_MAX_H * AR_KPITCH * 2 + AR_WARPS * 16 * (AR_MAX_H / 2) * 4 +
                        2 * AR_WARPS * AR_MAX_H * 4;
static_assert(AR_TILE_BYTES >= AR_WARPS * AR_MAX_H * AR_D * 4, "merge buffer must fit in the row tiles");

__device__ __forceinline__ void unpack8(const uint4& u, float (&v)[8]) {
  v[0] = bf16_lo(u.x); v[1] = bf16_hi(u.x); v[2] = bf16_lo(u.y); v[3] = bf16_hi(u.y);
  v[4] = bf16_lo(u.z); v[5] = bf16_hi(u.z); v[6] = bf16_lo(u.w); v[7] = bf16_hi(u.w);
}

// k'[r][h][i] = scale_log2 * sum_j q_r[h dh + j] W_K^R[h dh + j][i], q = hi + lo of the request query.
// Grid (ceil(B_R / 16), 8): thread i owns feature i for the CTA's 16 requests; heads >= H are zero.
__global__ void __launch_bounds__(AR_D) attn_req_kq_kernel(const __nv_bfloat16* __restrict__ Q, long long ldq,
                                                          const __nv_bfloat16* __restrict__ WK, int B_R, int H,
                                                          float scale_log2, __nv_bfloat16* __restrict__ Kq) {
  constexpr int D = AR_D;
  __shared__ float qs[AR_KQ_REQ][D];
  const int h = blockIdx.y, r0 = blockIdx.x * AR_KQ_REQ, i = threadIdx.x;
  const int nr = B_R - r0 < AR_KQ_REQ ? B_R - r0 : AR_KQ_REQ;
  if (h >= H) {
    for (int rr = 0; rr < nr; ++rr) {
      Kq[(long long)(r0 + rr) * AR_KQ_ELEMS + h * D + i] = __float2bfloat16_rn(0.f);
      Kq[(long long)(r0 + rr) * AR_KQ_ELEMS + AR_MAX_H * D + h * D + i] = __float2bfloat16_rn(0.f);
    }
    return;
  }
  const int dh = D / H;
  for (int idx = i; idx < AR_KQ_REQ * dh; idx += D) {
    const int rr = idx / dh, j = idx - rr * dh;
    float v = 0.f;
    if (rr < nr) {
      const __nv_bfloat16* q = Q + (long long)(r0 + rr) * ldq + h * dh + j;
      v = __bfloat162float(q[0]) + __bfloat162float(q[D]);
    }
    qs[rr][j] = v;
  }
  __syncthreads();
  float acc[AR_KQ_REQ];
#pragma unroll
  for (int rr = 0; rr < AR_KQ_REQ; ++rr) acc[rr] = 0.f;
  // (dh is a multiple of 16: sixteen independent weight loads in flight per step)
  for (int j0 = 0; j0 < dh; j0 += 16) {
    float w[16];
#pragma unroll
    for (int u = 0; u < 16; ++u) w[u] = __bfloat162float(WK[(long long)(h * dh + j0 + u) * D + i]);
#pragma unroll
    for (int rr = 0; rr < AR_KQ_REQ; ++rr)
#pragma unroll
      for (int u = 0; u < 16; ++u) acc[rr] = fmaf(qs[rr][j0 + u], w[u], acc[rr]);
  }
#pragma unroll
  for (int rr = 0; rr < AR_KQ_REQ; ++rr) {
    if (rr < nr) {
      const float v = acc[rr] * scale_log2;
      const __nv_bfloat16 hi = __float2bfloat16_rn(v);
      Kq[(long long)(r0 + rr) * AR_KQ_ELEMS + h * D + i] = hi;
      Kq[(long long)(r0 + rr) * AR_KQ_ELEMS + AR_MAX_H * D + h * D + i] = __float2bfloat16_rn(v - __bfloat162float(hi));
    }
  }
}

// One CTA per (request r, split p) over rows [p RS, min((p + 1) RS, L_r)) of S_r; writes the split's
// (m, l, s) to part[(r P + p)] (a split with no rows writes m = -inf, l = 0).
__global__ void __launch_bounds__(AR_WARPS * 32, 2) attn_req_kernel(
    const __nv_bfloat16* __restrict__ Kq, const __nv_bfloat16* __restrict__ S, int L_all, int P, int RS,
    float* __restrict__ part, const int32_t* __restrict__ kv_len, int* status) {
  constexpr int D = AR_D;
  extern __shared__ __align__(16) uint8_t ar_dyn[];
  uint8_t* tiles = ar_dyn;                                                   // [warp][stage][16][AR_PITCH]
  __nv_bfloat16* kbh = reinterpret_cast<__nv_bfloat16*>(ar_dyn + AR_TILE_BYTES);   // [8][AR_KPITCH]
  __nv_bfloat16* kbl = kbh + AR_MAX_H * AR_KPITCH;
  uint32_t* pbuf = reinterpret_cast<uint32_t*>(kbl + AR_MAX_H * AR_KPITCH);       // [warp][16][4] bf16 pairs
  float* wm = reinterpret_cast<float*>(pbuf + AR_WARPS * 16 * (AR_MAX_H / 2));    // [warp][8]
  float* wl = wm + AR_WARPS * AR_MAX_H;
  auto ws = reinterpret_cast<float (*)[AR_MAX_H][D]>(ar_dyn);                     // after the pass: [warp][8][D]

  const int r = blockIdx.x / P, p = blockIdx.x - r * P;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const __nv_bfloat16* Sr = S + (long long)r * L_all * D;
  // this request's rows: the first L of its L_all (a ragged history), L in [1, L_all]
  int L = kv_len != nullptr ? kv_len[r] : L_all;
  if (L < 1 || L > L_all) {
    if (tid == 0) set_status(status, ROCS_ERR_COUNTS);
    L = 0;   // the split then holds no rows; the output is not defined
  }
  const int t_begin = p * RS, t_end = L < t_begin + RS ? L : t_begin + RS;

  uint8_t* tile = tiles + warp * AR_STAGES * 16 * AR_PITCH;
  // chunk c of this warp: rows t_begin + (c AR_WARPS + warp) 16 .. + 15; one commit group per chunk
  // (empty past the end) so that "wait until 2 groups remain" always means "chunk c has landed".
  // Rows past the end of a last chunk are zeroed: their scores are -inf and p = 0 multiplies them.
  auto issue_chunk = [&](int c) {
    const int t0 = t_begin + (c * AR_WARPS + warp) * 16;
    if (t0 < t_end) {
      const int nrows = t_end - t0 < 16 ? t_end - t0 : 16;
      uint8_t* buf = tile + (c % AR_STAGES) * 16 * AR_PITCH;
      const uint32_t dst = smem_u32(buf) + lane * 16;
#pragma unroll
      for (int k = 0; k < 16; ++k) {
        if (k < nrows)
          asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(dst + k * AR_PITCH),
                       "l"(Sr + (long long)(t0 + k) * D + lane * 8)
                       : "memory");
        else
          *reinterpret_cast<uint4*>(buf + k * AR_PITCH + lane * 16) = make_uint4(0, 0, 0, 0);
      }
    }
    asm volatile("cp.async.commit_group;" ::: "memory");
  };
  issue_chunk(0);
  issue_chunk(1);
  // k' (hi, lo) into padded rows, 2 x 8 x 256 bf16 = 512 pieces of 16 bytes (the round trip
  // overlaps the first chunks')
#pragma unroll
  for (int k = tid; k < 2 * AR_MAX_H * (D / 8); k += AR_WARPS * 32) {
    const int half = k / (AR_MAX_H * (D / 8)), rem = k - half * (AR_MAX_H * (D / 8));
    const int h = rem / (D / 8), c = rem - h * (D / 8);
    const uint4 v = __ldg(reinterpret_cast<const uint4*>(Kq + (long long)r * AR_KQ_ELEMS + half * AR_MAX_H * D + h * D) + c);
    *reinterpret_cast<uint4*>((half ? kbl : kbh) + h * AR_KPITCH + c * 8) = v;
  }

  __syncthreads();   // k' rows are in shared memory

  // score B fragments: k' (8 heads x D) as hi and lo
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
  uint32_t* wp = pbuf + warp * 16 * (AR_MAX_H / 2);
  const uint32_t pbase = smem_u32(wp);

  for (int c = 0;; ++c) {
    const int t0 = t_begin + (c * AR_WARPS + warp) * 16;
    if (t0 >= t_end) break;
    const int nrows = t_end - t0 < 16 ? t_end - t0 : 16;
    // chunk c + 2 goes into the stage chunk c - 1 used (its reads ended at the last __syncwarp)
    issue_chunk(c + 2);
    asm volatile("cp.async.wait_group 2;" ::: "memory");
    __syncwarp();
    const uint32_t tbase = smem_u32(tile + (c % AR_STAGES) * 16 * AR_PITCH);
    // scores (16 rows x 8 heads): four independent accumulator chains (hi / lo x even / odd k-steps)
    float sc[4], sq[4][4];
#pragma unroll
    for (int a = 0; a < 4; ++a) sq[a][0] = sq[a][1] = sq[a][2] = sq[a][3] = 0.f;
#pragma unroll
    for (int ks = 0; ks < D / 16; ++ks) {
      uint32_t a4[4];
      load_a_frag(tbase, AR_PITCH, 0, ks * 16, a4);
      mma_bf16_16816(sq[ks & 1], a4, bh[ks][0], bh[ks][1]);
      mma_bf16_16816(sq[2 + (ks & 1)], a4, bl[ks][0], bl[ks][1]);
    }
#pragma unroll
    for (int e = 0; e < 4; ++e) sc[e] = (sq[0][e] + sq[1][e]) + (sq[2][e] + sq[3][e]);
    // rows past the chunk's end do not exist
    if (g8 >= nrows) sc[0] = sc[1] = -INFINITY;
    if (g8 + 8 >= nrows) sc[2] = sc[3] = -INFINITY;
    // online softmax for heads 2t (c = 0) and 2t + 1 (c = 1)
    float corr[2];
#pragma unroll
    for (int q = 0; q < 2; ++q) {
      float mx = fmaxf(sc[q], sc[q + 2]);
      mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 4));
      mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 8));
      mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 16));
      const float m_new = fmaxf(m[q], mx);
      corr[q] = m[q] == -INFINITY ? 0.f : exp2f(m[q] - m_new);
      sc[q] = exp2f(sc[q] - m_new);
      sc[q + 2] = exp2f(sc[q + 2] - m_new);
      float sum = sc[q] + sc[q + 2];
      sum += __shfl_xor_sync(0xffffffffu, sum, 4);
      sum += __shfl_xor_sync(0xffffffffu, sum, 8);
      sum += __shfl_xor_sync(0xffffffffu, sum, 16);
      l[q] = fmaf(l[q], corr[q], sum);
      m[q] = m_new;
    }
    // P (16 rows x 8 heads, bf16) through the warp's buffer, back as the B fragment
    wp[g8 * 4 + t4] = pack_bf16x2(sc[0], sc[1]);
    wp[(g8 + 8) * 4 + t4] = pack_bf16x2(sc[2], sc[3]);
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
    __syncwarp();   // this stage and the P buffer are read before they are written again
  }
  asm volatile("cp.async.wait_group 0;" ::: "memory");
  __syncthreads();   // every warp is done with its tiles: the region now holds the weighted sums

  // merge the warps' states (fragment layout: columns mt*16 + g8 (+8), heads 2t4, 2t4 + 1)
#pragma unroll
  for (int mt = 0; mt < D / 16; ++mt) {
    ws[warp][2 * t4][mt * 16 + g8] = accO[mt][0];
    ws[warp][2 * t4 + 1][mt * 16 + g8] = accO[mt][1];
    ws[warp][2 * t4][mt * 16 + g8 + 8] = accO[mt][2];
    ws[warp][2 * t4 + 1][mt * 16 + g8 + 8] = accO[mt][3];
  }
  if (g8 == 0) {
    wm[warp * AR_MAX_H + 2 * t4] = m[0];
    wm[warp * AR_MAX_H + 2 * t4 + 1] = m[1];
    wl[warp * AR_MAX_H + 2 * t4] = l[0];
    wl[warp * AR_MAX_H + 2 * t4 + 1] = l[1];
  }
  __syncthreads();
  float* out = part + (long long)blockIdx.x * AR_PART;
  for (int k = tid; k < AR_MAX_H * D; k += AR_WARPS * 32) {
    const int h = k / D, col = k - h * D;
    float M = -INFINITY;
#pragma unroll
    for (int w = 0; w < AR_WARPS; ++w) M = fmaxf(M, wm[w * AR_MAX_H + h]);
    float sum = 0.f;
#pragma unroll
    for (int w = 0; w < AR_WARPS; ++w) {
      const float mw = wm[w * AR_MAX_H + h];
      if (mw != -INFINITY) sum = fmaf(exp2f(mw - M), ws[w][h][col], sum);   // a warp with no rows adds nothing
    }
    out[k] = sum;
  }
  if (tid < AR_MAX_H) {
    const int h = tid;
    float M = -INFINITY, lsum = 0.f;
#pragma unroll
    for (int w = 0; w < AR_WARPS; ++w) M = fmaxf(M, wm[w * AR_MAX_H + h]);
#pragma unroll
    for (int w = 0; w < AR_WARPS; ++w) {
      const float mw = wm[w * AR_MAX_H + h];
      if (mw != -INFINITY) lsum = fmaf(exp2f(mw - M), wl[w * AR_MAX_H + h], lsum);
    }
    out[AR_MAX_H * D + h] = M;
    out[AR_MAX_H * D + AR_MAX_H + h] = lsum;
  }
}

// Merge request r's P split states for head h and project: A[r][o] = W_V^R[o] . s_h / l_h for the
// head's d_h outputs o.  One small CTA per (request, head), so thousands are resident and the few
// dependent round trips of each overlap; the head's W_V^R rows are in flight from the start.
__global__ void __launch_bounds__(AR_CMB_THREADS) attn_req_combine_kernel(
    const float* __restrict__ part, int P, const __nv_bfloat16* __restrict__ WV, int H, float* __restrict__ O,
    long long ldo, __nv_bfloat16* __restrict__ O2, long long ldo2) {
  constexpr int D = AR_D;
  __shared__ __align__(16) float s_m[D];
  __shared__ float fct[AR_MAX_SPLIT], lsp[AR_MAX_SPLIT];
  const int r = blockIdx.x, h = blockIdx.y;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int dh = D / H;
  const float* pr = part + (long long)r * P * AR_PART;
  // first eight of the warp's weight rows (rows h dh + warp + 4 k), a 16-byte slice per lane
  uint4 wr[8];
#pragma unroll
  for (int k = 0; k < 8; ++k) {
    const int o = warp + 4 * k;
    wr[k] = o < dh ? __ldg(reinterpret_cast<const uint4*>(WV + (long long)(h * dh + o) * D) + lane) : make_uint4(0, 0, 0, 0);
  }
  if (tid < P) {
    fct[tid] = pr[(long long)tid * AR_PART + AR_MAX_H * D + h];
    lsp[tid] = pr[(long long)tid * AR_PART + AR_MAX_H * D + AR_MAX_H + h];
  }
  float2 v[AR_MAX_SPLIT];
#pragma unroll
  for (int p = 0; p < AR_MAX_SPLIT; ++p)
    if (p < P) v[p] = reinterpret_cast<const float2*>(pr + (long long)p * AR_PART + h * D)[tid];
  __syncthreads();
  float M = -INFINITY;
  for (int p = 0; p < P; ++p) M = fmaxf(M, fct[p]);
  float lsum = 0.f, sx = 0.f, sy = 0.f;
#pragma unroll
  for (int p = 0; p < AR_MAX_SPLIT; ++p) {
    if (p < P) {
      const float mp = fct[p];
      const float f = mp == -INFINITY ? 0.f : exp2f(mp - M);   // a split with no rows adds nothing
      lsum = fmaf(f, lsp[p], lsum);
      sx = fmaf(f, v[p].x, sx);
      sy = fmaf(f, v[p].y, sy);
    }
  }
  const float inv_l = lsum > 0.f ? 1.0f / lsum : 0.f;
  reinterpret_cast<float2*>(s_m)[tid] = make_float2(sx, sy);
  __syncthreads();
  const float4 s0 = reinterpret_cast<const float4*>(s_m)[2 * lane];
  const float4 s1 = reinterpret_cast<const float4*>(s_m)[2 * lane + 1];
  for (int o0 = warp; o0 < dh; o0 += 32) {
    if (o0 > warp) {
#pragma unroll
      for (int k = 0; k < 8; ++k) {
        const int o = o0 + 4 * k;
        wr[k] = o < dh ? __ldg(reinterpret_cast<const uint4*>(WV + (long long)(h * dh + o) * D) + lane) : make_uint4(0, 0, 0, 0);
      }
    }
    float mine = 0.f;
#pragma unroll
    for (int k = 0; k < 8; ++k) {
      float w[8];
      unpack8(wr[k], w);
      float a = w[0] * s0.x;
      a = fmaf(w[1], s0.y, a); a = fmaf(w[2], s0.z, a); a = fmaf(w[3], s0.w, a);
      a = fmaf(w[4], s1.x, a); a = fmaf(w[5], s1.y, a); a = fmaf(w[6], s1.z, a); a = fmaf(w[7], s1.w, a);
#pragma unroll
      for (int off = 16; off > 0; off >>= 1) a += __shfl_xor_sync(0xffffffffu, a, off);
      if (lane == k) mine = a * inv_l;
    }
    const int o = o0 + 4 * lane;
    if (lane < 8 && o < dh) {
      O[r * ldo + h * dh + o] = mine;
      if (O2 != nullptr) O2[r * ldo2 + h * dh + o] = __float2bfloat16_rn(mine);
    }
  }
}

struct ArSplit {
  int P, RS;
};

// Row splits of each request's history: about 512 rows each (shorter splits pay the per-CTA start
// and merge more often: 256-row splits measured 15% slower, 128-row 70%), more (down to 64 rows)
// when there are too few requests to give each SM two CTAs twice over, at most 16.
ArSplit ar_split(int B_R, int L) {
  const int rows_per_round = AR_WARPS * 16;
  int P = (L + 511) / 512;
  const int want = (4 * 148 + B_R - 1) / (B_R > 0 ? B_R : 1);
  if (want > P) P = want;
  const int cap = (L + rows_per_round - 1) / rows_per_round;
  if (P > cap) P = cap;
  if (P > AR_MAX_SPLIT) P = AR_MAX_SPLIT;
  if (P < 1) P = 1;
  int RS = (L + P - 1) / P;
  RS = (RS + rows_per_round - 1) / rows_per_round * rows_per_round;
  P = (L + RS - 1) / RS;
  return {P, RS};
}

size_t align256(size_t b) { return (b + 255) & ~(size_t)255; }

}  // namespace

bool attention_req_absorbed_supported(int d, int H, int L) {
  return d == AR_D && H >= 1 && H <= AR_MAX_H && d % H == 0 && (d / H) % 16 == 0 && L >= 1;
}

size_t attention_req_absorbed_scratch(int B_R, int L) {
  if (B_R <= 0 || L <= 0) return 0;
  const ArSplit sp = ar_split(B_R, L);
  return align256((size_t)B_R * AR_KQ_ELEMS * 2) + align256((size_t)B_R * sp.P * AR_PART * 4);
}

rocs_status launch_attention_req_absorbed(rocs_context* ctx, const void* Q, long long ldq, const void* S,
                                          const void* WK, const void* WV, int B_R, int L, int d, int H, float scale,
                                          float* O, long long ldo, void* O2, long long ldo2, cudaStream_t s,
                                          const int32_t* kv_len, void* scratch) {
  if (B_R == 0) return ROCS_OK;
  if (!attention_req_absorbed_supported(d, H, L) || ((uintptr_t)S & 15) || ((uintptr_t)WV & 15) ||
      scratch == nullptr || ((uintptr_t)scratch & 15)) {
    set_error("request attention: unsupported d=%d H=%d L=%d (or scratch missing)", d, H, L);
    return ROCS_ERR_UNSUPPORTED;
  }
  const ArSplit sp = ar_split(B_R, L);
  __nv_bfloat16* Kq = (__nv_bfloat16*)scratch;
  float* part = (float*)((char*)scratch + align256((size_t)B_R * AR_KQ_ELEMS * 2));
  static bool attr[64] = {false};
  if (ctx->device < 64 && !attr[ctx->device]) {
    rocs_status st = cuda_check(
        cudaFuncSetAttribute(attn_req_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, AR_SMEM),
        "cudaFuncSetAttribute(attn_req)");
    if (st != ROCS_OK) return st;
    attr[ctx->device] = true;
  }
  {
    LaunchTimer lt_("attn_req_kq", s);
    attn_req_kq_kernel<<<dim3((B_R + AR_KQ_REQ - 1) / AR_KQ_REQ, AR_MAX_H), AR_D, 0, s>>>(
        (const __nv_bfloat16*)Q, ldq, (const __nv_bfloat16*)WK, B_R, H, scale * 1.4426950408889634f, Kq);
  }
  rocs_status st = cuda_check(cudaGetLastError(), "attn_req_kq_kernel");
  if (st != ROCS_OK) return st;
  {
    LaunchTimer lt_("attn_req", s);
    attn_req_kernel<<<(unsigned)((long long)B_R * sp.P), AR_WARPS * 32, AR_SMEM, s>>>(
        Kq, (const __nv_bfloat16*)S, L, sp.P, sp.RS, part, kv_len, ctx->d_status);
  }
  st = cuda_check(cudaGetLastError(), "attn_req_kernel");
  if (st != ROCS_OK) return st;
  {
    LaunchTimer lt_("attn_req_combine", s);
    attn_req_combine_kernel<<<dim3(B_R, H), AR_CMB_THREADS, 0, s>>>(part, sp.P, (const __nv_bfloat16*)WV, H, O, ldo,
                                                                  (__nv_bfloat16*)O2, ldo2);
  }
  return cuda_check(cudaGetLastError(), "attn_req_combine_kernel");
}

}  // namespace rocs
