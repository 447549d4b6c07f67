// FP8-weight (W8A16) linears on the 5th-generation tensor cores ("Compute Only Once:
// UG-Separation ...", §三 Stage 4 and the W8A16 table of §六: 8-bit floating-point weights, bf16
// activations, dequantisation cost negligible).
//
//   out[r, c] = act( 2^shift[r] * scale[c] * sum_k Xh[r, k] * q[c, k] + bias[c] + Z[gidx[r], c] )
//
// Xh is the activation in f16 with a per-row power-of-two shift (w8_xprep_kernel: exact, no
// overflow), q the E4M3 weight bytes [N, K] and scale one float per output channel.  A tcgen05
// MMA takes two operands of one 16-bit type, so the weights meet the tensor core as f16: every
// E4M3 value is an f16 value, and one cvt.rn.f16x2.e4m3x2 converts a pair exactly.  The weights
// cross HBM once, as bytes; the conversion happens in shared memory, between the TMA copy and the
// MMA, instead of in a bf16 copy of the whole matrix.
//
// One CTA per SM walks a static schedule of 128 x 128 output tiles (problem-major), 480 threads.
// Shared memory is one pool of 14 slots of 16 KiB, split per launch between three rings (more
// converted slots and fewer activation slots at small M, where the activation boxes are small):
//   warp 0       TMA producer of the weights: per 128 bytes of K (two MMA k blocks), the E4M3 tile
//                (128 rows x 128 bytes, unswizzled: each row request a whole 128-byte line).  A
//                weight slot is free again as soon as the converters have read it into registers.
//   warp 14      TMA producer of the activations: f16 boxes of 64 k values by `bma` rows (128-byte
//                swizzle), bma the power of two >= M up to 128.  A slot holds 128 / bma such boxes,
//                consecutive k blocks, so at small M one activation round trip covers up to 16 k
//                blocks.  The MMA still reads 128 rows per k block: the rows past bma are other data
//                of the pool, and their accumulator rows, past M, are never stored.
//   warp 1       allocates 256 TMEM columns (two 128 x 128 fp32 accumulators); one thread issues
//                tcgen05.mma kind::f16 (f16 x f16 -> f32, M = 128, N = 128, K = 16).
//   warps 2..9   converters: each weight tile's bytes to f16, written in the 128-byte-swizzled
//                K-major layout the MMA reads (64 k values per converted slot); each warp 16 rows.
//   warps 10..13 epilogue, one per TMEM lane quarter: tcgen05.ld, then the row shift, channel
//                scale, bias, request gather and activation, and vector stores.
// A phase trace of the first version (4 converter warps, 3 converted slots) showed the converters
// and the MMA in lockstep, each waiting on the other about half of every weight tile; the deeper
// converted ring and twice the converter warps remove that.
// Every wait is bounded; a wait that runs out sets ROCS_ERR_DEVICE_TIMEOUT and the CTA unwinds
// (copies and MMAs drained, TMEM released).  No cluster launch, no multicast.
#include <algorithm>
#include <cstring>

#include "common.cuh"
#include "internal.h"

namespace rocs {
namespace {

constexpr int W8_BM = 128;
constexpr int W8_BN = 128;
constexpr int W8_BK = 64;
constexpr int W8_WK = 128;           // k bytes per weight tile: two MMA k blocks
constexpr int W8_SLOT = 16384;       // every ring's slot: 16 KiB
constexpr int W8_SLOTS = 14;
constexpr int W8_MAX_A = 4, W8_MAX_C = 6, W8_MAX_W = 8;   // barrier arrays per ring
constexpr int W8_THREADS = 480;
constexpr int W8_TMEM_COLS = 256;
constexpr int W8_CONV_WARPS = 8;
constexpr int W8_EPI_WARP0 = 10;
constexpr int W8_APROD_WARP = 14;
constexpr int W8_NBARS = 2 * (W8_MAX_A + W8_MAX_C + W8_MAX_W) + 5;
constexpr int W8_SMEM = 1024 + W8_SLOTS * W8_SLOT + W8_NBARS * 8 + 16;
static_assert(W8_SMEM <= 232448, "shared memory");
constexpr int kMaxW8Problems = 3;

struct W8Problem {
  CUtensorMap tmA;   // Xh f16 [M, K]: box {64, bma}, 128-byte swizzle
  CUtensorMap tmW;   // q bytes [N, K]: box {128, 128}, unswizzled
  const int* shift;
  const float* scale;
  const float* bias;
  const float* Z;
  const int32_t* gidx;
  void* out;
  long long ldo, ldz;
  int M, N, K, out_bf16, act, gidx_bound;
  int n_tiles, k_blocks, tile_start;
  int bma, akb;   // activation rows per box, k blocks per activation slot (bma * akb = 128)
};

struct W8Params {
  W8Problem p[kMaxW8Problems];
  int nprob, total_tiles;
  int na, nc, nw;   // slots of the activation, converted and weight rings (na + nc + nw = 14)
  int* status;
};

// f16 x f16 -> f32, K-major A and B, M x N
constexpr uint32_t idesc_f16_f32(int M, int N) {
  return (1u << 4) | ((uint32_t)(N >> 3) << 17) | ((uint32_t)(M >> 4) << 24);
}

__device__ __forceinline__ void w8_decode(const W8Params& P, int t, int& pi, int& mb, int& nb) {
  pi = 0;
  while (pi + 1 < P.nprob && t >= P.p[pi + 1].tile_start) ++pi;
  const int local = t - P.p[pi].tile_start;
  mb = local / P.p[pi].n_tiles;
  nb = local - mb * P.p[pi].n_tiles;
}

__device__ __forceinline__ uint32_t e4m3x2_to_f16x2(uint32_t two_bytes) {
  uint32_t h;
  asm("cvt.rn.f16x2.e4m3x2 %0, %1;" : "=r"(h) : "h"((uint16_t)two_bytes));
  return h;
}

// Bounded wait with a short sleep between polls, for the warps that wait long (producers,
// converters, epilogue): polled without a pause, their waits would take issue slots from the one
// thread that issues the MMAs.
__device__ __forceinline__ bool mbar_wait_backoff(uint64_t* bar, uint32_t parity, int* status,
                                                  volatile int* abort_flag) {
  return mbar_wait_sleep(bar, parity, status, abort_flag, 64);
}

// A ring position: slot and the phase parity of its current use.
struct RingPos {
  int s = 0;
  uint32_t ph = 0;
  __device__ __forceinline__ void next(int n) {
    if (++s == n) {
      s = 0;
      ph ^= 1;
    }
  }
};

__global__ void __launch_bounds__(W8_THREADS, 1) gemm_w8_tc_kernel(const __grid_constant__ W8Params P) {
  extern __shared__ uint8_t w8_smem_raw[];
  uint8_t* base = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(w8_smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sA = base;                                  // [na] activation slots (1024-B aligned)
  uint8_t* sC = sA + P.na * W8_SLOT;                   // [nc] converted weights
  uint8_t* sW = sC + P.nc * W8_SLOT;                   // [nw] weight bytes
  uint64_t* bars = reinterpret_cast<uint64_t*>(base + W8_SLOTS * W8_SLOT);
  uint64_t* afull = bars;                              // activation TMA -> MMA
  uint64_t* aempty = afull + W8_MAX_A;                 // MMA -> activation TMA
  uint64_t* cfull = aempty + W8_MAX_A;                 // converters -> MMA
  uint64_t* cempty = cfull + W8_MAX_C;                 // MMA -> converters
  uint64_t* wfull = cempty + W8_MAX_C;                 // weight TMA -> converters
  uint64_t* wempty = wfull + W8_MAX_W;                 // converters -> weight TMA
  uint64_t* tfull = wempty + W8_MAX_W;                 // [2] MMA -> epilogue
  uint64_t* tempty = tfull + 2;                        // [2] epilogue -> MMA
  uint64_t* drain = tempty + 2;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(drain + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (threadIdx.x == 0) {
    for (int i = 0; i < W8_MAX_A; ++i) {
      mbar_init(&afull[i], 1);
      mbar_init(&aempty[i], 1);
    }
    for (int i = 0; i < W8_MAX_C; ++i) {
      mbar_init(&cfull[i], W8_CONV_WARPS);
      mbar_init(&cempty[i], 1);
    }
    for (int i = 0; i < W8_MAX_W; ++i) {
      mbar_init(&wfull[i], 1);
      mbar_init(&wempty[i], W8_CONV_WARPS);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&tfull[b], 1);
      mbar_init(&tempty[b], 128);
    }
    mbar_init(drain, 1);
    *abort_flag = 0;
    fence_barrier_init();
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, W8_TMEM_COLS);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;

  if (warp == 0 || warp == W8_APROD_WARP) {
    if (lane == 0) {
      // ---------------- TMA producers: weights (warp 0), activations (warp 14) ----------------
      // The first pass over a ring waits on parity 1 of fresh barriers, which counts as done.
      const bool wts = warp == 0;
      const int nst = wts ? P.nw : P.na;
      uint64_t* fb = wts ? wfull : afull;
      uint64_t* eb = wts ? wempty : aempty;
      for (int i = 0; i < P.nprob; ++i) prefetch_tensormap(wts ? &P.p[i].tmW : &P.p[i].tmA);
      RingPos r;
      int issued = 0;
      bool ok = true;
      for (int t = blockIdx.x; t < P.total_tiles && ok; t += gridDim.x) {
        int pi, mb, nb;
        w8_decode(P, t, pi, mb, nb);
        const W8Problem& pr = P.p[pi];
        const int kstep = wts ? 2 : pr.akb;   // a weight tile is two k blocks; an activation slot akb
        for (int kb = 0; kb < pr.k_blocks; kb += kstep) {
          if (!mbar_wait_backoff(&eb[r.s], r.ph ^ 1, P.status, abort_flag)) { ok = false; break; }
          if (wts) {
            mbar_arrive_expect_tx(&fb[r.s], W8_SLOT);
            tma_load_2d(sW + r.s * W8_SLOT, &pr.tmW, &fb[r.s], kb * W8_BK, nb * W8_BN);
          } else {
            const int nk = min(pr.akb, pr.k_blocks - kb);
            mbar_arrive_expect_tx(&fb[r.s], (uint32_t)(nk * pr.bma * 128));
            for (int j = 0; j < nk; ++j)
              tma_load_2d(sA + r.s * W8_SLOT + j * pr.bma * 128, &pr.tmA, &fb[r.s], (kb + j) * W8_BK, mb * W8_BM);
          }
          ++issued;
          r.next(nst);
        }
      }
      // no copy of this CTA may still be landing when it exits: the last min(issued, nst) slots
      for (int i = 0; i < nst && i < issued; ++i) {
        if (--r.s < 0) {
          r.s = nst - 1;
          r.ph ^= 1;
        }
        mbar_wait(&fb[r.s], r.ph, P.status, nullptr);
      }
    }
  } else if (warp == 1) {
    if (lane == 0) {
      // ---------------- MMA issuer ----------------
      RingPos ra, rc;
      int acc = 0;
      uint32_t acc_phase = 0;
      bool ok = true;
      for (int t = blockIdx.x; t < P.total_tiles && ok; t += gridDim.x) {
        int pi, mb, nb;
        w8_decode(P, t, pi, mb, nb);
        const W8Problem& pr = P.p[pi];
        if (!mbar_wait(&tempty[acc], acc_phase ^ 1, P.status, abort_flag)) break;
        tc_fence_after();
        const uint32_t d_tmem = tmem_base + (uint32_t)(acc * W8_BN);
        for (int kb = 0; kb < pr.k_blocks; ++kb) {
          const int sub = kb % pr.akb;   // k block within its activation slot
          if ((sub == 0 && !mbar_wait(&afull[ra.s], ra.ph, P.status, abort_flag)) ||
              !mbar_wait(&cfull[rc.s], rc.ph, P.status, abort_flag)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t a0 = smem_u32(sA + ra.s * W8_SLOT + sub * pr.bma * 128);
          const uint32_t b0 = smem_u32(sC + rc.s * W8_SLOT);
#pragma unroll
          for (int k = 0; k < W8_BK / 16; ++k)
            tc_mma_bf16(d_tmem, smem_desc_sw128(a0 + k * 32), smem_desc_sw128(b0 + k * 32),
                        idesc_f16_f32(W8_BM, W8_BN), (kb | k) != 0 ? 1u : 0u);
          tc_commit(&cempty[rc.s]);
          rc.next(P.nc);
          if (sub == pr.akb - 1 || kb == pr.k_blocks - 1) {   // the activation slot's last k block
            tc_commit(&aempty[ra.s]);
            ra.next(P.na);
          }
        }
        if (!ok) break;
        tc_commit(&tfull[acc]);
        acc ^= 1;
        if (acc == 0) acc_phase ^= 1;
      }
      // every MMA this thread issued has completed before TMEM is released
      tc_commit(drain);
      mbar_wait(drain, 0, P.status, nullptr);
    }
  } else if (warp < 2 + W8_CONV_WARPS) {
    // ---------------- converters: E4M3 weight bytes -> f16, 128-byte-swizzled K-major ----------------
    // Warp cw converts rows [16 cw, 16 cw + 16) of each weight tile, four rows (512 contiguous
    // bytes) per step: lane = (row r, 16-byte unit u of the 128-byte row).  Unit u holds k bytes
    // 16u .. 16u + 15, i.e. k block 2w + (u >> 2) of the tile pair, whose converted row r gets them
    // as its swizzled 16-byte units 2 (u & 3) and 2 (u & 3) + 1 (unit j of row r sits at j ^ (r & 7)).
    const int cw = warp - 2;
    const int u = lane & 7, uu = u & 3;
    RingPos rw, rc;
    bool ok = true;
    for (int t = blockIdx.x; t < P.total_tiles && ok; t += gridDim.x) {
      int pi, mb, nb;
      w8_decode(P, t, pi, mb, nb);
      const int pairs = P.p[pi].k_blocks / 2;
      for (int pp = 0; pp < pairs; ++pp) {
        RingPos rc1 = rc;
        rc1.next(P.nc);
        const bool got = mbar_wait_backoff(&wfull[rw.s], rw.ph, P.status, abort_flag) &&
                         mbar_wait_backoff(&cempty[rc.s], rc.ph ^ 1, P.status, abort_flag) &&
                         mbar_wait_backoff(&cempty[rc1.s], rc1.ph ^ 1, P.status, abort_flag);
        if (!__all_sync(0xffffffffu, got)) { ok = false; break; }
        const uint8_t* src = sW + rw.s * W8_SLOT;
        uint4 qv[4];
#pragma unroll
        for (int step = 0; step < 4; ++step)
          qv[step] = *reinterpret_cast<const uint4*>(src + (cw * 16 + step * 4 + (lane >> 3)) * W8_WK + u * 16);
        // the weight bytes are in registers: the slot goes back to the weight producer
        __syncwarp();
        if (lane == 0) mbar_arrive(&wempty[rw.s]);
        uint8_t* dst = sC + (u < 4 ? rc.s : rc1.s) * W8_SLOT;
#pragma unroll
        for (int step = 0; step < 4; ++step) {
          const int r = cw * 16 + step * 4 + (lane >> 3);
          const uint4 q = qv[step];
          const uint4 lo = make_uint4(e4m3x2_to_f16x2(q.x & 0xFFFFu), e4m3x2_to_f16x2(q.x >> 16),
                                      e4m3x2_to_f16x2(q.y & 0xFFFFu), e4m3x2_to_f16x2(q.y >> 16));
          const uint4 hi = make_uint4(e4m3x2_to_f16x2(q.z & 0xFFFFu), e4m3x2_to_f16x2(q.z >> 16),
                                      e4m3x2_to_f16x2(q.w & 0xFFFFu), e4m3x2_to_f16x2(q.w >> 16));
          uint8_t* row = dst + r * 128;
          *reinterpret_cast<uint4*>(row + (((2 * uu) ^ (r & 7)) << 4)) = lo;
          *reinterpret_cast<uint4*>(row + (((2 * uu + 1) ^ (r & 7)) << 4)) = hi;
        }
        fence_proxy_async_smem();   // the generic-proxy writes, visible to the tensor core
        __syncwarp();
        if (lane == 0) {
          mbar_arrive(&cfull[rc.s]);
          mbar_arrive(&cfull[rc1.s]);
        }
        rw.next(P.nw);
        rc = rc1;
        rc.next(P.nc);
      }
    }
  } else if (warp < W8_EPI_WARP0 + 4) {
    // ---------------- epilogue: one warp per TMEM lane quarter ----------------
    const int q = warp & 3;
    const int row_in_tile = q * 32 + lane;
    int acc = 0;
    uint32_t acc_phase = 0;
    for (int t = blockIdx.x; t < P.total_tiles; t += gridDim.x) {
      int pi, mb, nb;
      w8_decode(P, t, pi, mb, nb);
      const W8Problem& pr = P.p[pi];
      const long long grow = (long long)mb * W8_BM + row_in_tile;
      bool rvalid = grow < pr.M;
      float rmul = 0.f;
      const float* zrow = nullptr;
      if (rvalid) {
        rmul = __uint_as_float((uint32_t)(127 + pr.shift[grow]) << 23);
        if (pr.Z != nullptr) {
          const int zi = pr.gidx[grow];
          if (zi < 0 || zi >= pr.gidx_bound) {
            set_status(P.status, ROCS_ERR_INDEX);
            rvalid = false;
          } else {
            zrow = pr.Z + (long long)zi * pr.ldz;
          }
        }
      }
      if (!__all_sync(0xffffffffu, mbar_wait_backoff(&tfull[acc], acc_phase, P.status, abort_flag))) break;
      tc_fence_after();
      const uint32_t tbase = tmem_base + ((uint32_t)(q * 32) << 16) + (uint32_t)(acc * W8_BN);
#pragma unroll 1
      for (int ch = 0; ch < W8_BN / 32; ++ch) {
        uint32_t rr[32];
        tmem_ld_32x32b_x32(tbase + (uint32_t)(ch * 32), rr);
        tmem_ld_wait();
        if (ch == W8_BN / 32 - 1) {
          tc_fence_before();
          mbar_arrive(&tempty[acc]);
        }
        const int col0 = nb * W8_BN + ch * 32;
        if (!rvalid || col0 >= pr.N) continue;
        const int ncol = min(32, pr.N - col0);
        float v[32];
#pragma unroll
        for (int j = 0; j < 32; ++j) {
          const int col = col0 + j;
          float x = __uint_as_float(rr[j]) * rmul;
          if (j < ncol) {
            x *= __ldg(pr.scale + col);
            if (pr.bias != nullptr) x += __ldg(pr.bias + col);
            if (zrow != nullptr) x += zrow[col];
          }
          v[j] = x;
        }
        switch (pr.act) {
          case ROCS_ACT_RELU:
#pragma unroll
            for (int j = 0; j < 32; ++j) v[j] = fmaxf(v[j], 0.f);
            break;
          case ROCS_ACT_GELU:
#pragma unroll
            for (int j = 0; j < 32; ++j) v[j] = gelu_erf(v[j]);
            break;
          case ROCS_ACT_SIGMOID:
#pragma unroll
            for (int j = 0; j < 32; ++j) v[j] = sigmoid_fast(v[j]);
            break;
          default:
            break;
        }
        if (pr.out_bf16) {
          __nv_bfloat16* o = reinterpret_cast<__nv_bfloat16*>(pr.out) + grow * pr.ldo + col0;
          if (ncol == 32 && (pr.ldo % 8) == 0) {
#pragma unroll
            for (int j = 0; j < 32; j += 8)
              *reinterpret_cast<uint4*>(o + j) = make_uint4(pack_bf16x2(v[j], v[j + 1]), pack_bf16x2(v[j + 2], v[j + 3]),
                                                           pack_bf16x2(v[j + 4], v[j + 5]), pack_bf16x2(v[j + 6], v[j + 7]));
          } else {
#pragma unroll
            for (int j = 0; j < 32; ++j)
              if (j < ncol) o[j] = __float2bfloat16_rn(v[j]);
          }
        } else {
          float* o = reinterpret_cast<float*>(pr.out) + grow * pr.ldo + col0;
          if (ncol == 32 && (pr.ldo % 4) == 0) {
#pragma unroll
            for (int j = 0; j < 32; j += 4) *reinterpret_cast<float4*>(o + j) = make_float4(v[j], v[j + 1], v[j + 2], v[j + 3]);
          } else {
#pragma unroll
            for (int j = 0; j < 32; ++j)
              if (j < ncol) o[j] = v[j];
          }
        }
      }
      acc ^= 1;
      if (acc == 0) acc_phase ^= 1;
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem_base, W8_TMEM_COLS);
  }
}

typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                  const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

}  // namespace

bool w8_tc_supported(int K, int N) { return K >= W8_WK && K % W8_WK == 0 && N >= 1; }

rocs_status launch_gemm_w8(rocs_context* ctx, const W8GemmDesc* probs, int nprob, cudaStream_t s) {
  if (nprob < 1 || nprob > kMaxW8Problems) {
    set_error("w8 gemm: %d problems (1..%d supported)", nprob, kMaxW8Problems);
    return ROCS_ERR_INVALID_ARG;
  }
  static bool attr_set[64] = {false};
  if (ctx->device < 64 && !attr_set[ctx->device]) {
    rocs_status st = cuda_check(cudaFuncSetAttribute(gemm_w8_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                                     W8_SMEM),
                                "cudaFuncSetAttribute(gemm_w8_tc)");
    if (st != ROCS_OK) return st;
    attr_set[ctx->device] = true;
  }
  W8Params P;
  memset(&P, 0, sizeof(P));
  P.nprob = nprob;
  P.status = ctx->d_status;
  EncodeTiledFn fn = reinterpret_cast<EncodeTiledFn>(ctx->encode_fn);
  int tiles = 0;
  for (int i = 0; i < nprob; ++i) {
    const W8GemmDesc& g = probs[i];
    if (g.M < 1 || g.N < 1 || !w8_tc_supported(g.K, g.N) || g.ldx % 8 || ((uintptr_t)g.Xh & 15) ||
        ((uintptr_t)g.W8 & 15) || !g.shift || !g.scale || !g.out || (g.Z && !g.gidx) || g.ldo < g.N) {
      set_error("w8 gemm problem %d: unsupported shape/alignment (M=%d N=%d K=%d)", i, g.M, g.N, g.K);
      return ROCS_ERR_INVALID_ARG;
    }
    W8Problem& p = P.p[i];
    {
      cuuint64_t dims[2] = {(cuuint64_t)g.K, (cuuint64_t)g.M};
      cuuint64_t strides[1] = {(cuuint64_t)g.ldx * 2};
      p.bma = 8;
      while (p.bma < W8_BM && p.bma < g.M) p.bma *= 2;
      p.akb = W8_BM / p.bma;
      cuuint32_t box[2] = {(cuuint32_t)W8_BK, (cuuint32_t)p.bma};
      cuuint32_t estr[2] = {1, 1};
      if (fn(&p.tmA, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 2, const_cast<void*>(g.Xh), dims, strides, box, estr,
             CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
             CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS) {
        set_error("w8 gemm problem %d: cuTensorMapEncodeTiled (activations) failed", i);
        return ROCS_ERR_CUDA;
      }
    }
    {
      cuuint64_t dims[2] = {(cuuint64_t)g.K, (cuuint64_t)g.N};
      cuuint64_t strides[1] = {(cuuint64_t)g.K};
      cuuint32_t box[2] = {(cuuint32_t)W8_WK, (cuuint32_t)W8_BN};
      cuuint32_t estr[2] = {1, 1};
      if (fn(&p.tmW, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<uint8_t*>(g.W8), dims, strides, box, estr,
             CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
             CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS) {
        set_error("w8 gemm problem %d: cuTensorMapEncodeTiled (weights) failed", i);
        return ROCS_ERR_CUDA;
      }
    }
    p.shift = g.shift;
    p.scale = g.scale;
    p.bias = g.bias;
    p.Z = g.Z;
    p.gidx = g.gidx;
    p.gidx_bound = g.gidx_bound;
    p.out = g.out;
    p.ldo = g.ldo;
    p.ldz = g.ldz;
    p.M = g.M;
    p.N = g.N;
    p.K = g.K;
    p.out_bf16 = g.out_bf16;
    p.act = g.act;
    p.n_tiles = (g.N + W8_BN - 1) / W8_BN;
    p.k_blocks = g.K / W8_BK;
    p.tile_start = tiles;
    tiles += ((g.M + W8_BM - 1) / W8_BM) * p.n_tiles;
  }
  P.total_tiles = tiles;
  // ring split: small activation boxes (several k blocks per slot) need few activation slots
  int min_akb = W8_BM;
  for (int i = 0; i < nprob; ++i) min_akb = std::min(min_akb, P.p[i].akb);
  if (min_akb >= 4) {
    P.na = 2; P.nc = 5; P.nw = 7;
  } else if (min_akb == 2) {
    P.na = 3; P.nc = 5; P.nw = 6;
  } else {
    P.na = 4; P.nc = 4; P.nw = 6;
  }
  const int grid = std::min(tiles, ctx->num_sms);
  LaunchTimer lt_("gemm_w8_tc", s);
  gemm_w8_tc_kernel<<<grid, W8_THREADS, W8_SMEM, s>>>(P);
  return cuda_check(cudaGetLastError(), "gemm_w8_tc_kernel launch");
}

}  // namespace rocs
