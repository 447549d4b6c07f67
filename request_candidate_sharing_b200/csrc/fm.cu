// a4: block-masked factorization machine and token-axis linear compression (LCB).
//
// FM ([REV] §2.1 FM equation, Figure 2(c)): output group i interacts only with input groups
// j <= i, so
//   request:   F^R_r = E^R_r E^R_r^T                        (n_R x n_R, once per request)
//   candidate: F^C_c = E^C_c [E^R_{m_c} ; E^C_c]^T          (n_C x (n_R + n_C))
// The candidate kernel reads the request embeddings through the map m (no broadcast tensor):
// one warp per candidate stages T = [E^R_{m_c} ; E^C_c] in shared memory (re-staging E^R only
// when m changes along its run of consecutive candidates) and computes the products with
// m16n8k16 tensor-core fragments.
//
// Token LCB ([REV] §2.1 masked linear along the embedding-count axis; IKBO split of §2.4):
//   L^R_r = P_RR E^R_r,   Z^L_r = P_CR E^R_r   (request batch, fp32 Z^L in the workspace)
//   L^C_c = Z^L_{m_c} + P_CC E^C_c              (candidate batch)
#include "common.cuh"
#include "internal.h"
#include "mma_frag.cuh"

#include <cstring>

namespace rocs {
namespace {

constexpr int FM_WARPS = 4;
constexpr int FM_RUN = 8;   // consecutive candidates per warp
constexpr int LCB_OMAX_F = 8;
constexpr int NC_MAX = 16;   // candidate embeddings per candidate handled by the fused pass

__device__ __forceinline__ uint4 load8_as_bf16(const __nv_bfloat16* p) { return __ldg(reinterpret_cast<const uint4*>(p)); }
__device__ __forceinline__ uint4 load8_as_bf16(const float* p) {
  const float4 a = __ldg(reinterpret_cast<const float4*>(p));
  const float4 b = __ldg(reinterpret_cast<const float4*>(p) + 1);
  return make_uint4(pack_bf16x2(a.x, a.y), pack_bf16x2(a.z, a.w), pack_bf16x2(b.x, b.y), pack_bf16x2(b.z, b.w));
}

// rows x D (contiguous source rows, bf16 or fp32) -> bf16 shared rows of `pitch` bytes.
template <typename TIN>
__device__ __forceinline__ void stage_rows(uint8_t* dst, int pitch, const TIN* src, int rows, int D) {
  const int lane = threadIdx.x & 31;
  const int vpr = D / 8;
  for (int i = lane; i < rows * vpr; i += 32) {
    const int r = i / vpr, v = i - r * vpr;
    *reinterpret_cast<uint4*>(dst + r * pitch + v * 16) = load8_as_bf16(src + (long long)r * D + v * 8);
  }
}

__device__ __forceinline__ void zero_rows(uint8_t* dst, int pitch, int rows, int D) {
  const int lane = threadIdx.x & 31;
  const int vpr = D / 8;
  for (int i = lane; i < rows * vpr; i += 32) {
    const int r = i / vpr, v = i - r * vpr;
    *reinterpret_cast<uint4*>(dst + r * pitch + v * 16) = make_uint4(0, 0, 0, 0);
  }
}

__device__ __forceinline__ void store_bf16_pair(__nv_bfloat16* p, long long o, float a, float b, bool two) {
  if (two && (o & 1) == 0) {
    *reinterpret_cast<uint32_t*>(p) = pack_bf16x2(a, b);
  } else {
    p[0] = __float2bfloat16_rn(a);
    if (two) p[1] = __float2bfloat16_rn(b);
  }
}

// Writes one 16x8 fp32 C fragment (rows r0.., cols c0..) of a [rows_valid x cols_valid] output
// with row stride ld.  out_mode 0: fp32; 1: bf16; 2: bf16 hi at offset o and bf16 lo = value - hi
// at offset o + lo_off (fp32-precise activation for a following tensor-core GEMM).
__device__ __forceinline__ void store_c_frag(void* out, int out_mode, long long base, int ld, int r0, int c0,
                                             int rows_valid, int cols_valid, const float (&c)[4],
                                             long long lo_off = 0) {
  const int lane = threadIdx.x & 31;
  const int g = lane >> 2, t = lane & 3;
#pragma unroll
  for (int h = 0; h < 2; ++h) {
    const int r = r0 + g + 8 * h;
    const int col = c0 + 2 * t;
    if (r >= rows_valid || col >= cols_valid) continue;
    const long long o = base + (long long)r * ld + col;
    const bool two = col + 1 < cols_valid;
    if (out_mode == 1) {
      store_bf16_pair(reinterpret_cast<__nv_bfloat16*>(out) + o, o, c[2 * h], c[2 * h + 1], two);
    } else if (out_mode == 2) {
      const float h0 = __bfloat162float(__float2bfloat16_rn(c[2 * h]));
      const float h1 = __bfloat162float(__float2bfloat16_rn(c[2 * h + 1]));
      __nv_bfloat16* p = reinterpret_cast<__nv_bfloat16*>(out);
      store_bf16_pair(p + o, o, h0, h1, two);
      store_bf16_pair(p + o + lo_off, o + lo_off, c[2 * h] - h0, c[2 * h + 1] - h1, two);
    } else {
      float* p = reinterpret_cast<float*>(out) + o;
      if (col < cols_valid) p[0] = c[2 * h];
      if (col + 1 < cols_valid) p[1] = c[2 * h + 1];
    }
  }
}

// Gram products of one staged tile: out[i][j] = sum_k T[a0 + i][k] T[j][k] for i < mrows,
// j < ncols (ncols <= 64, multiple of 8 after padding; rows beyond the valid ones are zero).
__device__ __forceinline__ void gram_tile(uint32_t sbase, int pitch, int a0, int mrows, int ncols, int D, void* out,
                                          int out_mode, long long obase, int ld, long long lo_off) {
  const int mt = (mrows + 15) / 16;
  const int nt2 = (ncols + 15) / 16;   // pairs of 8-wide n-tiles
  for (int mi = 0; mi < mt; ++mi) {
    float acc[8][4];
#pragma unroll
    for (int i = 0; i < 8; ++i)
#pragma unroll
      for (int j = 0; j < 4; ++j) acc[i][j] = 0.f;
    for (int k0 = 0; k0 < D; k0 += 16) {
      uint32_t a[4];
      load_a_frag(sbase, pitch, a0 + mi * 16, k0, a);
#pragma unroll
      for (int p = 0; p < 4; ++p) {
        if (p < nt2) {
          uint32_t b[4];
          load_b_frag_nmajor_x2(sbase, pitch, p * 16, k0, b);
          mma_bf16_16816(acc[2 * p], a, b[0], b[1]);
          mma_bf16_16816(acc[2 * p + 1], a, b[2], b[3]);
        }
      }
    }
#pragma unroll
    for (int p = 0; p < 8; ++p)
      if (p * 8 < ncols) store_c_frag(out, out_mode, obase, ld, mi * 16, p * 8, mrows, ncols, acc[p], lo_off);
  }
}

// ---------------------------------------------------------------------------------------------
// Fused candidate pass of one GLM layer: reads each candidate's embeddings E^C_c ONCE and emits
//   F^C_c  = E^C_c [E^R_{m_c} ; E^C_c]^T             (masked FM, bf16 hi/lo pairs)
//   L^C_c  = Z^L_{m_c} + P_CC E^C_c                  (token LCB, fp32; Z^L = P_CR E^R per request)
//   t^C_c  = Z^Q_{m_c} + p_CC E^C_c                  (optional: the DCA query generator's one-token
//                                                      LCB of the same embeddings, bf16 hi/lo pairs)
// The LCB sums take fp32 embeddings as a bf16 hi + lo pair (bf16 ones as they are), the FM
// products their bf16 rounding; both run as m16n8k16 tensor-core fragments.
// ---------------------------------------------------------------------------------------------
// One CTA per SM walks a contiguous range of candidates.  Warp 0 streams each candidate's E^C rows
// (contiguous, n_C x D) into a ring of shared-memory stages with bulk async copies, FC_STAGES
// candidates ahead; consumer pair p (two warps sharing one tile) takes the candidates p,
// p + FC_PAIRS, ... of the range, so its loads are already in flight while it computes.  Splitting
// each candidate over two warps halves the registers a warp needs (its half of the features and of
// the Gram k-range) and doubles the warps that hide each other's latencies.
constexpr int FC_PAIRS = 7;                    // consumer warp pairs, one candidate tile each
constexpr int FC_CONSUMERS = 2 * FC_PAIRS;     // 15 warps in all: at most 128 registers per thread
constexpr int FC_STAGES = 12;
// A pair's next candidate (i + pairs) reuses the stage of candidate i + pairs - stages, which must
// already have been loaded (it is <= i) for the parity of its mbarrier wait to be unambiguous.
static_assert(FC_STAGES >= FC_PAIRS, "ring stages must cover the consumer pairs");
// Each pair's block of shared memory starts with one region per warp (1024-byte aligned, so a
// 128-byte-swizzled TMA box can start there).  Warp hf's region holds feature half hf of the
// candidate's lo rows (fp32 inputs), read only by warp hf's token LCB; after that the same bytes
// stage warp hf's L^C columns for a TMA store, and then its partial Gram sums for the exchange.
// The pair's tile [E^R rows ; E^C hi rows ; 0 pad] follows the two regions.
constexpr int FC_LO_PITCH = 144;                            // 64 bf16 + 16 bytes: conflict-free ldmatrix rows
constexpr int FC_HALF = 3072;                               // one warp's region
constexpr int FC_LO_BYTES = FC_HALF + NC_MAX * FC_LO_PITCH; // both regions (the second one ends early)
static_assert(NC_MAX * FC_LO_PITCH <= FC_HALF && FC_HALF % 1024 == 0, "lo-row regions");
static_assert(2 * 1024 <= NC_MAX * FC_LO_PITCH, "two 8 x 32 fp32 swizzled boxes per warp region");
static_assert(4 * 32 * 16 <= NC_MAX * FC_LO_PITCH, "exchange slot per warp region");

__host__ __device__ constexpr int fc_pair_bytes(int trows, int pitch) {
  return (FC_LO_BYTES + trows * pitch + 1023) / 1024 * 1024;
}

__device__ __forceinline__ void st_shared_f32x2(uint32_t addr, float a, float b) {
  asm volatile("st.shared.v2.f32 [%0], {%1, %2};" ::"r"(addr), "f"(a), "f"(b) : "memory");
}
__device__ __forceinline__ void st_shared_f32x4(uint32_t addr, float a, float b, float c, float d) {
  asm volatile("st.shared.v4.f32 [%0], {%1, %2, %3, %4};" ::"r"(addr), "f"(a), "f"(b), "f"(c), "f"(d) : "memory");
}
__device__ __forceinline__ float4 ld_shared_f32x4(uint32_t addr) {
  float4 v;
  asm volatile("ld.shared.v4.f32 {%0, %1, %2, %3}, [%4];" : "=f"(v.x), "=f"(v.y), "=f"(v.z), "=f"(v.w) : "r"(addr) : "memory");
  return v;
}

// Barrier `id` over the 64 threads of a consumer pair.
__device__ __forceinline__ void pair_sync(int id) { asm volatile("bar.sync %0, 64;" ::"r"(id) : "memory"); }
// The same barrier, returning the AND of v over the pair's threads (so both warps take one branch).
__device__ __forceinline__ bool pair_and(int id, bool v) {
  uint32_t r;
  asm volatile(
      "{\n\t.reg .pred p, q;\n\tsetp.ne.u32 p, %1, 0;\n\tbar.red.and.pred q, %2, 64, p;\n\tselp.u32 %0, 1, 0, q;\n\t}"
      : "=r"(r)
      : "r"((uint32_t)v), "r"(id)
      : "memory");
  return r != 0;
}

template <typename TIN>
__global__ void __launch_bounds__(32 * (1 + FC_CONSUMERS), 1) glm_cand_fused_kernel(
    const TIN* __restrict__ E_R, const TIN* __restrict__ E_C, const int32_t* __restrict__ req_idx, int B_R,
    long long B_C, long long per_block, int n_R, int n_C, int trows, int pitch, __nv_bfloat16* __restrict__ F_C,
    const __nv_bfloat16* __restrict__ P_CC, int o_C, const float* __restrict__ ZL, float* __restrict__ L_C,
    const __nv_bfloat16* __restrict__ q_pCC, const float* __restrict__ ZQ, __nv_bfloat16* __restrict__ tC,
    const __grid_constant__ CUtensorMap mapL, int l_tma, int* status) {
  constexpr int D = 128;
  extern __shared__ __align__(128) uint8_t fc_smem_raw[];
  uint8_t* fc_smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(fc_smem_raw) + 1023) & ~uintptr_t(1023));
  __shared__ float sP[LCB_OMAX_F * 64];
  __shared__ float sQ[64];
  __shared__ __align__(8) uint64_t full[FC_STAGES], empty[FC_STAGES];
  __shared__ int stage_r[FC_STAGES];   // request index of the candidate in each stage
  __shared__ int stage_c[FC_STAGES];   // the candidate (index in the range) each stage was last loaded for
  __shared__ int abort_flag_s;
  volatile int* abort_flag = &abort_flag_s;

  const long long c0 = (long long)blockIdx.x * per_block;
  const long long c1 = c0 + per_block < B_C ? c0 + per_block : B_C;
  if (c0 >= c1) return;
  const int n = (int)(c1 - c0);
  const uint32_t stage_bytes = (uint32_t)(n_C * D * sizeof(TIN));
  uint8_t* ring = fc_smem;
  static_assert(FC_STAGES * NC_MAX * D * sizeof(TIN) % 1024 == 0, "pair blocks start 1024-byte aligned");
  uint8_t* tiles = fc_smem + FC_STAGES * NC_MAX * D * sizeof(TIN);

  for (int i = threadIdx.x; i < o_C * n_C; i += blockDim.x) sP[i] = __bfloat162float(P_CC[i]);
  for (int i = threadIdx.x; i < n_C; i += blockDim.x) sQ[i] = q_pCC ? __bfloat162float(q_pCC[i]) : 0.f;
  if (threadIdx.x == 0) {
    for (int k = 0; k < FC_STAGES; ++k) {
      mbar_init(&full[k], 1);
      mbar_init(&empty[k], 64);   // both warps of a pair
    }
    abort_flag_s = 0;
    fence_barrier_init();
  }
  __syncthreads();
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  if (warp == 0) {
    if (lane == 0) {
      // ---------------- producer ----------------
      int issued = 0;
      for (int i = 0; i < n; ++i) {
        const int st = i % FC_STAGES, use = i / FC_STAGES;
        const int r = req_idx[c0 + i];   // loaded ahead of the consumers
        if (use > 0 && !mbar_wait(&empty[st], (use - 1) & 1, status, abort_flag)) break;
        stage_r[st] = r;
        stage_c[st] = i;
        mbar_arrive_expect_tx(&full[st], stage_bytes);
        bulk_load(ring + st * NC_MAX * D * sizeof(TIN), E_C + (c0 + i) * (long long)n_C * D, stage_bytes, &full[st]);
        issued = i + 1;
      }
      // no copy of this CTA may still be landing when it exits
      for (int i = issued - FC_STAGES < 0 ? 0 : issued - FC_STAGES; i < issued; ++i)
        mbar_wait(&full[i % FC_STAGES], (i / FC_STAGES) & 1, status, nullptr);
    }
    return;
  }

  // ---------------- consumers: warp pairs ----------------
  // Pair pr takes candidates pr, pr + FC_PAIRS, ... of the range; warp hf of the pair owns features
  // [64 hf, 64 hf + 64) of the token LCB and the k-half [64 hf, 64 hf + 64) of the Gram products,
  // whose partial sums the two warps exchange through their lo-row regions (each free once its
  // own warp's LCB has read it).  Named barrier 1 + pr synchronises the pair.
  const int cw = warp - 1, pr = cw >> 1, hf = cw & 1;
  const int bar_id = 1 + pr;
  uint8_t* TL = tiles + pr * fc_pair_bytes(trows, pitch);   // two warp regions, FC_HALF bytes apart
  uint8_t* TLh = TL + hf * FC_HALF;                         // this warp's region
  uint8_t* T = TL + FC_LO_BYTES;                            // [E^R rows ; E^C hi rows ; 0 pad]
  // exchange slots: [4 n-tile slots][32 lanes] at the start of each warp's region
  const uint32_t sbase = smem_u32(T);
  const int ncols = n_R + n_C;
  const int nt2 = (ncols + 15) / 16;                    // pairs of 8-wide Gram n-tiles
  const long long fsz = (long long)n_C * ncols;
  const int g8 = lane >> 2, t4 = lane & 3;
  const int f0 = hf * (D / 2);                          // this warp's first feature
  // Fragment row g8 (< 8) carries LCB output o(g8) = 2 (g8 mod 4) + g8 / 4: the first half-warp
  // holds the even outputs, the second the odd ones, so the swizzled staging of L^C below puts
  // each half-warp's 16 stores on 16 different 8-byte bank pairs.
  const int og = ((g8 & 3) << 1) | (g8 >> 2);
  // A operand of the token LCB (16 x 16 tokens): row g8 < 8 holds P_CC row o(g8) (zero beyond
  // o_C) and rows 8..15 each the query generator's one-token weights.  Constant for the whole
  // kernel.  The eight equal rows give every lane the query token for its n-tile g8, so the warp
  // writes its 64 features of t^C with one 128-byte store per half (hi, lo).
  uint32_t pa[4];
  {
    auto A = [&](int row, int k) -> float {
      if (k >= n_C) return 0.f;
      if (row >= 8) return sQ[k];
      const int o = ((row & 3) << 1) | (row >> 2);
      return o < o_C ? sP[o * n_C + k] : 0.f;
    };
    pa[0] = pack_bf16x2(A(g8, 2 * t4), A(g8, 2 * t4 + 1));
    pa[1] = pack_bf16x2(A(g8 + 8, 2 * t4), A(g8 + 8, 2 * t4 + 1));
    pa[2] = pack_bf16x2(A(g8, 2 * t4 + 8), A(g8, 2 * t4 + 9));
    pa[3] = pack_bf16x2(A(g8 + 8, 2 * t4 + 8), A(g8 + 8, 2 * t4 + 9));
  }
  // Z^L row o(g8) of the current request for this warp's features, in the C-fragment layout
  // (n-tile nt, columns f0 + nt*8 + 2*t4 and +1), and the Z^Q pair at columns f0 + g8*8 + 2*t4
  // and +1
  float zl[D / 16][2];
  float2 zq = make_float2(0.f, 0.f);
#pragma unroll
  for (int nt = 0; nt < D / 16; ++nt) zl[nt][0] = zl[nt][1] = 0.f;
  int staged = -1;
  if (hf == 0) zero_rows(T + (n_R + n_C) * pitch, pitch, trows - (n_R + n_C), D);
  for (int i = pr; i < n; i += FC_PAIRS) {
    const int st = i % FC_STAGES;
    // Candidate i's rows in stage st.  A pair waits only on every FC_PAIRS-th candidate, so the
    // phase parity alone is ambiguous if the stage's previous load (candidate i - FC_STAGES) were
    // still landing: then the completed phase before it has the same parity.  The stage's tag is
    // set to i only once that previous phase has completed and been consumed; after it reads i,
    // a second wait on the same parity can only mean candidate i's own phase.
    bool got = true;
    {
      volatile int* tag = stage_c;
      const long long t0 = clock64();
      while (true) {
        got = mbar_wait(&full[st], (i / FC_STAGES) & 1, status, abort_flag);
        if (!got) break;
        if (tag[st] == i) {
          got = mbar_wait(&full[st], (i / FC_STAGES) & 1, status, abort_flag);
          break;
        }
        if (clock64() - t0 > kWaitBudgetCycles) {
          set_status(status, ROCS_ERR_DEVICE_TIMEOUT);
          *abort_flag = 1;
          got = false;
          break;
        }
      }
    }
    // both warps agree (and synchronise: the pair's reads of the previous candidate's tile and
    // exchange buffer are done)
    if (!pair_and(bar_id, got)) break;
    const long long c = c0 + i;
    // this candidate's rows from the stage into the tile as bf16 (hi, and lo = E - hi for fp32
    // inputs); warp hf converts rows hf, hf + 2, ...; lane j features 4j..4j+3
    const TIN* ec = reinterpret_cast<const TIN*>(ring + st * NC_MAX * D * sizeof(TIN));
#pragma unroll
    for (int k = 0; k < NC_MAX / 2; ++k) {
      const int t = 2 * k + hf;
      if (t < n_C) {
        if constexpr (sizeof(TIN) == 4) {
          const float4 v = reinterpret_cast<const float4*>(ec + t * D)[lane];
          const uint32_t h01 = pack_bf16x2(v.x, v.y), h23 = pack_bf16x2(v.z, v.w);
          *reinterpret_cast<uint2*>(T + (n_R + t) * pitch + lane * 8) = make_uint2(h01, h23);
          *reinterpret_cast<uint2*>(TL + (lane >> 4) * FC_HALF + t * FC_LO_PITCH + (lane & 15) * 8) =
              make_uint2(pack_bf16x2(v.x - bf16_lo(h01), v.y - bf16_hi(h01)),
                         pack_bf16x2(v.z - bf16_lo(h23), v.w - bf16_hi(h23)));
        } else {
          *reinterpret_cast<uint2*>(T + (n_R + t) * pitch + lane * 8) = reinterpret_cast<const uint2*>(ec + t * D)[lane];
        }
      } else if constexpr (sizeof(TIN) == 4) {
        // padding token rows of the lo tile meet zero LCB weights but must be finite: the staged
        // L^C and the exchange of the previous candidate overwrote them
        *reinterpret_cast<uint2*>(TL + (lane >> 4) * FC_HALF + t * FC_LO_PITCH + (lane & 15) * 8) = make_uint2(0, 0);
      }
    }
    const int r = stage_r[st];
    mbar_arrive(&empty[st]);
    if (r < 0 || r >= B_R) {   // the same r for both warps: both skip
      if (lane == 0 && hf == 0) set_status(status, ROCS_ERR_INDEX);
      continue;
    }
    if (r != staged) {
      // a new request run: its rows into the tile (warp hf rows hf, hf + 2, ...), this warp's
      // Z^L and Z^Q columns into registers
      const int nrw = (n_R - hf + 1) / 2;
      for (int k = lane; k < nrw * (D / 8); k += 32) {
        const int rr = hf + 2 * (k / (D / 8)), v = k % (D / 8);
        *reinterpret_cast<uint4*>(T + rr * pitch + v * 16) = load8_as_bf16(E_R + ((long long)r * n_R + rr) * D + v * 8);
      }
#pragma unroll
      for (int nt = 0; nt < D / 16; ++nt) {
        if (og < o_C) {
          const float2 z = __ldg(reinterpret_cast<const float2*>(ZL + ((long long)r * o_C + og) * D + f0 + nt * 8 + 2 * t4));
          zl[nt][0] = z.x;
          zl[nt][1] = z.y;
        }
      }
      if (tC != nullptr) zq = __ldg(reinterpret_cast<const float2*>(ZQ + (long long)r * D + f0 + g8 * 8 + 2 * t4));
      staged = r;
    }
    pair_sync(bar_id);   // the tile is complete
    {
      // token LCB on the tensor cores for this warp's 64 features: [P_CC ; p_CC] (16 x 16) times
      // E^C (16 tokens x 64), the fp32 embeddings as hi + lo bf16 parts
      float acc[D / 16][4];
#pragma unroll
      for (int nt = 0; nt < D / 16; ++nt) acc[nt][0] = acc[nt][1] = acc[nt][2] = acc[nt][3] = 0.f;
#pragma unroll
      for (int p = 0; p < D / 32; ++p) {
        uint32_t b[4];
        load_b_frag_kmajor_x2(sbase, pitch, n_R, f0 + p * 16, b);
        mma_bf16_16816(acc[2 * p], pa, b[0], b[1]);
        mma_bf16_16816(acc[2 * p + 1], pa, b[2], b[3]);
        if constexpr (sizeof(TIN) == 4) {
          load_b_frag_kmajor_x2(smem_u32(TLh), FC_LO_PITCH, 0, p * 16, b);
          mma_bf16_16816(acc[2 * p], pa, b[0], b[1]);
          mma_bf16_16816(acc[2 * p + 1], pa, b[2], b[3]);
        }
      }
      // L^C = Z^L + P_CC E^C (fp32): output o(g8) in fragment row g8 of every n-tile.  With the
      // TMA path, the warp's 64 columns go to its region as two boxes of o_C rows x 32 floats in
      // the 128-byte swizzle (the 16-byte unit u of row o at u ^ o), and one lane hands the boxes
      // to the tensor-store engine.  The region's lo rows were this warp's alone, and its LCB
      // products above have consumed them.
      if (l_tma) {
        if (og < o_C) {
          const uint32_t sl = smem_u32(TLh) + (og << 7) + ((t4 & 1) << 3);
          const uint32_t x = (uint32_t)((t4 >> 1) ^ og);
#pragma unroll
          for (int nt = 0; nt < D / 16; ++nt)
            st_shared_f32x2(sl + ((nt >> 2) << 10) + ((x ^ ((nt & 3) << 1)) << 4), acc[nt][0] + zl[nt][0],
                            acc[nt][1] + zl[nt][1]);
        }
        fence_proxy_async_smem();
        __syncwarp();
        if (lane == 0) {
          tma_store_2d(&mapL, TLh, f0, (int32_t)(c * o_C));
          tma_store_2d(&mapL, TLh + 1024, f0 + 32, (int32_t)(c * o_C));
          bulk_commit_group();
        }
      } else if (og < o_C) {
        float* lp = L_C + (c * o_C + og) * (long long)D + f0 + 2 * t4;
#pragma unroll
        for (int nt = 0; nt < D / 16; ++nt)
          *reinterpret_cast<float2*>(lp + nt * 8) = make_float2(acc[nt][0] + zl[nt][0], acc[nt][1] + zl[nt][1]);
      }
      // t^C = Z^Q + p_CC E^C as a bf16 hi/lo pair: fragment row 8 + g8 holds it for every g8, and
      // lane (g8, t4) writes n-tile g8's columns 2*t4 and +1
      if (tC != nullptr) {
        float a0 = acc[0][2], a1 = acc[0][3];
#pragma unroll
        for (int nt = 1; nt < D / 16; ++nt)
          if (g8 == nt) {
            a0 = acc[nt][2];
            a1 = acc[nt][3];
          }
        const float v0 = a0 + zq.x, v1 = a1 + zq.y;
        const uint32_t h = pack_bf16x2(v0, v1);
        __nv_bfloat16* tp = tC + c * 2LL * D + f0 + g8 * 8 + 2 * t4;
        *reinterpret_cast<uint32_t*>(tp) = h;
        *reinterpret_cast<uint32_t*>(tp + D) = pack_bf16x2(v0 - bf16_lo(h), v1 - bf16_hi(h));
      }
    }
    // F^C = E^C [E^R ; E^C]^T: this warp's k-half for every n-tile, then the pair exchange; warp hf
    // finishes the n-tiles nt with nt % 2 == hf
    float acc[8][4];
#pragma unroll
    for (int q = 0; q < 8; ++q) acc[q][0] = acc[q][1] = acc[q][2] = acc[q][3] = 0.f;
#pragma unroll
    for (int k0 = 0; k0 < D / 2; k0 += 16) {
      uint32_t a[4];
      load_a_frag(sbase, pitch, n_R, f0 + k0, a);
#pragma unroll
      for (int p = 0; p < 4; ++p) {
        if (p < nt2) {
          uint32_t b[4];
          load_b_frag_nmajor_x2(sbase, pitch, p * 16, f0 + k0, b);
          mma_bf16_16816(acc[2 * p], a, b[0], b[1]);
          mma_bf16_16816(acc[2 * p + 1], a, b[2], b[3]);
        }
      }
    }
    // the exchange slot is this warp's region: the tensor store must have read the staged L^C
    if (l_tma) {
      if (lane == 0) bulk_wait_read_all();
      __syncwarp();
    }
#pragma unroll
    for (int q = 0; q < 8; ++q)
      if (q < 2 * nt2 && (q & 1) != hf)
        st_shared_f32x4(smem_u32(TLh) + (((q >> 1) * 32 + lane) << 4), acc[q][0], acc[q][1], acc[q][2], acc[q][3]);
    pair_sync(bar_id);
#pragma unroll
    for (int q = 0; q < 8; ++q) {
      if (q < 2 * nt2 && (q & 1) == hf && q * 8 < ncols) {
        const float4 o = ld_shared_f32x4(smem_u32(TL) + (1 - hf) * FC_HALF + (((q >> 1) * 32 + lane) << 4));
        acc[q][0] += o.x;
        acc[q][1] += o.y;
        acc[q][2] += o.z;
        acc[q][3] += o.w;
        store_c_frag(F_C, 2, c * fsz * 2, ncols, 0, q * 8, n_C, ncols, acc[q], fsz);
      }
    }
  }
  // the CTA's last tensor stores complete before it exits
  if (l_tma && lane == 0) bulk_wait_all();
}


// Shared tile rows: n_R request rows, then n_C candidate rows, padded with zeros up to TROWS.
// TROWS >= max(n_R + roundup16(n_C), roundup16(n_R + n_C), roundup16(n_R)).
template <typename TIN>
__global__ void __launch_bounds__(FM_WARPS * 32) fm_cand_kernel(const TIN* __restrict__ E_R, const TIN* __restrict__ E_C,
                                                               const int32_t* __restrict__ req_idx, int B_R,
                                                               long long B_C, int n_R, int n_C, int D, int trows,
                                                               int pitch, void* F_C, int out_mode, int* status) {
  extern __shared__ __align__(16) uint8_t fm_smem[];
  const int warp = threadIdx.x >> 5;
  uint8_t* T = fm_smem + warp * trows * pitch;
  const uint32_t sbase = smem_u32(T);
  const long long c_begin = ((long long)blockIdx.x * FM_WARPS + warp) * FM_RUN;
  const int ncols = n_R + n_C;
  int staged = -1;
  // zero the padding rows once
  zero_rows(T + (n_R + n_C) * pitch, pitch, trows - (n_R + n_C), D);
  for (int i = 0; i < FM_RUN; ++i) {
    const long long c = c_begin + i;
    if (c >= B_C) break;
    const int r = req_idx[c];
    if (r < 0 || r >= B_R) {
      if ((threadIdx.x & 31) == 0) set_status(status, ROCS_ERR_INDEX);
      continue;
    }
    __syncwarp();
    if (r != staged) {
      stage_rows(T, pitch, E_R + (long long)r * n_R * D, n_R, D);
      staged = r;
    }
    stage_rows(T + n_R * pitch, pitch, E_C + c * n_C * D, n_C, D);
    __syncwarp();
    const long long fsz = (long long)n_C * ncols;   // one candidate's F^C; split rows hold [hi | lo]
    gram_tile(sbase, pitch, n_R, n_C, ncols, D, F_C, out_mode, c * fsz * (out_mode == 2 ? 2 : 1), ncols, fsz);
  }
}

template <typename TIN>
__global__ void __launch_bounds__(FM_WARPS * 32) fm_req_kernel(const TIN* __restrict__ E_R, int B_R, int n_R, int D,
                                                              int trows, int pitch, void* F_R, int out_mode) {
  extern __shared__ __align__(16) uint8_t fm_smem[];
  const int warp = threadIdx.x >> 5;
  const int r = blockIdx.x * FM_WARPS + warp;
  if (r >= B_R) return;
  uint8_t* T = fm_smem + warp * trows * pitch;
  zero_rows(T + n_R * pitch, pitch, trows - n_R, D);
  stage_rows(T, pitch, E_R + (long long)r * n_R * D, n_R, D);
  __syncwarp();
  const long long fsz = (long long)n_R * n_R;
  gram_tile(smem_u32(T), pitch, 0, n_R, n_R, D, F_R, out_mode, r * fsz * (out_mode == 2 ? 2 : 1), n_R, fsz);
}

// ---------------------------------------------------------------------------------------------
// token LCB (SIMT; P is tiny).  Inputs bf16 or fp32; out_mode 0 fp32, 1 bf16, 2 bf16 hi/lo pair
// (the low half at +lo_off elements within the row).
// ---------------------------------------------------------------------------------------------
__device__ __forceinline__ float ld_f(const float* p) { return __ldg(p); }
__device__ __forceinline__ float ld_f(const __nv_bfloat16* p) { return __bfloat162float(*p); }

__device__ __forceinline__ void store_val(void* out, long long off, float v, int out_mode, long long lo_off) {
  if (out_mode == 0) {
    reinterpret_cast<float*>(out)[off] = v;
  } else {
    const __nv_bfloat16 h = __float2bfloat16_rn(v);
    reinterpret_cast<__nv_bfloat16*>(out)[off] = h;
    if (out_mode == 2) reinterpret_cast<__nv_bfloat16*>(out)[off + lo_off] = __float2bfloat16_rn(v - __bfloat162float(h));
  }
}

// Request side: one block per request, thread per (o, d).
template <typename TIN>
__global__ void lcb_req_kernel(const TIN* __restrict__ E_R, long long ld_ER, int n_R, int D,
                               const __nv_bfloat16* __restrict__ P_RR, const __nv_bfloat16* __restrict__ P_CR,
                               int o_R, int o_C, void* L_R, long long ld_LR, int out_mode, long long lo_off,
                               float* __restrict__ ZL) {
  const int r = blockIdx.x;
  const TIN* e = E_R + (long long)r * ld_ER;
  for (int i = threadIdx.x; i < (o_R + o_C) * D; i += blockDim.x) {
    const int o = i / D, d = i - o * D;
    const bool req = o < o_R;
    const __nv_bfloat16* p = req ? P_RR + (long long)o * n_R : P_CR + (long long)(o - o_R) * n_R;
    float acc = 0.f;
    for (int t = 0; t < n_R; ++t) acc = fmaf(__bfloat162float(p[t]), ld_f(e + t * D + d), acc);
    if (req) store_val(L_R, (long long)r * ld_LR + (long long)o * D + d, acc, out_mode, lo_off);
    else ZL[((long long)r * o_C + (o - o_R)) * D + d] = acc;
  }
}

// The same with the request's rows and the weights staged in shared memory first (as floats),
// so the token loop reads shared memory instead of re-reading global memory for every output
// row.  Same accumulation order, so the same bits.
template <typename TIN>
__global__ void lcb_req_staged_kernel(const TIN* __restrict__ E_R, long long ld_ER, int n_R, int D,
                                      const __nv_bfloat16* __restrict__ P_RR, const __nv_bfloat16* __restrict__ P_CR,
                                      int o_R, int o_C, void* L_R, long long ld_LR, int out_mode, long long lo_off,
                                      float* __restrict__ ZL) {
  extern __shared__ float lcb_sm[];
  float* sE = lcb_sm;              // [n_R][D]
  float* sP = sE + n_R * D;        // [o_R + o_C][n_R]
  const int r = blockIdx.x;
  const TIN* e = E_R + (long long)r * ld_ER;
  for (int i = threadIdx.x; i < n_R * D; i += blockDim.x) sE[i] = ld_f(e + i);
  for (int i = threadIdx.x; i < (o_R + o_C) * n_R; i += blockDim.x) {
    const int o = i / n_R, t = i - o * n_R;
    sP[i] = __bfloat162float(o < o_R ? P_RR[(long long)o * n_R + t] : P_CR[(long long)(o - o_R) * n_R + t]);
  }
  __syncthreads();
  for (int i = threadIdx.x; i < (o_R + o_C) * D; i += blockDim.x) {
    const int o = i / D, d = i - o * D;
    const float* p = sP + o * n_R;
    float acc = 0.f;
    for (int t = 0; t < n_R; ++t) acc = fmaf(p[t], sE[t * D + d], acc);
    if (o < o_R) store_val(L_R, (long long)r * ld_LR + (long long)o * D + d, acc, out_mode, lo_off);
    else ZL[((long long)r * o_C + (o - o_R)) * D + d] = acc;
  }
}

// Candidate side: one warp per candidate; lane owns features d = lane + 32 j (j < DPL).
constexpr int LCB_OMAX = 8;

template <typename TIN, int DPL>
__global__ void lcb_cand_kernel(const TIN* __restrict__ E_C, long long ld_EC, const int32_t* __restrict__ req_idx,
                                int B_R, long long B_C, int n_C, int D, const __nv_bfloat16* __restrict__ P_CC, int o_C,
                                const float* __restrict__ ZL, void* L_C, long long ld_LC, int out_mode,
                                long long lo_off, int* status) {
  __shared__ float sP[LCB_OMAX * 64];
  for (int i = threadIdx.x; i < o_C * n_C; i += blockDim.x) sP[i] = __bfloat162float(P_CC[i]);
  __syncthreads();
  const long long c = ((long long)blockIdx.x * blockDim.x + threadIdx.x) >> 5;
  const int lane = threadIdx.x & 31;
  if (c >= B_C) return;
  const int r = req_idx[c];
  if (r < 0 || r >= B_R) {
    if (lane == 0) set_status(status, ROCS_ERR_INDEX);
    return;
  }
  float acc[LCB_OMAX][DPL];
#pragma unroll
  for (int o = 0; o < LCB_OMAX; ++o)
#pragma unroll
    for (int j = 0; j < DPL; ++j) {
      const int d = lane + 32 * j;
      acc[o][j] = (o < o_C && d < D) ? ZL[((long long)r * o_C + o) * D + d] : 0.f;
    }
  const TIN* ec = E_C + c * ld_EC;
  for (int t = 0; t < n_C; ++t) {
    float e[DPL];
#pragma unroll
    for (int j = 0; j < DPL; ++j) {
      const int d = lane + 32 * j;
      e[j] = d < D ? ld_f(ec + t * D + d) : 0.f;
    }
#pragma unroll
    for (int o = 0; o < LCB_OMAX; ++o) {
      if (o < o_C) {
        const float p = sP[o * n_C + t];
#pragma unroll
        for (int j = 0; j < DPL; ++j) acc[o][j] = fmaf(p, e[j], acc[o][j]);
      }
    }
  }
#pragma unroll
  for (int o = 0; o < LCB_OMAX; ++o) {
    if (o >= o_C) continue;
#pragma unroll
    for (int j = 0; j < DPL; ++j) {
      const int d = lane + 32 * j;
      if (d < D) store_val(L_C, c * ld_LC + (long long)o * D + d, acc[o][j], out_mode, lo_off);
    }
  }
}

int fm_trows(int n_R, int n_C) {
  auto r16 = [](int x) { return (x + 15) / 16 * 16; };
  int t = n_R + r16(n_C);
  t = t > r16(n_R + n_C) ? t : r16(n_R + n_C);
  t = t > r16(n_R) ? t : r16(n_R);
  return t;
}

template <typename TIN>
rocs_status fm_launch(rocs_context* ctx, const TIN* E_R, const TIN* E_C, const int32_t* req_idx, int B_R, long long B_C,
                      int n_R, int n_C, int D, void* F_R, void* F_C, int out_mode, cudaStream_t s) {
  const int pitch = D * 2 + 16;
  const int trows = fm_trows(n_R, n_C);
  const int smem = FM_WARPS * trows * pitch;
  static bool attr[64] = {false};
  if (ctx->device < 64 && !attr[ctx->device]) {
    rocs_status st = cuda_check(cudaFuncSetAttribute(fm_cand_kernel<TIN>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                                     227 * 1024),
                                "cudaFuncSetAttribute(fm_cand)");
    if (st != ROCS_OK) return st;
    st = cuda_check(cudaFuncSetAttribute(fm_req_kernel<TIN>, cudaFuncAttributeMaxDynamicSharedMemorySize, 227 * 1024),
                    "cudaFuncSetAttribute(fm_req)");
    if (st != ROCS_OK) return st;
    attr[ctx->device] = true;
  }
  if (F_R != nullptr && B_R > 0) {
    LaunchTimer lt_("fm_req", s);
    fm_req_kernel<TIN><<<(B_R + FM_WARPS - 1) / FM_WARPS, FM_WARPS * 32, smem, s>>>(E_R, B_R, n_R, D, trows, pitch, F_R,
                                                                                  out_mode);
    rocs_status st = cuda_check(cudaGetLastError(), "fm_req_kernel");
    if (st != ROCS_OK) return st;
  }
  if (B_C > 0) {
    const long long per_block = (long long)FM_WARPS * FM_RUN;
    const long long blocks = (B_C + per_block - 1) / per_block;
    LaunchTimer lt_("fm_cand", s);
    fm_cand_kernel<TIN><<<(unsigned)blocks, FM_WARPS * 32, smem, s>>>(E_R, E_C, req_idx, B_R, B_C, n_R, n_C, D, trows,
                                                                     pitch, F_C, out_mode, ctx->d_status);
    return cuda_check(cudaGetLastError(), "fm_cand_kernel");
  }
  return ROCS_OK;
}

template <typename TIN>
rocs_status lcb_launch(rocs_context* ctx, const TIN* E_R, long long ld_ER, const TIN* E_C, long long ld_EC,
                       const int32_t* req_idx, int B_R, long long B_C, int n_R, int n_C, int D, const void* P_RR,
                       const void* P_CR, const void* P_CC, int o_R, int o_C, void* L_R, long long ld_LR, void* L_C,
                       long long ld_LC, int out_mode, long long lo_R, long long lo_C, float* ws_Z, cudaStream_t s) {
  if (B_R > 0 && (o_R + o_C) > 0) {
    LaunchTimer lt_("lcb_req", s);
    const size_t sm_bytes = ((size_t)n_R * D + (size_t)(o_R + o_C) * n_R) * sizeof(float);
    if (sm_bytes <= 48 * 1024)
      lcb_req_staged_kernel<TIN><<<B_R, 256, sm_bytes, s>>>(E_R, ld_ER, n_R, D, (const __nv_bfloat16*)P_RR,
                                                             (const __nv_bfloat16*)P_CR, o_R, o_C, L_R, ld_LR,
                                                             out_mode, lo_R, ws_Z);
    else
      lcb_req_kernel<TIN><<<B_R, 256, 0, s>>>(E_R, ld_ER, n_R, D, (const __nv_bfloat16*)P_RR,
                                              (const __nv_bfloat16*)P_CR, o_R, o_C, L_R, ld_LR, out_mode, lo_R, ws_Z);
    rocs_status st = cuda_check(cudaGetLastError(), "lcb_req_kernel");
    if (st != ROCS_OK) return st;
  }
  if (B_C > 0 && o_C > 0) {
    const long long threads = B_C * 32;
    const unsigned blocks = (unsigned)((threads + 255) / 256);
    const int dpl = (D + 31) / 32;
    LaunchTimer lt_("lcb_cand", s);
    if (dpl <= 4)
      lcb_cand_kernel<TIN, 4><<<blocks, 256, 0, s>>>(E_C, ld_EC, req_idx, B_R, B_C, n_C, D, (const __nv_bfloat16*)P_CC,
                                                     o_C, ws_Z, L_C, ld_LC, out_mode, lo_C, ctx->d_status);
    else
      lcb_cand_kernel<TIN, 8><<<blocks, 256, 0, s>>>(E_C, ld_EC, req_idx, B_R, B_C, n_C, D, (const __nv_bfloat16*)P_CC,
                                                     o_C, ws_Z, L_C, ld_LC, out_mode, lo_C, ctx->d_status);
    return cuda_check(cudaGetLastError(), "lcb_cand_kernel");
  }
  return ROCS_OK;
}

// Dynamic shared memory of the fused pass: the ring, the pair blocks and 1 KB to align them.  The
// cap leaves room under the 227 KB per block for the kernel's static arrays.
constexpr size_t FC_SMEM_MAX = 223 * 1024;
size_t fused_smem_bytes(int n_R, int n_C, int in_f32) {
  const int D = 128, pitch = D * 2 + 16;
  return 1024 + (size_t)FC_STAGES * NC_MAX * D * (in_f32 ? 4 : 2) + (size_t)FC_PAIRS * fc_pair_bytes(fm_trows(n_R, n_C), pitch);
}

typedef CUresult (*EncodeTiledFnFm)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                    const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                    CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

template <typename TIN>
rocs_status fused_launch(rocs_context* ctx, const TIN* E_R, const TIN* E_C, const int32_t* req_idx, int B_R,
                         long long B_C, int n_R, int n_C, void* F_C, const void* P_CC, int o_C, const float* ZL,
                         float* L_C, const void* q_pCC, const float* ZQ, void* tC, cudaStream_t s) {
  const int D = 128;
  const int pitch = D * 2 + 16;
  const int trows = fm_trows(n_R, n_C);
  const size_t smem = fused_smem_bytes(n_R, n_C, sizeof(TIN) == 4);
  if (n_C > NC_MAX || o_C < 1 || o_C > LCB_OMAX_F || smem > FC_SMEM_MAX) {
    set_error("fused candidate pass: unsupported n_R=%d n_C=%d o_C=%d", n_R, n_C, o_C);
    return ROCS_ERR_UNSUPPORTED;
  }
  static bool attr[64] = {false};
  if (ctx->device < 64 && !attr[ctx->device]) {
    rocs_status st = cuda_check(cudaFuncSetAttribute(glm_cand_fused_kernel<TIN>,
                                                     cudaFuncAttributeMaxDynamicSharedMemorySize, (int)FC_SMEM_MAX),
                                "cudaFuncSetAttribute(glm_cand_fused)");
    if (st != ROCS_OK) return st;
    attr[ctx->device] = true;
  }
  if (B_C == 0) return ROCS_OK;
  // L^C [B_C * o_C, D] fp32 through TMA stores: boxes of o_C rows x 32 floats, 128-byte swizzle.
  // A base address off the 16-byte grid takes the plain stores.
  CUtensorMap mapL;
  memset(&mapL, 0, sizeof(mapL));
  int l_tma = 0;
  if ((reinterpret_cast<uintptr_t>(L_C) & 15) == 0 && B_C * o_C < (1LL << 31)) {
    EncodeTiledFnFm fn = reinterpret_cast<EncodeTiledFnFm>(ctx->encode_fn);
    cuuint64_t dims[2] = {(cuuint64_t)D, (cuuint64_t)(B_C * o_C)};
    cuuint64_t strides[1] = {(cuuint64_t)D * 4};
    cuuint32_t box[2] = {32, (cuuint32_t)o_C};
    cuuint32_t estr[2] = {1, 1};
    l_tma = fn(&mapL, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 2, L_C, dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
               CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_NONE,
               CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
  }
  // one CTA per SM, each over a contiguous candidate range (runs of a request stay together)
  const long long blocks = B_C < ctx->num_sms ? B_C : ctx->num_sms;
  const long long per_block = (B_C + blocks - 1) / blocks;
  LaunchTimer lt_("glm_cand_fused", s);
  glm_cand_fused_kernel<TIN><<<(unsigned)blocks, 32 * (1 + FC_CONSUMERS), smem, s>>>(
      E_R, E_C, req_idx, B_R, B_C, per_block, n_R, n_C, trows, pitch, (__nv_bfloat16*)F_C,
      (const __nv_bfloat16*)P_CC, o_C, ZL, L_C, (const __nv_bfloat16*)q_pCC, ZQ, (__nv_bfloat16*)tC, mapL, l_tma,
      ctx->d_status);
  return cuda_check(cudaGetLastError(), "glm_cand_fused_kernel");
}

}  // namespace

bool glm_cand_fused_fits(int D, int n_R, int n_C, int o_C, int in_f32) {
  return D == 128 && n_C <= NC_MAX && o_C >= 1 && o_C <= LCB_OMAX_F && fused_smem_bytes(n_R, n_C, in_f32) <= FC_SMEM_MAX;
}

rocs_status launch_glm_cand_fused(rocs_context* ctx, const void* E_R, const void* E_C, const int32_t* req_idx,
                                  int B_R, long long B_C, int n_R, int n_C, int in_f32, void* F_C, const void* P_CC,
                                  int o_C, const float* ZL, float* L_C, const void* q_pCC, const float* ZQ, void* tC,
                                  cudaStream_t s) {
  if (in_f32)
    return fused_launch<float>(ctx, (const float*)E_R, (const float*)E_C, req_idx, B_R, B_C, n_R, n_C, F_C, P_CC, o_C,
                               ZL, L_C, q_pCC, ZQ, tC, s);
  return fused_launch<__nv_bfloat16>(ctx, (const __nv_bfloat16*)E_R, (const __nv_bfloat16*)E_C, req_idx, B_R, B_C,
                                     n_R, n_C, F_C, P_CC, o_C, ZL, L_C, q_pCC, ZQ, tC, s);
}

rocs_status launch_fm(rocs_context* ctx, const void* E_R, const void* E_C, const int32_t* req_idx, int B_R,
                      long long B_C, int n_R, int n_C, int D, void* F_R, void* F_C, int in_f32, int out_mode,
                      cudaStream_t s) {
  if (in_f32)
    return fm_launch<float>(ctx, (const float*)E_R, (const float*)E_C, req_idx, B_R, B_C, n_R, n_C, D, F_R, F_C,
                            out_mode, s);
  return fm_launch<__nv_bfloat16>(ctx, (const __nv_bfloat16*)E_R, (const __nv_bfloat16*)E_C, req_idx, B_R, B_C, n_R,
                                  n_C, D, F_R, F_C, out_mode, s);
}

rocs_status launch_token_lcb(rocs_context* ctx, const void* E_R, long long ld_ER, const void* E_C, long long ld_EC,
                             const int32_t* req_idx, int B_R, long long B_C, int n_R, int n_C, int D,
                             const void* P_RR, const void* P_CR, const void* P_CC, int o_R, int o_C, void* L_R,
                             long long ld_LR, void* L_C, long long ld_LC, int in_f32, int out_mode, long long lo_R,
                             long long lo_C, float* ws_Z, cudaStream_t s) {
  if (in_f32)
    return lcb_launch<float>(ctx, (const float*)E_R, ld_ER, (const float*)E_C, ld_EC, req_idx, B_R, B_C, n_R, n_C, D,
                             P_RR, P_CR, P_CC, o_R, o_C, L_R, ld_LR, L_C, ld_LC, out_mode, lo_R, lo_C, ws_Z, s);
  return lcb_launch<__nv_bfloat16>(ctx, (const __nv_bfloat16*)E_R, ld_ER, (const __nv_bfloat16*)E_C, ld_EC, req_idx,
                                   B_R, B_C, n_R, n_C, D, P_RR, P_CR, P_CC, o_R, o_C, L_R, ld_LR, L_C, ld_LC, out_mode,
                                   lo_R, lo_C, ws_Z, s);
}

}  // namespace rocs
