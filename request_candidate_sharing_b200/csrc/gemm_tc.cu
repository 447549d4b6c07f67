// Persistent grouped GEMM on the 5th-generation tensor cores (tcgen05 + TMEM + TMA), with the
// IKBO epilogue: bias, the request-map gather Z[m_i] and the activation are applied to the
// accumulator tile in registers and only the final output is written
// ([REV] §2.4: "the candidate GEMM's epilogue looks up m_i, loads the request contribution
// and adds it in registers").
//
// Design (B200, one CTA per SM, 192 threads):
//   warp 0      TMA producer: A tile 128x64 and B tile BNx64 (bf16, 128-B swizzle) per stage,
//               4-stage ring of mbarriers (full: TMA -> MMA, empty: MMA -> TMA).
//   warp 1      allocates 512 TMEM columns (two 128x256 fp32 accumulators); lane 0 issues
//               tcgen05.mma (M=128, N=BN, K=16) and commits to the ring / accumulator barriers.
//   warps 2..9  epilogue: two warps per TMEM lane quarter, splitting the tile's 32-column
//               chunks between them; tcgen05.ld 32 columns at a time (each thread owns one
//               output row), + bias + Z[gidx[row]] + act, bf16/fp32 stores.  The second
//               accumulator lets the epilogue of tile i overlap the main loop of tile i+1 (the
//               Blackwell form of the pages' producer / ping-pong consumer warp specialisation).
// Tiles of all problems form one static round-robin schedule over the persistent CTAs; when
// every problem has the same M, tiles are interleaved per 128-row block so the problems that
// share the A operand read it from L2 rather than HBM.
// No cluster launch, no multicast: each CTA loads its own operand tiles.
#include <algorithm>
#include <cstring>

#include "common.cuh"
#include "internal.h"

namespace rocs {
namespace {

constexpr int BM = 128;
constexpr int BK = 64;
constexpr int BN_MAX = 256;
constexpr int STAGES = 4;
constexpr int A_STAGE = BM * BK * 2;       // 16 KiB
constexpr int B_STAGE = BN_MAX * BK * 2;   // 32 KiB
constexpr int THREADS = 320;
constexpr int EPI_THREADS = 256;
constexpr int TMEM_COLS = 512;
constexpr int EPI_BUF = 4096;              // per epilogue warp: one 32x32 output chunk (fp32, or bf16 hi + lo)
constexpr int SMEM_BYTES = 1024 + STAGES * (A_STAGE + B_STAGE) + (EPI_THREADS / 32) * EPI_BUF + 256;

struct Problem {
  CUtensorMap tmA;
  CUtensorMap tmB;
  CUtensorMap tmO;     // output [M, N] (out_mode 2: the hi half), box 32 x 32, stored by TMA
  CUtensorMap tmOlo;   // out_mode 2: the lo half at column offset lo_off
  const float* bias;
  const float* scale;   // optional per-column factor on the accumulator (FP8 weights' channel scales)
  const float* Z;
  const int32_t* gidx;
  void* out;
  long long ldo, ldz;
  int M, N, K, BN;
  int out_mode, act, gidx_bound, vec_ok, tma_out;
  int m_tiles, n_tiles, k_blocks, b_kblocks, tile_start, n_start;
  long long lo_off;   // out_mode 2: column offset of the low half
  // Request/candidate tiles in one launch (the IKBO mega-kernel): flag_role 1 = this problem
  // publishes each finished tile in flags[mb * n_tiles + nb] (one increment per epilogue warp);
  // flag_role 2 = this problem's Z rows come from such a problem in the same launch, whose tile
  // (zi / BM, nb) must have published before they are read (flag_ntiles = its n_tiles).
  int* flags;
  int flag_role, flag_ntiles;
};

struct Params {
  Problem p[kMaxGemmProblems];
  int nprob;
  int total_tiles;
  int interleave;     // 1: tile order (m block, problem, n block); 0: problem-major
  int n_per_m;        // sum of n_tiles over problems (interleave mode)
  int* status;
  long long flag_budget;   // clock64 cycles a completion-flag wait may take
  int withhold_flag;       // test hook: this completion flag is never published (-1: none)
};

__device__ __forceinline__ void decode_tile(const Params& P, int t, int& pi, int& mb, int& nb) {
  if (P.interleave) {
    mb = t / P.n_per_m;
    int r = t - mb * P.n_per_m;
    pi = 0;
    while (pi + 1 < P.nprob && r >= P.p[pi + 1].n_start) ++pi;
    nb = r - P.p[pi].n_start;
  } else {
    pi = 0;
    while (pi + 1 < P.nprob && t >= P.p[pi + 1].tile_start) ++pi;
    int local = t - P.p[pi].tile_start;
    mb = local / P.p[pi].n_tiles;
    nb = local - mb * P.p[pi].n_tiles;
  }
}

// Spin (bounded by `budget` cycles) until *flag >= target, with acquire ordering for the reads
// that follow.
__device__ __forceinline__ bool wait_flag(const int* flag, int target, long long budget, int* status,
                                          volatile int* abort_flag) {
  const long long t0 = clock64();
  while (true) {
    int v;
    asm volatile("ld.acquire.gpu.global.b32 %0, [%1];" : "=r"(v) : "l"(flag) : "memory");
    if (v >= target) return true;
    if (abort_flag && *abort_flag) return false;
    if (clock64() - t0 > budget) {
      set_status(status, ROCS_ERR_DEVICE_TIMEOUT);
      if (abort_flag) *abort_flag = 1;
      return false;
    }
    __nanosleep(64);
  }
}

__device__ __forceinline__ void store_bf16_32(__nv_bfloat16* o, int ncol, bool vec, const float (&v)[32]) {
  if (ncol == 32 && vec) {
    uint4* o4 = reinterpret_cast<uint4*>(o);
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      uint4 w;
      w.x = pack_bf16x2(v[8 * j + 0], v[8 * j + 1]);
      w.y = pack_bf16x2(v[8 * j + 2], v[8 * j + 3]);
      w.z = pack_bf16x2(v[8 * j + 4], v[8 * j + 5]);
      w.w = pack_bf16x2(v[8 * j + 6], v[8 * j + 7]);
      o4[j] = w;
    }
  } else {
#pragma unroll
    for (int j = 0; j < 32; ++j)
      if (j < ncol) o[j] = __float2bfloat16_rn(v[j]);
  }
}

// out_mode 0: fp32; 1: bf16; 2: bf16 pair -- hi = bf16(v) at column c, lo = bf16(v - hi) at
// column c + lo_off (activations carried as hi + lo keep ~16 mantissa bits for the next GEMM).
__device__ __forceinline__ void store_chunk(const Problem& pr, long long grow, int col0, float (&v)[32]) {
  const int ncol = min(32, pr.N - col0);
  if (pr.out_mode == 1) {
    store_bf16_32(reinterpret_cast<__nv_bfloat16*>(pr.out) + grow * pr.ldo + col0, ncol, pr.vec_ok, v);
  } else if (pr.out_mode == 2) {
    __nv_bfloat16* o = reinterpret_cast<__nv_bfloat16*>(pr.out) + grow * pr.ldo + col0;
    float lo[32];
#pragma unroll
    for (int j = 0; j < 32; ++j) {
      const float h = __bfloat162float(__float2bfloat16_rn(v[j]));
      lo[j] = v[j] - h;
      v[j] = h;
    }
    store_bf16_32(o, ncol, pr.vec_ok, v);
    store_bf16_32(o + pr.lo_off, ncol, pr.vec_ok, lo);
  } else {
    float* o = reinterpret_cast<float*>(pr.out) + grow * pr.ldo + col0;
    if (ncol == 32 && pr.vec_ok) {
      float4* o4 = reinterpret_cast<float4*>(o);
#pragma unroll
      for (int j = 0; j < 8; ++j) o4[j] = make_float4(v[4 * j], v[4 * j + 1], v[4 * j + 2], v[4 * j + 3]);
    } else {
#pragma unroll
      for (int j = 0; j < 32; ++j)
        if (j < ncol) o[j] = v[j];
    }
  }
}

// bias, the request contribution Z[gidx[row]] and the activation on one thread's 32 values.  Z
// written by the same launch (flag_role 2) is read with ordinary loads, ordered after the flag's
// acquire, never through the non-coherent read-only path.
__device__ __forceinline__ void epilogue_math(const Problem& pr, const float* zrow, int col0, float (&v)[32]) {
  const bool full32 = (col0 + 32 <= pr.N) && pr.vec_ok;
  if (pr.scale != nullptr) {
#pragma unroll
    for (int j = 0; j < 32; ++j) v[j] *= col0 + j < pr.N ? __ldg(pr.scale + col0 + j) : 0.f;
  }
  if (pr.bias != nullptr) {
    if (full32) {
      const float4* b4 = reinterpret_cast<const float4*>(pr.bias + col0);
#pragma unroll
      for (int j = 0; j < 8; ++j) {
        float4 b = __ldg(b4 + j);
        v[4 * j] += b.x; v[4 * j + 1] += b.y; v[4 * j + 2] += b.z; v[4 * j + 3] += b.w;
      }
    } else {
#pragma unroll
      for (int j = 0; j < 32; ++j)
        if (col0 + j < pr.N) v[j] += pr.bias[col0 + j];
    }
  }
  if (zrow != nullptr) {
    if (full32) {
      const float4* z4 = reinterpret_cast<const float4*>(zrow + col0);
#pragma unroll
      for (int j = 0; j < 8; ++j) {
        const float4 z = pr.flag_role == 2 ? z4[j] : __ldg(z4 + j);
        v[4 * j] += z.x; v[4 * j + 1] += z.y; v[4 * j + 2] += z.z; v[4 * j + 3] += z.w;
      }
    } else {
#pragma unroll
      for (int j = 0; j < 32; ++j)
        if (col0 + j < pr.N) v[j] += zrow[col0 + j];
    }
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
}

// bf16 outputs (out_mode 1) go out in 32 x 64 boxes instead: a warp stages two adjacent chunks
// (128-byte rows, 128-byte swizzle) and issues one store for both.  The epilogue is bound by the
// number of output copies, not their bytes: halving them cut the short-K GEMMs by 9-14%.
//
// One warp's 32 x 32 output chunk (lane = row) through shared memory and one TMA store: rows are
// written into `buf` in the layout of the output map's swizzle (128-byte rows for fp32, 64-byte
// rows for bf16: the 16-byte unit j of row r sits at j ^ (r & 7), resp. j ^ ((r >> 1) & 3)),
// so the shared-memory writes are free of bank conflicts and the global write is whole lines.
__device__ __forceinline__ void store_chunk_tma(const Problem& pr, uint8_t* buf, int row0, int col0,
                                                const float (&v)[32]) {
  const int lane = threadIdx.x & 31;
  if (lane == 0) bulk_wait_read_all();   // the previous chunk's copy has read the buffer
  __syncwarp();
  if (pr.out_mode == 0) {
    uint8_t* rowp = buf + lane * 128;
#pragma unroll
    for (int j = 0; j < 8; ++j)
      *reinterpret_cast<float4*>(rowp + ((j ^ (lane & 7)) << 4)) =
          make_float4(v[4 * j], v[4 * j + 1], v[4 * j + 2], v[4 * j + 3]);
  } else {
    uint8_t* rowp = buf + lane * 64;
    const int sw = (lane >> 1) & 3;
    uint32_t hi[16], lo[16];
#pragma unroll
    for (int j = 0; j < 16; ++j) {
      hi[j] = pack_bf16x2(v[2 * j], v[2 * j + 1]);
      if (pr.out_mode == 2) lo[j] = pack_bf16x2(v[2 * j] - bf16_lo(hi[j]), v[2 * j + 1] - bf16_hi(hi[j]));
    }
#pragma unroll
    for (int j = 0; j < 4; ++j)
      *reinterpret_cast<uint4*>(rowp + ((j ^ sw) << 4)) = make_uint4(hi[4 * j], hi[4 * j + 1], hi[4 * j + 2], hi[4 * j + 3]);
    if (pr.out_mode == 2) {
#pragma unroll
      for (int j = 0; j < 4; ++j)
        *reinterpret_cast<uint4*>(rowp + 2048 + ((j ^ sw) << 4)) =
            make_uint4(lo[4 * j], lo[4 * j + 1], lo[4 * j + 2], lo[4 * j + 3]);
    }
  }
  fence_proxy_async_smem();
  __syncwarp();
  if (lane == 0) {
    tma_store_2d(&pr.tmO, buf, col0, row0);
    if (pr.out_mode == 2) tma_store_2d(&pr.tmOlo, buf + 2048, col0, row0);
    bulk_commit_group();
  }
}

template <bool PLAIN>
__global__ void __launch_bounds__(THREADS, 1) gemm_tc_kernel(const __grid_constant__ Params P) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* base = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sA = base;
  uint8_t* sB = base + STAGES * A_STAGE;
  uint8_t* sEpi = sB + STAGES * B_STAGE;   // 1024-B aligned
  uint64_t* bars = reinterpret_cast<uint64_t*>(sEpi + (EPI_THREADS / 32) * EPI_BUF);
  uint64_t* full = bars;
  uint64_t* empty = bars + STAGES;
  uint64_t* tfull = bars + 2 * STAGES;
  uint64_t* tempty = tfull + 2;
  uint64_t* drain = tempty + 2;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(drain + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;

  if (threadIdx.x == 0) {
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&tfull[b], 1);
      mbar_init(&tempty[b], EPI_THREADS);
    }
    mbar_init(drain, 1);
    *abort_flag = 0;
    fence_barrier_init();
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, TMEM_COLS);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;

  if (warp == 0) {
    if (lane == 0) {
      // ---------------- TMA producer ----------------
      for (int i = 0; i < P.nprob; ++i) {
        prefetch_tensormap(&P.p[i].tmA);
        prefetch_tensormap(&P.p[i].tmB);
      }
      int stage = 0;
      uint32_t phase = 0;
      long long issued = 0;
      bool ok = true;
      for (int t = blockIdx.x; t < P.total_tiles && ok; t += gridDim.x) {
        int pi, mb, nb;
        decode_tile(P, t, pi, mb, nb);
        const Problem& pr = P.p[pi];
        for (int kb = 0; kb < pr.k_blocks; ++kb) {
          if (!mbar_wait(&empty[stage], phase ^ 1, P.status, abort_flag)) { ok = false; break; }
          mbar_arrive_expect_tx(&full[stage], A_STAGE + pr.BN * BK * 2);
          tma_load_2d(sA + stage * A_STAGE, &pr.tmA, &full[stage], kb * BK, mb * BM);
          // split operands: A rows are [hi | lo], B's k blocks repeat for the low half
          const int kbB = kb < pr.b_kblocks ? kb : kb - pr.b_kblocks;
          tma_load_2d(sB + stage * B_STAGE, &pr.tmB, &full[stage], kbB * BK, nb * pr.BN);
          ++issued;
          if (++stage == STAGES) { stage = 0; phase ^= 1; }
        }
      }
      // Make sure no copy issued by this CTA is still landing in shared memory at exit.
      for (int i = 0; i < STAGES && i < issued; ++i) {
        if (--stage < 0) { stage = STAGES - 1; phase ^= 1; }
        mbar_wait(&full[stage], phase, P.status, nullptr);
      }
    }
  } else if (warp == 1) {
    if (lane == 0) {
      // ---------------- MMA issuer ----------------
      int stage = 0;
      uint32_t phase = 0;
      int acc = 0;
      uint32_t acc_phase = 0;
      bool ok = true;
      for (int t = blockIdx.x; t < P.total_tiles && ok; t += gridDim.x) {
        int pi, mb, nb;
        decode_tile(P, t, pi, mb, nb);
        const Problem& pr = P.p[pi];
        if (!mbar_wait(&tempty[acc], acc_phase ^ 1, P.status, abort_flag)) break;
        tc_fence_after();
        const uint32_t d_tmem = tmem_base + (uint32_t)(acc * BN_MAX);
        const uint32_t idesc = idesc_bf16_f32(BM, pr.BN);
        for (int kb = 0; kb < pr.k_blocks; ++kb) {
          if (!mbar_wait(&full[stage], phase, P.status, abort_flag)) { ok = false; break; }
          tc_fence_after();
          const uint32_t a0 = smem_u32(sA + stage * A_STAGE);
          const uint32_t b0 = smem_u32(sB + stage * B_STAGE);
#pragma unroll
          for (int k = 0; k < BK / 16; ++k)
            tc_mma_bf16(d_tmem, smem_desc_sw128(a0 + k * 32), smem_desc_sw128(b0 + k * 32), idesc,
                        (kb | k) != 0 ? 1u : 0u);
          tc_commit(&empty[stage]);
          if (++stage == STAGES) { stage = 0; phase ^= 1; }
        }
        if (!ok) break;
        tc_commit(&tfull[acc]);
        acc ^= 1;
        if (acc == 0) acc_phase ^= 1;
      }
      // Drain: every MMA this thread issued has completed before TMEM is released.
      tc_commit(drain);
      mbar_wait(drain, 0, P.status, nullptr);
    }
  } else {
    if constexpr (PLAIN) {
      // ---------------- epilogue warps, bf16 output with nothing to add or apply ----------------
      // (the encoder's projections): both chunks of a pair are loaded from TMEM before one wait
      // and go straight to bf16.  A kernel of its own, so the general epilogue's state does not
      // crowd its registers.
      const int q = warp & 3, half = (warp - 2) >> 2;
      int acc = 0;
      uint32_t acc_phase = 0;
      uint8_t* buf = sEpi + (warp - 2) * EPI_BUF;
      uint8_t* rowp = buf + lane * 128;
      for (int t = blockIdx.x; t < P.total_tiles; t += gridDim.x) {
        int pi, mb, nb;
        decode_tile(P, t, pi, mb, nb);
        const Problem& pr = P.p[pi];
        if (!mbar_wait(&tfull[acc], acc_phase, P.status, abort_flag)) break;
        tc_fence_after();
        const uint32_t tbase = tmem_base + ((uint32_t)(q * 32) << 16) + (uint32_t)(acc * BN_MAX);
        const int nchunks = pr.BN / 32, npairs = (nchunks + 1) / 2;
        const int lp = npairs - 1 - ((npairs - 1 - half) & 1);   // this warp's last pair (< 0: none)
        if (lp < 0) mbar_arrive(&tempty[acc]);
        for (int pp = half; pp < npairs; pp += 2) {
          if (lane == 0) bulk_wait_read_all();   // the previous copy has read the buffer
          __syncwarp();
          const bool two = 2 * pp + 1 < nchunks;
          uint32_t r0[32], r1[32];
          tmem_ld_32x32b_x32(tbase + (uint32_t)(2 * pp * 32), r0);
          if (two) tmem_ld_32x32b_x32(tbase + (uint32_t)((2 * pp + 1) * 32), r1);
          tmem_ld_wait();
          if (pp == lp) {
            tc_fence_before();
            mbar_arrive(&tempty[acc]);
          }
          // 128-byte rows, 128-byte swizzle: 16-byte unit j of row r at j ^ (r & 7)
#pragma unroll
          for (int u = 0; u < 4; ++u)
            *reinterpret_cast<uint4*>(rowp + ((u ^ (lane & 7)) << 4)) =
                make_uint4(pack_bf16x2(__uint_as_float(r0[8 * u]), __uint_as_float(r0[8 * u + 1])),
                           pack_bf16x2(__uint_as_float(r0[8 * u + 2]), __uint_as_float(r0[8 * u + 3])),
                           pack_bf16x2(__uint_as_float(r0[8 * u + 4]), __uint_as_float(r0[8 * u + 5])),
                           pack_bf16x2(__uint_as_float(r0[8 * u + 6]), __uint_as_float(r0[8 * u + 7])));
          if (two) {
#pragma unroll
            for (int u = 0; u < 4; ++u)
              *reinterpret_cast<uint4*>(rowp + (((4 + u) ^ (lane & 7)) << 4)) =
                  make_uint4(pack_bf16x2(__uint_as_float(r1[8 * u]), __uint_as_float(r1[8 * u + 1])),
                             pack_bf16x2(__uint_as_float(r1[8 * u + 2]), __uint_as_float(r1[8 * u + 3])),
                             pack_bf16x2(__uint_as_float(r1[8 * u + 4]), __uint_as_float(r1[8 * u + 5])),
                             pack_bf16x2(__uint_as_float(r1[8 * u + 6]), __uint_as_float(r1[8 * u + 7])));
          }
          fence_proxy_async_smem();
          __syncwarp();
          if (lane == 0) {
            if (mb * BM + q * 32 < pr.M) tma_store_2d(&pr.tmO, buf, nb * pr.BN + 64 * pp, mb * BM + q * 32);
            bulk_commit_group();
          }
        }
        acc ^= 1;
        if (acc == 0) acc_phase ^= 1;
      }
      // this warp's output stores have landed before the CTA (and its staging memory) goes away
      if (lane == 0) bulk_wait_all();
      __syncwarp();
    } else {
      // ---------------- epilogue warps ----------------
      const int q = warp & 3;            // TMEM lane quarter this warp may access
      const int half = (warp - 2) >> 2;  // which of the two warps on this quarter
      const int row = q * 32 + lane;
      int acc = 0;
      uint32_t acc_phase = 0;
      // this row's request index in a tile, read one tile ahead of its use
      auto load_gidx = [&](int tt) -> int {
        if (tt >= P.total_tiles) return -1;
        int pn, mn, nn;
        decode_tile(P, tt, pn, mn, nn);
        const Problem& q2 = P.p[pn];
        const long long gn = (long long)mn * BM + row;
        return (q2.Z != nullptr && gn < q2.M) ? __ldg(q2.gidx + gn) : -1;
      };
      int zi_next = load_gidx(blockIdx.x);
      unsigned long long seen = 0;   // request tiles this warp has seen published (fused launches)
      for (int t = blockIdx.x; t < P.total_tiles; t += gridDim.x) {
        int pi, mb, nb;
        decode_tile(P, t, pi, mb, nb);
        const Problem& pr = P.p[pi];
        const long long grow = (long long)mb * BM + row;
        bool rvalid = grow < pr.M;
        const float* zrow = nullptr;
        const int zi = zi_next;
        zi_next = load_gidx(t + gridDim.x);
        if (rvalid && pr.Z != nullptr) {
          if (zi < 0 || zi >= pr.gidx_bound) {
            set_status(P.status, ROCS_ERR_INDEX);
            rvalid = false;
          } else {
            zrow = pr.Z + (long long)zi * pr.ldz;
            // this warp's chunks of the row's Z into L1 before the wait for the accumulator (the
            // gathered rows were the epilogue's longest latency at short K); Z that this launch
            // writes only once it is published (below)
            if (pr.flag_role != 2)
              for (int c = half; c < pr.BN / 32; c += 2)
                if (nb * pr.BN + c * 32 < pr.N)
                  asm volatile("prefetch.global.L1 [%0];" ::"l"(zrow + nb * pr.BN + c * 32));
          }
        }
        if (pr.flag_role == 2) {
          // the request tiles holding this warp's rows' Z must have published (their tiles precede
          // every candidate tile in each CTA's order, so they never wait on this one)
          const int lo = __reduce_min_sync(0xffffffffu, zrow != nullptr ? zi : 0x7fffffff);
          const int hi = __reduce_max_sync(0xffffffffu, zrow != nullptr ? zi : -1);
          bool ok = true;
          for (int mbr = hi >= 0 ? lo / BM : 1, mend = hi >= 0 ? hi / BM : 0; mbr <= mend && ok; ++mbr) {
            // a tile seen published stays published: later tiles skip its flag (the first 64)
            const int fi = mbr * pr.flag_ntiles + nb;
            if (fi < 64 && ((seen >> fi) & 1ull)) continue;
            if (lane == 0) ok = wait_flag(pr.flags + fi, EPI_THREADS / 32, P.flag_budget, P.status, abort_flag);
            ok = __shfl_sync(0xffffffffu, ok, 0);
            if (ok && fi < 64) seen |= 1ull << fi;
          }
          if (!ok) {
            rvalid = false;   // timed out: the status says so; this row is not written
            zrow = nullptr;
          } else if (zrow != nullptr) {
            for (int c = half; c < pr.BN / 32; c += 2)
              if (nb * pr.BN + c * 32 < pr.N)
                asm volatile("prefetch.global.L1 [%0];" ::"l"(zrow + nb * pr.BN + c * 32));
          }
        }
        if (!mbar_wait(&tfull[acc], acc_phase, P.status, abort_flag)) break;
        tc_fence_after();
        // a row with a bad request index is skipped, not written: such a warp stores element-wise
        const bool use_tma = pr.tma_out && !__any_sync(0xffffffffu, grow < pr.M && !rvalid);
        const uint32_t tbase = tmem_base + ((uint32_t)(q * 32) << 16) + (uint32_t)(acc * BN_MAX);
        const int nchunks = pr.BN / 32;
        // this warp takes chunks half, half + 2, ... (bf16 output through TMA: adjacent pairs of
        // chunks 2p, 2p + 1 for p = half, half + 2, ..., one 32 x 64 store per pair); it releases the
        // accumulator after its last load
        const bool pair_path = use_tma && pr.out_mode == 1;
        const int npairs = (nchunks + 1) / 2;
        const int lp = npairs - 1 - ((npairs - 1 - half) & 1);
        const int last = pair_path ? (lp < 0 ? -1 : (2 * lp + 1 < nchunks ? 2 * lp + 1 : nchunks - 1))
                                   : nchunks - 1 - ((nchunks - 1 - half) & 1);
        if (last < 0) {
          mbar_arrive(&tempty[acc]);
        }
        if (pair_path) {
          uint8_t* buf = sEpi + (warp - 2) * EPI_BUF;
          uint8_t* rowp = buf + lane * 128;
          for (int pp = half; pp < npairs; pp += 2) {
            if (lane == 0) bulk_wait_read_all();   // the previous copy has read the buffer
            __syncwarp();
  #pragma unroll 1
            for (int hh = 0; hh < 2; ++hh) {
              const int c = 2 * pp + hh;
              if (c >= nchunks) break;
              uint32_t r[32];
              tmem_ld_32x32b_x32(tbase + (uint32_t)(c * 32), r);
              tmem_ld_wait();
              if (c == last) {
                tc_fence_before();
                mbar_arrive(&tempty[acc]);
              }
              const int col0 = nb * pr.BN + c * 32;
              float v[32];
  #pragma unroll
              for (int j = 0; j < 32; ++j) v[j] = __uint_as_float(r[j]);
              if (rvalid) epilogue_math(pr, zrow, col0, v);
              // 128-byte rows, 128-byte swizzle: 16-byte unit j of row r at j ^ (r & 7)
  #pragma unroll
              for (int u = 0; u < 4; ++u)
                *reinterpret_cast<uint4*>(rowp + (((4 * hh + u) ^ (lane & 7)) << 4)) =
                    make_uint4(pack_bf16x2(v[8 * u], v[8 * u + 1]), pack_bf16x2(v[8 * u + 2], v[8 * u + 3]),
                               pack_bf16x2(v[8 * u + 4], v[8 * u + 5]), pack_bf16x2(v[8 * u + 6], v[8 * u + 7]));
            }
            fence_proxy_async_smem();
            __syncwarp();
            if (lane == 0) {
              if (mb * BM + q * 32 < pr.M) tma_store_2d(&pr.tmO, buf, nb * pr.BN + 64 * pp, mb * BM + q * 32);
              bulk_commit_group();
            }
          }
        } else
        for (int c = half; c < nchunks; c += 2) {
          uint32_t r[32];
          __syncwarp();
          tmem_ld_32x32b_x32(tbase + (uint32_t)(c * 32), r);
          tmem_ld_wait();
          if (c == last) {
            tc_fence_before();
            mbar_arrive(&tempty[acc]);
          }
          const int col0 = nb * pr.BN + c * 32;
          if (use_tma && col0 < pr.N && mb * BM + q * 32 < pr.M) {
            // every lane takes part in the staged store; rows past M are clipped by the copy
            float v[32];
  #pragma unroll
            for (int j = 0; j < 32; ++j) v[j] = __uint_as_float(r[j]);
            if (rvalid) epilogue_math(pr, zrow, col0, v);
            store_chunk_tma(pr, sEpi + (warp - 2) * EPI_BUF, mb * BM + q * 32, col0, v);
          } else if (!use_tma && rvalid && col0 < pr.N) {
            float v[32];
  #pragma unroll
            for (int j = 0; j < 32; ++j) v[j] = __uint_as_float(r[j]);
            const bool full32 = (col0 + 32 <= pr.N) && pr.vec_ok;
            if (pr.scale != nullptr) {
  #pragma unroll
              for (int j = 0; j < 32; ++j) v[j] *= col0 + j < pr.N ? __ldg(pr.scale + col0 + j) : 0.f;
            }
            if (pr.bias != nullptr) {
              if (full32) {
                const float4* b4 = reinterpret_cast<const float4*>(pr.bias + col0);
  #pragma unroll
                for (int j = 0; j < 8; ++j) {
                  float4 b = __ldg(b4 + j);
                  v[4 * j] += b.x; v[4 * j + 1] += b.y; v[4 * j + 2] += b.z; v[4 * j + 3] += b.w;
                }
              } else {
  #pragma unroll
                for (int j = 0; j < 32; ++j)
                  if (col0 + j < pr.N) v[j] += pr.bias[col0 + j];
              }
            }
            if (zrow != nullptr) {
              if (full32) {
                const float4* z4 = reinterpret_cast<const float4*>(zrow + col0);
  #pragma unroll
                for (int j = 0; j < 8; ++j) {
                  float4 z = __ldg(z4 + j);
                  v[4 * j] += z.x; v[4 * j + 1] += z.y; v[4 * j + 2] += z.z; v[4 * j + 3] += z.w;
                }
              } else {
  #pragma unroll
                for (int j = 0; j < 32; ++j)
                  if (col0 + j < pr.N) v[j] += zrow[col0 + j];
              }
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
            store_chunk(pr, grow, col0, v);
          }
        }
        if (pr.flag_role == 1) {
          // this warp's part of the tile is stored (plain stores): publish it device-wide
          __threadfence();
          __syncwarp();
          const int fi = mb * pr.n_tiles + nb;
          if (lane == 0 && fi != P.withhold_flag) atomicAdd(pr.flags + fi, 1);
        }
        acc ^= 1;
        if (acc == 0) acc_phase ^= 1;
      }
      // this warp's output stores have landed before the CTA (and its staging memory) goes away
      if (lane == 0) bulk_wait_all();
      __syncwarp();
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem_base, TMEM_COLS);
  }
}

typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                  const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

bool encode_bf16_kmajor(rocs_context* ctx, CUtensorMap* map, const void* ptr, long long rows, int K, long long ld,
                        int box_rows) {
  EncodeTiledFn fn = reinterpret_cast<EncodeTiledFn>(ctx->encode_fn);
  cuuint64_t dims[2] = {(cuuint64_t)K, (cuuint64_t)rows};
  cuuint64_t strides[1] = {(cuuint64_t)ld * 2};
  cuuint32_t box[2] = {(cuuint32_t)BK, (cuuint32_t)box_rows};
  cuuint32_t estr[2] = {1, 1};
  CUresult r = fn(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(ptr), dims, strides, box, estr,
                  CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                  CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

// Output map for the TMA-store epilogue: [rows, cols] with row stride ld elements, box 32 x 32,
// swizzled to match store_chunk_tma's shared-memory layout.
bool encode_out(rocs_context* ctx, CUtensorMap* map, void* ptr, long long rows, int cols, long long ld, bool f32,
                bool wide = false) {
  EncodeTiledFn fn = reinterpret_cast<EncodeTiledFn>(ctx->encode_fn);
  const int es = f32 ? 4 : 2;
  cuuint64_t dims[2] = {(cuuint64_t)cols, (cuuint64_t)rows};
  cuuint64_t strides[1] = {(cuuint64_t)ld * es};
  cuuint32_t box[2] = {wide ? 64u : 32u, 32};
  cuuint32_t estr[2] = {1, 1};
  CUresult r = fn(map, f32 ? CU_TENSOR_MAP_DATA_TYPE_FLOAT32 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, ptr, dims, strides,
                  box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                  (f32 || wide) ? CU_TENSOR_MAP_SWIZZLE_128B : CU_TENSOR_MAP_SWIZZLE_64B,
                  CU_TENSOR_MAP_L2_PROMOTION_NONE, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

}  // namespace

rocs_status launch_gemm_bf16(rocs_context* ctx, const GemmDesc* probs, int nprob, cudaStream_t s) {
  if (nprob < 1 || nprob > kMaxGemmProblems) {
    set_error("gemm: %d problems (1..%d supported)", nprob, kMaxGemmProblems);
    return ROCS_ERR_INVALID_ARG;
  }
  static bool attr_set[64] = {false};
  if (ctx->device < 64 && !attr_set[ctx->device]) {
    rocs_status st = cuda_check(
        cudaFuncSetAttribute(gemm_tc_kernel<false>, cudaFuncAttributeMaxDynamicSharedMemorySize, SMEM_BYTES),
        "cudaFuncSetAttribute(gemm)");
    if (st == ROCS_OK)
      st = cuda_check(
          cudaFuncSetAttribute(gemm_tc_kernel<true>, cudaFuncAttributeMaxDynamicSharedMemorySize, SMEM_BYTES),
          "cudaFuncSetAttribute(gemm)");
    if (st != ROCS_OK) return st;
    attr_set[ctx->device] = true;
  }
  Params P;
  memset(&P, 0, sizeof(P));
  P.nprob = nprob;
  P.status = ctx->d_status;
  P.flag_budget = ctx->test_flag_budget > 0 ? ctx->test_flag_budget : kWaitBudgetCycles;
  P.withhold_flag = ctx->test_withhold_flag;
  int tiles = 0;
  bool same_m = true;
  int nstart = 0;
  for (int i = 0; i < nprob; ++i) {
    const GemmDesc& g = probs[i];
    const int kA = g.split_a ? 2 * g.K : g.K;   // A columns read
    if (g.M < 1 || g.N < 1 || g.K < 1 || g.K % 8 || g.lda % 8 || g.ldb % 8 || g.lda < kA || g.ldb < g.K ||
        (g.split_a && g.K % BK) || ((uintptr_t)g.A & 15) || ((uintptr_t)g.B & 15) || g.out == nullptr ||
        (g.Z && !g.gidx) || g.ldo < (g.out_mode == 2 ? 2LL * g.N : g.N)) {
      set_error("gemm problem %d: unsupported shape/alignment (M=%d N=%d K=%d lda=%lld ldb=%lld)", i, g.M, g.N, g.K,
                g.lda, g.ldb);
      return ROCS_ERR_INVALID_ARG;
    }
    Problem& p = P.p[i];
    p.BN = g.N >= BN_MAX ? BN_MAX : ((g.N + 31) / 32) * 32;
    if (!encode_bf16_kmajor(ctx, &p.tmA, g.A, g.M, kA, g.lda, BM) ||
        !encode_bf16_kmajor(ctx, &p.tmB, g.B, g.N, g.K, g.ldb, p.BN)) {
      set_error("gemm problem %d: cuTensorMapEncodeTiled failed", i);
      return ROCS_ERR_CUDA;
    }
    p.bias = g.bias;
    p.scale = g.scale;
    p.Z = g.Z;
    p.gidx = g.gidx;
    p.gidx_bound = g.gidx_bound;
    p.out = g.out;
    p.ldo = g.ldo;
    p.ldz = g.ldz;
    p.M = g.M;
    p.N = g.N;
    p.K = g.K;
    p.out_mode = g.out_mode;
    p.act = g.act;
    p.lo_off = g.N;
    p.flags = g.flags;
    p.flag_role = g.flag_role;
    const int ve = g.out_mode == 0 ? 4 : 8;
    p.vec_ok = (g.ldo % ve == 0) && (((uintptr_t)g.out & 15) == 0) && (!g.bias || ((uintptr_t)g.bias & 15) == 0) &&
               (!g.Z || (((uintptr_t)g.Z & 15) == 0 && g.ldz % 4 == 0)) && (g.out_mode != 2 || g.N % 8 == 0);
    // TMA-store epilogue when the output rows are 16-byte aligned (and, for hi/lo pairs, the
    // low half starts on a 16-byte boundary); element stores otherwise
    {
      const bool f32 = g.out_mode == 0;
      const int es = f32 ? 4 : 2;
      bool ok = ((uintptr_t)g.out & 15) == 0 && (g.ldo * es) % 16 == 0 && (g.out_mode != 2 || (g.N * 2) % 16 == 0);
      ok = ok && encode_out(ctx, &p.tmO, g.out, g.M, g.N, g.ldo, f32, g.out_mode == 1);
      if (ok && g.out_mode == 2)
        ok = encode_out(ctx, &p.tmOlo, reinterpret_cast<__nv_bfloat16*>(g.out) + g.N, g.M, g.N, g.ldo, false);
      // a publishing problem stores with plain stores, so that a fence orders them before its flag
      p.tma_out = ok && g.flag_role != 1 ? 1 : 0;
    }
    p.m_tiles = (g.M + BM - 1) / BM;
    p.n_tiles = (g.N + p.BN - 1) / p.BN;
    p.b_kblocks = (g.K + BK - 1) / BK;
    p.k_blocks = g.split_a ? 2 * p.b_kblocks : p.b_kblocks;
    p.tile_start = tiles;
    p.n_start = nstart;
    tiles += p.m_tiles * p.n_tiles;
    nstart += p.n_tiles;
    if (g.M != probs[0].M) same_m = false;
  }
  P.total_tiles = tiles;
  bool any_flags = false;
  for (int i = 0; i < nprob; ++i) any_flags = any_flags || probs[i].flag_role != 0;
  // with completion flags the order stays problem-major: every publishing tile first
  P.interleave = same_m && !any_flags ? 1 : 0;
  P.n_per_m = nstart;
  // completion flags: one publishing problem, its readers with the same N; publishing tiles
  // must come before every reading tile (problem-major order with the publisher first)
  int producer = -1;
  bool flagged = false;
  for (int i = 0; i < nprob; ++i)
    if (probs[i].flag_role == 1) {
      if (producer >= 0 || probs[i].flags == nullptr) {
        set_error("gemm: one publishing problem with a flags array expected");
        return ROCS_ERR_INVALID_ARG;
      }
      producer = i;
    }
  for (int i = 0; i < nprob; ++i)
    if (probs[i].flag_role == 2) {
      if (producer < 0 || producer > i || probs[i].flags != probs[producer].flags || probs[i].N != probs[producer].N) {
        set_error("gemm problem %d: reads flags of no earlier publishing problem of the same N", i);
        return ROCS_ERR_INVALID_ARG;
      }
      P.p[i].flag_ntiles = P.p[producer].n_tiles;
      flagged = true;
    }
  const int grid = std::min(tiles, ctx->num_sms);
  LaunchTimer lt_("gemm_tc", s);
  if (!flagged) {
    // bf16 outputs stored through TMA with nothing to add or apply take the lean epilogue
    bool plain = true;
    for (int i = 0; i < nprob; ++i) {
      const Problem& p = P.p[i];
      plain = plain && p.out_mode == 1 && p.tma_out && p.bias == nullptr && p.Z == nullptr && p.scale == nullptr &&
              p.act == ROCS_ACT_NONE;
    }
    if (plain)
      gemm_tc_kernel<true><<<grid, THREADS, SMEM_BYTES, s>>>(P);
    else
      gemm_tc_kernel<false><<<grid, THREADS, SMEM_BYTES, s>>>(P);
    return cuda_check(cudaGetLastError(), "gemm_tc_kernel launch");
  }
  // readers spin on tiles other CTAs publish: launch cooperatively (all CTAs resident)
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(grid);
  cfg.blockDim = dim3(THREADS);
  cfg.dynamicSmemBytes = SMEM_BYTES;
  cfg.stream = s;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeCooperative;
  attr[0].val.cooperative = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cuda_check(cudaLaunchKernelEx(&cfg, gemm_tc_kernel<false>, P), "gemm_tc_kernel cooperative launch");
}

}  // namespace rocs
