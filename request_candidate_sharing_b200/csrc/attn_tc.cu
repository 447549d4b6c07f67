// a7/a9: attention against per-request shared K/V on the 5th-generation tensor cores.
//
// [REV] §2.2: S_i and its K/V are computed once per request and every query of that request
// (the request's own history positions for the encoder, its candidates for the grouped
// cross-attention) reads the same K/V; [REV] §2.4 (IKBO-DCA): the kernel consumes request-batch
// K/V directly, never a per-candidate copy.
//
// Persistent: one CTA per SM, each over its share of the (request, head) items, dealt out in
// alternating directions.  G query-tile groups (2 or 3) of one softmax warpgroup each, blocks of
// TK keys (128 or 64), one control warpgroup; 128 (G + 1) threads:
//   warp 0      producer, one polling loop over three jobs: the item's K and V (L x d_h bf16)
//               into shared memory ONCE, in blocks of TK keys, block j of the next item loaded
//               as soon as the groups that read block j of the current one are done with it (so
//               items follow each other without a pipeline drain, and the CTA's startup is paid
//               once per SM); passing each block on to the groups that read it once it has
//               landed (one barrier per block and group); and the query tiles (bf16, or a hi/lo
//               pair) of the CTA's items, which go to the groups in turn, each with a small
//               descriptor (rows, head, keys) in shared memory.
//   warps 1..G  one MMA issuer per group; one thread issues, for each key block j,
//                 S_j = Q K_j^T       (tcgen05.mma M=128, N=TK, K=d_h; one S buffer per group)
//                 O  += P_j V_j       (M=128, N=d_h, K=TK; V read as an MN-major operand; O
//                                      accumulates in TMEM across the key blocks)
//               issuing the next S block before it waits on the current P, so the group's
//               exponentials overlap the other groups' tensor-core work.
//   warps 4..   the softmax warpgroups, one thread per query row (TMEM lane): the S row is read
//               from TMEM in one batch, its maximum and exp2 taken in registers (no shuffles; part
//               of the exponentials on the FMA pipe as a polynomial), P_j written back to TMEM as
//               bf16 pairs (tcgen05.st), where it is the A operand of P_j V_j; the row sum is an MMA
//               of the same P_j against a ones tile.  The row's reference maximum moves only when a
//               block exceeds it by more than 2^8 (then the warp rescales its O and l rows in
//               TMEM); at the end O is read once and divided by the row sum.
//   setmaxnreg moves registers from the control warpgroup (72) to the softmax warpgroups (216 for
//   two groups, 144 for three).
// All waits are bounded; a wait that runs out sets ROCS_ERR_DEVICE_TIMEOUT and the CTA unwinds
// (in-flight copies and MMAs drained, TMEM released) instead of spinning.
#include "common.cuh"
#include "internal.h"
#include "softmax_math.cuh"

namespace rocs {
namespace {

constexpr int TQ = 128;         // query rows per tile (MMA M)
constexpr int AT_TMEM_COLS = 512;
constexpr int AT_MAX_L = 1024;  // keys staged in shared memory at most
constexpr int AT_FIFO = 8;      // K/V copies issued and not yet passed on, at most
// (query-tile groups, keys per block).  Three groups of 64-key blocks give each sub-partition a
// third softmax warp and were 4.5% faster on the encoder (one bf16 query per row); with hi/lo
// queries (twice the S MMAs per block, and twice the blocks) they were 1% slower, so those keep
// two groups of 128-key blocks, as does d_h = 64 (whose registers would not fit three groups).
constexpr int kAtGroups32 = 3, kAtKeys32 = 64;
constexpr int kAtGroupsSplit = 2, kAtKeysSplit = 128;
constexpr int kAtGroups64 = 2, kAtKeys64 = 128;

struct AttnTcParams {
  CUtensorMap tmQ;   // queries [rows, cols] bf16: box {d_h, 128}
  CUtensorMap tmK;   // keys    [B_R * L, H * d_h]: box {d_h, TK}
  CUtensorMap tmV;   // values  same layout
  const int32_t* offsets;
  long long rows;
  int B_R, H, L, nkb;
  long long q_lo_col;   // column of the low half in a query row (hi/lo queries)
  float scale_log2;
  void* O;
  long long ldo;
  int out_bf16;
  __nv_bfloat16* O2;
  long long ldo2;
  const int32_t* out_rows;   // optional: query row q is written to output row out_rows[q]
  const int32_t* kv_len;     // optional: request r has kv_len[r] keys (1..L), the rest are padding
  int q_by_kv;               // with kv_len: request r's queries are also only its first kv_len[r] rows
  const int32_t* order;      // optional: the item list takes the requests in this order (a permutation;
                             // heaviest first spreads them evenly over the CTAs)
  int* status;
};

__host__ __device__ constexpr uint32_t idesc_bf16(int M, int N, bool b_mn_major) {
  return (1u << 4) | (1u << 7) | (1u << 10) | (b_mn_major ? (1u << 16) : 0u) | ((uint32_t)(N >> 3) << 17) |
         ((uint32_t)(M >> 4) << 24);
}

// Shared-memory matrix descriptor: swizzle `layout` (2 = 128 B, 4 = 64 B), stride between 8-row
// groups `sbo` bytes.
__device__ __forceinline__ uint64_t sdesc(uint32_t saddr, uint32_t sbo, uint32_t layout) {
  return (uint64_t)((saddr >> 4) & 0x3FFF) | ((uint64_t)1 << 16) | ((uint64_t)(sbo >> 4) << 32) | ((uint64_t)1 << 46) |
         ((uint64_t)layout << 61);
}


__device__ __forceinline__ void tc_mma_ss(uint32_t d, uint64_t a, uint64_t b, uint32_t idesc, uint32_t acc) {
  asm volatile(
      "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(d),
      "l"(a), "l"(b), "r"(idesc), "r"(acc)
      : "memory");
}

__device__ __forceinline__ void tmem_st_32x32b_x32(uint32_t taddr, const uint32_t (&r)[32]) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x32.b32 [%0], "
      "{%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16,"
      "%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31,%32};" ::"r"(taddr),
      "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7]), "r"(r[8]),
      "r"(r[9]), "r"(r[10]), "r"(r[11]), "r"(r[12]), "r"(r[13]), "r"(r[14]), "r"(r[15]), "r"(r[16]),
      "r"(r[17]), "r"(r[18]), "r"(r[19]), "r"(r[20]), "r"(r[21]), "r"(r[22]), "r"(r[23]), "r"(r[24]),
      "r"(r[25]), "r"(r[26]), "r"(r[27]), "r"(r[28]), "r"(r[29]), "r"(r[30]), "r"(r[31])
      : "memory");
}
__device__ __forceinline__ void tmem_st_wait() { asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory"); }

__device__ __forceinline__ void tmem_st_32x32b_x16(uint32_t taddr, const uint32_t (&r)[16]) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x16.b32 [%0], "
      "{%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16};" ::"r"(taddr),
      "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7]), "r"(r[8]),
      "r"(r[9]), "r"(r[10]), "r"(r[11]), "r"(r[12]), "r"(r[13]), "r"(r[14]), "r"(r[15])
      : "memory");
}

// D[tmem] (+)= A[tmem] * B[smem]: the A operand (M rows in TMEM lanes, two bf16 of K per column)
// is read from tensor memory.
__device__ __forceinline__ void tc_mma_ts(uint32_t d, uint32_t a_tmem, uint64_t b, uint32_t idesc, uint32_t acc) {
  asm volatile(
      "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, p;\n\t}" ::"r"(d),
      "r"(a_tmem), "l"(b), "r"(idesc), "r"(acc)
      : "memory");
}

__device__ __forceinline__ void tmem_ld_32x32b_x1(uint32_t taddr, uint32_t& r) {
  asm volatile("tcgen05.ld.sync.aligned.32x32b.x1.b32 {%0}, [%1];" : "=r"(r) : "r"(taddr));
}
__device__ __forceinline__ void tmem_st_32x32b_x1(uint32_t taddr, uint32_t r) {
  asm volatile("tcgen05.st.sync.aligned.32x32b.x1.b32 [%0], {%1};" ::"r"(taddr), "r"(r) : "memory");
}

__device__ __forceinline__ float fmax3(float a, float b, float c) {
  float d;
  asm("max.f32 %0, %1, %2, %3;" : "=f"(d) : "f"(a), "f"(b), "f"(c));
  return d;
}

// A row's running maximum is only moved when a block's maximum exceeds it by more than this
// (log2 units): exponentials stay <= 2^8, and the O accumulator in TMEM is rescaled rarely.
constexpr float kLazyRescaleLog2 = 8.0f;

// G query-tile groups (one softmax warpgroup and one MMA issuer each, one tile in flight each)
// and TK keys per block.
template <int DH, int G, int TK>
struct AtCfg {
  static constexpr int MAX_KB = AT_MAX_L / TK;       // key blocks at most
  static constexpr bool SUM_MMA = DH == 32;          // row sums by an MMA of P against ones
  static constexpr int THREADS = 128 + 128 * G;
  static constexpr int REG_LAUNCH = 65536 / THREADS / 8 * 8;
  static constexpr int REG_CTRL = 72;                // producer / MMA warpgroup after setmaxnreg.dec
  static constexpr int REG_SOFTMAX = (65536 - 128 * REG_CTRL) / (128 * G) / 8 * 8;
  static_assert(128 * REG_CTRL + 128 * G * REG_SOFTMAX <= THREADS * REG_LAUNCH, "register split");
  static_assert(G >= 2 && G <= 3 && TK % 64 == 0 && AT_MAX_L % TK == 0 && MAX_KB <= 16, "tile shape");
  // tensor memory per group: S (TK fp32 columns) | P (TK / 2 columns of bf16 pairs) | O (DH) | row sum (16)
  static constexpr int S_COL = 0, P_COL = G * TK, O_COL = P_COL + G * (TK / 2), L_COL = O_COL + G * DH;
  static_assert(L_COL + (SUM_MMA ? G * 16 : 0) <= AT_TMEM_COLS, "tensor memory columns");
};

constexpr int AT_DESC = 4;   // tile descriptors in flight per softmax warpgroup
constexpr unsigned kKvPollSleepNs = 32;   // the K/V producer's pause between polls that found nothing to do

// Non-blocking check whether the phase with the given parity has completed.
__device__ __forceinline__ bool mbar_test(uint64_t* bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.test_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(smem_u32(bar)), "r"(parity)
      : "memory");
  return ok != 0;
}

// One query tile of a softmax warpgroup, published by the query producer.  The MMA issuer and
// the softmax warpgroup of that group read it; the softmax reads it again when it writes the
// tile's output, one tile later.
struct AtTile {
  long long q0;      // first query row of the tile's request
  long long q1;      // end of the request's query rows
  int tile;          // tile index within the request; -1 closes the group's tile stream
  int h;             // head
  int Lr;            // keys of the request
  int nkb;           // key blocks of the request
  uint32_t flags;    // AT_LAST
};
constexpr uint32_t AT_LAST = 1;   // the group's last tile of this request

// Work item n of the list (request rb in processing order, head h), its query rows and keys.
struct AtItem {
  long long q0, q1;
  int r, h, Lr, nkb, ntiles;
};

// Geometry of item idx = rb * H + h.  An item whose offsets or key count are invalid gets
// ntiles = 0 and `bad` the status to report.
template <int TK, bool RAGGED>
__device__ __forceinline__ void at_item(const AttnTcParams& P, int idx, AtItem& it, int& bad) {
  const int rb = idx / P.H;
  it.h = idx - rb * P.H;
  it.r = P.order != nullptr ? P.order[rb] : rb;
  it.ntiles = 0;
  it.nkb = 0;
  bad = 0;
  if (it.r < 0 || it.r >= P.B_R) {
    bad = ROCS_ERR_INDEX;
    return;
  }
  it.q0 = P.offsets[it.r];
  it.q1 = P.offsets[it.r + 1];
  if (it.q0 < 0 || it.q1 < it.q0 || it.q1 > P.rows) {
    bad = ROCS_ERR_INDEX;
    return;
  }
  // the request's keys: the first Lr rows of its L-row K/V (a ragged history), Lr in [1, L]
  it.Lr = RAGGED ? P.kv_len[it.r] : P.L;
  if (RAGGED && (it.Lr < 1 || it.Lr > P.L)) {
    bad = ROCS_ERR_COUNTS;
    return;
  }
  // a ragged self-attention: the padding rows are no queries either
  if (RAGGED && P.q_by_kv && it.q1 > it.q0 + it.Lr) it.q1 = it.q0 + it.Lr;
  it.ntiles = (int)((it.q1 - it.q0 + TQ - 1) / TQ);
  it.nkb = RAGGED ? (it.Lr + TK - 1) / TK : P.nkb;
}

// Item index of pass `pass` for this CTA: the list is dealt out in alternating directions
// (CTA c of n takes items c, 2n - 1 - c, 2n + c, ...), so that a list sorted heaviest first
// spreads evenly over the CTAs.  Returns -1 past the end of the list.
__device__ __forceinline__ int at_item_index(int pass, int n_items) {
  const int n = (int)gridDim.x, c = (int)blockIdx.x;
  const long long idx = (long long)pass * n + ((pass & 1) ? n - 1 - c : c);
  return idx < n_items ? (int)idx : -1;
}

template <int DH, bool SPLIT, bool RAGGED, int G, int TK>
__global__ void __launch_bounds__(AtCfg<DH, G, TK>::THREADS, 1) attn_tc_kernel(const __grid_constant__ AttnTcParams P) {
  using C = AtCfg<DH, G, TK>;
  constexpr int GROUPS = G;
  constexpr int MAX_KB = C::MAX_KB;
  constexpr uint32_t GMASK = (1u << G) - 1u;
  constexpr int ROWB = DH * 2;                        // bytes per K/V/Q row
  constexpr uint32_t SW = DH == 32 ? 4u : 2u;         // 64-B or 128-B swizzle for K/V/Q
  constexpr uint32_t SBO = 8 * ROWB;                  // 8-row group stride
  constexpr int KV_BLOCK = TK * ROWB;                 // bytes of one key block
  constexpr int Q_TILE = TQ * ROWB;
  constexpr int NQ = SPLIT ? 2 : 1;
  constexpr int ONES_BYTES = 2048;                    // 16 rows x 64 bf16 ones (128-byte rows)
  constexpr int CH = TK / 64;                         // 32-key chunks per half block
  constexpr uint32_t IDESC_S = idesc_bf16(TQ, TK, false);
  constexpr uint32_t IDESC_O = idesc_bf16(TQ, DH, true);
  constexpr uint32_t IDESC_L = idesc_bf16(TQ, 16, false);
  const int n_items = P.B_R * P.H;

  extern __shared__ uint8_t at_smem_raw[];
  uint8_t* base = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(at_smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sK = base;
  uint8_t* sV = sK + P.nkb * KV_BLOCK;
  uint8_t* sQ = sV + P.nkb * KV_BLOCK;                // [GROUPS][NQ][Q_TILE]
  uint8_t* sOnes = sQ + GROUPS * NQ * Q_TILE;         // 1024-B aligned (Q tiles are 8 KiB multiples)
  AtTile* descs = reinterpret_cast<AtTile*>(sOnes + ONES_BYTES);   // [GROUPS][AT_DESC]
  uint64_t* bars = reinterpret_cast<uint64_t*>(descs + GROUPS * AT_DESC);
  uint64_t* kv_full = bars;                           // [MAX_KB]: block j's copy landed (producer only)
  uint64_t* kv_ready = kv_full + MAX_KB;              // [MAX_KB][GROUPS]: block j ready for group g
  uint64_t* kv_empty = kv_ready + MAX_KB * GROUPS;    // [MAX_KB][GROUPS]: group g done with block j
  uint64_t* q_full = kv_empty + MAX_KB * GROUPS;      // [GROUPS] each
  uint64_t* q_free = q_full + GROUPS;
  uint64_t* s_full = q_free + GROUPS;
  uint64_t* s_free = s_full + GROUPS;
  uint64_t* p_full = s_free + GROUPS;                 // [GROUPS][2]: P half h of the block written
  uint64_t* o_full = p_full + 2 * GROUPS;             // [GROUPS][2]: P half h times V consumed
  uint64_t* drain = o_full + 2 * GROUPS;              // [GROUPS]
  uint64_t* d_full = drain + GROUPS;                  // [GROUPS][AT_DESC]: tile descriptor written
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(d_full + GROUPS * AT_DESC);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (threadIdx.x == 0) {
    for (int i = 0; i < MAX_KB; ++i) {
      mbar_init(&kv_full[i], 1);
      for (int g = 0; g < GROUPS; ++g) {
        mbar_init(&kv_ready[i * GROUPS + g], 1);
        mbar_init(&kv_empty[i * GROUPS + g], 1);
      }
    }
    for (int g = 0; g < GROUPS; ++g) {
      mbar_init(&q_full[g], 1);
      mbar_init(&q_free[g], 1);
      mbar_init(&s_full[g], 1);
      mbar_init(&s_free[g], TQ);
      for (int hh = 0; hh < 2; ++hh) {
        mbar_init(&p_full[2 * g + hh], TQ);
        mbar_init(&o_full[2 * g + hh], 1);
      }
      mbar_init(&drain[g], 1);
      for (int s = 0; s < AT_DESC; ++s) mbar_init(&d_full[g * AT_DESC + s], 1);
    }
    *abort_flag = 0;
    fence_barrier_init();
  }
  if (C::SUM_MMA && threadIdx.x < ONES_BYTES / 16) {
    reinterpret_cast<uint4*>(sOnes)[threadIdx.x] = make_uint4(0x3F803F80u, 0x3F803F80u, 0x3F803F80u, 0x3F803F80u);
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");   // visible to the tensor core
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, AT_TMEM_COLS);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;

  if (warp < 4) {
    asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;" ::"n"(C::REG_CTRL));
    if (warp == 0) {
      // ---------------- producer (the whole warp; lane 0 issues copies and arrivals) ----------------
      // One polling loop with three jobs, none of which may hold up the others:
      //  * K/V copies: block j of the next item is loaded as soon as every group that read block
      //    j of the previous copy has handed it back (kv_empty), so a group that runs out of
      //    tiles of one item starts the next a block behind the others instead of waiting.
      //  * passing blocks on: the warp observes every copy it issued, in order (kv_full), and
      //    only then passes the block to the groups that read the item (kv_ready, one barrier
      //    per block and group).  A group that skips an item would otherwise wait on a copy
      //    barrier that may be two phases from the one it saw last, where parity alone is
      //    ambiguous.  Keys past Lr have P = 0, but their V rows still enter the P V product,
      //    where non-finite padding would give 0 * inf = NaN: the last block's padding rows are
      //    zeroed (whole rows: the swizzle permutes 16-byte units within a row) before it is
      //    passed on.
      //  * query tiles: the tiles of the CTA's items go to the groups in turn; each gets a small
      //    descriptor (rows, head, keys) in one of the group's AT_DESC slots and its queries in
      //    the group's query buffer, once the group has released the previous tile's queries
      //    (q_free).  A slot is rewritten only after that release three tiles later, by which
      //    time the softmax has written that tile's output (it does so during the next tile).
      if (lane == 0) {
        prefetch_tensormap(&P.tmK);
        prefetch_tensormap(&P.tmV);
        prefetch_tensormap(&P.tmQ);
      }
      uint32_t kv_par = 0;   // bit j: parity of kv_full[j] for block j's oldest copy not yet passed on
      uint64_t pend = 0;     // bit GROUPS j + g: group g reads block j's last copy and has not handed it back
      uint64_t e_par = 0;    // bit GROUPS j + g: parity of kv_empty[j][g]'s next completion
      // copies issued and not yet passed on, oldest first, 16 bits each: block (4 bits), groups
      // (3 bits), padding rows of the block (7 bits); at most AT_FIFO
      uint64_t fq_lo = 0, fq_hi = 0;
      int fn = 0;
      AtItem it;
      int pass = 0, jn = 0, tcount = 0;
      bool have = false, more = true;   // an item with blocks left to issue; items left in the list
      uint32_t used = 0;                // the groups that read the current item
      // query side: its own walk over the same items
      AtItem qi;
      int qpass = 0, qt = 0, qcount = 0, closed = 0;
      bool qhave = false, qmore = true;
      int kq[GROUPS];
#pragma unroll
      for (int g = 0; g < GROUPS; ++g) kq[g] = 0;
      long long t_idle = clock64();
      bool ok = true;
      while (ok) {
        bool progress = false;
        // ---- K/V copies
        while (!have && more) {
          if ((long long)pass * gridDim.x >= n_items) {
            more = false;
            break;
          }
          const int idx = at_item_index(pass++, n_items);
          if (idx < 0) continue;
          int bad;
          at_item<TK, RAGGED>(P, idx, it, bad);
          if (it.ntiles == 0) continue;
          used = 0;
          for (int t = 0; t < it.ntiles && t < GROUPS; ++t) used |= 1u << ((tcount + t) % GROUPS);
          tcount += it.ntiles;
          jn = 0;
          have = true;
        }
        if (have && fn < AT_FIFO) {
          const int j = jn;
          bool free_blk = true;
#pragma unroll
          for (int g = 0; g < GROUPS; ++g) {
            const int b = GROUPS * j + g;
            if ((pend >> b) & 1u) free_blk = free_blk && mbar_test(&kv_empty[b], (uint32_t)((e_par >> b) & 1u));
          }
          free_blk = __shfl_sync(0xffffffffu, free_blk, 0);
          if (free_blk) {
            e_par ^= pend & ((uint64_t)GMASK << (GROUPS * j));
            if (lane == 0) {
              const int kv_row = it.r * P.L + j * TK;
              mbar_arrive_expect_tx(&kv_full[j], 2 * KV_BLOCK);
              tma_load_2d(sK + j * KV_BLOCK, &P.tmK, &kv_full[j], it.h * DH, kv_row);
              tma_load_2d(sV + j * KV_BLOCK, &P.tmV, &kv_full[j], it.h * DH, kv_row);
            }
            pend = (pend & ~((uint64_t)GMASK << (GROUPS * j))) | ((uint64_t)used << (GROUPS * j));
            const uint32_t pad = j == it.nkb - 1 ? (uint32_t)(it.nkb * TK - it.Lr) : 0u;
            const uint64_t e = (uint64_t)(j | (used << 4) | (pad << 7));
            if (fn < 4) fq_lo |= e << (16 * fn);
            else fq_hi |= e << (16 * (fn - 4));
            ++fn;
            if (++jn == it.nkb) have = false;
            progress = true;
          }
        }
        // ---- passing landed blocks on
        if (fn > 0) {
          const uint32_t e = (uint32_t)(fq_lo & 0xFFFFu);
          const int j = (int)(e & 15u);
          const bool landed = __shfl_sync(0xffffffffu, mbar_test(&kv_full[j], (kv_par >> j) & 1u), 0);
          if (landed) {
            const int pad = (int)((e >> 7) & 127u);
            if (pad > 0) {
              uint8_t* vb = sV + j * KV_BLOCK + (TK - pad) * ROWB;
              for (int i = lane; i < pad * ROWB / 16; i += 32) reinterpret_cast<uint4*>(vb)[i] = make_uint4(0, 0, 0, 0);
              asm volatile("fence.proxy.async.shared::cta;" ::: "memory");   // visible to the tensor core
              __syncwarp();
            }
            if (lane == 0) {
#pragma unroll
              for (int g = 0; g < GROUPS; ++g)
                if ((e >> (4 + g)) & 1u) mbar_arrive(&kv_ready[GROUPS * j + g]);
            }
            kv_par ^= 1u << j;
            fq_lo = (fq_lo >> 16) | (fq_hi << 48);
            fq_hi >>= 16;
            --fn;
            progress = true;
          }
        }
        // ---- query tiles
        while (!qhave && qmore) {
          if ((long long)qpass * gridDim.x >= n_items) {
            qmore = false;
            break;
          }
          const int idx = at_item_index(qpass++, n_items);
          if (idx < 0) continue;
          int bad;
          at_item<TK, RAGGED>(P, idx, qi, bad);
          if (bad != 0 && lane == 0) set_status(P.status, bad);
          if (qi.ntiles == 0) continue;
          qt = 0;
          qhave = true;
        }
        if (qhave || closed < GROUPS) {
          const int g = qhave ? qcount % GROUPS : closed;
          const int k = kq[g];
          const bool q_ok = __shfl_sync(0xffffffffu, k == 0 || mbar_test(&q_free[g], (k - 1) & 1), 0);
          if (q_ok) {
            const int slot = g * AT_DESC + (k % AT_DESC);
            if (lane == 0) {
              AtTile& d = descs[slot];
              if (qhave) {
                d.q0 = qi.q0;
                d.q1 = qi.q1;
                d.tile = qt;
                d.h = qi.h;
                d.Lr = qi.Lr;
                d.nkb = qi.nkb;
                d.flags = qt + GROUPS >= qi.ntiles ? AT_LAST : 0u;
                mbar_arrive(&d_full[slot]);
                mbar_arrive_expect_tx(&q_full[g], NQ * Q_TILE);
                const int qrow = (int)(qi.q0 + (long long)qt * TQ);
                tma_load_2d(sQ + (g * NQ) * Q_TILE, &P.tmQ, &q_full[g], qi.h * DH, qrow);
                if (SPLIT) tma_load_2d(sQ + (g * NQ + 1) * Q_TILE, &P.tmQ, &q_full[g], (int)P.q_lo_col + qi.h * DH, qrow);
              } else {
                d.tile = -1;   // the group's tile stream is closed
                mbar_arrive(&d_full[slot]);
              }
            }
            if (qhave) {
              kq[g] = k + 1;
              ++qcount;
              if (++qt == qi.ntiles) qhave = false;
            } else {
              ++closed;
            }
            progress = true;
          }
        }
        if (!have && !more && fn == 0 && !qhave && !qmore && closed == GROUPS) break;
        if (progress) {
          t_idle = clock64();
        } else if (*abort_flag) {
          ok = false;
        } else if (clock64() - t_idle > kWaitBudgetCycles) {
          if (lane == 0) set_status(P.status, ROCS_ERR_DEVICE_TIMEOUT);
          *abort_flag = 1;
          ok = false;
        } else if (kKvPollSleepNs != 0) {
          __nanosleep(kKvPollSleepNs);
        }
        ok = __shfl_sync(0xffffffffu, ok, 0);
      }
      // no copy of this CTA may still be landing when it exits (after an abort, the queue holds
      // the K/V copies issued and not passed on, and a group's last query copy may be in flight)
      while (fn > 0) {
        const int j = (int)(fq_lo & 15u);
        if (lane == 0) mbar_wait(&kv_full[j], (kv_par >> j) & 1u, P.status, nullptr);
        kv_par ^= 1u << j;
        fq_lo = (fq_lo >> 16) | (fq_hi << 48);
        fq_hi >>= 16;
        --fn;
      }
      if (lane == 0)
        for (int g = 0; g < GROUPS; ++g)
          if (kq[g] > 0) mbar_wait(&q_full[g], (kq[g] - 1) & 1, P.status, nullptr);
    } else if (warp <= GROUPS && lane == 0) {
      // ---------------- MMA issuer of query-tile group g = warp - 1 ----------------
      // Per key block i of the group's tile stream:  S_i = Q K_j^T once the softmax has read
      // S_{i-1} (s_free); then, for the previous block, O += P V_j and l += P 1 in two halves,
      // each once the softmax has written that half of P (p_full).  After the group's last tile
      // of an item, each block's P V is followed by a commit that hands the block back to the
      // producer (kv_empty).  Each group's MMAs touch only its own TMEM columns.
      const int g = warp - 1;
      auto issue_pv = [&](int ib, int hh, int j, uint32_t fl, int nkb) -> bool {
        if (!mbar_wait(&p_full[2 * g + hh], ib & 1, P.status, abort_flag)) return false;
        tc_fence_after();
        const uint32_t va = smem_u32(sV + j * KV_BLOCK);
#pragma unroll
        for (int kq2 = 0; kq2 < TK / 32; ++kq2) {
          const int ks = hh * (TK / 32) + kq2;
          const uint32_t pa = tmem_base + C::P_COL + g * (TK / 2) + ks * 8;
          tc_mma_ts(tmem_base + C::O_COL + g * DH, pa, sdesc(va + ks * 16 * ROWB, SBO, SW), IDESC_O,
                    (ks > 0 || j > 0) ? 1u : 0u);
          if (C::SUM_MMA)
            tc_mma_ts(tmem_base + C::L_COL + g * 16, pa, sdesc(smem_u32(sOnes), 1024, 2), IDESC_L,
                      (ks > 0 || j > 0) ? 1u : 0u);
        }
        tc_commit(&o_full[2 * g + hh]);
        if (hh == 1 && (fl & AT_LAST)) tc_commit(&kv_empty[GROUPS * j + g]);
        return true;
      };
      // S_i = Q K_j^T into the group's S buffer, once the softmax has read S_{i-1}
      auto issue_s = [&](int ib, int j, uint32_t qa, int nkb) -> bool {
        if (ib > 0 && !mbar_wait(&s_free[g], (ib - 1) & 1, P.status, abort_flag)) return false;
        tc_fence_after();
        const uint32_t ka = smem_u32(sK + j * KV_BLOCK);
#pragma unroll
        for (int ks = 0; ks < DH / 16; ++ks) {
          tc_mma_ss(tmem_base + C::S_COL + g * TK, sdesc(qa + ks * 32, SBO, SW), sdesc(ka + ks * 32, SBO, SW),
                    IDESC_S, ks > 0 ? 1u : 0u);
          if (SPLIT)
            tc_mma_ss(tmem_base + C::S_COL + g * TK, sdesc(qa + Q_TILE + ks * 32, SBO, SW),
                      sdesc(ka + ks * 32, SBO, SW), IDESC_S, 1u);
        }
        tc_commit(&s_full[g]);
        if (j == nkb - 1) tc_commit(&q_free[g]);   // this tile's queries are no longer read
        return true;
      };
      const uint32_t qa = smem_u32(sQ + (g * NQ) * Q_TILE);
      bool ok = true;
      int k = 0, i = 0;
      bool pend_pv = false;   // block i - 1's P V is not issued yet
      int pj = 0, pnkb = 0;   // that block's index and its item's block count
      uint32_t pfl = 0;       // and its tile's flags
      uint32_t rpar = 0;      // bit j: parity of kv_ready[j][g] for the next item this group reads
      for (;;) {
        const int slot = g * AT_DESC + (k % AT_DESC);
        if (!mbar_wait(&d_full[slot], (k / AT_DESC) & 1, P.status, abort_flag)) {
          ok = false;
          break;
        }
        const int tile = descs[slot].tile;
        if (tile < 0) break;
        const int nkb = descs[slot].nkb;
        const uint32_t fl = descs[slot].flags;
        if (!mbar_wait(&q_full[g], k & 1, P.status, abort_flag)) {
          ok = false;
          break;
        }
        for (int j = 0; j < nkb; ++j) {
          if (!mbar_wait(&kv_ready[GROUPS * j + g], (rpar >> j) & 1u, P.status, abort_flag) || !issue_s(i, j, qa, nkb) ||
              (pend_pv && !(issue_pv(i - 1, 0, pj, pfl, pnkb) && issue_pv(i - 1, 1, pj, pfl, pnkb)))) {
            ok = false;
            break;
          }
          pj = j;
          pfl = fl;
          pnkb = nkb;
          pend_pv = true;
          ++i;
        }
        if (!ok) break;
        // The group's last tile of an item: its last P V (and the hand-back of the last block)
        // is issued now, not after the next tile's first S, which may wait for the next item's
        // K/V, whose load waits for this hand-back.
        if (fl & AT_LAST) {
          rpar ^= (1u << nkb) - 1u;   // the group is done with this item's blocks
          if (!(issue_pv(i - 1, 0, pj, pfl, pnkb) && issue_pv(i - 1, 1, pj, pfl, pnkb))) {
            ok = false;
            break;
          }
          pend_pv = false;
        }
        ++k;
      }
      if (ok && pend_pv) ok = issue_pv(i - 1, 0, pj, pfl, pnkb) && issue_pv(i - 1, 1, pj, pfl, pnkb);
      tc_commit(&drain[g]);
      mbar_wait(&drain[g], 0, P.status, nullptr);
    }
  } else {
    asm volatile("setmaxnreg.inc.sync.aligned.u32 %0;" ::"n"(C::REG_SOFTMAX));
    // ---------------- softmax warpgroups: thread = query row = TMEM lane ----------------
    const int g = (warp - 4) >> 2;
    const int quarter = warp & 3;
    const int row = quarter * 32 + lane;
    const uint32_t lane_addr = tmem_base + ((uint32_t)(quarter * 32) << 16);
    const uint32_t saddr = lane_addr + C::S_COL + g * TK;
    const uint32_t paddr = lane_addr + C::P_COL + g * (TK / 2);
    const uint32_t oaddr = lane_addr + C::O_COL + g * DH;
    const uint32_t laddr = lane_addr + C::L_COL + g * 16;
    // the group's tile descriptors, re-read where needed (kept out of the registers)
    volatile AtTile* dq = descs + g * AT_DESC;
    const float sl2 = P.scale_log2;
    float m_cur = -INFINITY, l_reg = 0.f;

    // O of the group's finished tile kt, divided by its row sum, to global memory
    auto emit_row = [&](int kt) {
      float out[DH];
#pragma unroll
      for (int c = 0; c < DH / 32; ++c) {
        uint32_t w[32];
        tmem_ld_32x32b_x32(oaddr + c * 32, w);
        tmem_ld_wait();
#pragma unroll
        for (int k = 0; k < 32; ++k) out[c * 32 + k] = __uint_as_float(w[k]);
      }
      float l_final = l_reg;
      if (C::SUM_MMA) {
        uint32_t lw;
        tmem_ld_32x32b_x1(laddr, lw);
        tmem_ld_wait();
        l_final = __uint_as_float(lw);
      }
      volatile AtTile& d = dq[kt % AT_DESC];
      const long long qrow0 = d.q0 + (long long)d.tile * TQ + row;
      if (qrow0 >= d.q1) return;
      const int h = d.h;
      const long long qrow = P.out_rows != nullptr ? (long long)P.out_rows[qrow0] : qrow0;
      const float inv = 1.0f / l_final;
#pragma unroll
      for (int e = 0; e < DH; ++e) out[e] *= inv;
      if (P.out_bf16) {
        __nv_bfloat16* o = reinterpret_cast<__nv_bfloat16*>(P.O) + qrow * P.ldo + h * DH;
#pragma unroll
        for (int e = 0; e < DH; e += 8)
          *reinterpret_cast<uint4*>(o + e) = make_uint4(pack_bf16x2(out[e], out[e + 1]), pack_bf16x2(out[e + 2], out[e + 3]),
                                                       pack_bf16x2(out[e + 4], out[e + 5]), pack_bf16x2(out[e + 6], out[e + 7]));
      } else {
        float* o = reinterpret_cast<float*>(P.O) + qrow * P.ldo + h * DH;
#pragma unroll
        for (int e = 0; e < DH; e += 4) *reinterpret_cast<float4*>(o + e) = make_float4(out[e], out[e + 1], out[e + 2], out[e + 3]);
      }
      if (P.O2 != nullptr) {
        __nv_bfloat16* o = P.O2 + qrow * P.ldo2 + h * DH;
#pragma unroll
        for (int e = 0; e < DH; e += 8)
          *reinterpret_cast<uint4*>(o + e) = make_uint4(pack_bf16x2(out[e], out[e + 1]), pack_bf16x2(out[e + 2], out[e + 3]),
                                                       pack_bf16x2(out[e + 4], out[e + 5]), pack_bf16x2(out[e + 6], out[e + 7]));
      }
    };

    bool ok = true;
    int k = 0, i = 0;
    for (;;) {
      if (!__all_sync(0xffffffffu, mbar_wait(&d_full[g * AT_DESC + (k % AT_DESC)], (k / AT_DESC) & 1, P.status,
                                             abort_flag))) {
        ok = false;
        break;
      }
      if (dq[k % AT_DESC].tile < 0) break;
      const int nkb = dq[k % AT_DESC].nkb;
      for (int j = 0; j < nkb; ++j, ++i) {
        if (!__all_sync(0xffffffffu, mbar_wait(&s_full[g], i & 1, P.status, abort_flag))) { ok = false; break; }
        tc_fence_after();
        // the whole S row into registers with one wait, then the S accumulator is released
        uint32_t v[TK / 32][32];
#pragma unroll
        for (int c = 0; c < TK / 32; ++c) tmem_ld_32x32b_x32(saddr + c * 32, v[c]);
        tmem_ld_wait();
        tc_fence_before();
        mbar_arrive(&s_free[g]);
        const int valid = dq[k % AT_DESC].Lr - j * TK;   // keys of this block that exist (>= 1)
        if (valid < TK) {
#pragma unroll
          for (int c = 0; c < TK / 32; ++c)
#pragma unroll
            for (int kk = 0; kk < 32; ++kk)
              if (c * 32 + kk >= valid) v[c][kk] = __float_as_uint(-INFINITY);
        }
        // row maximum: eight chains of three-input max
        float mt[8];
#pragma unroll
        for (int t = 0; t < 8; ++t) mt[t] = fmaxf(__uint_as_float(v[0][t]), __uint_as_float(v[0][t + 8]));
#pragma unroll
        for (int e = 16; e < TK; e += 16)
#pragma unroll
          for (int t = 0; t < 8; ++t)
            mt[t] = fmax3(mt[t], __uint_as_float(v[(e + t) >> 5][(e + t) & 31]),
                          __uint_as_float(v[(e + 8 + t) >> 5][(e + 8 + t) & 31]));
        const float mx = fmax3(fmax3(mt[0], mt[1], mt[2]), fmax3(mt[3], mt[4], mt[5]), fmaxf(mt[6], mt[7])) * sl2;
        // the first block sets the row's reference maximum; later blocks move it only when some
        // row of the warp would otherwise produce exponentials above 2^8 (warp-uniform, since the
        // rescale is a warp-wide TMEM access)
        float m_new = m_cur, corr = 1.0f;
        const bool rescale = j != 0 && __any_sync(0xffffffffu, mx > m_cur + kLazyRescaleLog2);
        if (j == 0) {
          m_new = mx;
        } else if (rescale) {
          m_new = fmaxf(m_cur, mx);
          corr = ex2_approx(m_cur - m_new);
        }
        // O is read (finished tile) or rescaled only once both halves of the previous block's P V
        // have completed.  Otherwise those waits come later, just before each half of P is
        // overwritten, so that the exponentials of the half are computed while the tensor core is
        // still reading it.
        const bool need_o = i > 0 && (j == 0 || rescale);
        if (need_o) {
          if (!__all_sync(0xffffffffu, mbar_wait(&o_full[2 * g], (i - 1) & 1, P.status, abort_flag) &&
                                           mbar_wait(&o_full[2 * g + 1], (i - 1) & 1, P.status, abort_flag))) {
            ok = false;
            break;
          }
          tc_fence_after();
          if (j == 0) {
            emit_row(k - 1);
          } else if (rescale) {
#pragma unroll
            for (int c = 0; c < DH / 32; ++c) {
              uint32_t w[32];
              tmem_ld_32x32b_x32(oaddr + c * 32, w);
              tmem_ld_wait();
#pragma unroll
              for (int kk = 0; kk < 32; ++kk) w[kk] = __float_as_uint(__uint_as_float(w[kk]) * corr);
              tmem_st_32x32b_x32(oaddr + c * 32, w);
            }
            if (C::SUM_MMA) {
              uint32_t lw;
              tmem_ld_32x32b_x1(laddr, lw);
              tmem_ld_wait();
              tmem_st_32x32b_x1(laddr, __float_as_uint(__uint_as_float(lw) * corr));
            }
          }
        }
        // exponentials: three pairs in eight on the FMA pipe (polynomial), the rest on MUFU; P_i
        // as bf16 pairs into TMEM, one half block at a time (32 keys per store), each half handed
        // to the tensor core as soon as it is written
        const float neg_m = -m_new;
        float rs = 0.f;
#pragma unroll
        for (int hh = 0; hh < 2; ++hh) {
          uint32_t pk[CH][16];
#pragma unroll
          for (int cc = 0; cc < CH; ++cc) {
            const int c = CH * hh + cc;
#pragma unroll
            for (int kk = 0; kk < 32; kk += 2) {
              float x0, x1, p0, p1;
              ffma2(__uint_as_float(v[c][kk]), __uint_as_float(v[c][kk + 1]), sl2, neg_m, x0, x1);
              if (((kk >> 1) & 7) >= 5) {
                exp2_poly2(x0, x1, p0, p1);
                if (valid < TK) {   // masked keys (x = -inf) must give exactly zero
                  p0 = x0 == -INFINITY ? 0.f : p0;
                  p1 = x1 == -INFINITY ? 0.f : p1;
                }
              } else {
                p0 = ex2_approx(x0);
                p1 = ex2_approx(x1);
              }
              if (!C::SUM_MMA) rs += p0 + p1;
              pk[cc][kk >> 1] = pack_bf16x2(p0, p1);
            }
          }
          // this half of P may be overwritten once the previous block's P V of it has completed
          if (i > 0 && !need_o) {
            if (!__all_sync(0xffffffffu, mbar_wait(&o_full[2 * g + hh], (i - 1) & 1, P.status, abort_flag))) {
              ok = false;
              break;
            }
            tc_fence_after();
          }
#pragma unroll
          for (int cc = 0; cc < CH; ++cc) tmem_st_32x32b_x16(paddr + (CH * hh + cc) * 16, pk[cc]);
          if (hh == 0) {
            tmem_st_wait();
            tc_fence_before();
            mbar_arrive(&p_full[2 * g]);
          }
        }
        if (!ok) break;
        tmem_st_wait();
        tc_fence_before();
        mbar_arrive(&p_full[2 * g + 1]);
        if (!C::SUM_MMA) l_reg = j == 0 ? rs : fmaf(l_reg, corr, rs);
        m_cur = m_new;
      }
      if (!ok) break;
      ++k;
    }
    if (ok && i > 0 && __all_sync(0xffffffffu, mbar_wait(&o_full[2 * g], (i - 1) & 1, P.status, abort_flag) &&
                                              mbar_wait(&o_full[2 * g + 1], (i - 1) & 1, P.status, abort_flag))) {
      tc_fence_after();
      emit_row(k - 1);
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    __syncwarp();
    tc_fence_after();
    tmem_dealloc(tmem_base, AT_TMEM_COLS);
  }
}

template <int DH, bool SPLIT, int G, int TK>
size_t at_smem_bytes(int nkb) {
  using C = AtCfg<DH, G, TK>;
  return 1024 + (size_t)2 * nkb * TK * DH * 2 + (size_t)G * (SPLIT ? 2 : 1) * TQ * DH * 2 + 2048 +
         G * AT_DESC * sizeof(AtTile) + (size_t)(C::MAX_KB * (1 + 2 * G) + G * (9 + AT_DESC)) * 8 + 16;
}

typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                  const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

bool encode_rows(rocs_context* ctx, CUtensorMap* map, const void* ptr, long long rows, long long cols, long long ld,
                 int dh, int box_rows) {
  EncodeTiledFn fn = reinterpret_cast<EncodeTiledFn>(ctx->encode_fn);
  cuuint64_t dims[2] = {(cuuint64_t)cols, (cuuint64_t)rows};
  cuuint64_t strides[1] = {(cuuint64_t)ld * 2};
  cuuint32_t box[2] = {(cuuint32_t)dh, (cuuint32_t)box_rows};
  cuuint32_t estr[2] = {1, 1};
  return fn(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(ptr), dims, strides, box, estr,
            CU_TENSOR_MAP_INTERLEAVE_NONE, dh == 32 ? CU_TENSOR_MAP_SWIZZLE_64B : CU_TENSOR_MAP_SWIZZLE_128B,
            CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

template <int DH, bool SPLIT, bool RAGGED, int G, int TK>
rocs_status at_launch(rocs_context* ctx, AttnTcParams& P, const void* K, const void* V, long long ldkv,
                      long long kv_rows, int B_R, int H, cudaStream_t s) {
  using C = AtCfg<DH, G, TK>;
  P.nkb = (P.L + TK - 1) / TK;
  const size_t smem = at_smem_bytes<DH, SPLIT, G, TK>(P.nkb);
  if (smem > 232448) {
    set_error("tcgen05 attention: L=%d needs %zu B of shared memory", P.L, smem);
    return ROCS_ERR_UNSUPPORTED;
  }
  if (!encode_rows(ctx, &P.tmK, K, kv_rows, (long long)H * DH, ldkv, DH, TK) ||
      !encode_rows(ctx, &P.tmV, V, kv_rows, (long long)H * DH, ldkv, DH, TK)) {
    set_error("tcgen05 attention: cuTensorMapEncodeTiled failed");
    return ROCS_ERR_CUDA;
  }
  static bool attr[64] = {false};
  if (ctx->device < 64 && !attr[ctx->device]) {
    rocs_status st = cuda_check(cudaFuncSetAttribute(attn_tc_kernel<DH, SPLIT, RAGGED, G, TK>,
                                                     cudaFuncAttributeMaxDynamicSharedMemorySize, 232448),
                                "cudaFuncSetAttribute(attn_tc)");
    if (st != ROCS_OK) return st;
    // the softmax warpgroups raise their register limit out of the block's launch allocation;
    // refuse to launch if the compiled kernel was given fewer registers than that split needs
    cudaFuncAttributes fa;
    st = cuda_check(cudaFuncGetAttributes(&fa, attn_tc_kernel<DH, SPLIT, RAGGED, G, TK>),
                    "cudaFuncGetAttributes(attn_tc)");
    if (st != ROCS_OK) return st;
    if (fa.numRegs < C::REG_LAUNCH) {
      set_error("tcgen05 attention: kernel compiled with %d registers per thread, below the warpgroup split",
                fa.numRegs);
      return ROCS_ERR_UNSUPPORTED;
    }
    attr[ctx->device] = true;
  }
  // persistent: one CTA per SM (shared memory allows no second), each over its share of the
  // (request, head) items
  const long long items = (long long)B_R * H;
  const unsigned grid = (unsigned)(items < ctx->num_sms ? items : ctx->num_sms);
  attn_tc_kernel<DH, SPLIT, RAGGED, G, TK><<<grid, C::THREADS, smem, s>>>(P);
  return cuda_check(cudaGetLastError(), "attn_tc_kernel");
}

template <int DH, int G, int TK, int GS, int TKS>
rocs_status at_dispatch(rocs_context* ctx, AttnTcParams& P, bool split, bool rag, const void* K, const void* V,
                        long long ldkv, long long kv_rows, int B_R, int H, cudaStream_t s) {
  if (split)
    return rag ? at_launch<DH, true, true, GS, TKS>(ctx, P, K, V, ldkv, kv_rows, B_R, H, s)
               : at_launch<DH, true, false, GS, TKS>(ctx, P, K, V, ldkv, kv_rows, B_R, H, s);
  return rag ? at_launch<DH, false, true, G, TK>(ctx, P, K, V, ldkv, kv_rows, B_R, H, s)
             : at_launch<DH, false, false, G, TK>(ctx, P, K, V, ldkv, kv_rows, B_R, H, s);
}

}  // namespace

rocs_status launch_attention_tc(rocs_context* ctx, const void* Q, long long ldq, int q_split, const void* K,
                                const void* V, long long ldkv, long long kv_rows, const int32_t* offsets, int B_R,
                                long long rows, int L, int H, int d_h, float scale, void* O, long long ldo,
                                int out_bf16, void* O2, long long ldo2, cudaStream_t s, const int32_t* out_rows,
                                const int32_t* kv_len, int q_by_kv, const int32_t* order) {
  if (B_R == 0 || rows == 0) return ROCS_OK;
  if ((d_h != 32 && d_h != 64) || L < 1 || (long long)L * d_h > 32768 || L > AT_MAX_L ||
      (long long)B_R * H > 2147483647LL ||
      ((uintptr_t)Q & 15) || ((uintptr_t)K & 15) || ((uintptr_t)V & 15) || ldq % 8 || ldkv % 8 ||
      (q_split && (ldq < 2LL * H * d_h)) || ldkv < (long long)H * d_h || ((uintptr_t)O & 15) ||
      (O2 && ((uintptr_t)O2 & 15)) || ldo % 8 || (O2 && ldo2 % 8)) {
    set_error("tcgen05 attention: unsupported shape or alignment (d_h=%d L=%d)", d_h, L);
    return ROCS_ERR_UNSUPPORTED;
  }
  AttnTcParams P;
  memset(&P, 0, sizeof(P));
  const long long qcols = q_split ? 2LL * H * d_h : (long long)H * d_h;
  if (!encode_rows(ctx, &P.tmQ, Q, rows, qcols, ldq, d_h, TQ)) {
    set_error("tcgen05 attention: cuTensorMapEncodeTiled failed");
    return ROCS_ERR_CUDA;
  }
  P.offsets = offsets;
  P.rows = rows;
  P.B_R = B_R;
  P.H = H;
  P.L = L;
  P.q_lo_col = (long long)H * d_h;
  P.scale_log2 = scale * 1.4426950408889634f;
  P.O = O;
  P.ldo = ldo;
  P.out_bf16 = out_bf16;
  P.O2 = (__nv_bfloat16*)O2;
  P.ldo2 = ldo2;
  P.out_rows = out_rows;
  P.kv_len = kv_len;
  P.q_by_kv = kv_len != nullptr && q_by_kv ? 1 : 0;
  P.order = order;
  P.status = ctx->d_status;
  LaunchTimer lt_("attn_tc", s);
  const bool rag = kv_len != nullptr;
  if (d_h == 32)
    return at_dispatch<32, kAtGroups32, kAtKeys32, kAtGroupsSplit, kAtKeysSplit>(ctx, P, q_split != 0, rag, K, V, ldkv,
                                                                               kv_rows, B_R, H, s);
  return at_dispatch<64, kAtGroups64, kAtKeys64, kAtGroups64, kAtKeys64>(ctx, P, q_split != 0, rag, K, V, ldkv,
                                                                         kv_rows, B_R, H, s);
}

}  // namespace rocs
