// Candidates in any order: a stable counting sort by request index, and the row gather/scatter
// that lets the segment path (candidates grouped by request, [REV] §2.4's map m) serve them.
//
// Counting sort over the keys m[c] in [0, B_R) (an index outside that range is an error: it sorts
// after every valid candidate, as key B_R, and sets ROCS_ERR_INDEX):
//   1. the candidates are cut into chunks of `chunk` in order; one warp per chunk counts its keys
//      into H[key][chunk] (warp-aggregated: lanes with equal keys add once);
//   2. one warp per key turns its row of H into a running total over the chunks (H[key][chunk] =
//      that key's candidates in earlier chunks) and writes the key's count into offsets[key]; one
//      CTA then turns offsets[0..B_R] into its own running total, so offsets[key] + H[key][chunk]
//      is the first sorted position of that chunk's candidates of that key;
//   3. one warp per chunk walks its candidates in order, 32 at a time: lanes with equal keys
//      (__match_any_sync) take consecutive positions in lane order, then the key's position moves
//      past them.  With up to SMEM_KEYS keys the warp first copies its column of H into shared
//      memory and moves the positions there; otherwise it keeps the most recent key's position in
//      registers and reads and writes H for the others (grouped input then touches H only at
//      request boundaries).
// Stability: within a chunk by the walk's order, across chunks by the key-major total.
#include "common.cuh"
#include "internal.h"

namespace rocs {
namespace {

constexpr int SORT_BLOCK = 256;   // 8 warps, one chunk each
constexpr int SCAN_T = 1024;
constexpr int SMEM_WARPS = 4;     // shared-memory scatter: 4 warps (chunks) per block
constexpr int SMEM_KEYS = 6144;   // keys (B_R + 1) whose positions fit: 4 x 24 KiB

__device__ __forceinline__ int sort_key(const int32_t* req_idx, long long i, int B_R, bool& bad) {
  const int k = req_idx[i];
  if (k < 0 || k >= B_R) {
    bad = true;
    return B_R;
  }
  return k;
}

__global__ void __launch_bounds__(SORT_BLOCK) sort_hist_kernel(const int32_t* __restrict__ req_idx, long long B_C,
                                                               int B_R, int chunk, int nchunks, int32_t* __restrict__ H,
                                                               int* status) {
  const int w = (int)((blockIdx.x * (long long)blockDim.x + threadIdx.x) >> 5), lane = threadIdx.x & 31;
  if (w >= nchunks) return;
  const long long c0 = (long long)w * chunk, c1 = min(c0 + chunk, B_C);
  bool bad = false;
  for (long long i0 = c0; i0 < c1; i0 += 32) {
    const long long i = i0 + lane;
    const bool act = i < c1;
    const unsigned am = __ballot_sync(0xffffffffu, act);
    if (act) {
      const int k = sort_key(req_idx, i, B_R, bad);
      const unsigned grp = __match_any_sync(am, k);
      if (__ffs(grp) - 1 == lane) atomicAdd(H + (long long)k * nchunks + w, __popc(grp));
    }
  }
  if (__any_sync(0xffffffffu, bad) && lane == 0) set_status(status, ROCS_ERR_INDEX);
}

// One warp per key: H[key][0..nchunks) -> its exclusive running total; the key's count -> T[key].
__global__ void sort_rowscan_kernel(int32_t* __restrict__ H, int nchunks, int keys, int32_t* __restrict__ T) {
  const long long k = ((long long)blockIdx.x * blockDim.x + threadIdx.x) >> 5;
  const int lane = threadIdx.x & 31;
  if (k >= keys) return;
  int32_t* row = H + k * nchunks;
  int carry = 0;
  for (int c0 = 0; c0 < nchunks; c0 += 32) {
    const int c = c0 + lane;
    const int v = c < nchunks ? row[c] : 0;
    int incl = v;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int t = __shfl_up_sync(0xffffffffu, incl, o);
      if (lane >= o) incl += t;
    }
    if (c < nchunks) row[c] = carry + incl - v;
    carry += __shfl_sync(0xffffffffu, incl, 31);
  }
  if (lane == 0) T[k] = carry;
}

// T[0..n) -> its exclusive running total, in place (one CTA, SCAN_ITEMS entries per thread per pass).
constexpr int SCAN_ITEMS = 8;
__global__ void __launch_bounds__(SCAN_T) sort_scan_kernel(int32_t* __restrict__ T, long long n) {
  __shared__ int warp_tot[32];
  __shared__ int carry_s;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  if (tid == 0) carry_s = 0;
  __syncthreads();
  for (long long base = 0; base < n; base += (long long)SCAN_T * SCAN_ITEMS) {
    const long long j0 = base + (long long)tid * SCAN_ITEMS;
    int v[SCAN_ITEMS];
    int tsum = 0;
#pragma unroll
    for (int e = 0; e < SCAN_ITEMS; ++e) {
      v[e] = j0 + e < n ? T[j0 + e] : 0;
      tsum += v[e];
    }
    int incl = tsum;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int t = __shfl_up_sync(0xffffffffu, incl, o);
      if (lane >= o) incl += t;
    }
    if (lane == 31) warp_tot[warp] = incl;
    __syncthreads();
    if (warp == 0) {
      const int wt = warp_tot[lane];
      int wi = wt;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const int t = __shfl_up_sync(0xffffffffu, wi, o);
        if (lane >= o) wi += t;
      }
      warp_tot[lane] = wi - wt;
    }
    __syncthreads();
    int run = carry_s + warp_tot[warp] + incl - tsum;
#pragma unroll
    for (int e = 0; e < SCAN_ITEMS; ++e) {
      if (j0 + e < n) T[j0 + e] = run;
      run += v[e];
    }
    __syncthreads();
    if (tid == SCAN_T - 1) carry_s = run;
    __syncthreads();
  }
}

__global__ void __launch_bounds__(SORT_BLOCK) sort_scatter_kernel(const int32_t* __restrict__ req_idx, long long B_C,
                                                                  int B_R, int chunk, int nchunks,
                                                                  int32_t* __restrict__ H,
                                                                  const int32_t* __restrict__ offsets,
                                                                  int32_t* __restrict__ perm) {
  const int w = (int)((blockIdx.x * (long long)blockDim.x + threadIdx.x) >> 5), lane = threadIdx.x & 31;
  if (w >= nchunks) return;
  const long long c0 = (long long)w * chunk, c1 = min(c0 + chunk, B_C);
  int ck = -1, cv = 0;   // cached key (warp-uniform) and its next sorted position
  bool bad = false;
  for (long long i0 = c0; i0 < c1; i0 += 32) {
    const long long i = i0 + lane;
    const bool act = i < c1;
    const unsigned am = __ballot_sync(0xffffffffu, act);
    int k = -1, base = 0, size = 0;
    if (act) {
      k = sort_key(req_idx, i, B_R, bad);
      const unsigned grp = __match_any_sync(am, k);
      const int leader = __ffs(grp) - 1;
      size = __popc(grp);
      if (k == ck) {
        base = cv;
      } else {
        int* hp = H + (long long)k * nchunks + w;
        if (lane == leader) {
          base = offsets[k] + *hp;
          *hp = base - offsets[k] + size;   // written through: only the cached key's position lives in registers
        }
        base = __shfl_sync(grp, base, leader);
      }
      perm[base + __popc(grp & ((1u << lane) - 1u))] = (int32_t)i;
    }
    // the last candidate's key becomes the cached one; the evicted key's position goes back to H
    const int last = 31 - __clz(am);
    const int nk = __shfl_sync(0xffffffffu, k, last);
    const int nv = __shfl_sync(0xffffffffu, base + size, last);
    const int add = __reduce_max_sync(0xffffffffu, (act && k == ck) ? size : 0);
    if (nk != ck && ck >= 0 && lane == 0) H[(long long)ck * nchunks + w] = cv + add - offsets[ck];
    ck = nk;
    cv = nv;
    __syncwarp();
  }
  (void)bad;
}

// The scatter of step 3 with the warp's column of positions in shared memory.
__global__ void __launch_bounds__(SMEM_WARPS * 32) sort_scatter_smem_kernel(const int32_t* __restrict__ req_idx,
                                                                         long long B_C, int B_R, int chunk,
                                                                         int nchunks, const int32_t* __restrict__ H,
                                                                         const int32_t* __restrict__ offsets,
                                                                         int32_t* __restrict__ perm) {
  extern __shared__ int32_t pos_all[];
  const int wl = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int w = blockIdx.x * SMEM_WARPS + wl;
  if (w >= nchunks) return;
  int32_t* pos = pos_all + wl * (B_R + 1);
  for (int k = lane; k <= B_R; k += 32) pos[k] = offsets[k] + H[(long long)k * nchunks + w];
  __syncwarp();
  const long long c0 = (long long)w * chunk, c1 = min(c0 + chunk, B_C);
  bool bad = false;
  for (long long i0 = c0; i0 < c1; i0 += 32) {
    const long long i = i0 + lane;
    const bool act = i < c1;
    const unsigned am = __ballot_sync(0xffffffffu, act);
    if (act) {
      const int k = sort_key(req_idx, i, B_R, bad);
      const unsigned grp = __match_any_sync(am, k);
      const int leader = __ffs(grp) - 1;
      int base = 0;
      if (lane == leader) {
        base = pos[k];
        pos[k] = base + __popc(grp);
      }
      base = __shfl_sync(grp, base, leader);
      perm[base + __popc(grp & ((1u << lane) - 1u))] = (int32_t)i;
    }
    __syncwarp();
  }
  (void)bad;
}

// gather rows: dst[k] = src[perm[k]] (16-byte units per row)
__global__ void gather_rows_kernel(const uint4* __restrict__ src, long long ld_src, const int32_t* __restrict__ perm,
                                   long long n, int row_units, uint4* __restrict__ dst, long long ld_dst) {
  const long long k = ((long long)blockIdx.x * blockDim.x + threadIdx.x) >> 5;
  const int lane = threadIdx.x & 31;
  if (k >= n) return;
  const long long s = perm[k];
  for (int u = lane; u < row_units; u += 32) dst[k * ld_dst + u] = src[s * ld_src + u];
}

// scatter rows src[k] -> dst[perm[k]] for k < *count (4-byte words per row)
__global__ void scatter_rows_kernel(const uint32_t* __restrict__ src, long long ld_src,
                                    const int32_t* __restrict__ perm, const int32_t* __restrict__ count, long long n,
                                    int row_words, uint32_t* __restrict__ dst, long long ld_dst) {
  const long long k = ((long long)blockIdx.x * blockDim.x + threadIdx.x) >> 5;
  const int lane = threadIdx.x & 31;
  if (k >= n || k >= *count) return;
  const long long d = perm[k];
  for (int u = lane; u < row_words; u += 32) dst[d * ld_dst + u] = src[k * ld_src + u];
}

}  // namespace

SortPlan plan_sort(int B_R, long long B_C) {
  SortPlan p;
  p.chunk = 512;
  // keep the histogram matrix under 2^24 entries
  const long long keys = (long long)B_R + 1;
  while (((B_C + p.chunk - 1) / p.chunk) * keys > (1LL << 24)) p.chunk *= 2;
  p.nchunks = (int)((B_C + p.chunk - 1) / p.chunk);
  p.h_ints = (long long)p.nchunks * keys;
  return p;
}

rocs_status launch_sort_by_request(rocs_context* ctx, const int32_t* req_idx, int B_R, long long B_C, int32_t* perm,
                                   int32_t* offsets, int32_t* H, cudaStream_t s) {
  if (B_C == 0) return cuda_check(cudaMemsetAsync(offsets, 0, (size_t)(B_R + 1) * 4, s), "zero offsets");
  const SortPlan p = plan_sort(B_R, B_C);
  rocs_status st = cuda_check(cudaMemsetAsync(H, 0, (size_t)p.h_ints * 4, s), "zero sort histogram");
  if (st != ROCS_OK) return st;
  const unsigned blocks = (unsigned)((p.nchunks * 32LL + SORT_BLOCK - 1) / SORT_BLOCK);
  {
    LaunchTimer lt_("sort_hist", s);
    sort_hist_kernel<<<blocks, SORT_BLOCK, 0, s>>>(req_idx, B_C, B_R, p.chunk, p.nchunks, H, ctx->d_status);
    st = cuda_check(cudaGetLastError(), "sort_hist_kernel");
    if (st != ROCS_OK) return st;
  }
  {
    LaunchTimer lt_("sort_rowscan", s);
    const long long threads = (long long)(B_R + 1) * 32;
    sort_rowscan_kernel<<<(unsigned)((threads + 255) / 256), 256, 0, s>>>(H, p.nchunks, B_R + 1, offsets);
    st = cuda_check(cudaGetLastError(), "sort_rowscan_kernel");
    if (st != ROCS_OK) return st;
  }
  {
    LaunchTimer lt_("sort_scan", s);
    sort_scan_kernel<<<1, SCAN_T, 0, s>>>(offsets, (long long)B_R + 1);
    st = cuda_check(cudaGetLastError(), "sort_scan_kernel");
    if (st != ROCS_OK) return st;
  }
  LaunchTimer lt_("sort_scatter", s);
  if (B_R + 1 <= SMEM_KEYS) {
    const size_t smem = (size_t)SMEM_WARPS * (B_R + 1) * 4;
    static bool attr[64] = {false};
    if (ctx->device < 64 && !attr[ctx->device]) {
      st = cuda_check(cudaFuncSetAttribute(sort_scatter_smem_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                           SMEM_WARPS * SMEM_KEYS * 4),
                      "cudaFuncSetAttribute(sort_scatter_smem)");
      if (st != ROCS_OK) return st;
      attr[ctx->device] = true;
    }
    sort_scatter_smem_kernel<<<(unsigned)((p.nchunks + SMEM_WARPS - 1) / SMEM_WARPS), SMEM_WARPS * 32, smem, s>>>(
        req_idx, B_C, B_R, p.chunk, p.nchunks, H, offsets, perm);
    return cuda_check(cudaGetLastError(), "sort_scatter_smem_kernel");
  }
  sort_scatter_kernel<<<blocks, SORT_BLOCK, 0, s>>>(req_idx, B_C, B_R, p.chunk, p.nchunks, H, offsets, perm);
  return cuda_check(cudaGetLastError(), "sort_scatter_kernel");
}

rocs_status launch_gather_rows(const void* src, long long ld_src_bytes, const int32_t* perm, long long n,
                               int row_bytes, void* dst, long long ld_dst_bytes, cudaStream_t s) {
  if (n == 0) return ROCS_OK;
  LaunchTimer lt_("gather_rows", s);
  const long long threads = n * 32;
  gather_rows_kernel<<<(unsigned)((threads + 255) / 256), 256, 0, s>>>(
      (const uint4*)src, ld_src_bytes / 16, perm, n, row_bytes / 16, (uint4*)dst, ld_dst_bytes / 16);
  return cuda_check(cudaGetLastError(), "gather_rows_kernel");
}

rocs_status launch_scatter_rows(const void* src, long long ld_src_bytes, const int32_t* perm, const int32_t* count,
                                long long n, int row_bytes, void* dst, long long ld_dst_bytes, cudaStream_t s) {
  if (n == 0) return ROCS_OK;
  LaunchTimer lt_("scatter_rows", s);
  const long long threads = n * 32;
  scatter_rows_kernel<<<(unsigned)((threads + 255) / 256), 256, 0, s>>>(
      (const uint32_t*)src, ld_src_bytes / 4, perm, count, n, row_bytes / 4, (uint32_t*)dst, ld_dst_bytes / 4);
  return cuda_check(cudaGetLastError(), "scatter_rows_kernel");
}

// Requests by descending query count, ties by index: order[k] is the request of rank k.  The rank of
// request r counts the requests that precede it in that strict total order, so order is a
// permutation of [0, B_R) whatever the offsets hold.  One thread per request, the counts staged
// 256 at a time in shared memory: O(B_R^2) comparisons, for up to kRequestOrderMax requests.
static __global__ void __launch_bounds__(256) request_order_kernel(const int32_t* __restrict__ offsets, int B_R,
                                                                   int32_t* __restrict__ order) {
  __shared__ int keys[256];
  const int r = blockIdx.x * 256 + threadIdx.x;
  const int mine = r < B_R ? offsets[r + 1] - offsets[r] : 0;
  int rank = 0;
  for (int s0 = 0; s0 < B_R; s0 += 256) {
    const int j = s0 + threadIdx.x;
    keys[threadIdx.x] = j < B_R ? offsets[j + 1] - offsets[j] : 0;
    __syncthreads();
    const int n = B_R - s0 < 256 ? B_R - s0 : 256;
    if (r < B_R)
      for (int k = 0; k < n; ++k) {
        const int key = keys[k];
        rank += (key > mine) || (key == mine && s0 + k < r);
      }
    __syncthreads();
  }
  if (r < B_R) order[rank] = r;
}

rocs_status launch_request_order(const int32_t* offsets, int B_R, int32_t* order, cudaStream_t s) {
  if (B_R <= 0) return ROCS_OK;
  if (B_R > kRequestOrderMax) {
    set_error("request order: %d requests (at most %d)", B_R, kRequestOrderMax);
    return ROCS_ERR_UNSUPPORTED;
  }
  LaunchTimer lt_("request_order", s);
  request_order_kernel<<<(B_R + 255) / 256, 256, 0, s>>>(offsets, B_R, order);
  return cuda_check(cudaGetLastError(), "request_order_kernel");
}

}  // namespace rocs
