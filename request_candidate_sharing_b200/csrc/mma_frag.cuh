// Register-fragment tensor-core helpers (m16n8k16 bf16 -> fp32) and ldmatrix loads, used by
// the kernels whose contractions are many tiny per-candidate products (masked FM) or short
// query tiles against shared K/V (cross-attention), where a 128-row tcgen05 tile would be
// mostly empty.
#pragma once
#include <stdint.h>

namespace rocs {

// Fragment layout (g = lane / 4, t = lane % 4):
//   A 16x16 row-major: a0 = A[g][2t..2t+1], a1 = A[g+8][2t..], a2 = A[g][2t+8..], a3 = A[g+8][2t+8..]
//   B 16x8 (k x n):    b0 = B[2t..2t+1][g], b1 = B[2t+8..2t+9][g]
//   C 16x8 fp32:       c0,c1 = C[g][2t..2t+1], c2,c3 = C[g+8][2t..2t+1]
__device__ __forceinline__ void mma_bf16_16816(float (&c)[4], const uint32_t (&a)[4], uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
      "{%0,%1,%2,%3};"
      : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

// The same fragments with f16 operands (both A and B f16).
__device__ __forceinline__ void mma_f16_16816(float (&c)[4], const uint32_t (&a)[4], uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
      "{%0,%1,%2,%3};"
      : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

__device__ __forceinline__ void ldsm_x4(uint32_t saddr, uint32_t& r0, uint32_t& r1, uint32_t& r2, uint32_t& r3) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0,%1,%2,%3}, [%4];"
               : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
               : "r"(saddr));
}

__device__ __forceinline__ void ldsm_x4_trans(uint32_t saddr, uint32_t& r0, uint32_t& r1, uint32_t& r2,
                                              uint32_t& r3) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0,%1,%2,%3}, [%4];"
               : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
               : "r"(saddr));
}

// A fragment (16 rows x 16 k) of a row-major bf16 tile in shared memory with row pitch `pitch`
// bytes, rows r0..r0+15, columns k0..k0+15.
__device__ __forceinline__ void load_a_frag(uint32_t base, int pitch, int r0, int k0, uint32_t (&a)[4]) {
  const int lane = threadIdx.x & 31;
  const int j = lane >> 3;
  const int row = r0 + ((j & 1) << 3) + (lane & 7);
  const int col = k0 + ((j >> 1) << 3);
  ldsm_x4(base + row * pitch + col * 2, a[0], a[1], a[2], a[3]);
}

// B fragments for two adjacent n-tiles (n0..n0+7 and n0+8..n0+15) x 16 k, where the operand is
// stored n-major (row n holds its k values contiguously): b[0],b[1] for tile n0; b[2],b[3] for
// tile n0+8.
__device__ __forceinline__ void load_b_frag_nmajor_x2(uint32_t base, int pitch, int n0, int k0, uint32_t (&b)[4]) {
  const int lane = threadIdx.x & 31;
  const int j = lane >> 3;
  const int row = n0 + ((j >> 1) << 3) + (lane & 7);
  const int col = k0 + ((j & 1) << 3);
  ldsm_x4(base + row * pitch + col * 2, b[0], b[1], b[2], b[3]);
}

// B fragments for two adjacent n-tiles x 16 k, where the operand is stored k-major (row k holds
// its n values contiguously, e.g. V[key][dim] with k = key): uses the transposing load.
__device__ __forceinline__ void load_b_frag_kmajor_x2(uint32_t base, int pitch, int k0, int n0, uint32_t (&b)[4]) {
  const int lane = threadIdx.x & 31;
  const int j = lane >> 3;
  const int row = k0 + ((j & 1) << 3) + (lane & 7);
  const int col = n0 + ((j >> 1) << 3);
  ldsm_x4_trans(base + row * pitch + col * 2, b[0], b[1], b[2], b[3]);
}

}  // namespace rocs
