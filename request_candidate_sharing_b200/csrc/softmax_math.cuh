// The attention softmax's per-score arithmetic on the FMA pipe, shared by the tcgen05 attention
// kernel and the exponential-throughput probe (probe.cu) that measures its ceiling.
#pragma once
#include <stdint.h>

namespace rocs {

// (a0, a1) * (b, b) + (c, c) on the packed fp32x2 FMA path.
__device__ __forceinline__ void ffma2(float a0, float a1, float b, float c, float& d0, float& d1) {
  uint64_t av, bv, cv, dv;
  asm("mov.b64 %0, {%1, %2};" : "=l"(av) : "f"(a0), "f"(a1));
  asm("mov.b64 %0, {%1, %1};" : "=l"(bv) : "f"(b));
  asm("mov.b64 %0, {%1, %1};" : "=l"(cv) : "f"(c));
  asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(dv) : "l"(av), "l"(bv), "l"(cv));
  asm("mov.b64 {%0, %1}, %2;" : "=f"(d0), "=f"(d1) : "l"(dv));
}

__device__ __forceinline__ uint64_t dup2(float c) {
  uint64_t v;
  asm("mov.b64 %0, {%1, %1};" : "=l"(v) : "f"(c));
  return v;
}

// 2^x0, 2^x1 on the FMA pipe: x = n + f with n = round(x) by the 1.5 * 2^23 shifter, 2^f by a
// degree-3 minimax polynomial on [-1/2, 1/2] (max relative error 7.5e-5, coefficients from
// gen_exp2_poly.py), 2^n added into the exponent field.  Valid for x < 128 (the softmax keeps
// x <= 8); arguments below -126 are raised to -126.
__device__ __forceinline__ void exp2_poly2(float x0, float x1, float& y0, float& y1) {
  x0 = fmaxf(x0, -126.0f);
  x1 = fmaxf(x1, -126.0f);
  uint64_t xv, tv, nv, fv, pv;
  const uint64_t shifter = dup2(12582912.0f);   // 1.5 * 2^23 in both halves
  asm("mov.b64 %0, {%1, %2};" : "=l"(xv) : "f"(x0), "f"(x1));
  asm("add.rn.f32x2 %0, %1, %2;" : "=l"(tv) : "l"(xv), "l"(shifter));
  asm("sub.rn.f32x2 %0, %1, %2;" : "=l"(nv) : "l"(tv), "l"(shifter));
  asm("sub.rn.f32x2 %0, %1, %2;" : "=l"(fv) : "l"(xv), "l"(nv));
  const uint64_t c3 = dup2(0.0551716685f), c2 = dup2(0.242611125f), c1 = dup2(0.693260968f), c0 = dup2(0.999928057f);
  asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(pv) : "l"(c3), "l"(fv), "l"(c2));
  asm("fma.rn.f32x2 %0, %0, %1, %2;" : "+l"(pv) : "l"(fv), "l"(c1));
  asm("fma.rn.f32x2 %0, %0, %1, %2;" : "+l"(pv) : "l"(fv), "l"(c0));
  uint32_t t0, t1, p0, p1;
  asm("mov.b64 {%0, %1}, %2;" : "=r"(t0), "=r"(t1) : "l"(tv));
  asm("mov.b64 {%0, %1}, %2;" : "=r"(p0), "=r"(p1) : "l"(pv));
  // the shifter's low 9 bits are zero, so bits(t) * 2^23 is exactly n << 23 (mod 2^32)
  uint32_t r0, r1;
  asm("mad.lo.u32 %0, %1, 8388608, %2;" : "=r"(r0) : "r"(t0), "r"(p0));
  asm("mad.lo.u32 %0, %1, 8388608, %2;" : "=r"(r1) : "r"(t1), "r"(p1));
  y0 = __uint_as_float(r0);
  y1 = __uint_as_float(r1);
}

}  // namespace rocs
