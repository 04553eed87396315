// quant_div.h -- the quantizers' division, scalar form: the definition the
// pre-pass kernels follow (they run the same three steps on two lanes per
// fp32-pair instruction, each lane rounded as here) and that the host
// program checks against IEEE division bit for bit.
//
// The quantizers need x / delta rounded to nearest ([SA2++] "核心公式":
// A_hat = round(A / delta), delta_V = colmax|V| / V_r), one division per
// element with one delta per block (or channel).  Instead of a division per
// element, the kernels take r = RN(1/delta) once and correct the product:
//   q = RN(x * r)            (within about one ulp of x / delta)
//   rem = RN(x - q * delta)  (exact: one fused multiply-add)
//   RN(q + rem * r)          (the correctly rounded quotient)
// -- Markstein's correction step (P. Markstein, "Computation of elementary
// functions on the IBM RISC System/6000 processor", IBM J. Res. Dev. 34(1),
// 1990).  Valid away from overflow and underflow of the quotient and the
// remainder, which the quantizers' ranges (|x| <= 127 delta, or V_r delta)
// never reach.  Compiled as host code (g++, no contraction of a * b + c)
// the same functions give the same bits, which is how they are tested.
#pragma once

#include <math.h>

#if defined(__CUDACC__)
#define SAGE_HD __host__ __device__ __forceinline__
#else
#define SAGE_HD inline
#endif

namespace sage {

// fp32 product and fused multiply-add, each rounded once to nearest even
SAGE_HD float mul_rn(float a, float b) {
#if defined(__CUDA_ARCH__)
  return __fmul_rn(a, b);  // never contracted into an fma
#else
  return a * b;
#endif
}
SAGE_HD float fma_rn(float a, float b, float c) {
#if defined(__CUDA_ARCH__)
  return __fmaf_rn(a, b, c);
#else
  return fmaf(a, b, c);
#endif
}

// RN(x / d) given r = RN(1/d).  The correction's additions turn a -0
// quotient into +0; with d > 0 the quotient carries the sign of x, which
// copysign restores (E4M3 encodes -0 as 0x80).
SAGE_HD float div_rn_by(float x, float d, float r) {
  const float q = mul_rn(x, r);
  const float rem = fma_rn(-q, d, x);
  return copysignf(fma_rn(rem, r, q), x);
}

// RN(x / d) given r = RN(1/d) without the sign fix of div_rn_by (for int8
// codes, where -0 and +0 coincide).
SAGE_HD float div_rn_nosign(float x, float d, float r) {
  const float q = mul_rn(x, r);
  const float rem = fma_rn(-q, d, x);
  return fma_rn(rem, r, q);
}

}  // namespace sage
