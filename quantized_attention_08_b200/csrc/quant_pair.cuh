// quant_pair.cuh -- fp32-pair arithmetic of the pre-pass kernels, and the
// quantizers' division on two lanes at a time.  Device only.  The division
// follows quant_div.h's scalar definition lane by lane; a device program
// (tests/c/div_check_gpu.cu) compares these functions with IEEE division
// over every fp16 input the quantizers can see.
#pragma once

#include <cuda_fp16.h>
#include <stdint.h>

namespace sage {

// ---------------------------------------------------------------- fp32 pairs
// Lane-wise IEEE fp32 operations on two values (each lane rounded to nearest
// even, exactly as the scalar operation), two per instruction.  A product
// must not feed f2_add / f2_sub directly: ptxas contracts that pair into a
// fused multiply-add whatever the rounding qualifiers (measured), which
// rounds once instead of twice.
__device__ __forceinline__ uint64_t f2_pack(float lo, float hi) {
  uint64_t r;
  asm("mov.b64 %0, {%1, %2};" : "=l"(r) : "f"(lo), "f"(hi));
  return r;
}
__device__ __forceinline__ float2 f2_unpack(uint64_t v) {
  float2 r;
  asm("mov.b64 {%0, %1}, %2;" : "=f"(r.x), "=f"(r.y) : "l"(v));
  return r;
}
__device__ __forceinline__ uint64_t f2_mul(uint64_t a, uint64_t b) {
  uint64_t d;
  asm("mul.rn.f32x2 %0, %1, %2;" : "=l"(d) : "l"(a), "l"(b));
  return d;
}
__device__ __forceinline__ uint64_t f2_add(uint64_t a, uint64_t b) {
  uint64_t d;
  asm("add.rn.f32x2 %0, %1, %2;" : "=l"(d) : "l"(a), "l"(b));
  return d;
}
__device__ __forceinline__ uint64_t f2_sub(uint64_t a, uint64_t b) {
  uint64_t d;
  asm("sub.rn.f32x2 %0, %1, %2;" : "=l"(d) : "l"(a), "l"(b));
  return d;
}
__device__ __forceinline__ uint64_t f2_fma(uint64_t a, uint64_t b, uint64_t c) {
  uint64_t d;
  asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(d) : "l"(a), "l"(b), "l"(c));
  return d;
}
// the two fp16 values of w as fp32 (exact)
__device__ __forceinline__ uint64_t f2_from_h2(uint32_t w) {
  const float2 f = __half22float2(*reinterpret_cast<const __half2*>(&w));
  return f2_pack(f.x, f.y);
}
__device__ __forceinline__ uint32_t prmt(uint32_t a, uint32_t b, uint32_t sel) {
  uint32_t d;
  asm("prmt.b32 %0, %1, %2, %3;" : "=r"(d) : "r"(a), "r"(b), "r"(sel));
  return d;
}
// RN(x / d) of two lanes given r = RN(1/d) and nd = -d (div_rn_nosign of
// quant_div.h lane-wise: q = RN(x r), the remainder fma(q, -d, x) -- the
// same exact value as fma(-q, d, x) -- then RN(q + rem r)).  A -0 quotient
// can come out as +0.
__device__ __forceinline__ uint64_t div2_rn(uint64_t x, uint64_t nd, uint64_t r) {
  const uint64_t q = f2_mul(x, r);
  return f2_fma(f2_fma(q, nd, x), r, q);
}

// int8 codes of four x values (two lanes each), delta > 0, r = RN(1/delta),
// nd = -delta: y = RN(x / delta) by div2_rn, then rounded half-even to an
// integer: adding 1.5 * 2^23 leaves it in the low mantissa bits, whose low
// byte is the two's-complement code; bytes in lane order.  No clamp is
// needed: |x| <= absmax and delta = RN(absmax / 127) >= absmax / 127 *
// (1 - 2^-24), so |y| <= 127 * (1 + 2^-22) rounds to at most 127; -0 and
// +0 both give code 0.
__device__ __forceinline__ uint32_t codes4(uint64_t x01, uint64_t x23, uint64_t nd2, uint64_t r2) {
  const uint64_t magic2 = f2_pack(12582912.f, 12582912.f);
  const uint64_t y01 = div2_rn(x01, nd2, r2), y23 = div2_rn(x23, nd2, r2);
  const uint64_t c01 = f2_add(y01, magic2), c23 = f2_add(y23, magic2);
  const uint32_t lo = prmt(static_cast<uint32_t>(c01), static_cast<uint32_t>(c01 >> 32), 0x0040u);
  const uint32_t hi = prmt(static_cast<uint32_t>(c23), static_cast<uint32_t>(c23 >> 32), 0x0040u);
  return prmt(lo, hi, 0x5410u);
}

}  // namespace sage
