// device_utils.cuh -- small sm_100a device helpers (conversions, mma.sync, loads).
#pragma once

#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <stdint.h>

namespace moe {

__device__ __forceinline__ uint4 ldg_nc_v4(const void *p) {
  uint4 r;
  asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0,%1,%2,%3}, [%4];"
               : "=r"(r.x), "=r"(r.y), "=r"(r.z), "=r"(r.w)
               : "l"(p));
  return r;
}

__device__ __forceinline__ uint4 ldg_v4(const void *p) {
  uint4 r;
  asm volatile("ld.global.v4.u32 {%0,%1,%2,%3}, [%4];"
               : "=r"(r.x), "=r"(r.y), "=r"(r.z), "=r"(r.w)
               : "l"(p));
  return r;
}

// Four E2M1 pairs (the four bytes of w) -> four f16x2 registers, exact.
// Byte i's low nibble becomes the low half of out[i].
__device__ __forceinline__ void e2m1x8_to_f16x2(uint32_t w, uint32_t out[4]) {
  asm("{\n\t.reg .b8 b0, b1, b2, b3;\n\t"
      "mov.b32 {b0, b1, b2, b3}, %4;\n\t"
      "cvt.rn.f16x2.e2m1x2 %0, b0;\n\t"
      "cvt.rn.f16x2.e2m1x2 %1, b1;\n\t"
      "cvt.rn.f16x2.e2m1x2 %2, b2;\n\t"
      "cvt.rn.f16x2.e2m1x2 %3, b3;\n\t}"
      : "=r"(out[0]), "=r"(out[1]), "=r"(out[2]), "=r"(out[3])
      : "r"(w));
}

// Two E4M3 codes (low byte first) -> f16x2, exact.
__device__ __forceinline__ uint32_t e4m3x2_to_f16x2(uint16_t v) {
  uint32_t r;
  asm("cvt.rn.f16x2.e4m3x2 %0, %1;" : "=r"(r) : "h"(v));
  return r;
}

__device__ __forceinline__ uint32_t hmul2_u32(uint32_t a, uint32_t b) {
  __half2 r = __hmul2(*reinterpret_cast<__half2 *>(&a), *reinterpret_cast<__half2 *>(&b));
  return *reinterpret_cast<uint32_t *>(&r);
}

// f16x2 with both halves equal to 2^d (d <= 0); 0 when 2^d is below half the
// smallest f16 subnormal.
__device__ __forceinline__ uint32_t f16x2_pow2(int d) {
  d = max(d, -30);
  float f = __int_as_float((d + 127) << 23);
  __half2 h = __float2half2_rn(f);
  return *reinterpret_cast<uint32_t *>(&h);
}

__device__ __forceinline__ uint32_t dup_lo16(uint32_t v) { return __byte_perm(v, 0, 0x1010); }
__device__ __forceinline__ uint32_t dup_hi16(uint32_t v) { return __byte_perm(v, 0, 0x3232); }

// D = A(16x16, row) * B(16x8, col) + C, f16 inputs, fp32 accumulate.
__device__ __forceinline__ void mma_f16(float d[4], const uint32_t a[4], uint32_t b0, uint32_t b1,
                                        const float c[4]) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
      "{%10,%11,%12,%13};"
      : "=f"(d[0]), "=f"(d[1]), "=f"(d[2]), "=f"(d[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1), "f"(c[0]), "f"(c[1]),
        "f"(c[2]), "f"(c[3]));
}

__device__ __forceinline__ void mma_bf16(float d[4], const uint32_t a[4], uint32_t b0, uint32_t b1,
                                         const float c[4]) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
      "{%10,%11,%12,%13};"
      : "=f"(d[0]), "=f"(d[1]), "=f"(d[2]), "=f"(d[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1), "f"(c[0]), "f"(c[1]),
        "f"(c[2]), "f"(c[3]));
}

__device__ __forceinline__ float bf16_bits_to_float(uint16_t b) {
  return __uint_as_float(static_cast<uint32_t>(b) << 16);
}

// Chunk scale exponent c with amax * 2^-c in [2^14, 2^15): keeps the chunk's
// largest value inside the f16 normal range with maximum precision.
__device__ __forceinline__ int chunk_exponent(float amax) {
  if (!(amax > 0.0f)) return 0;
  int e = ((__float_as_uint(amax) >> 23) & 0xFF) - 127;   // floor(log2) for normal amax
  if (e == -127) e = -126;                                  // subnormal amax
  int c = e - 14;
  return max(-126, min(126, c));
}

__device__ __forceinline__ float pow2f(int c) { return __int_as_float((c + 127) << 23); }

// silu(a) = a / (1 + e^-a) with the fast exponential and division intrinsics
// (branch-free, a few ulp): the result feeds bf16-precision h or its E4M3
// pieces.  For a < -87 the denominator passes 2^126 and the quotient is 0.
__device__ __forceinline__ float silu_f(float a) { return __fdividef(a, 1.0f + __expf(-a)); }

__device__ __forceinline__ uint16_t f16_bits(float v) {
  __half h = __float2half_rn(v);
  return *reinterpret_cast<uint16_t *>(&h);
}

__device__ __forceinline__ uint16_t bf16_bits(float v) {
  __nv_bfloat16 h = __float2bfloat16_rn(v);
  return *reinterpret_cast<uint16_t *>(&h);
}

}  // namespace moe
