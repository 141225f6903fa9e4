// pieces.cuh -- the two-piece E4M3 form of activations used by the EXACT
// tensor-core path: v = 2^e1 * q1 + 2^e2 * q2 per block of 32, with
// e1 = floor(log2(max|v|)) - 7 and e2 from the largest remainder, q = RN_E4M3.
#pragma once

#include "checks.cuh"
#include "device_utils.cuh"
#include "moe_internal.h"

namespace moe {

__device__ __forceinline__ int floor_log2_pos(float v) {   // v > 0 finite; subnormals give -127
  const int ex = (int)((__float_as_uint(v) >> 23) & 0xFF);
  return ex == 0 ? -127 : ex - 127;
}

__device__ __forceinline__ float exp2_int(int e) {          // 2^e for e in [-126, 127]
  return __int_as_float((e + 127) << 23);
}

// Two E4M3 codes: `lo` in bits 0..7, `hi` in bits 8..15.
__device__ __forceinline__ uint32_t e4m3x2(float lo, float hi) {
  uint16_t r;
  asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;" : "=h"(r) : "f"(hi), "f"(lo));
  return r;
}

__device__ __forceinline__ float e4m3_value(uint32_t code) {
  const uint32_t h2 = e4m3x2_to_f16x2((uint16_t)(code & 0xFFu));
  return __half2float(__ushort_as_half((unsigned short)(h2 & 0xFFFFu)));
}

// Block exponents of the split.  e1 from the block maximum of |v|; e2
// (absolute) from the maximum of the remainders, in the units of 2^e1.
__device__ __forceinline__ int split_e1(float amax) {
  return amax > 0.0f ? max(-127, floor_log2_pos(amax) - 7) : 0;
}
__device__ __forceinline__ int split_e2rel(float rmax, int e1) {
  if (!(rmax > 0.0f)) return 0;
  int e = floor_log2_pos(rmax) - 7;
  e = max(e, -120);
  return max(e, -127 - e1);
}

// One warp writes the two pieces of token j of tile `tile` (rows
// kTcSlotRows * tile + 2j, + 1) and their scale bytes; lane handles 32-blocks
// lane, lane + 32, ...
__device__ __forceinline__ void tc_quant_x_slot(const TcQuantArgs &q, size_t row0, int token);

__device__ __forceinline__ void tc_quant_x_row(const TcQuantArgs &q, int tile, int j) {
  const TileInfo ti = q.tiles[tile];
  if (j >= ti.nrows) return;
  tc_quant_x_slot(q, (size_t)tile * kTcSlotRows + 2 * j,
                  checked_index(q.prow_token[ti.prow0 + j], 0, q.db.n_tokens, 0, q.db.err, kChkToken));
}

// Pieces of token `token` into activation rows row0 (first piece) and row0 + 1.
__device__ __forceinline__ void tc_quant_x_slot(const TcQuantArgs &q, size_t row0, int token) {
  const int lane = threadIdx.x & 31;
  const int H = q.H, nsf = H / 32;
  const uint16_t *xr = q.x + (size_t)token * H;
  const bool vec = ((reinterpret_cast<uintptr_t>(xr) & 15u) == 0);
  for (int b = lane; b < nsf; b += 32) {
    float v[32];
    if (vec) {
      const uint4 *src = reinterpret_cast<const uint4 *>(xr + b * 32);
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const uint4 u = __ldg(src + i);
        const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
        for (int c = 0; c < 4; ++c) {
          v[8 * i + 2 * c] = __uint_as_float(w[c] << 16);
          v[8 * i + 2 * c + 1] = __uint_as_float(w[c] & 0xFFFF0000u);
        }
      }
    } else {
#pragma unroll
      for (int i = 0; i < 32; ++i) v[i] = bf16_bits_to_float(xr[b * 32 + i]);
    }
    float amax = 0.0f;
#pragma unroll
    for (int i = 0; i < 32; ++i) amax = fmaxf(amax, fabsf(v[i]));
    const int e1 = split_e1(amax);
    const float inv1 = exp2_int(-e1);
    uint32_t c1[8];
    float rmax = 0.0f;
#pragma unroll
    for (int i = 0; i < 16; ++i) {
      const float w0 = v[2 * i] * inv1, w1 = v[2 * i + 1] * inv1;
      const uint32_t pr = e4m3x2(w0, w1);
      const float r0 = w0 - e4m3_value(pr), r1 = w1 - e4m3_value(pr >> 8);
      v[2 * i] = r0;
      v[2 * i + 1] = r1;
      rmax = fmaxf(rmax, fmaxf(fabsf(r0), fabsf(r1)));
      if (i & 1) c1[i >> 1] |= pr << 16;
      else c1[i >> 1] = pr;
    }
    const int e2r = split_e2rel(rmax, e1);
    const float inv2 = exp2_int(-e2r);
    uint32_t c2[8];
#pragma unroll
    for (int i = 0; i < 16; ++i) {
      const uint32_t pr = e4m3x2(v[2 * i] * inv2, v[2 * i + 1] * inv2);
      if (i & 1) c2[i >> 1] |= pr << 16;
      else c2[i >> 1] = pr;
    }
    uint4 *d1 = reinterpret_cast<uint4 *>(q.xq + row0 * H + b * 32);
    uint4 *d2 = reinterpret_cast<uint4 *>(q.xq + (row0 + 1) * H + b * 32);
    d1[0] = make_uint4(c1[0], c1[1], c1[2], c1[3]);
    d1[1] = make_uint4(c1[4], c1[5], c1[6], c1[7]);
    d2[0] = make_uint4(c2[0], c2[1], c2[2], c2[3]);
    d2[1] = make_uint4(c2[4], c2[5], c2[6], c2[7]);
    q.xsf[sf_offset(nsf, (int)row0, b)] = (uint8_t)(e1 + 127);
    q.xsf[sf_offset(nsf, (int)row0 + 1, b)] = (uint8_t)(e1 + e2r + 127);
  }
}

}  // namespace moe
