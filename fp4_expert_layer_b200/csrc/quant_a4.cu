// quant_a4.cu -- activation quantisation of the opt-in A4 numerics.
//
// A4 quantises the expert GEMM activations (x before gate/up, h before down)
// to the experts' own 4-bit format so that the tensor core runs FP4 x FP4
// block-scaled MMA; "ro99/strata" sets four bits as the floor for anything it
// stores, and exact mode is never replaced silently, so A4 is a separate mode
// the caller asks for.  The rules (no formula on the pages):
//  * MXFP4, per block of 32 along K (OCP MX conversion): scale exponent
//    X = floor(log2(amax)) - 2 stored as E8M0 clamp(X + 127, 1, 254) (1 when
//    amax = 0); code = round-to-nearest-even E2M1 of v * 2^-X, saturating.
//  * NVFP4, per row: G = 2^ceil(log2(amax_row / (6 * 448))) (1 when amax = 0);
//    per block of 16: s = RN_E4M3((amax_block / 6) / G), code = RNE_E2M1(
//    v * (1 / (s * G))) (0 when s = 0).
// Every step is taken in fp32 in this order (the two divisions and the
// reciprocal correctly rounded) so the CPU oracle takes the same decisions.
//
// One warp per padded row; rows past the padded count exit, pad rows are
// written as zero codes.
#include "checks.cuh"
#include "device_utils.cuh"
#include "moe_internal.h"

namespace moe {

namespace {

__device__ __forceinline__ uint32_t e2m1x2_from_f32(float lo, float hi) {
  uint32_t r;
  asm("{\n\t.reg .b8 b;\n\t"
      "cvt.rn.satfinite.e2m1x2.f32 b, %2, %1;\n\t"
      "cvt.u32.u8 %0, b;\n\t}"
      : "=r"(r)
      : "f"(lo), "f"(hi));
  return r;
}

__device__ __forceinline__ uint32_t e4m3_from_f32(float v) {
  uint16_t r;
  asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;" : "=h"(r) : "f"(0.0f), "f"(v));
  return r & 0xFFu;
}

__device__ __forceinline__ float e4m3_to_f32(uint32_t code) {
  const uint32_t h2 = e4m3x2_to_f16x2((uint16_t)code);
  return __half2float(__ushort_as_half((unsigned short)(h2 & 0xFFFFu)));
}

// The N source values k0 .. k0 + N - 1 of a row (token `src` of x, or row `row`
// of h; zeros for a pad row): 16-byte loads when the source allows them (h
// always, x when its base is 16-byte aligned), else one element at a time.
template <int N>
__device__ __forceinline__ void load_block(const QuantArgs &q, int src, int row, int k0, bool vec, float (&v)[N]) {
  if (src < 0) {
#pragma unroll
    for (int i = 0; i < N; ++i) v[i] = 0.0f;
    return;
  }
  if (q.src_bf16) {
    const uint16_t *p = q.src_bf16 + (size_t)src * q.K + k0;
    if (vec) {
#pragma unroll
      for (int c = 0; c < N / 8; ++c) {
        const uint4 u = __ldg(reinterpret_cast<const uint4 *>(p) + c);
        const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          v[8 * c + 2 * j] = __uint_as_float(w[j] << 16);
          v[8 * c + 2 * j + 1] = __uint_as_float(w[j] & 0xFFFF0000u);
        }
      }
    } else {
#pragma unroll
      for (int i = 0; i < N; ++i) v[i] = bf16_bits_to_float(p[i]);
    }
  } else {
    const float4 *p = reinterpret_cast<const float4 *>(q.src_f32 + (size_t)row * q.K + k0);
#pragma unroll
    for (int c = 0; c < N / 4; ++c) {
      const float4 f = __ldg(p + c);
      v[4 * c] = f.x; v[4 * c + 1] = f.y; v[4 * c + 2] = f.z; v[4 * c + 3] = f.w;
    }
  }
}

}  // namespace

__global__ void __launch_bounds__(256) quant_rows_kernel(const QuantArgs q) {
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int row = blockIdx.x * 8 + warp;
  if (row >= q.max_rows || row >= *q.n_rows) return;
  const int K = q.K;
  int src = -1;
  if (q.src_bf16) {
    src = checked_index(q.row_token[row], -1, q.db.n_tokens, -1, q.db.err, kChkToken);
  } else {
    const int p = checked_index(q.row_pair[row], -1, q.db.n_pairs, -1, q.db.err, kChkPair);
    if (p >= 0) {
      // expert not in this pass: its h is not ready
      if (q.loc && load_loc(q.loc, q.ids[p], q.db) == kLocAbsent) return;
      src = row;
    }
  }
  uint8_t *codes = q.codes + (size_t)row * (K / 2);
  const bool vec = q.src_f32 != nullptr || (reinterpret_cast<uintptr_t>(q.src_bf16) & 15u) == 0;

  if (q.fmt == MOE_FMT_MXFP4) {
    const int nsf = K / 32;
    for (int b = lane; b < nsf; b += 32) {
      float v[32];
      load_block<32>(q, src, row, b * 32, vec, v);
      float amax = 0.0f;
#pragma unroll
      for (int i = 0; i < 32; ++i) amax = fmaxf(amax, fabsf(v[i]));
      int code = 1;
      if (amax > 0.0f) {
        const int ex = (int)((__float_as_uint(amax) >> 23) & 0xFF);
        const int fl = (ex == 0) ? -127 : ex - 127;        // floor(log2(amax))
        code = min(254, max(1, fl - 2 + 127));
      }
      const float inv = __int_as_float((254 - code) << 23);   // 2^(127 - code), code <= 252 in fp32
      uint32_t w[4];
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        uint32_t word = 0;
#pragma unroll
        for (int j = 0; j < 4; ++j)
          word |= e2m1x2_from_f32(v[i * 8 + 2 * j] * inv, v[i * 8 + 2 * j + 1] * inv) << (8 * j);
        w[i] = word;
      }
      *reinterpret_cast<uint4 *>(codes + b * 16) = make_uint4(w[0], w[1], w[2], w[3]);
      q.sf[sf_offset(nsf, row, b)] = (uint8_t)code;
    }
  } else {
    const int nsf = K / 16;
    // row maximum: 16-byte loads spread over the lanes (the block pass below
    // reads the same bytes again, from L1)
    float amax = 0.0f;
    if (src >= 0) {
      if (q.src_f32) {
        const float4 *p = reinterpret_cast<const float4 *>(q.src_f32 + (size_t)row * K);
        for (int i = lane; i < K / 4; i += 32) {
          const float4 f = __ldg(p + i);
          amax = fmaxf(amax, fmaxf(fmaxf(fabsf(f.x), fabsf(f.y)), fmaxf(fabsf(f.z), fabsf(f.w))));
        }
      } else if (vec) {
        const uint4 *p = reinterpret_cast<const uint4 *>(q.src_bf16 + (size_t)src * K);
        for (int i = lane; i < K / 8; i += 32) {
          const uint4 u = __ldg(p + i);
          const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
          for (int j = 0; j < 4; ++j)
            amax = fmaxf(amax, fmaxf(fabsf(__uint_as_float(w[j] << 16)), fabsf(__uint_as_float(w[j] & 0xFFFF0000u))));
        }
      } else {
        for (int k = lane; k < K; k += 32) amax = fmaxf(amax, fabsf(bf16_bits_to_float(q.src_bf16[(size_t)src * K + k])));
      }
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, o));
    float G = 1.0f;
    if (amax > 0.0f) {
      const double r = (double)amax / (6.0 * 448.0);
      int ex;
      const double f = frexp(r, &ex);
      const int c = (f == 0.5) ? ex - 1 : ex;                 // ceil(log2(r))
      G = ldexpf(1.0f, c);
    }
    if (lane == 0) q.G[row] = G;
    for (int b = lane; b < nsf; b += 32) {
      float v[16];
      load_block<16>(q, src, row, b * 16, vec, v);
      float bmax = 0.0f;
#pragma unroll
      for (int i = 0; i < 16; ++i) bmax = fmaxf(bmax, fabsf(v[i]));
      const float t = __fdiv_rn(__fdiv_rn(bmax, 6.0f), G);
      const uint32_t sc = e4m3_from_f32(t);
      uint32_t w[2] = {0u, 0u};
      if (sc != 0u) {
        const float denom = e4m3_to_f32(sc) * G;
        const float inv = __fdiv_rn(1.0f, denom);
#pragma unroll
        for (int i = 0; i < 2; ++i) {
          uint32_t word = 0;
#pragma unroll
          for (int j = 0; j < 4; ++j)
            word |= e2m1x2_from_f32(v[i * 8 + 2 * j] * inv, v[i * 8 + 2 * j + 1] * inv) << (8 * j);
          w[i] = word;
        }
      }
      *reinterpret_cast<uint2 *>(codes + b * 8) = make_uint2(w[0], w[1]);
      q.sf[sf_offset(nsf, row, b)] = (uint8_t)sc;
    }
  }
}

void launch_quant(const QuantArgs &q, cudaStream_t s) {
  const int blocks = (q.max_rows + 7) / 8;
  if (blocks > 0) quant_rows_kernel<<<blocks, 256, 0, s>>>(q);
}

}  // namespace moe
