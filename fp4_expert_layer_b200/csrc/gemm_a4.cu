// gemm_a4.cu -- grouped expert GEMM on tcgen05 block-scaled FP4 MMA (A4 numerics).
//
// One CTA computes, for one token tile (up to 128 rows of one expert in the
// padded expert-sorted order) and one block of 128 weight rows, the full-K
// product  D[128 x 128] = W[rows, K] . X[tokens, K]^T  with both operands E2M1
// and per-block scales (MXFP4: UE8M0 per 32; NVFP4: UE4M3 per 16) applied by
// the tensor core (kind::mxf4 / kind::mxf4nvf4).  Gate/up runs two
// accumulators (gate and up rows of the same block) so the SwiGLU epilogue
// needs no second pass.  Weights are the A operand (M = 128), tokens the B
// operand (N = 128); both are K-major FP4 tiles loaded by TMA with 128-byte
// swizzle, 256 K elements (128 bytes per row) per stage, 4 stages.  Scale
// factors arrive as 512-byte blocks (128 rows x 4 scales) by bulk copy and are
// moved to TMEM with tcgen05.cp before the MMAs that read them.
//
// Warp roles: warp 0 issues the copies, warp 1 allocates TMEM and one lane
// issues every MMA, warps 4..7 (one per TMEM lane quadrant) read the
// accumulators back with tcgen05.ld.  All mbarrier waits are bounded.
//
// TMEM columns: accumulators at 0 and 128 (128 fp32 columns each), scale
// factors of stage s at 256 + s * (4 per block).
#include "checks.cuh"
#include "device_utils.cuh"
#include "moe_internal.h"
#include "tcgen05.cuh"
#include "tma.cuh"

namespace moe {

namespace {
constexpr int kGStages = 4;

// Two E2M1 codes (round to nearest even, saturating): `lo` in bits 0..3.
__device__ __forceinline__ uint32_t e2m1x2_pack(float lo, float hi) {
  uint32_t r;
  asm("{\n\t.reg .b8 b;\n\t"
      "cvt.rn.satfinite.e2m1x2.f32 b, %2, %1;\n\t"
      "cvt.u32.u8 %0, b;\n\t}"
      : "=r"(r)
      : "f"(lo), "f"(hi));
  return r;
}
constexpr int kTileBytes = 128 * 128;   // 128 rows x 128 bytes (256 FP4 per row)
constexpr int kGThreads = 256;
}  // namespace

template <int WF, int MODE>
struct GemmGeom {
  static constexpr int NMAT = (MODE == MODE_GATEUP) ? 2 : 1;
  static constexpr int NBLK = (WF == WF_MX) ? 2 : 4;            // scale blocks per 128 rows per stage
  static constexpr int SF_BYTES = NBLK * 512;
  static constexpr int B_OFF = NMAT * kTileBytes;
  static constexpr int SF_OFF = (NMAT + 1) * kTileBytes;
  static constexpr int STAGE = SF_OFF + (NMAT + 1) * SF_BYTES;  // multiple of 1024
  static constexpr int SF_COLS = (NMAT + 1) * NBLK * 4;          // TMEM columns per stage
};

template <int WF, int MODE>
__global__ void __launch_bounds__(kGThreads, 1) gemm_a4_kernel(const __grid_constant__ A4GemmArgs a) {
  using Geo = GemmGeom<WF, MODE>;
  constexpr int NMAT = Geo::NMAT;
  static_assert(Geo::STAGE % 1024 == 0, "stage must keep 1024-byte alignment");
  extern __shared__ __align__(1024) uint8_t gsmem_raw[];
  __shared__ __align__(8) uint64_t full_bar[kGStages];
  __shared__ __align__(8) uint64_t empty_bar[kGStages];
  __shared__ __align__(8) uint64_t acc_bar;
  __shared__ uint32_t tmem_base_s;
  // epilogue: per-column activation scale, pair index and gate of the tile,
  // loaded once (the output stores would otherwise order every such load)
  __shared__ float col_bs[128];
  __shared__ int col_pair[128];
  __shared__ float col_gate[128];
  // MXFP4 gate/up with h quantised in the epilogue: per epilogue warp, the
  // codes and block scales of 32 tokens before they go out
  __shared__ __align__(16) uint8_t hq_stage[4][32][16];
  __shared__ uint8_t sf_stage[4][32];

  uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(gsmem_raw) + 1023) & ~uintptr_t(1023));
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int rb = blockIdx.x % a.n_rowblocks;
  const int tile = blockIdx.x / a.n_rowblocks;
  if (tile >= *a.n_tiles) return;
  const TileInfo ti = a.tiles[tile];
  const int loc = load_loc(a.loc, ti.expert, a.db);
  if (loc == kLocAbsent) return;
  const int prow0 = ti.prow0, nrows = ti.nrows;
  const bool in_slot = loc >= 0;
  const int bidx = in_slot ? loc : (-2 - loc);
  const int region = in_slot ? 0 : 1;
  const uint8_t *blob = (in_slot ? a.slots : a.staging) + (size_t)bidx * a.blob_bytes;
  const int K = a.K;
  const int nk = (K + 255) / 256;            // K is a multiple of 128: the last stage may be half full
  const int G = (WF == WF_MX) ? 32 : 16;
  const int nsf = K / G;

  if (threadIdx.x == 0) {
    for (int s = 0; s < kGStages; ++s) {
      mbar_init(smem_u32(&full_bar[s]), 1);
      mbar_init(smem_u32(&empty_bar[s]), 1);
    }
    mbar_init(smem_u32(&acc_bar), 1);
    mbar_fence_init();
  }
  if (warp == 1) {
    tmem_alloc(smem_u32(&tmem_base_s), 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = tmem_base_s;

  if (warp == 0) {
    // ---------------- producer
    if (lane == 0) {
      int s = 0, issued = 0;
      uint32_t ph = 0;
      for (int it = 0; it < nk; ++it) {
        if (it >= kGStages && !mbar_wait(smem_u32(&empty_bar[s]), ph ^ 1u, a.err, 12)) break;
        ++issued;
        const uint32_t bar = smem_u32(&full_bar[s]);
        const uint32_t st = smem_u32(smem + (size_t)s * Geo::STAGE);
        // a half stage (last 128 K elements) carries half the scale blocks; the
        // code tiles are full boxes whose out-of-range half TMA fills with zeros
        const int sfb = (min(256, K - it * 256) / G) / 4 * 512;
        mbar_arrive_expect_tx(bar, (uint32_t)((NMAT + 1) * kTileBytes + (NMAT + 1) * sfb));
        const int col0 = it * (256 / G);                           // first scale column of this stage
#pragma unroll
        for (int j = 0; j < NMAT; ++j) {
          const int m = (MODE == MODE_GATEUP) ? j : 2;
          tma_load_3d(st + j * kTileBytes, &a.maps.w[region][m], bar, it * 128, rb * 128, bidx);
          bulk_load(st + Geo::SF_OFF + j * Geo::SF_BYTES, blob + a.L.scales[m] + sf_offset(nsf, rb * 128, col0),
                    (uint32_t)sfb, bar);
        }
        tma_load_2d(st + Geo::B_OFF, &a.maps.act[a.act_map], bar, it * 128, prow0);
        bulk_load(st + Geo::SF_OFF + NMAT * Geo::SF_BYTES, a.bsf + sf_offset(nsf, prow0, col0), (uint32_t)sfb, bar);
        if (++s == kGStages) { s = 0; ph ^= 1u; }
      }
      // the last copies issued have landed before the CTA exits: at once on a
      // normal run (the MMA lane waited for them), and also when a wait gave up
      int s2 = 0;
      uint32_t ph2 = 0;
      for (int i = 0; i < issued; ++i) {
        if (i >= issued - kGStages) mbar_drain(smem_u32(&full_bar[s2]), ph2);
        if (++s2 == kGStages) { s2 = 0; ph2 ^= 1u; }
      }
    }
  } else if (warp == 1) {
    // ---------------- MMA issuer (one lane)
    if (lane == 0) {
      int s = 0;
      uint32_t ph = 0;
      for (int it = 0; it < nk; ++it) {
        mbar_wait(smem_u32(&full_bar[s]), ph, a.err, 11);
        tc_fence_after();
        const uint32_t st = smem_u32(smem + (size_t)s * Geo::STAGE);
        const uint32_t sf_t = tmem + 256 + (uint32_t)(s * Geo::SF_COLS);
        const int kmma = min(256, K - it * 256) / 64;              // 4, or 2 in a half stage
        const int nblk = (WF == WF_MX) ? kmma / 2 : kmma;          // valid scale blocks per operand
#pragma unroll
        for (int mat = 0; mat <= NMAT; ++mat)
          for (int b = 0; b < nblk; ++b)
            tc_cp_sf_block(sf_t + 4 * (mat * Geo::NBLK + b), st + Geo::SF_OFF + mat * Geo::SF_BYTES + 512 * b);
#pragma unroll
        for (int k = 0; k < 4; ++k) {                              // K = 64 per MMA
          if (k >= kmma) break;
          const int blk = (WF == WF_MX) ? (k >> 1) : k;
          const uint32_t byte = (WF == WF_MX) ? (uint32_t)(2 * (k & 1)) : 0u;
          const uint64_t bdesc = umma_desc(st + Geo::B_OFF + k * 32, 16, 1024, 2);
          const uint32_t sfb = (sf_t + (uint32_t)((NMAT * Geo::NBLK + blk) * 4)) | (byte << 30);
          const uint32_t idesc = idesc_fp4_block(128, 128, WF == WF_MX, byte, byte);
#pragma unroll
          for (int j = 0; j < NMAT; ++j) {
            const uint64_t adesc = umma_desc(st + j * kTileBytes + k * 32, 16, 1024, 2);
            const uint32_t sfa = (sf_t + (uint32_t)((j * Geo::NBLK + blk) * 4)) | (byte << 30);
            const uint32_t acc = (it > 0 || k > 0) ? 1u : 0u;
            if constexpr (WF == WF_MX) umma_mxf4(tmem + 128 * j, adesc, bdesc, idesc, sfa, sfb, acc);
            else umma_nvf4(tmem + 128 * j, adesc, bdesc, idesc, sfa, sfb, acc);
          }
        }
        tc_commit(smem_u32(&empty_bar[s]));                        // stage free once these MMAs finish
        if (++s == kGStages) { s = 0; ph ^= 1u; }
      }
      tc_commit(smem_u32(&acc_bar));                               // accumulators complete
      // this lane waits for them too: no MMA may still run when the CTA frees
      // TMEM and leaves, even if the epilogue's wait gave up
      mbar_drain(smem_u32(&acc_bar), 0);
    }
  } else if (warp >= 4) {
    // ---------------- epilogue: warp w reads TMEM lanes 32*(w%4) .. +31
    const int quad = warp & 3;
    {
      const int c = threadIdx.x - 128;                               // 0..127 over warps 4..7
      if (c < nrows) {
        col_bs[c] = (WF == WF_NV) ? __ldg(a.bG + prow0 + c) : 1.0f;
        if constexpr (MODE == MODE_DOWN) {
          const int p = checked_index(__ldg(a.prow_pair + prow0 + c), 0, a.db.n_pairs, 0, a.db.err, kChkPair);
          col_pair[c] = p;
          col_gate[c] = __ldg(a.gates + p);
        }
      }
      named_bar_sync(1, 128);
    }
    mbar_wait(smem_u32(&acc_bar), 0, a.err, 13);
    tc_fence_after();
    const int r_local = 32 * quad + lane;
    const int row = rb * 128 + r_local;                            // weight row (I or H index)
    float wsc[2] = {1.0f, 1.0f};
    if constexpr (WF == WF_NV) {
#pragma unroll
      for (int j = 0; j < NMAT; ++j) {
        const int m = (MODE == MODE_GATEUP) ? j : 2;
        wsc[j] = reinterpret_cast<const float *>(blob + a.L.glob)[m];
      }
    }
    bool quantised = false;
    if constexpr (WF == WF_MX && MODE == MODE_GATEUP) {
      if (a.hq_out) {
        quantised = true;
        // h quantised here for the down pass (MXFP4 rule of the activation
        // quantiser: per 32 consecutive h columns of a token, E8M0 exponent
        // clamp(floor(log2 amax) - 2 + 127, 1, 254), codes RNE E2M1 of
        // h * 2^(127 - e), saturating).  A warp holds 32 consecutive columns
        // (one block) of each token; 32 tokens at a time so that the block
        // maxima of different tokens reduce in parallel.
        const int I = a.rows;
        const int blk = (rb * 128 + 32 * quad) / 32;
        uint8_t(*qs)[16] = hq_stage[quad];                       // [token][16 code bytes] of this warp
        for (int cb = 0; cb < 4; ++cb) {
          if (32 * cb >= nrows) break;                           // warp-uniform
          uint32_t d0[32], d1[32];
          tmem_ld32(tmem + ((uint32_t)(32 * quad) << 16) + 32 * cb, d0);
          tmem_ld32(tmem + ((uint32_t)(32 * quad) << 16) + 128 + 32 * cb, d1);
          tmem_ld_wait();
#pragma unroll
          for (int jj = 0; jj < 32; ++jj) {
            const float h = silu_f(__uint_as_float(d0[jj])) * __uint_as_float(d1[jj]);
            // block maximum of |h| over the warp's 32 columns (non-negative
            // floats order like their bit patterns)
            const uint32_t am = __reduce_max_sync(0xffffffffu, __float_as_uint(fabsf(h)));
            int code = 1;
            if (am != 0u) {
              const int ex = (int)((am >> 23) & 0xFF);
              code = min(254, max(1, (ex == 0 ? -127 : ex - 127) - 2 + 127));
            }
            const float v = h * __int_as_float((254 - code) << 23);   // h * 2^(127 - code)
            const float vn = __shfl_down_sync(0xffffffffu, v, 1);
            if ((lane & 1) == 0) qs[jj][lane >> 1] = (uint8_t)(e2m1x2_pack(v, vn) & 0xFFu);
            if (lane == 0) sf_stage[quad][jj] = (uint8_t)code;
          }
          __syncwarp();
          // lane j writes token j of the chunk: 16 code bytes and one scale
          const int col = 32 * cb + lane;
          if (col < nrows) {
            const size_t prow = (size_t)(prow0 + col);
            *reinterpret_cast<uint4 *>(a.hq_out + prow * (I / 2) + (rb * 128 + 32 * quad) / 2) =
                *reinterpret_cast<const uint4 *>(qs[lane]);
            a.hsf_out[sf_offset(I / 32, (int)prow, blk)] = sf_stage[quad][lane];
          }
          __syncwarp();
        }
      }
    }
    for (int cb = 0; cb < 4 && !quantised; ++cb) {
      uint32_t d0[32], d1[32];
      tmem_ld32(tmem + ((uint32_t)(32 * quad) << 16) + 32 * cb, d0);
      if constexpr (NMAT == 2) tmem_ld32(tmem + ((uint32_t)(32 * quad) << 16) + 128 + 32 * cb, d1);
      tmem_ld_wait();
#pragma unroll
      for (int jj = 0; jj < 32; ++jj) {
        const int col = 32 * cb + jj;
        if (col >= nrows) continue;
        const int prow = prow0 + col;
        const float bs = col_bs[col];
        if constexpr (MODE == MODE_GATEUP) {
          const float av = __uint_as_float(d0[jj]) * (wsc[0] * bs);
          const float uv = __uint_as_float(d1[jj]) * (wsc[1] * bs);
          a.h_out[(size_t)prow * a.rows + row] = silu_f(av) * uv;
        } else {
          a.o_out[(size_t)col_pair[col] * a.rows + row] = __uint_as_float(d0[jj]) * (wsc[0] * bs) * col_gate[col];
        }
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

template <int WF, int MODE>
static void launch_gemm_one(const A4GemmArgs &a, int grid_tiles, cudaStream_t s) {
  using Geo = GemmGeom<WF, MODE>;
  const size_t smem = (size_t)kGStages * Geo::STAGE + 1024;
  auto fn = gemm_a4_kernel<WF, MODE>;
  cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  fn<<<grid_tiles * a.n_rowblocks, kGThreads, smem, s>>>(a);
}

void launch_gemm_a4(int wf, int mode, const A4GemmArgs &a, int grid_tiles, cudaStream_t s) {
  if (grid_tiles <= 0) return;
  if (wf == WF_MX) {
    if (mode == MODE_GATEUP) launch_gemm_one<WF_MX, MODE_GATEUP>(a, grid_tiles, s);
    else launch_gemm_one<WF_MX, MODE_DOWN>(a, grid_tiles, s);
  } else {
    if (mode == MODE_GATEUP) launch_gemm_one<WF_NV, MODE_GATEUP>(a, grid_tiles, s);
    else launch_gemm_one<WF_NV, MODE_DOWN>(a, grid_tiles, s);
  }
}

}  // namespace moe
