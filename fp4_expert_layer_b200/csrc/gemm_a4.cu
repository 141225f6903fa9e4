// gemm_a4.cu -- grouped expert GEMM on tcgen05 block-scaled FP4 MMA (A4 numerics).
//
// A work item is one token tile (up to 128 rows of one expert in the padded
// expert-sorted order) and one block of 128 weight rows; it computes the
// full-K product  D[128 x 128] = W[rows, K] . X[tokens, K]^T  with both
// operands E2M1 and per-block scales (MXFP4: UE8M0 per 32; NVFP4: UE4M3 per
// 16) applied by the tensor core (kind::mxf4 / kind::mxf4nvf4).  Weights are
// the A operand (M = 128), tokens the B operand (N = 128); both are K-major
// FP4 tiles loaded by TMA with 128-byte swizzle, 256 K elements (128 bytes per
// row) per stage.  Scale factors arrive as 512-byte blocks (128 rows x 4
// scales) by bulk copy and are moved to TMEM with tcgen05.cp before the MMAs
// that read them.
//
// Gate/up: an A4 layer's blob holds gate and up as one matrix of 2I rows,
// interleaved per 64 rows (64 gate rows, the same 64 up rows, ...), so one
// 128-row block carries both halves of 64 h columns: the item's single
// accumulator has the gate rows in TMEM lanes 0..63 and the up rows in lanes
// 64..127, and the SwiGLU epilogue meets them through shared memory.  With
// one 128-column accumulator per item the accumulators are double-buffered in
// TMEM, so an item's epilogue overlaps the next item's main loop.
//
// Persistent, one CTA per SM, work items taken from a counter in index order.
// Warp roles: warp 0 takes the items and issues the copies, warp 1 allocates
// TMEM and issues every MMA (both whole warps with one elected lane issuing),
// warps 2..9 read the
// accumulators back with tcgen05.ld (warp w the lanes of quadrant w % 4; warps
// 2..5 tokens 0..63 of an item, warps 6..9 tokens 64..127).  All mbarrier
// waits are bounded.
//
// TMEM columns: accumulators at 0 and 128; the A and B scale blocks of stage
// s at 256 + s * SF_COLS (16 columns per stage for MXFP4, 32 for NVFP4).
#include "checks.cuh"
#include "device_utils.cuh"
#include "launch.cuh"
#include "moe_internal.h"
#include "tcgen05.cuh"
#include "tma.cuh"

namespace moe {

namespace {

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

__device__ __forceinline__ TileInfo load_tile_a4(const TileInfo *p) {
  const int4 v = __ldcg(reinterpret_cast<const int4 *>(p));
  return TileInfo{v.x, v.y, v.z, v.w};
}

constexpr int kTileBytes = 128 * 128;   // 128 rows x 128 bytes (256 FP4 per row)
constexpr int kGThreads = 320;          // warp 0 copies, warp 1 MMA, warps 2..9 epilogue
constexpr int kGEpi = 256;              // epilogue threads
constexpr int kGSched = 4;
constexpr int kGSchedReaders = 9;       // MMA lane + 8 epilogue warps

}  // namespace

template <int WF>
struct GemmGeom {
  static constexpr int NBLK = (WF == WF_MX) ? 2 : 4;      // scale blocks per operand per 256 K
  static constexpr int SF_BYTES = NBLK * 512;
  static constexpr int B_OFF = kTileBytes;
  static constexpr int SF_OFF = 2 * kTileBytes;
  static constexpr int STAGE = SF_OFF + 2 * SF_BYTES;     // 34 KB (MXFP4) / 36 KB (NVFP4)
  static constexpr int STAGES = (WF == WF_MX) ? 6 : 5;
  static constexpr int NBUF = 2;
  static constexpr int SF_COLS = 2 * NBLK * 4;            // TMEM columns per stage (A and B scales)
  static constexpr int SF_TMEM = NBUF * 128;
  static constexpr size_t SMEM = (size_t)STAGES * STAGE + 1024;
  static_assert(STAGE % 1024 == 0, "stages keep the 1024-byte swizzle alignment");
  static_assert(SF_TMEM + STAGES * SF_COLS <= 512, "TMEM budget");
  static_assert(SMEM + 22 * 1024 <= 227 * 1024, "shared-memory budget");
};

template <int WF, int MODE>
__global__ void __launch_bounds__(kGThreads, 1) gemm_a4_kernel(const __grid_constant__ A4GemmArgs a) {
  using Geo = GemmGeom<WF>;
  constexpr int S = Geo::STAGES;
  constexpr int NBUF = Geo::NBUF;
  extern __shared__ __align__(1024) uint8_t gsmem_raw[];
  __shared__ __align__(8) uint64_t full_bar[S];
  __shared__ __align__(8) uint64_t empty_bar[S];
  __shared__ __align__(8) uint64_t accf_bar[NBUF];
  __shared__ __align__(8) uint64_t acce_bar[NBUF];
  __shared__ __align__(8) uint64_t quiesce_bar;      // all MMAs of the CTA done (before TMEM is freed)
  __shared__ __align__(8) uint64_t sched_full[kGSched];
  __shared__ __align__(8) uint64_t sched_empty[kGSched];
  __shared__ int sched_item[kGSched];
  __shared__ TileInfo sched_ti[kGSched];
  __shared__ int sched_loc[kGSched];
  __shared__ uint32_t tmem_base_s;
  // epilogue: per-column activation scale, pair index and gate of the item's
  // tile, loaded once (the output stores would otherwise order every such load)
  __shared__ float col_bs[128];
  __shared__ int col_pair[128];
  __shared__ float col_gate[128];
  // gate/up, per epilogue group: gate values of the second 16 tokens of a
  // 32-token chunk (for the up warps) and up values of the first 16 (for the
  // gate warps), 64 rows each
  __shared__ float xg[2][64][17];
  __shared__ float xu[2][64][17];
  // MXFP4 gate/up with h quantised in the epilogue: per epilogue warp, the
  // codes and block scales of its 16 tokens before they go out
  __shared__ __align__(16) uint8_t hq_stage[8][16][16];
  __shared__ uint8_t sf_stage[8][16];

  uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(gsmem_raw) + 1023) & ~uintptr_t(1023));
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int K = a.K;
  const int nk = (K + 255) / 256;            // K is a multiple of 128: the last stage may be half full
  const int G = (WF == WF_MX) ? 32 : 16;
  const int nsf = K / G;
  const int ipt = a.n_rowblocks;

  if (threadIdx.x == 0) {
    for (int s = 0; s < S; ++s) {
      mbar_init(smem_u32(&full_bar[s]), 1);
      mbar_init(smem_u32(&empty_bar[s]), 1);
    }
    for (int b = 0; b < NBUF; ++b) {
      mbar_init(smem_u32(&accf_bar[b]), 1);
      mbar_init(smem_u32(&acce_bar[b]), kGEpi / 32);
    }
    for (int q = 0; q < kGSched; ++q) {
      mbar_init(smem_u32(&sched_full[q]), 1);
      mbar_init(smem_u32(&sched_empty[q]), kGSchedReaders);
    }
    mbar_init(smem_u32(&quiesce_bar), 1);
    mbar_fence_init();
  }
  if (warp == 1) {
    tmem_alloc(smem_u32(&tmem_base_s), 512);
    tmem_relinquish();
  }
  wait_prior_grid();                                   // tiles, locations and activations come from earlier kernels
  const int n_items = __ldcg(a.n_tiles) * ipt;
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = tmem_base_s;

  if (warp == 0) {
    // ---------------- copies: work items, weight + activation tiles and their
    // scales.  The whole warp runs the loop (warp-uniform waits, values
    // broadcast from lane 0) and one elected lane issues the copies: a copy
    // issued from a one-lane loop behind a lane test costs about twice as much.
    int s = 0, issued = 0;
    uint32_t ph = 0;
    int q = 0;
    uint32_t qph = 0;
    bool failed = false;
    const int m = (MODE == MODE_GATEUP) ? 0 : 2;
    for (int j = 0; !failed; ++j) {
      int item = 0;
      if (lane == 0) item = atomicAdd(a.work_ctr, 1);
      item = __shfl_sync(0xffffffffu, item, 0);
      TileInfo ti{};
      int loc = kLocAbsent;
      if (item < n_items) {
        ti = load_tile_a4(a.tiles + item / ipt);
        loc = load_loc(a.loc, ti.expert, a.db);
      }
      if (j >= kGSched && !mbar_wait_warp(smem_u32(&sched_empty[q]), qph ^ 1u, a.err, 14)) { failed = true; break; }
      const bool done = item >= n_items;
      if (lane == 0) {
        sched_item[q] = done ? -1 : item;
        sched_ti[q] = ti;
        sched_loc[q] = loc;
        mbar_arrive(smem_u32(&sched_full[q]));
      }
      __syncwarp();
      if (++q == kGSched) { q = 0; qph ^= 1u; }
      if (done) break;
      if (loc == kLocAbsent) continue;
      const int rb = item % ipt;
      const bool in_slot = loc >= 0;
      const int bidx = in_slot ? loc : (-2 - loc);
      const int region = in_slot ? 0 : 1;
      const uint8_t *blob = (in_slot ? a.slots : a.staging) + (size_t)bidx * a.blob_bytes;
      for (int it = 0; it < nk; ++it) {
        if (issued >= S && !mbar_wait_warp(smem_u32(&empty_bar[s]), ph ^ 1u, a.err, 12)) { failed = true; break; }
        const uint32_t bar = smem_u32(&full_bar[s]);
        const uint32_t st = smem_u32(smem + (size_t)s * Geo::STAGE);
        // a half stage (last 128 K elements) carries half the scale blocks; the
        // code tiles are full boxes whose out-of-range half TMA fills with zeros
        const int sfb = (min(256, K - it * 256) / G) / 4 * 512;
        const int col0 = it * (256 / G);                         // first scale column of this stage
        if (elect_one()) {
          mbar_arrive_expect_tx(bar, (uint32_t)(2 * kTileBytes + 2 * sfb));
          tma_load_3d(st, &a.maps.w[region][m], bar, it * 128, rb * 128, bidx);
          bulk_load(st + Geo::SF_OFF, blob + a.L.scales[m] + sf_offset(nsf, rb * 128, col0), (uint32_t)sfb, bar);
          tma_load_2d(st + Geo::B_OFF, &a.maps.act[a.act_map], bar, it * 128, ti.prow0);
          bulk_load(st + Geo::SF_OFF + Geo::SF_BYTES, a.bsf + sf_offset(nsf, ti.prow0, col0), (uint32_t)sfb, bar);
        }
        __syncwarp();
        ++issued;
        if (++s == S) { s = 0; ph ^= 1u; }
      }
    }
    // the last copies issued have landed before the CTA exits: at once on a
    // normal run (the MMA warp waited for them), and also when a wait gave up
    if (lane == 0) {
      int s2 = 0;
      uint32_t ph2 = 0;
      for (int i = 0; i < issued; ++i) {
        if (i >= issued - S) mbar_drain(smem_u32(&full_bar[s2]), ph2);
        if (++s2 == S) { s2 = 0; ph2 ^= 1u; }
      }
    }
  } else if (warp == 1) {
    // ---------------- MMA issuer: the whole warp runs the loop (every wait
    // warp-uniform) and one elected lane issues the scale copies, the MMAs and
    // the commits, so that their operands stay in uniform registers
    int s = 0, n = 0;
    uint32_t ph = 0;
    int q = 0;
    uint32_t qph = 0;
    while (true) {
      if (!mbar_wait_warp(smem_u32(&sched_full[q]), qph, a.err, 15)) break;
      // broadcast from lane 0: values the compiler knows to be warp-uniform
      const int item = __shfl_sync(0xffffffffu, sched_item[q], 0);
      const int loc = __shfl_sync(0xffffffffu, sched_loc[q], 0);
      if (lane == 0) mbar_arrive(smem_u32(&sched_empty[q]));
      if (++q == kGSched) { q = 0; qph ^= 1u; }
      if (item < 0) break;
      if (loc == kLocAbsent) continue;
      const int buf = n % NBUF;
      if (n >= NBUF && !mbar_wait_warp(smem_u32(&acce_bar[buf]), ((n / NBUF) - 1) & 1, a.err, 16)) break;
      tc_fence_after();
      const uint32_t acc = tmem + (uint32_t)(buf * 128);
      bool failed = false;
      for (int it = 0; it < nk; ++it) {
        if (!mbar_wait_warp(smem_u32(&full_bar[s]), ph, a.err, 11)) { failed = true; break; }
        tc_fence_after();
        const uint32_t st = smem_u32(smem + (size_t)s * Geo::STAGE);
        const uint32_t sf_t = tmem + (uint32_t)(Geo::SF_TMEM + s * Geo::SF_COLS);
        const int kmma = min(256, K - it * 256) / 64;                // 4, or 2 in a half stage
        const int nblk = (WF == WF_MX) ? kmma / 2 : kmma;            // valid scale blocks per operand
        if (elect_one()) {
#pragma unroll
          for (int mat = 0; mat < 2; ++mat)
            for (int b = 0; b < nblk; ++b)
              tc_cp_sf_block(sf_t + 4 * (mat * Geo::NBLK + b), st + Geo::SF_OFF + mat * Geo::SF_BYTES + 512 * b);
#pragma unroll
          for (int k = 0; k < 4; ++k) {                              // K = 64 per MMA
            if (k >= kmma) break;
            const int blk = (WF == WF_MX) ? (k >> 1) : k;
            const uint32_t byte = (WF == WF_MX) ? (uint32_t)(2 * (k & 1)) : 0u;
            const uint64_t adesc = umma_desc(st + k * 32, 16, 1024, 2);
            const uint64_t bdesc = umma_desc(st + Geo::B_OFF + k * 32, 16, 1024, 2);
            const uint32_t sfa = (sf_t + (uint32_t)(blk * 4)) | (byte << 30);
            const uint32_t sfb = (sf_t + (uint32_t)((Geo::NBLK + blk) * 4)) | (byte << 30);
            const uint32_t idesc = idesc_fp4_block(128, 128, WF == WF_MX, byte, byte);
            const uint32_t accum = (it > 0 || k > 0) ? 1u : 0u;
            if constexpr (WF == WF_MX) umma_mxf4(acc, adesc, bdesc, idesc, sfa, sfb, accum);
            else umma_nvf4(acc, adesc, bdesc, idesc, sfa, sfb, accum);
          }
          tc_commit(smem_u32(&empty_bar[s]));                        // stage free once these MMAs finish
        }
        __syncwarp();
        if (++s == S) { s = 0; ph ^= 1u; }
      }
      if (failed) break;
      if (elect_one()) tc_commit(smem_u32(&accf_bar[buf]));         // this item's accumulator complete
      __syncwarp();
      ++n;
    }
    // every MMA issued above has completed before the CTA frees TMEM and
    // leaves (also after a wait gave up and the loop was left early)
    __syncwarp();
    if (elect_one()) tc_commit(smem_u32(&quiesce_bar));
    __syncwarp();
    mbar_drain(smem_u32(&quiesce_bar), 0);
  } else {
    // ---------------- epilogue: warp w reads TMEM lanes 32*(w%4) .. +31; the
    // warps 2..5 (group 0) take tokens 0..63 of an item, warps 6..9 (group 1)
    // tokens 64..127
    const int quad = warp & 3;
    const int grp = (warp - 2) >> 2;
    const int wslot = warp - 2;
    const int et = threadIdx.x - 64;                                 // 0..255 over warps 2..9
    int n = 0;
    bool ok = true;
    int q = 0;
    uint32_t qph = 0;
    while (ok) {
      int okw = 1;
      if (lane == 0) okw = mbar_wait(smem_u32(&sched_full[q]), qph, a.err, 17) ? 1 : 0;
      okw = __shfl_sync(0xffffffffu, okw, 0);
      __syncwarp();
      const int item = okw ? sched_item[q] : -1;
      const TileInfo ti = sched_ti[q];
      const int loc = sched_loc[q];
      __syncwarp();
      if (okw && lane == 0) mbar_arrive(smem_u32(&sched_empty[q]));
      if (++q == kGSched) { q = 0; qph ^= 1u; }
      // the eight warps stop together (each takes every named barrier below)
      if (!named_bar_and(1, kGEpi, okw != 0 && item >= 0)) break;
      if (loc == kLocAbsent) continue;
      const int rb = item % ipt;
      const int prow0 = ti.prow0, nrows = ti.nrows;
      const int buf = n % NBUF;
      const uint8_t *blob = (loc >= 0 ? a.slots : a.staging) + (size_t)(loc >= 0 ? loc : (-2 - loc)) * a.blob_bytes;
      if (et < nrows && et < 128) {
        col_bs[et] = (WF == WF_NV) ? __ldg(a.bG + prow0 + et) : 1.0f;
        if constexpr (MODE == MODE_DOWN) {
          const int p = checked_index(__ldg(a.prow_pair + prow0 + et), 0, a.db.n_pairs, 0, a.db.err, kChkPair);
          col_pair[et] = p;
          col_gate[et] = __ldg(a.gates + p);
        }
      }
      ok = mbar_wait(smem_u32(&accf_bar[buf]), (n / NBUF) & 1, a.err, 13);
      ok = named_bar_and(1, kGEpi, ok);                               // also publishes col_*
      tc_fence_after();
      const uint32_t acc = tmem + (uint32_t)(buf * 128) + ((uint32_t)(32 * quad) << 16);
      if constexpr (MODE == MODE_GATEUP) {
        // lanes 0..63: gate rows, 64..127: up rows of h columns rb*64 .. +63.
        // A gate warp and the up warp of the same 32 columns split each
        // 32-token chunk: the gate warp computes tokens 0..15, the up warp
        // 16..31, each handing the other the values it needs
        const bool is_up = quad >= 2;
        const int half = quad & 1;
        const int I = a.rows;
        const int hrow = 32 * half + lane;                           // h column within the item's 64
        const int hcol = rb * 64 + hrow;
        const float wsc = (WF == WF_NV) ? reinterpret_cast<const float *>(blob + a.L.glob)[is_up ? 1 : 0] : 1.0f;
        const bool quantise = (WF == WF_MX) && a.hq_out != nullptr;
        const int j0 = is_up ? 16 : 0;                               // this warp's tokens in a chunk
        for (int cc = 0; cc < 2; ++cc) {
          const int cb = 2 * grp + cc;
          if (32 * cb >= nrows) break;                               // uniform over the group
          uint32_t d[32];
          tmem_ld32(acc + (uint32_t)(32 * cb), d);
          tmem_ld_wait();
          float v[32];
#pragma unroll
          for (int jj = 0; jj < 32; ++jj) v[jj] = __uint_as_float(d[jj]) * (wsc * col_bs[32 * cb + jj]);
          if (ok) {
#pragma unroll
            for (int jj = 0; jj < 16; ++jj) {
              if (is_up) xu[grp][hrow][jj] = v[jj];                  // up of tokens 0..15 for the gate warp
              else xg[grp][hrow][jj] = v[16 + jj];                   // gate of tokens 16..31 for the up warp
            }
          }
          named_bar_sync(2 + grp, 128);
          if (ok) {
            float h[16];
#pragma unroll
            for (int jj = 0; jj < 16; ++jj)
              h[jj] = is_up ? silu_f(xg[grp][hrow][jj]) * v[16 + jj] : silu_f(v[jj]) * xu[grp][hrow][jj];
            if (quantise) {
              // h quantised for the down pass (MXFP4 rule of the activation
              // quantiser: per 32 consecutive h columns of a token, E8M0
              // exponent clamp(floor(log2 amax) - 2 + 127, 1, 254), codes RNE
              // E2M1 of h * 2^(127 - e), saturating).  The warp's 32 lanes are
              // one block of 32 h columns of each token.
              uint8_t(*qs)[16] = hq_stage[wslot];
#pragma unroll
              for (int jj = 0; jj < 16; ++jj) {
                // block maximum of |h| (non-negative floats order like their bit patterns)
                const uint32_t am = __reduce_max_sync(0xffffffffu, __float_as_uint(fabsf(h[jj])));
                int code = 1;
                if (am != 0u) {
                  const int ex = (int)((am >> 23) & 0xFF);
                  code = min(254, max(1, (ex == 0 ? -127 : ex - 127) - 2 + 127));
                }
                const float qv = h[jj] * __int_as_float((254 - code) << 23);   // h * 2^(127 - code)
                const float qn = __shfl_down_sync(0xffffffffu, qv, 1);
                if ((lane & 1) == 0) qs[jj][lane >> 1] = (uint8_t)(e2m1x2_pack(qv, qn) & 0xFFu);
                if (lane == 0) sf_stage[wslot][jj] = (uint8_t)code;
              }
              __syncwarp();
              // lane t < 16 writes token j0 + t of the chunk: 16 code bytes and one scale
              const int col = 32 * cb + j0 + lane;
              if (lane < 16 && col < nrows) {
                const size_t prow = (size_t)(prow0 + col);
                const int c0 = rb * 64 + 32 * half;
                *reinterpret_cast<uint4 *>(a.hq_out + prow * (I / 2) + c0 / 2) =
                    *reinterpret_cast<const uint4 *>(qs[lane]);
                a.hsf_out[sf_offset(I / 32, (int)prow, c0 / 32)] = sf_stage[wslot][lane];
              }
              __syncwarp();
            } else {
#pragma unroll
              for (int jj = 0; jj < 16; ++jj) {
                const int col = 32 * cb + j0 + jj;
                if (col < nrows) a.h_out[(size_t)(prow0 + col) * I + hcol] = h[jj];   // warp-uniform test
              }
            }
          }
          named_bar_sync(2 + grp, 128);                                // xg / xu are rewritten by the next chunk
        }
      } else {
        const float wsc = (WF == WF_NV) ? reinterpret_cast<const float *>(blob + a.L.glob)[2] : 1.0f;
        const int row = rb * 128 + 32 * quad + lane;                   // output row (H index)
        for (int cc = 0; cc < 2; ++cc) {
          const int cb = 2 * grp + cc;
          if (32 * cb >= nrows) break;
          uint32_t d[32];
          tmem_ld32(acc + (uint32_t)(32 * cb), d);
          tmem_ld_wait();
          if (!ok) continue;
#pragma unroll
          for (int jj = 0; jj < 32; ++jj) {
            const int col = 32 * cb + jj;
            if (col >= nrows) continue;
            a.o_out[(size_t)col_pair[col] * a.rows + row] =
                __uint_as_float(d[jj]) * (wsc * col_bs[col]) * col_gate[col];
          }
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(smem_u32(&acce_bar[buf]));
      named_bar_sync(1, kGEpi);                                        // col_* are rewritten by the next item
      ++n;
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
static void launch_gemm_one(const A4GemmArgs &a, cudaStream_t s) {
  using Geo = GemmGeom<WF>;
  auto fn = gemm_a4_kernel<WF, MODE>;
  cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)Geo::SMEM);
  launch_dependent(fn, a.grid, kGThreads, Geo::SMEM, s, a);
}

void launch_gemm_a4(int wf, int mode, const A4GemmArgs &a, cudaStream_t s) {
  if (a.grid <= 0) return;
  if (wf == WF_MX) {
    if (mode == MODE_GATEUP) launch_gemm_one<WF_MX, MODE_GATEUP>(a, s);
    else launch_gemm_one<WF_MX, MODE_DOWN>(a, s);
  } else {
    if (mode == MODE_GATEUP) launch_gemm_one<WF_NV, MODE_GATEUP>(a, s);
    else launch_gemm_one<WF_NV, MODE_DOWN>(a, s);
  }
}

}  // namespace moe
