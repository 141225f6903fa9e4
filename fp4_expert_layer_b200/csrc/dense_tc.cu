// dense_tc.cu -- the always-on bf16 shared expert on the tcgen05 tensor core
// (kind::f16, bf16 x bf16 -> fp32 in TMEM) for prefill-sized batches.
//
// The shared expert is applied to every token with weight 1 ("Strata,
// Explained", section 2: routed experts plus one shared expert that stays
// in VRAM); s = W_down . (silu(W_gate . x) * (W_up . x)), h kept in bf16.
// Persistent CTAs walk work items (tile of NBOX tokens, 256 weight rows):
// gate/up items hold 128 gate and the same 128 up rows (two accumulators),
// down items 256 output rows.  Warp 0 streams 64-element K slabs of both
// operands by TMA (bf16, 128-byte swizzle, rows past T read as zeros), warp 1
// issues the MMAs (M = 128, N = tokens rounded up to 16, K = 16 each), warps
// 2..5 read the double-buffered accumulators back: gate/up writes h (bf16
// [T, I_s]), down writes s (fp32 [T, H]) for the ordered combine.
// All mbarrier waits are bounded.
#include <cooperative_groups.h>

#include "device_utils.cuh"
#include "launch.cuh"
#include "moe_internal.h"
#include "tcgen05.cuh"
#include "tma.cuh"

namespace cg = cooperative_groups;

namespace moe {

namespace {
constexpr int kDenseThreads = 192;

template <int NBOX>
struct DenseGeom {
  static constexpr int STAGES = NBOX <= 32 ? 5 : 4;
  static constexpr int A_BYTES = 2 * 128 * 128;   // two 128-row x 64-element bf16 tiles
  static constexpr int B_OFF = A_BYTES;
  static constexpr int B_BYTES = NBOX * 128;      // NBOX token rows x 64 bf16
  static constexpr int STAGE = ((B_OFF + B_BYTES) + 1023) / 1024 * 1024;
  static constexpr int NBUF = 2;
  static constexpr int COLS = NBUF * 2 * NBOX;
  static constexpr int TMEM_COLS = COLS <= 128 ? 128 : (COLS <= 256 ? 256 : 512);
  static constexpr size_t SMEM = (size_t)STAGES * STAGE + 1024;
  static_assert(COLS <= 512, "TMEM budget");
};

// kind::f16 instruction descriptor: fp32 accumulator, bf16 A and B, K-major.
__device__ __forceinline__ uint32_t idesc_bf16(int M, int N) {
  uint32_t d = 0;
  d |= 1u << 4;    // C: F32
  d |= 1u << 7;    // A: BF16
  d |= 1u << 10;   // B: BF16
  d |= (uint32_t)(N >> 3) << 17;
  d |= (uint32_t)(M >> 4) << 24;
  return d;
}

__device__ __forceinline__ void umma_bf16(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc, uint32_t idesc,
                                          uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
      "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate)
      : "memory");
}
}  // namespace

template <int MODE, int NBOX>
__global__ void __launch_bounds__(kDenseThreads, 1) dense_tc_kernel(const __grid_constant__ DenseTcArgs a) {
  using Geo = DenseGeom<NBOX>;
  constexpr int S = Geo::STAGES;
  constexpr int NBUF = Geo::NBUF;
  extern __shared__ __align__(1024) uint8_t dn_smem_raw[];
  __shared__ __align__(8) uint64_t full_bar[S];
  __shared__ __align__(8) uint64_t empty_bar[S];
  __shared__ __align__(8) uint64_t accf_bar[NBUF];
  __shared__ __align__(8) uint64_t acce_bar[NBUF];
  __shared__ __align__(8) uint64_t quiesce_bar;   // all MMAs of the CTA done (before TMEM is freed)
  __shared__ uint32_t tmem_base_s;

  uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(dn_smem_raw) + 1023) & ~uintptr_t(1023));
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int nslab = a.K / 64;
  const int ipt = a.n_rowblocks;
  const int n_tiles = (a.T + NBOX - 1) / NBOX;
  const int n_items = n_tiles * ipt;

  if (threadIdx.x == 0) {
    for (int s = 0; s < S; ++s) {
      mbar_init(smem_u32(&full_bar[s]), 1);
      mbar_init(smem_u32(&empty_bar[s]), 1);
    }
    for (int b = 0; b < NBUF; ++b) {
      mbar_init(smem_u32(&accf_bar[b]), 1);
      mbar_init(smem_u32(&acce_bar[b]), 4);
    }
    mbar_init(smem_u32(&quiesce_bar), 1);
    mbar_fence_init();
  }
  if (warp == 1) {
    tmem_alloc(smem_u32(&tmem_base_s), Geo::TMEM_COLS);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = tmem_base_s;
  wait_prior_grid();                                   // x / h come from earlier kernels

  if (warp == 0) {
    // ---------------- producer: the whole warp runs the loop (warp-uniform
    // waits) and one elected lane issues the copies
    {
      int s = 0, issued = 0;
      uint32_t ph = 0;
      bool failed = false;
      for (int item = blockIdx.x; item < n_items && !failed; item += gridDim.x) {
        const int tile = item / ipt, rb = item % ipt;
        for (int slab = 0; slab < nslab; ++slab) {
          if (issued >= S && !mbar_wait_warp(smem_u32(&empty_bar[s]), ph ^ 1u, a.err, 42)) { failed = true; break; }
          const uint32_t bar = smem_u32(&full_bar[s]);
          const uint32_t st = smem_u32(smem + (size_t)s * Geo::STAGE);
          if (elect_one()) {
            mbar_arrive_expect_tx(bar, (uint32_t)(Geo::A_BYTES + Geo::B_BYTES));
            if constexpr (MODE == MODE_GATEUP) {
              tma_load_2d(st, &a.wmap[0], bar, slab * 64, rb * 128);
              tma_load_2d(st + 16384, &a.wmap[1], bar, slab * 64, rb * 128);
            } else {
              tma_load_2d(st, &a.wmap[0], bar, slab * 64, rb * 256);
              tma_load_2d(st + 16384, &a.wmap[0], bar, slab * 64, rb * 256 + 128);
            }
            tma_load_2d(st + Geo::B_OFF, &a.xmap, bar, slab * 64, tile * NBOX);
          }
          __syncwarp();
          ++issued;
          if (++s == S) { s = 0; ph ^= 1u; }
        }
      }
      {
        // the last copies issued have landed before the CTA exits: at once on
        // a normal run (their consumers waited for them), and also when a
        // consumer gave up waiting
        int s2 = 0;
        uint32_t ph2 = 0;
        for (int i = 0; i < issued; ++i) {
          if (i >= issued - S) mbar_drain(smem_u32(&full_bar[s2]), ph2);
          if (++s2 == S) { s2 = 0; ph2 ^= 1u; }
        }
      }
    }
  } else if (warp == 1) {
    // ---------------- MMA issuer: the whole warp runs the loop (every wait
    // warp-uniform) and one elected lane issues, so that the MMA operands stay
    // in uniform registers
    int s = 0, n = 0;
    uint32_t ph = 0;
    bool failed = false;
    for (int item = blockIdx.x; item < n_items && !failed; item += gridDim.x) {
      const int tile = item / ipt;
      const int ntok = min(NBOX, a.T - tile * NBOX);
      const int N = max(16, (ntok + 15) & ~15);
      const int buf = n % NBUF;
      if (n >= NBUF && !mbar_wait_warp(smem_u32(&acce_bar[buf]), ((n / NBUF) - 1) & 1, a.err, 44)) break;
      tc_fence_after();
      const uint32_t acc = tmem + (uint32_t)(buf * 2 * NBOX);
      const uint32_t idesc = idesc_bf16(128, N);
      for (int slab = 0; slab < nslab; ++slab) {
        if (!mbar_wait_warp(smem_u32(&full_bar[s]), ph, a.err, 41)) { failed = true; break; }
        tc_fence_after();
        const uint32_t st = smem_u32(smem + (size_t)s * Geo::STAGE);
        if (elect_one()) {
#pragma unroll
          for (int kk = 0; kk < 4; ++kk) {                 // K = 16 per MMA
            const uint64_t bdesc = umma_desc(st + Geo::B_OFF + 32 * kk, 16, 1024, 2);
#pragma unroll
            for (int h = 0; h < 2; ++h) {
              const uint64_t adesc = umma_desc(st + h * 16384 + 32 * kk, 16, 1024, 2);
              umma_bf16(acc + (uint32_t)(h * NBOX), adesc, bdesc, idesc, (slab > 0 || kk > 0) ? 1u : 0u);
            }
          }
          tc_commit(smem_u32(&empty_bar[s]));
        }
        __syncwarp();
        if (++s == S) { s = 0; ph ^= 1u; }
      }
      if (failed) break;
      if (elect_one()) tc_commit(smem_u32(&accf_bar[buf]));
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
    // ---------------- epilogue: warp w reads TMEM lanes 32*(w%4) .. +31
    const int quad = warp & 3;
    int n = 0;
    bool ok = true;
    for (int item = blockIdx.x; item < n_items && ok; item += gridDim.x) {
      const int tile = item / ipt, rb = item % ipt;
      const int t0 = tile * NBOX;
      const int ntok = min(NBOX, a.T - t0);
      const int buf = n % NBUF;
      ok = mbar_wait(smem_u32(&accf_bar[buf]), (n / NBUF) & 1, a.err, 43);
      ok = named_bar_and(1, 128, ok);
      tc_fence_after();
      const uint32_t acc = tmem + (uint32_t)(buf * 2 * NBOX) + ((uint32_t)(32 * quad) << 16);
      if constexpr (MODE == MODE_GATEUP) {
        const int Is = a.rows;
        const int r = rb * 128 + 32 * quad + lane;
        for (int c0 = 0; c0 < ntok; c0 += 32) {
          uint32_t g[32], u[32];
          tmem_ld32(acc + (uint32_t)c0, g);
          tmem_ld32(acc + (uint32_t)(NBOX + c0), u);
          tmem_ld_wait();
          if (!ok) continue;
          // all 32 columns without a branch (columns past the tile's tokens
          // are not stored), so that different tokens' exp / reciprocal
          // chains overlap
          uint16_t hv[32];
#pragma unroll
          for (int jj = 0; jj < 32; ++jj) hv[jj] = bf16_bits(silu_f(__uint_as_float(g[jj])) * __uint_as_float(u[jj]));
          const int nj = min(32, ntok - c0);
#pragma unroll
          for (int jj = 0; jj < 32; ++jj)
            if (jj < nj) a.h_out[(size_t)(t0 + c0 + jj) * Is + r] = hv[jj];
        }
      } else {
        const int H = a.rows;
        for (int hh = 0; hh < 2; ++hh) {
          const int r = rb * 256 + hh * 128 + 32 * quad + lane;
          for (int c0 = 0; c0 < ntok; c0 += 32) {
            uint32_t d[32];
            tmem_ld32(acc + (uint32_t)(hh * NBOX + c0), d);
            tmem_ld_wait();
            if (!ok) continue;
#pragma unroll
            for (int jj = 0; jj < 32; ++jj) {
              if (c0 + jj >= ntok) continue;
              a.s_out[(size_t)(t0 + c0 + jj) * H + r] = __uint_as_float(d[jj]);
            }
          }
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(smem_u32(&acce_bar[buf]));
      ++n;
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, Geo::TMEM_COLS);
  }
}

template <int MODE, int NBOX>
static void launch_dense_one(const DenseTcArgs &a, cudaStream_t s) {
  using Geo = DenseGeom<NBOX>;
  auto fn = dense_tc_kernel<MODE, NBOX>;
  cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)Geo::SMEM);
  launch_dependent(fn, a.grid, kDenseThreads, Geo::SMEM, s, a);
}

void launch_dense_tc(int mode, const DenseTcArgs &a, cudaStream_t s) {
  if (a.grid <= 0) return;
  if (mode == MODE_GATEUP) launch_dense_one<MODE_GATEUP, 128>(a, s);
  else launch_dense_one<MODE_DOWN, 128>(a, s);
}

// ---------------------------------------------------------------------------
// Decode-sized batches (T <= 128): the weight stream is what costs, and one
// CTA per row block would leave most SMs idle, so K is split over a
// thread-block cluster of S CTAs.  CTA ks of the cluster for row block rb
// accumulates its 128 gate + 128 up rows (or 256 down rows) over the K slabs
// [ks * nslab / S, (ks + 1) * nslab / S) for all T tokens at once (N = T
// rounded up to 16; TMA zero-fills the rows past T).  Once every CTA of the
// cluster is done with its stages, each pushes its partial accumulators into
// the shared memory of the CTA that finishes those rows (distributed shared
// memory stores, one slot per source rank, over the stage memory), and each
// CTA sums the slots of its 128 / S rows in rank order (the same order every
// run, so the result does not depend on timing).
// Roles: warp 0 TMA producer, warp 1 MMA issuer, warps 2..5 epilogue.
// ---------------------------------------------------------------------------
namespace {
template <int NP>
struct SplitGeom {
  static constexpr int STAGES = NP <= 32 ? 6 : (NP <= 64 ? 5 : 4);
  static constexpr int A_BYTES = 2 * 128 * 128;   // two 128-row x 64-element bf16 tiles
  static constexpr int B_OFF = A_BYTES;
  static constexpr int B_BYTES = NP * 128;
  static constexpr int STAGE = (A_BYTES + B_BYTES + 1023) / 1024 * 1024;
  static constexpr int COLS = 2 * NP;
  static constexpr int TMEM_COLS = COLS <= 32 ? 32 : (COLS <= 64 ? 64 : (COLS <= 128 ? 128 : 256));
  // received partial accumulators, fp32: S slots x 2 halves x ceil(128 / S) rows, at most S = 7
  static constexpr int RED_BYTES = 7 * 2 * 19 * NP * 4;
  static constexpr size_t SMEM = (size_t)(STAGES * STAGE > RED_BYTES ? STAGES * STAGE : RED_BYTES) + 1024;
  static_assert(SMEM <= 227 * 1024, "shared-memory budget");
};
}  // namespace

template <int MODE, int NP>
__global__ void __launch_bounds__(kDenseThreads, 1) dense_splitk_kernel(const __grid_constant__ DenseTcArgs a) {
  using Geo = SplitGeom<NP>;
  constexpr int SN = Geo::STAGES;
  extern __shared__ __align__(1024) uint8_t sk_smem_raw[];
  __shared__ __align__(8) uint64_t full_bar[SN];
  __shared__ __align__(8) uint64_t empty_bar[SN];
  __shared__ __align__(8) uint64_t accf_bar;
  __shared__ uint32_t tmem_base_s;
  __shared__ int ok_s;

  uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(sk_smem_raw) + 1023) & ~uintptr_t(1023));
  // partials received from the cluster's ranks: [source rank][half][128 / S rows][NP],
  // over the stages once every CTA of the cluster is done with them
  float *recv = reinterpret_cast<float *>(smem);
  cg::cluster_group cluster = cg::this_cluster();
  const int S = (int)cluster.num_blocks();
  const int ks = (int)cluster.block_rank();
  const int rb = blockIdx.x / S;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int nslab = a.K / 64;
  const int s0 = ks * nslab / S, s1 = (ks + 1) * nslab / S;

  if (threadIdx.x == 0) {
    for (int s = 0; s < SN; ++s) {
      mbar_init(smem_u32(&full_bar[s]), 1);
      mbar_init(smem_u32(&empty_bar[s]), 1);
    }
    mbar_init(smem_u32(&accf_bar), 1);
    mbar_fence_init();
    ok_s = 1;
  }
  if (warp == 1) {
    tmem_alloc(smem_u32(&tmem_base_s), Geo::TMEM_COLS);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = tmem_base_s;
  wait_prior_grid();                                   // x / h come from earlier kernels

  if (warp == 0) {
    // producer: the whole warp runs the loop (warp-uniform waits) and one
    // elected lane issues the copies
    {
      int s = 0, issued = 0;
      uint32_t ph = 0;
      bool failed = false;
      for (int slab = s0; slab < s1; ++slab) {
        if (issued >= SN && !mbar_wait_warp(smem_u32(&empty_bar[s]), ph ^ 1u, a.err, 46)) { failed = true; break; }
        const uint32_t bar = smem_u32(&full_bar[s]);
        const uint32_t st = smem_u32(smem + (size_t)s * Geo::STAGE);
        if (elect_one()) {
          mbar_arrive_expect_tx(bar, (uint32_t)(Geo::A_BYTES + Geo::B_BYTES));
          if constexpr (MODE == MODE_GATEUP) {
            tma_load_2d(st, &a.wmap[0], bar, slab * 64, rb * 128);
            tma_load_2d(st + 16384, &a.wmap[1], bar, slab * 64, rb * 128);
          } else {
            tma_load_2d(st, &a.wmap[0], bar, slab * 64, rb * 256);
            tma_load_2d(st + 16384, &a.wmap[0], bar, slab * 64, rb * 256 + 128);
          }
          tma_load_2d(st + Geo::B_OFF, &a.xmap, bar, slab * 64, 0);
        }
        __syncwarp();
        ++issued;
        if (++s == SN) { s = 0; ph ^= 1u; }
      }
      {
        // the last copies issued have landed before the CTA exits: at once on
        // a normal run (their consumers waited for them), and also when a
        // consumer gave up waiting
        int s2 = 0;
        uint32_t ph2 = 0;
        for (int i = 0; i < issued; ++i) {
          if (i >= issued - SN) mbar_drain(smem_u32(&full_bar[s2]), ph2);
          if (++s2 == SN) { s2 = 0; ph2 ^= 1u; }
        }
      }
    }
  } else if (warp == 1) {
    // MMA issuer: the whole warp runs the loop (every wait warp-uniform) and
    // one elected lane issues
    int s = 0;
    uint32_t ph = 0;
    bool failed = false;
    const uint32_t idesc = idesc_bf16(128, NP);
    for (int slab = s0; slab < s1; ++slab) {
      if (!mbar_wait_warp(smem_u32(&full_bar[s]), ph, a.err, 47)) { failed = true; break; }
      tc_fence_after();
      const uint32_t st = smem_u32(smem + (size_t)s * Geo::STAGE);
      if (elect_one()) {
#pragma unroll
        for (int kk = 0; kk < 4; ++kk) {
          const uint64_t bdesc = umma_desc(st + Geo::B_OFF + 32 * kk, 16, 1024, 2);
#pragma unroll
          for (int h = 0; h < 2; ++h) {
            const uint64_t adesc = umma_desc(st + h * 16384 + 32 * kk, 16, 1024, 2);
            umma_bf16(tmem + (uint32_t)(h * NP), adesc, bdesc, idesc, (slab > s0 || kk > 0) ? 1u : 0u);
          }
        }
        tc_commit(smem_u32(&empty_bar[s]));
      }
      __syncwarp();
      if (++s == SN) { s = 0; ph ^= 1u; }
    }
    // completes once every MMA above has (or at once, with none issued); the
    // warp also waits for it, so that no MMA is still running when the
    // cluster's final barrier lets the CTA free TMEM and leave
    __syncwarp();
    if (elect_one()) tc_commit(smem_u32(&accf_bar));
    __syncwarp();
    mbar_drain(smem_u32(&accf_bar), 0);
    if (failed && lane == 0) ok_s = 0;
  }
  bool ok = true;
  if (warp >= 2) {
    ok = mbar_wait(smem_u32(&accf_bar), 0, a.err, 48);
    if (!ok) ok_s = 0;
  }
  tc_fence_before();
  cluster.sync();                                      // every rank is done with its stage memory
  // rank q finishes rows [q * 128 / S, (q + 1) * 128 / S) of both halves
  const int rmax = (128 + S - 1) / S;                  // rows of the largest range (receive slot size)
  const int r0 = ks * 128 / S, r1 = (ks + 1) * 128 / S;
  if (warp >= 2) {
    // push this rank's partials (rows 32*quad + lane) into the receive slot
    // [ks] of the rank that finishes them
    tc_fence_after();
    const int quad = warp & 3;
    const int row = 32 * quad + lane;
    const int owner = ((row + 1) * S + 127) / 128 - 1;   // the q whose range holds row
    const int rl = row - owner * 128 / S;
    float *dst = cluster.map_shared_rank(recv, owner);
#pragma unroll
    for (int h = 0; h < 2; ++h) {
#pragma unroll
      for (int c0 = 0; c0 < NP; c0 += 16) {
        uint32_t v[16];
        tmem_ld16(tmem + (uint32_t)(h * NP + c0) + ((uint32_t)(32 * quad) << 16), v);
        tmem_ld_wait();
        float4 *d4 = reinterpret_cast<float4 *>(dst + (((size_t)ks * 2 + h) * rmax + rl) * NP + c0);
#pragma unroll
        for (int j = 0; j < 4; ++j)
          d4[j] = ok ? make_float4(__uint_as_float(v[4 * j]), __uint_as_float(v[4 * j + 1]),
                                   __uint_as_float(v[4 * j + 2]), __uint_as_float(v[4 * j + 3]))
                     : make_float4(0.0f, 0.0f, 0.0f, 0.0f);
      }
    }
  }
  cluster.sync();                                      // every partial is in its owner's shared memory
  // this rank finishes rows [ks * 128 / S, (ks + 1) * 128 / S) of both halves,
  // summing the slots in rank order (local shared memory only)
  for (int i = threadIdx.x; i < (r1 - r0) * NP; i += blockDim.x) {
    const int rl = i / NP, c = i % NP;
    const int r = r0 + rl;
    float v0 = 0.0f, v1 = 0.0f;
    for (int q = 0; q < S; ++q) {
      v0 += recv[(((size_t)q * 2 + 0) * rmax + rl) * NP + c];
      v1 += recv[(((size_t)q * 2 + 1) * rmax + rl) * NP + c];
    }
    if (c >= a.T) continue;
    if constexpr (MODE == MODE_GATEUP) {
      a.h_out[(size_t)c * a.rows + rb * 128 + r] = bf16_bits(silu_f(v0) * v1);
    } else {
      a.s_out[(size_t)c * a.rows + rb * 256 + r] = v0;
      a.s_out[(size_t)c * a.rows + rb * 256 + 128 + r] = v1;
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, Geo::TMEM_COLS);
  }
}

// Clusters of S CTAs of this kernel that the device runs at once (0 if the
// query fails); cached per kernel and S.
template <int MODE, int NP>
static int splitk_max_clusters(int S) {
  static int cache[9] = {-1, -1, -1, -1, -1, -1, -1, -1, -1};   // by S = 1..8
  if (cache[S] >= 0) return cache[S];
  using Geo = SplitGeom<NP>;
  auto fn = dense_splitk_kernel<MODE, NP>;
  cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)Geo::SMEM);
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((unsigned)S);
  cfg.blockDim = dim3(kDenseThreads);
  cfg.dynamicSmemBytes = Geo::SMEM;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = (unsigned)S;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  int n = 0;
  if (cudaOccupancyMaxActiveClusters(&n, fn, &cfg) != cudaSuccess) {
    cudaGetLastError();
    n = 0;
  }
  cache[S] = n;
  return n;
}

// Cluster size for n_rowblocks row blocks: the largest S in 8..2 that leaves
// each CTA at least 4 K slabs and lets all n_rowblocks clusters run at once
// (a cluster left for a second round would double the pass), else 1.
template <int MODE, int NP>
static int splitk_ways(int n_rowblocks, int K) {
  for (int S = 8; S > 1; --S)
    if ((K / 64) >= 4 * S && splitk_max_clusters<MODE, NP>(S) >= n_rowblocks) return S;
  return 1;
}

template <int MODE, int NP>
static void launch_splitk_one(const DenseTcArgs &a, cudaStream_t s) {
  using Geo = SplitGeom<NP>;
  auto fn = dense_splitk_kernel<MODE, NP>;
  const int S = splitk_ways<MODE, NP>(a.n_rowblocks, a.K);
  cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)Geo::SMEM);
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((unsigned)(a.n_rowblocks * S));
  cfg.blockDim = dim3(kDenseThreads);
  cfg.dynamicSmemBytes = Geo::SMEM;
  cfg.stream = s;
  cudaLaunchAttribute attr[2];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = (unsigned)S;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[1].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 2;
  cudaLaunchKernelEx(&cfg, fn, a);
}

void launch_dense_splitk(int mode, const DenseTcArgs &a, cudaStream_t s) {
  const int np = dense_splitk_rows(a.T);
#define MOE_SPLITK(NP)                                              \
  if (mode == MODE_GATEUP) launch_splitk_one<MODE_GATEUP, NP>(a, s); \
  else launch_splitk_one<MODE_DOWN, NP>(a, s);
  if (np == 16) { MOE_SPLITK(16) }
  else if (np == 32) { MOE_SPLITK(32) }
  else if (np == 64) { MOE_SPLITK(64) }
  else { MOE_SPLITK(128) }
#undef MOE_SPLITK
}

}  // namespace moe
