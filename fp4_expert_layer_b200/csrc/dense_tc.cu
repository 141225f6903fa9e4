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
#include "device_utils.cuh"
#include "launch.cuh"
#include "moe_internal.h"
#include "tcgen05.cuh"
#include "tma.cuh"

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
    // ---------------- producer
    if (lane == 0) {
      int s = 0, issued = 0;
      uint32_t ph = 0;
      bool failed = false;
      for (int item = blockIdx.x; item < n_items && !failed; item += gridDim.x) {
        const int tile = item / ipt, rb = item % ipt;
        for (int slab = 0; slab < nslab; ++slab) {
          if (issued >= S && !mbar_wait(smem_u32(&empty_bar[s]), ph ^ 1u, a.err, 42)) { failed = true; break; }
          const uint32_t bar = smem_u32(&full_bar[s]);
          const uint32_t st = smem_u32(smem + (size_t)s * Geo::STAGE);
          mbar_arrive_expect_tx(bar, (uint32_t)(Geo::A_BYTES + Geo::B_BYTES));
          if constexpr (MODE == MODE_GATEUP) {
            tma_load_2d(st, &a.wmap[0], bar, slab * 64, rb * 128);
            tma_load_2d(st + 16384, &a.wmap[1], bar, slab * 64, rb * 128);
          } else {
            tma_load_2d(st, &a.wmap[0], bar, slab * 64, rb * 256);
            tma_load_2d(st + 16384, &a.wmap[0], bar, slab * 64, rb * 256 + 128);
          }
          tma_load_2d(st + Geo::B_OFF, &a.xmap, bar, slab * 64, tile * NBOX);
          ++issued;
          if (++s == S) { s = 0; ph ^= 1u; }
        }
      }
      if (failed) {
        int s2 = 0;
        uint32_t ph2 = 0;
        for (int i = 0; i < issued; ++i) {
          if (i >= issued - S) mbar_drain(smem_u32(&full_bar[s2]), ph2);
          if (++s2 == S) { s2 = 0; ph2 ^= 1u; }
        }
      }
    }
  } else if (warp == 1) {
    // ---------------- MMA issuer
    if (lane == 0) {
      int s = 0, n = 0;
      uint32_t ph = 0;
      bool failed = false;
      for (int item = blockIdx.x; item < n_items && !failed; item += gridDim.x) {
        const int tile = item / ipt;
        const int ntok = min(NBOX, a.T - tile * NBOX);
        const int N = max(16, (ntok + 15) & ~15);
        const int buf = n % NBUF;
        if (n >= NBUF && !mbar_wait(smem_u32(&acce_bar[buf]), ((n / NBUF) - 1) & 1, a.err, 44)) break;
        tc_fence_after();
        const uint32_t acc = tmem + (uint32_t)(buf * 2 * NBOX);
        const uint32_t idesc = idesc_bf16(128, N);
        for (int slab = 0; slab < nslab; ++slab) {
          if (!mbar_wait(smem_u32(&full_bar[s]), ph, a.err, 41)) { failed = true; break; }
          tc_fence_after();
          const uint32_t st = smem_u32(smem + (size_t)s * Geo::STAGE);
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
          if (++s == S) { s = 0; ph ^= 1u; }
        }
        tc_commit(smem_u32(&accf_bar[buf]));
        ++n;
      }
    }
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
#pragma unroll
          for (int jj = 0; jj < 32; ++jj) {
            if (c0 + jj >= ntok) continue;
            const float h = silu_f(__uint_as_float(g[jj])) * __uint_as_float(u[jj]);
            a.h_out[(size_t)(t0 + c0 + jj) * Is + r] = bf16_bits(h);
          }
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

}  // namespace moe
