// expert_dq.cu -- EXACT numerics for NVFP4 experts on the tcgen05 tensor core at
// prefill-sized batches.
//
// The pages' engines decode E2M1 to BF16 in registers for mma.sync
// ("ro99/strata", description of the SM86 kernel).  On sm_100a the
// block-scaled MMA kinds cannot take an NVFP4 weight against a 16-bit
// activation: kind::mxf4nvf4 (the one that reads E4M3 block scales) wants
// FP4 on both sides, and kind::mxf8f6f4 takes only UE8M0 per-32 scales.  So
// each weight tile is decoded ONCE per token tile into TMEM as bf16 (f16 for
// the gate/up pass) and multiplied with tcgen05.mma kind::f16 (fp32 in TMEM):
//   * an E2M1 value (at most 2 significant bits) times its E4M3 block scale
//     (4 significant bits, 2^-9 .. 448) has at most 6 significant bits and lies
//     in [2^-10, 2688]: exact in f16 and in bf16;
//   * the per-tensor fp32 scale G multiplies the fp32 accumulator in the
//     epilogue;
//   * the gate/up activations are the bf16 x rows themselves (exact), the down
//     activations are h = silu(G_g a) * (G_u u) rounded to bf16.
// The decode cost of a weight tile is shared by the up to NB tokens of a tile.
//
// The decoded weight tile is the MMA's A operand in TMEM (tcgen05.st by the
// decoders, one lane per weight row), not in shared memory: a bf16 tile
// written to and read back from shared memory would cost 64 KB of
// shared-memory traffic per 64-wide K slab of 256 rows on top of the MMAs'
// own reads of the activations, more than the 128 bytes per clock shared
// memory serves; from TMEM only the activation tile (B) and the packed raw
// codes pass through shared memory.
//
// Kernel expert_dq_kernel<MODE, NB>: persistent, one CTA per SM, work items
// (tile of up to NB tokens, 256 weight rows: 128 gate + the same 128 up rows,
// or 256 down rows) taken from a counter in index order.  Roles:
//   warp 0       producer: per 64-element K slab, one TMA box of the packed
//                codes (32 bytes x 128 or 256 rows) per matrix and the
//                512-byte E4M3 scale-factor blocks by bulk copy, into a ring
//                of raw stages (whole warp, one elected lane issuing);
//   warps 1, 15  MMA issuers (whole warps, one elected lane issuing; one
//                accumulator each: gate and up, or the two 128-row halves of
//                down): M = 128, N = tokens rounded up to 16, K = 16, A from
//                TMEM, B from shared memory;
//   warps 2..5   epilogue: TMEM -> SwiGLU -> h (bf16, padded-row order), or
//                G_d * gate * acc -> O' (fp32, pair order), each warp's
//                32 x 32 chunk turned into token rows in shared memory and
//                stored 16 bytes a lane;
//   warps 6..13  decoders: raw stage -> weight rows in TMEM, in two groups
//                of four warps taking alternate slabs (warp w the rows of TMEM
//                lane quadrant w % 4 of both 128-row halves; NVFP4: hardware
//                E2M1 -> f16x2 and an f16 multiply by the scale, widened to
//                bf16 for the down pass); every warp on every slab, one row a
//                thread, was slower (all eight then wait on the same stages);
//   warp 14      activation loader: the tile's 16-bit rows of this K slab
//                (x rows gathered into the padded expert order beforehand,
//                or h) by TMA in 64-row boxes, 128-byte swizzled K-major as
//                the B descriptor reads them (whole warp, one elected lane).
// TMEM: accumulators (2 x NB columns per buffer; two buffers when NB = 64),
// then 4 A stages of 64 columns (32 per 128-row half: 64 bf16 of a row).
// Every mbarrier wait is bounded (error word, then the kernel runs out).
#include "checks.cuh"
#include "device_utils.cuh"
#include "launch.cuh"
#include "moe_internal.h"
#include "tcgen05.cuh"
#include "tma.cuh"

namespace moe {

namespace {

constexpr int kDqThreads = 512;
constexpr int kDqDecoders = 256;   // warps 6..13 (warp 14 loads the activations)
constexpr int kDqSched = 8;
// arrivals that free a hand-over slot: 2 MMA lanes, 4 epilogue warps, 8 decoder warps, the loader warp
constexpr int kDqSchedReaders = 15;
// Raw stage of one 64-element K slab of 256 weight rows, per weight format:
//   DQ_NV  NVFP4: codes 256 rows x 32 bytes, then two 512-byte E4M3 scale blocks
//          (rows 0..127, 128..255; 4 scales per row);
//   DQ_I4  INT4 group-128: codes 256 rows x 32 bytes, then two 256-byte bf16
//          scale blocks (one scale per row: the group of 128 holding the slab);
//   DQ_F8  FP8 E4M3 block-128: codes 256 rows x 64 bytes (the fp32 block
//          scales, one per 128 rows, are read from the blob by the decoders).
template <int F>
struct DqRaw;
template <>
struct DqRaw<DQ_NV> {
  static constexpr int BYTES = 256 * 32 + 2 * 512;
};
template <>
struct DqRaw<DQ_I4> {
  static constexpr int BYTES = 256 * 32 + 2 * 256;
};
template <>
struct DqRaw<DQ_F8> {
  static constexpr int BYTES = 256 * 64;
};

template <int NB, int F>
struct DqGeom {
  static constexpr int B_BYTES = NB * 128;                 // NB token rows x 64 bf16
  static constexpr int OP_STAGE = B_BYTES;                 // multiple of 1024
  static constexpr int OP_STAGES = 4;
  static constexpr int A_COLS = 64;                        // TMEM columns of one stage's A (2 halves x 32)
  static constexpr int ACC_COLS = 2 * NB;                  // gate + up (or the two down halves)
  static constexpr int NBUF = (512 - OP_STAGES * A_COLS) / ACC_COLS >= 2 ? 2 : 1;
  static constexpr int A_TMEM = NBUF * ACC_COLS;           // first A column
  static constexpr int TMEM_COLS = 512;
  static constexpr int RAW_OFF = OP_STAGES * OP_STAGE;
  static constexpr int RAW_BYTES = DqRaw<F>::BYTES;
  // raw stages in what is left of 227 KB (1 KB alignment slack, 20 KB for the
  // static part: the epilogue's transpose tiles and the hand-over slots)
  static constexpr int RAW_FIT = (227 * 1024 - 1024 - 20 * 1024 - RAW_OFF) / RAW_BYTES;
  static constexpr int RAW_STAGES = RAW_FIT < 12 ? RAW_FIT : 12;
  static constexpr size_t SMEM = (size_t)RAW_OFF + (size_t)RAW_STAGES * RAW_BYTES + 1024;
  static_assert(OP_STAGE % 1024 == 0, "operand stages must keep the 1024-byte swizzle alignment");
  static_assert(RAW_BYTES % 512 == 0, "raw stages keep 128-byte TMA destinations");
  static_assert(RAW_STAGES >= 3, "raw ring depth");
  static_assert(A_TMEM + OP_STAGES * A_COLS <= TMEM_COLS, "TMEM budget");
  static_assert(SMEM + 20 * 1024 <= 227 * 1024, "shared-memory budget");
};

// kind::f16 instruction descriptor: fp32 accumulator, A and B both f16 or
// both bf16, K-major.
__device__ __forceinline__ uint32_t idesc_16_dq(int M, int N, bool f16) {
  uint32_t d = 0;
  d |= 1u << 4;                     // C: F32
  d |= (f16 ? 0u : 1u) << 7;        // A: F16 / BF16
  d |= (f16 ? 0u : 1u) << 10;       // B: F16 / BF16
  d |= (uint32_t)(N >> 3) << 17;
  d |= (uint32_t)(M >> 4) << 24;
  return d;
}

// D (TMEM) += A (TMEM: lane = row, two bf16 per column, lower K in the low
// half) x B (shared memory, descriptor).
__device__ __forceinline__ void umma_bf16_ts(uint32_t d_tmem, uint32_t a_tmem, uint64_t bdesc, uint32_t idesc,
                                             uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, p;\n\t}" ::"r"(d_tmem),
      "r"(a_tmem), "l"(bdesc), "r"(idesc), "r"(accumulate)
      : "memory");
}


__device__ __forceinline__ TileInfo load_tile_dq(const TileInfo *p) {
  const int4 v = __ldcg(reinterpret_cast<const int4 *>(p));
  return TileInfo{v.x, v.y, v.z, v.w};
}

__device__ __forceinline__ uint32_t bf16x2_fma(uint32_t a, uint32_t b, uint32_t c) {
  uint32_t r;
  asm("fma.rn.bf16x2 %0, %1, %2, %3;" : "=r"(r) : "r"(a), "r"(b), "r"(c));
  return r;
}

// f16x2 -> bf16x2 for values exactly representable in bf16 (no rounding
// happens): the two halves widen to fp32 on the FMA pipe and one conversion
// packs them, so the decode spends two integer-pipe instructions per pair
// (this one and the E2M1 conversion) and three on the otherwise idle FMA pipe.
__device__ __forceinline__ uint32_t f16x2_to_bf16x2(uint32_t h) {
  const float lo = __half2float(__ushort_as_half((unsigned short)(h & 0xFFFFu)));
  const float hi = __half2float(__ushort_as_half((unsigned short)(h >> 16)));
  uint32_t r;
  asm("cvt.rn.bf16x2.f32 %0, %1, %2;" : "=r"(r) : "f"(hi), "f"(lo));
  return r;
}

// Eight E2M1 codes (one 32-bit word, element 2i in the low nibble of byte i)
// times one E4M3 scale (f16x2 with the scale in both halves) -> eight f16, or
// eight bf16 (F16 = false): the f16 product is exact (at most 6 significant
// bits, in [2^-10, 2688]) and so is its bf16.
template <bool F16>
__device__ __forceinline__ uint4 decode8(uint32_t w, uint32_t sc2) {
  uint32_t f[4];
  e2m1x8_to_f16x2(w, f);
  uint4 o;
  if constexpr (F16) {
    o.x = hmul2_u32(f[0], sc2);
    o.y = hmul2_u32(f[1], sc2);
    o.z = hmul2_u32(f[2], sc2);
    o.w = hmul2_u32(f[3], sc2);
  } else {
    o.x = f16x2_to_bf16x2(hmul2_u32(f[0], sc2));
    o.y = f16x2_to_bf16x2(hmul2_u32(f[1], sc2));
    o.z = f16x2_to_bf16x2(hmul2_u32(f[2], sc2));
    o.w = f16x2_to_bf16x2(hmul2_u32(f[3], sc2));
  }
  return o;
}

// Eight INT4 codes (two's complement nibbles, element 2i in the low nibble of
// byte i) times one bf16 scale (both halves of sc2) -> eight bf16, each the
// product q * s rounded to nearest even.  q + 8 (0..15) is placed in the
// mantissa of bf16 128.0 (0x4300), so that the bf16 value is 136 + q exactly;
// one fma removes the 136 (exact), the next multiplies by the scale (one
// rounding).
__device__ __forceinline__ uint4 decode8_int4(uint32_t w, uint32_t sc2) {
  const uint32_t x = w ^ 0x88888888u;                      // q + 8 per nibble
  const uint32_t one2 = 0x3F803F80u, m136 = 0xC308C308u, nzero = 0x80008000u;   // 1.0, -136.0, -0.0
  uint32_t o[4];
#pragma unroll
  for (int b = 0; b < 4; ++b) {
    const uint32_t byte = (x >> (8 * b)) & 0xFFu;
    const uint32_t bits = 0x43004300u | (byte & 0xFu) | ((byte >> 4) << 16);
    const uint32_t q2 = bf16x2_fma(bits, one2, m136);
    o[b] = bf16x2_fma(q2, sc2, nzero);
  }
  return make_uint4(o[0], o[1], o[2], o[3]);
}

// Eight E4M3 codes (two 32-bit words, element i in byte i) times an fp32
// block scale -> eight bf16: each code is exact in f16 and in fp32, the
// product is rounded to fp32 and then to bf16 (nearest even).
__device__ __forceinline__ uint4 decode8_fp8(uint32_t w0, uint32_t w1, float s) {
  const uint32_t ws[2] = {w0, w1};
  uint32_t o[4];
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const uint32_t h2 = e4m3x2_to_f16x2((uint16_t)((ws[i >> 1] >> (16 * (i & 1))) & 0xFFFFu));
    const float lo = __half2float(__ushort_as_half((unsigned short)(h2 & 0xFFFFu))) * s;
    const float hi = __half2float(__ushort_as_half((unsigned short)(h2 >> 16))) * s;
    asm("cvt.rn.bf16x2.f32 %0, %1, %2;" : "=r"(o[i]) : "f"(hi), "f"(lo));
  }
  return make_uint4(o[0], o[1], o[2], o[3]);
}

}  // namespace

template <int MODE, int NB, int F>
__global__ void __launch_bounds__(kDqThreads, 1) expert_dq_kernel(const __grid_constant__ DqArgs a) {
  using Geo = DqGeom<NB, F>;
  // NVFP4 gate/up multiplies in f16: the weights need no widening to bf16
  // (one conversion and one f16 multiply per pair of codes) and x comes as
  // f16 rows with a power-of-two scale per token (act_scale)
  constexpr bool kF16 = F == DQ_NV && MODE == MODE_GATEUP;
  constexpr int kRawBytes = Geo::RAW_BYTES;
  constexpr int SO = Geo::OP_STAGES;
  constexpr int SR = Geo::RAW_STAGES;
  constexpr int NBUF = Geo::NBUF;
  extern __shared__ __align__(1024) uint8_t dq_smem_raw[];
  __shared__ __align__(8) uint64_t raw_full[SR];    // packed codes + scales landed (TMA / bulk)
  __shared__ __align__(8) uint64_t raw_empty[SR];   // decoders done with a raw stage
  __shared__ __align__(8) uint64_t op_full[SO];     // weights of a slab decoded into a TMEM A stage
  __shared__ __align__(8) uint64_t b_full[SO];      // activation rows of the slab landed (TMA)
  __shared__ __align__(8) uint64_t op_empty[SO];    // MMAs done with an operand stage
  __shared__ __align__(8) uint64_t accf_bar[NBUF];
  __shared__ __align__(8) uint64_t acce_bar[NBUF];
  __shared__ __align__(8) uint64_t quiesce_bar;     // all MMAs of the CTA done (before TMEM is freed)
  __shared__ uint32_t tmem_base_s;
  __shared__ __align__(8) uint64_t sched_full[kDqSched];
  __shared__ __align__(8) uint64_t sched_empty[kDqSched];
  __shared__ int sched_item[kDqSched];
  __shared__ TileInfo sched_ti[kDqSched];
  __shared__ int sched_loc[kDqSched];
  __shared__ int tok_pair[NB];
  __shared__ float tok_gate[NB];
  // per epilogue warp: its 32 rows x 32 tokens of a chunk, turned from one
  // row per lane into token rows so that the stores go out 16 bytes a lane
  __shared__ __align__(16) uint32_t epi_tile[4][32 * 32];

  uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(dq_smem_raw) + 1023) & ~uintptr_t(1023));
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int K = a.K;
  const int nslab = K / 64;
  const int ipt = a.n_rowblocks;
  const int nsf = K / 16;                              // E4M3 scale columns per weight row

  if (threadIdx.x == 0) {
    for (int s = 0; s < SR; ++s) {
      mbar_init(smem_u32(&raw_full[s]), 1);
      mbar_init(smem_u32(&raw_empty[s]), kDqDecoders / 64);     // one slab group
    }
    for (int s = 0; s < SO; ++s) {
      mbar_init(smem_u32(&op_full[s]), kDqDecoders / 64);
      mbar_init(smem_u32(&op_empty[s]), 2);               // both MMA issuers
      mbar_init(smem_u32(&b_full[s]), 1);
    }
    for (int b = 0; b < NBUF; ++b) {
      mbar_init(smem_u32(&accf_bar[b]), 2);
      mbar_init(smem_u32(&acce_bar[b]), 4);
    }
    for (int q = 0; q < kDqSched; ++q) {
      mbar_init(smem_u32(&sched_full[q]), 1);
      mbar_init(smem_u32(&sched_empty[q]), kDqSchedReaders);
    }
    mbar_init(smem_u32(&quiesce_bar), 2);
    mbar_fence_init();
  }
  if (warp == 1) {
    tmem_alloc(smem_u32(&tmem_base_s), Geo::TMEM_COLS);
    tmem_relinquish();
  }
  wait_prior_grid();                                   // routing, h and locations come from earlier kernels
  const int n_items = __ldcg(a.n_tiles) * ipt;
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = tmem_base_s;

  if (warp == 0) {
    // ---------------- producer: work items and the raw weight stream.  The
    // whole warp runs the loop (warp-uniform waits, values broadcast from lane
    // 0) and one elected lane issues the copies: a copy issued from a one-lane
    // loop behind a lane test costs about twice as much.
    int r = 0, issued = 0;
    uint32_t ph = 0;
    int q = 0;
    uint32_t qph = 0;
    bool failed = false;
    for (int j = 0; !failed; ++j) {
      int item = 0;
      if (lane == 0) item = atomicAdd(a.work_ctr, 1);
      item = __shfl_sync(0xffffffffu, item, 0);
      TileInfo ti{};
      int loc = kLocAbsent;
      if (item < n_items) {
        ti = load_tile_dq(a.tiles + item / ipt);
        loc = load_loc(a.loc, ti.expert, a.db);
      }
      if (j >= kDqSched && !mbar_wait_warp(smem_u32(&sched_empty[q]), qph ^ 1u, a.err, 58)) { failed = true; break; }
      const bool done = item >= n_items;
      if (lane == 0) {
        sched_item[q] = done ? -1 : item;
        sched_ti[q] = ti;
        sched_loc[q] = loc;
        mbar_arrive(smem_u32(&sched_full[q]));
      }
      __syncwarp();
      if (++q == kDqSched) { q = 0; qph ^= 1u; }
      if (done) break;
      if (loc == kLocAbsent) continue;
      const int rb = item % ipt;
      const bool in_slot = loc >= 0;
      const int bidx = in_slot ? loc : (-2 - loc);
      const uint8_t *blob = (in_slot ? a.slots : a.staging) + (size_t)bidx * a.blob_bytes;
      const CUtensorMap *maps = in_slot ? a.maps.slot : a.maps.stage;
      for (int slab = 0; slab < nslab; ++slab) {
        if (issued >= SR && !mbar_wait_warp(smem_u32(&raw_empty[r]), ph ^ 1u, a.err, 52)) { failed = true; break; }
        const uint32_t bar = smem_u32(&raw_full[r]);
        const uint32_t st = smem_u32(smem + Geo::RAW_OFF + (size_t)r * kRawBytes);
        if (elect_one()) {
          mbar_arrive_expect_tx(bar, (uint32_t)kRawBytes);
          // codes of the slab (TMA boxes of 32 bytes = 64 nibbles, or 64
          // bytes = 64 E4M3), then the scales the decoders need
          constexpr int cw = F == DQ_F8 ? 64 : 32;              // code bytes per row per slab
          if constexpr (MODE == MODE_GATEUP) {
            tma_load_3d(st, &maps[0], bar, slab * cw, rb * 128, bidx);
            tma_load_3d(st + 128 * cw, &maps[1], bar, slab * cw, rb * 128, bidx);
          } else {
            tma_load_3d(st, &maps[2], bar, slab * cw, rb * 256, bidx);
          }
          if constexpr (F == DQ_NV) {
            const int m0 = MODE == MODE_GATEUP ? 0 : 2, m1 = MODE == MODE_GATEUP ? 1 : 2;
            const int r0 = MODE == MODE_GATEUP ? rb * 128 : rb * 256;
            const int r1 = MODE == MODE_GATEUP ? rb * 128 : rb * 256 + 128;
            bulk_load(st + 8192, blob + a.L.scales[m0] + sf_offset(nsf, r0, slab * 4), 512, bar);
            bulk_load(st + 8704, blob + a.L.scales[m1] + sf_offset(nsf, r1, slab * 4), 512, bar);
          } else if constexpr (F == DQ_I4) {
            // 256-byte blocks of 128 rows' bf16 scales per group of 128 along K
            const int m0 = MODE == MODE_GATEUP ? 0 : 2, m1 = MODE == MODE_GATEUP ? 1 : 2;
            const int b0 = MODE == MODE_GATEUP ? rb : 2 * rb, b1 = MODE == MODE_GATEUP ? rb : 2 * rb + 1;
            const int ng = K / 128;
            bulk_load(st + 8192, blob + a.L.scales[m0] + ((size_t)b0 * ng + slab / 2) * 256, 256, bar);
            bulk_load(st + 8448, blob + a.L.scales[m1] + ((size_t)b1 * ng + slab / 2) * 256, 256, bar);
          }
        }
        __syncwarp();
        ++issued;
        if (++r == SR) { r = 0; ph ^= 1u; }
      }
    }
    // the last copies issued have landed before the CTA exits: at once on a
    // normal run (their consumers waited for them), and also when a consumer
    // gave up waiting
    if (lane == 0) {
      int r2 = 0;
      uint32_t ph2 = 0;
      for (int i = 0; i < issued; ++i) {
        if (i >= issued - SR) mbar_drain(smem_u32(&raw_full[r2]), ph2);
        if (++r2 == SR) { r2 = 0; ph2 ^= 1u; }
      }
    }
  } else if (warp == 1 || warp == 15) {
    // ---------------- MMA issuers: warp 1 issues the MMAs of the first
    // accumulator (gate, or the first 128 down rows), warp 15 those of the
    // second; each K slab is 4 MMAs of K = 16 per issuer.  The whole warp runs
    // the loop (every wait warp-uniform) and one elected lane issues, so that
    // the descriptors, advanced from ones computed up front, stay in uniform
    // registers.
    const int h = warp == 1 ? 0 : 1;
    int s = 0, n = 0;
    uint32_t ph = 0;
    int q = 0;
    uint32_t qph = 0;
    const uint64_t bdesc0 = umma_desc(smem_u32(smem), 16, 1024, 2);
    while (true) {
      if (!mbar_wait_warp(smem_u32(&sched_full[q]), qph, a.err, 59)) break;
      // broadcast from lane 0: values the compiler knows to be warp-uniform
      const int item = __shfl_sync(0xffffffffu, sched_item[q], 0);
      const int nrows = __shfl_sync(0xffffffffu, sched_ti[q].nrows, 0);
      const int loc = __shfl_sync(0xffffffffu, sched_loc[q], 0);
      if (lane == 0) mbar_arrive(smem_u32(&sched_empty[q]));
      if (++q == kDqSched) { q = 0; qph ^= 1u; }
      if (item < 0) break;
      if (loc == kLocAbsent) continue;
      const int N = max(16, (nrows + 15) & ~15);
      const int buf = n % NBUF;
      if (n >= NBUF && !mbar_wait_warp(smem_u32(&acce_bar[buf]), ((n / NBUF) - 1) & 1, a.err, 54)) break;
      tc_fence_after();
      const uint32_t acc = tmem + (uint32_t)(buf * Geo::ACC_COLS + h * NB);
      const uint32_t idesc = idesc_16_dq(128, N, kF16);
      bool failed = false;
      for (int slab = 0; slab < nslab; ++slab) {
        if (!mbar_wait_warp(smem_u32(&op_full[s]), ph, a.err, 51) ||
            !mbar_wait_warp(smem_u32(&b_full[s]), ph, a.err, 50)) {
          failed = true;
          break;
        }
        tc_fence_after();
        const uint64_t bd = bdesc0 + (uint64_t)(((uint32_t)s * (uint32_t)Geo::OP_STAGE) >> 4);
        const uint32_t at = tmem + (uint32_t)(Geo::A_TMEM + s * Geo::A_COLS + h * 32);
        if (elect_one()) {
#pragma unroll
          for (int kk = 0; kk < 4; ++kk)                     // K = 16 per MMA (8 TMEM columns of A, 32 B of B)
            umma_bf16_ts(acc, at + (uint32_t)(8 * kk), bd + (uint64_t)(2 * kk), idesc, (slab > 0 || kk > 0) ? 1u : 0u);
          tc_commit(smem_u32(&op_empty[s]));                 // stage free once both issuers' MMAs finish
        }
        __syncwarp();
        if (++s == SO) { s = 0; ph ^= 1u; }
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
  } else if (warp >= 6 && warp < 14) {
    // ---------------- decoders: raw codes + scales -> weight rows in TMEM.
    // Two groups of four warps take alternate slabs (group g the slabs n of
    // the CTA's sequence with n % 2 == g), so that one group's TMEM stores
    // drain while the other decodes; a thread decodes rows rr and 128 + rr.
    const int quad = warp & 3;                               // TMEM lane quadrant of this warp
    const int grp = warp >= 10 ? 1 : 0;
    const int rr = 32 * quad + lane;                         // row within each 128-row half
    const uint32_t tlane = (uint32_t)(32 * quad) << 16;
    int r = 0, s = 0, n_slabs = 0;
    uint32_t rph = 0, sph = 0;
    int q = 0;
    uint32_t qph = 0;
    bool failed = false;
    while (!failed) {
      int okw = 1;
      if (lane == 0) okw = mbar_wait(smem_u32(&sched_full[q]), qph, a.err, 60) ? 1 : 0;
      okw = __shfl_sync(0xffffffffu, okw, 0);
      if (!okw) break;
      __syncwarp();
      const int item = sched_item[q];
      const int loc = sched_loc[q];
      __syncwarp();
      if (lane == 0) mbar_arrive(smem_u32(&sched_empty[q]));
      if (++q == kDqSched) { q = 0; qph ^= 1u; }
      if (item < 0) break;
      if (loc == kLocAbsent) continue;
      // FP8: base of each half's fp32 block scales (one per 128 K) in the blob
      const float *bsp[2] = {nullptr, nullptr};
      if constexpr (F == DQ_F8) {
        const uint8_t *blob = (loc >= 0 ? a.slots : a.staging) + (size_t)(loc >= 0 ? loc : (-2 - loc)) * a.blob_bytes;
#pragma unroll
        for (int hh = 0; hh < 2; ++hh) {
          const int m = MODE == MODE_GATEUP ? hh : 2;
          const int rbk = MODE == MODE_GATEUP ? item % ipt : 2 * (item % ipt) + hh;
          bsp[hh] = reinterpret_cast<const float *>(blob + a.L.scales[m]) + (size_t)rbk * (K / 128);
        }
      }
      for (int slab = 0; slab < nslab; ++slab) {
        if ((n_slabs & 1) == grp) {
          int ok = 1;
          if (lane == 0) {
            ok = mbar_wait(smem_u32(&raw_full[r]), rph, a.err, 53) ? 1 : 0;
            if (ok && n_slabs >= SO) ok = mbar_wait(smem_u32(&op_empty[s]), sph ^ 1u, a.err, 55) ? 1 : 0;
          }
          ok = __shfl_sync(0xffffffffu, ok, 0);
          if (!ok) { failed = true; break; }
          tc_fence_after();
          const uint8_t *raw = smem + Geo::RAW_OFF + (size_t)r * kRawBytes;
#pragma unroll
          for (int hh = 0; hh < 2; ++hh) {
            const int row = 128 * hh + rr;                   // row of the 256 in the raw stage
            uint32_t v[32];
            if constexpr (F == DQ_F8) {
              const float sblk = __ldg(bsp[hh] + slab / 2);
#pragma unroll
              for (int c4 = 0; c4 < 4; ++c4) {
                const uint4 cv = *reinterpret_cast<const uint4 *>(raw + row * 64 + c4 * 16);
                const uint4 o0 = decode8_fp8(cv.x, cv.y, sblk), o1 = decode8_fp8(cv.z, cv.w, sblk);
                v[8 * c4 + 0] = o0.x; v[8 * c4 + 1] = o0.y; v[8 * c4 + 2] = o0.z; v[8 * c4 + 3] = o0.w;
                v[8 * c4 + 4] = o1.x; v[8 * c4 + 5] = o1.y; v[8 * c4 + 6] = o1.z; v[8 * c4 + 7] = o1.w;
              }
            } else {
              const uint4 c0 = *reinterpret_cast<const uint4 *>(raw + row * 32);
              const uint4 c1 = *reinterpret_cast<const uint4 *>(raw + row * 32 + 16);
              const uint32_t w[8] = {c0.x, c0.y, c0.z, c0.w, c1.x, c1.y, c1.z, c1.w};
              if constexpr (F == DQ_NV) {
                const uint32_t sf4 =
                    *reinterpret_cast<const uint32_t *>(raw + 8192 + hh * 512 + 16 * (rr & 31) + 4 * (rr >> 5));
                const uint32_t s01 = e4m3x2_to_f16x2((uint16_t)(sf4 & 0xFFFFu));
                const uint32_t s23 = e4m3x2_to_f16x2((uint16_t)(sf4 >> 16));
                const uint32_t sc[4] = {dup_lo16(s01), dup_hi16(s01), dup_lo16(s23), dup_hi16(s23)};
#pragma unroll
                for (int c = 0; c < 8; ++c) {
                  const uint4 o = decode8<kF16>(w[c], sc[c >> 1]);
                  v[4 * c + 0] = o.x; v[4 * c + 1] = o.y; v[4 * c + 2] = o.z; v[4 * c + 3] = o.w;
                }
              } else {
                const uint32_t sb = *reinterpret_cast<const uint16_t *>(raw + 8192 + hh * 256 + rr * 2);
                const uint32_t sc2 = sb | (sb << 16);
#pragma unroll
                for (int c = 0; c < 8; ++c) {
                  const uint4 o = decode8_int4(w[c], sc2);
                  v[4 * c + 0] = o.x; v[4 * c + 1] = o.y; v[4 * c + 2] = o.z; v[4 * c + 3] = o.w;
                }
              }
            }
            tmem_st32(tmem + tlane + (uint32_t)(Geo::A_TMEM + s * Geo::A_COLS + 32 * hh), v);
          }
          tmem_st_wait();
          tc_fence_before();
          __syncwarp();
          if (lane == 0) {
            mbar_arrive(smem_u32(&raw_empty[r]));
            mbar_arrive(smem_u32(&op_full[s]));
          }
        }
        ++n_slabs;
        if (++r == SR) { r = 0; rph ^= 1u; }
        if (++s == SO) { s = 0; sph ^= 1u; }
      }
    }
  } else if (warp == 14) {
    // ---------------- activation loader: the tile's 16-bit rows of each K
    // slab (x or h in padded-row order) by TMA, 64-row boxes, into the
    // 128-byte swizzled K-major layout of the B descriptor
    int s = 0, n_slabs = 0, issued = 0;
    uint32_t sph = 0;
    int q = 0;
    uint32_t qph = 0;
    bool failed = false;
    while (!failed) {
      // the whole warp runs the loop (warp-uniform waits, values broadcast
      // from lane 0) and one elected lane issues the copies
      if (!mbar_wait_warp(smem_u32(&sched_full[q]), qph, a.err, 61)) break;
      const int item = __shfl_sync(0xffffffffu, sched_item[q], 0);
      const int prow0 = __shfl_sync(0xffffffffu, sched_ti[q].prow0, 0);
      const int loc = __shfl_sync(0xffffffffu, sched_loc[q], 0);
      if (lane == 0) mbar_arrive(smem_u32(&sched_empty[q]));
      if (++q == kDqSched) { q = 0; qph ^= 1u; }
      if (item < 0) break;
      if (loc == kLocAbsent) continue;
      for (int slab = 0; slab < nslab; ++slab) {
        if (n_slabs >= SO && !mbar_wait_warp(smem_u32(&op_empty[s]), sph ^ 1u, a.err, 56)) { failed = true; break; }
        const uint32_t bst = smem_u32(smem + (size_t)s * Geo::OP_STAGE);
        const uint32_t bar = smem_u32(&b_full[s]);
        if (elect_one()) {
          mbar_arrive_expect_tx(bar, (uint32_t)Geo::B_BYTES);
#pragma unroll
          for (int bx = 0; bx < NB / 64; ++bx) tma_load_2d(bst + 8192 * bx, &a.maps.act, bar, slab * 64, prow0 + 64 * bx);
        }
        __syncwarp();
        ++issued;
        ++n_slabs;
        if (++s == SO) { s = 0; sph ^= 1u; }
      }
    }
    // the last copies issued have landed before the CTA exits (also when a
    // wait gave up)
    if (lane == 0) {
      int s2 = 0;
      uint32_t ph2 = 0;
      for (int i = 0; i < issued; ++i) {
        if (i >= issued - SO) mbar_drain(smem_u32(&b_full[s2]), ph2);
        if (++s2 == SO) { s2 = 0; ph2 ^= 1u; }
      }
    }
  } else {
    // ---------------- epilogue: warp w reads TMEM lanes 32*(w%4) .. +31
    const int quad = warp & 3;
    int n = 0;
    bool ok = true;
    int q = 0;
    uint32_t qph = 0;
    while (ok) {
      int okw = 1;
      if (lane == 0) okw = mbar_wait(smem_u32(&sched_full[q]), qph, a.err, 62) ? 1 : 0;
      okw = __shfl_sync(0xffffffffu, okw, 0);
      __syncwarp();
      const int item = okw ? sched_item[q] : -1;
      const TileInfo ti = sched_ti[q];
      const int loc = sched_loc[q];
      __syncwarp();
      if (okw && lane == 0) mbar_arrive(smem_u32(&sched_empty[q]));
      if (++q == kDqSched) { q = 0; qph ^= 1u; }
      if (!named_bar_and(1, 128, okw != 0 && item >= 0)) break;
      if (loc == kLocAbsent) continue;
      const int rb = item % ipt;
      const int ntok = ti.nrows;
      const int buf = n % NBUF;
      const int et = threadIdx.x - 64;                       // 0..127 over warps 2..5
      const uint8_t *blob = (loc >= 0 ? a.slots : a.staging) + (size_t)(loc >= 0 ? loc : (-2 - loc)) * a.blob_bytes;
      // NVFP4: the per-tensor fp32 scales of gate, up and down; other formats carry none
      const float one3[3] = {1.0f, 1.0f, 1.0f};
      const float *gsc = F == DQ_NV ? reinterpret_cast<const float *>(blob + a.L.glob) : one3;
      // down: each token's pair and gate; f16 gate/up: each token's x scale
      int my_pair = 0;
      float my_gate = 0.0f;
      if (MODE == MODE_DOWN && et < ntok) {
        my_pair = checked_index(__ldg(a.prow_pair + ti.prow0 + et), 0, a.db.n_pairs, 0, a.db.err, kChkPair);
        my_gate = __ldg(a.gates + my_pair);
      }
      if (kF16 && et < ntok) my_gate = __ldg(a.act_scale + ti.prow0 + et);
      ok = mbar_wait(smem_u32(&accf_bar[buf]), (n / NBUF) & 1, a.err, 57);
      if ((MODE == MODE_DOWN || kF16) && et < ntok) {
        tok_pair[et] = my_pair;
        tok_gate[et] = my_gate;
      }
      ok = named_bar_and(1, 128, ok);
      tc_fence_after();
      const uint32_t acc = tmem + (uint32_t)(buf * 2 * NB) + ((uint32_t)(32 * quad) << 16);
      if constexpr (MODE == MODE_GATEUP) {
        const float gg = gsc[0], gu = gsc[1];
        const int I = a.rows;
        uint32_t *tile = epi_tile[quad];
        uint16_t *tile16 = reinterpret_cast<uint16_t *>(tile);
        const int hcol0 = rb * 128 + 32 * quad;              // first h column of this warp
        for (int c0 = 0; c0 < ntok; c0 += 32) {
          uint32_t g[32], u[32];
          tmem_ld32(acc + (uint32_t)c0, g);
          tmem_ld32(acc + (uint32_t)(NB + c0), u);
          tmem_ld_wait();
          if (!ok) continue;
          // all 32 columns without a branch (columns past the tile's tokens
          // hold values of no one and are not stored), so that the dependent
          // exp / reciprocal chains of different tokens overlap
          uint32_t hv[16];
#pragma unroll
          for (int jj = 0; jj < 32; jj += 2) {
            float hh[2];
#pragma unroll
            for (int e = 0; e < 2; ++e) {
              const float ts = kF16 ? tok_gate[c0 + jj + e] : 1.0f;   // f16 x rows: their power-of-two scale
              const float av = __uint_as_float(g[jj + e]) * (gg * ts);
              const float uv = __uint_as_float(u[jj + e]) * (gu * ts);
              hh[e] = silu_f(av) * uv;
            }
            hv[jj / 2] = (uint32_t)bf16_bits(hh[0]) | ((uint32_t)bf16_bits(hh[1]) << 16);
          }
          // token row jj of the tile holds this warp's 32 h columns (64 bytes)
#pragma unroll
          for (int jj = 0; jj < 32; ++jj) tile16[jj * 32 + lane] = (uint16_t)(hv[jj / 2] >> (16 * (jj & 1)));
          __syncwarp();
          const int nj = min(32, ntok - c0);
#pragma unroll
          for (int i = 0; i < 4; ++i) {                      // 8 token rows per pass, 4 lanes a row
            const int r = (lane >> 2) + 8 * i;
            if (r < nj)
              *reinterpret_cast<uint4 *>(a.h_out + (size_t)(ti.prow0 + c0 + r) * I + hcol0 + 8 * (lane & 3)) =
                  *reinterpret_cast<const uint4 *>(tile16 + r * 32 + 8 * (lane & 3));
          }
          __syncwarp();                                      // the tile is rewritten by the next chunk
        }
      } else {
        const float gd = gsc[2];
        const int H = a.rows;
        uint32_t *tile = epi_tile[quad];
        for (int hh = 0; hh < 2; ++hh) {
          const int orow0 = rb * 256 + hh * 128 + 32 * quad;  // first output row of this warp
          for (int c0 = 0; c0 < ntok; c0 += 32) {
            uint32_t dv[32];
            tmem_ld32(acc + (uint32_t)(hh * NB + c0), dv);
            tmem_ld_wait();
            if (!ok) continue;
            // token row jj of the tile holds this warp's 32 output values of
            // that pair (the column index is rotated by the row against bank
            // conflicts)
#pragma unroll
            for (int jj = 0; jj < 32; ++jj)
              tile[jj * 32 + ((lane + jj) & 31)] = __float_as_uint(__uint_as_float(dv[jj]) * gd * tok_gate[c0 + jj]);
            __syncwarp();
            const int nj = min(32, ntok - c0);
#pragma unroll
            for (int i = 0; i < 4; ++i) {                    // 4 pair rows per pass, 8 lanes a row
#pragma unroll
              for (int i2 = 0; i2 < 2; ++i2) {
                const int r = (lane >> 3) + 4 * (2 * i + i2);
                if (r < nj) {
                  const int c = 4 * (lane & 7);
                  float4 v;
                  v.x = __uint_as_float(tile[r * 32 + ((c + 0 + r) & 31)]);
                  v.y = __uint_as_float(tile[r * 32 + ((c + 1 + r) & 31)]);
                  v.z = __uint_as_float(tile[r * 32 + ((c + 2 + r) & 31)]);
                  v.w = __uint_as_float(tile[r * 32 + ((c + 3 + r) & 31)]);
                  *reinterpret_cast<float4 *>(a.o_out + (size_t)tok_pair[c0 + r] * H + orow0 + c) = v;
                }
              }
            }
            __syncwarp();                                    // the tile is rewritten by the next chunk
          }
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(smem_u32(&acce_bar[buf]));
      named_bar_sync(1, 128);                                // tok_pair / tok_gate are rewritten next item
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

// The gate/up activations in the padded expert order: padded row r is token
// prow_token[r]'s x row (pad rows, token -1, are left as they are: their
// columns are never stored), as bf16 (to_f16 = 0) or as f16 multiplied by a
// power of two 2^p that puts the token's largest magnitude in [2^14, 2^15)
// (every element within 2^31 of the row's maximum converts exactly: f16 keeps
// 11 significant bits, bf16 has 8; smaller ones land on the f16 subnormal
// grid, off by less than 2^-25 of the maximum), xs[r] = 2^-p.  The expert
// pass then reads each tile's rows as one contiguous box per K slab.  One warp
// per padded row, 16-byte loads and stores (H a multiple of 256).
__global__ void __launch_bounds__(256) gather_rows_kernel(const uint16_t *x, int H, const int *prow_token,
                                                          const int *n_rows, int max_rows, int to_f16,
                                                          uint16_t *xg, float *xs, DevBounds db) {
  wait_prior_grid();
  const int row = blockIdx.x * 8 + (threadIdx.x >> 5), lane = threadIdx.x & 31;
  if (row >= max_rows || row >= __ldcg(n_rows)) return;
  const int tok = checked_index(__ldcg(prow_token + row), -1, db.n_tokens, -1, db.err, kChkToken);
  if (tok < 0) return;
  const uint4 *src = reinterpret_cast<const uint4 *>(x + (size_t)tok * H);
  uint4 *dst = reinterpret_cast<uint4 *>(xg + (size_t)row * H);
  const int n8 = H / 8;
  if (!to_f16) {
    for (int i = lane; i < n8; i += 32) dst[i] = src[i];
    return;
  }
  uint32_t am = 0;                                    // largest |bf16| bit pattern (orders like the magnitude)
  for (int i = lane; i < n8; i += 32) {
    const uint4 v = src[i];
    const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
    for (int k = 0; k < 4; ++k) am = max(am, max(w[k] & 0x7FFFu, (w[k] >> 16) & 0x7FFFu));
  }
  am = __reduce_max_sync(0xffffffffu, am);
  const int e = am >= 0x80u ? (int)(am >> 7) - 127 : -127;   // floor(log2 max), bf16 exponent field
  const int p = min(127, max(-126, 14 - e));
  const float sc = __int_as_float((p + 127) << 23);
  for (int i = lane; i < n8; i += 32) {
    const uint4 v = src[i];
    const uint32_t w[4] = {v.x, v.y, v.z, v.w};
    uint32_t o[4];
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      const float lo = __uint_as_float(w[k] << 16) * sc, hi = __uint_as_float(w[k] & 0xFFFF0000u) * sc;
      asm("cvt.rn.f16x2.f32 %0, %1, %2;" : "=r"(o[k]) : "f"(hi), "f"(lo));
    }
    dst[i] = make_uint4(o[0], o[1], o[2], o[3]);
  }
  if (lane == 0) xs[row] = __int_as_float((127 - p) << 23);
}

void launch_gather_rows(const uint16_t *x, int H, const int *prow_token, const int *n_rows, int max_rows,
                        int to_f16, uint16_t *xg, float *xs, const DevBounds &db, cudaStream_t s) {
  if (max_rows <= 0) return;
  launch_dependent(gather_rows_kernel, (max_rows + 7) / 8, 256, 0, s, x, H, prow_token, n_rows, max_rows, to_f16,
                   xg, xs, db);
}

template <int MODE, int NB, int F>
static void launch_dq_one(const DqArgs &a, cudaStream_t s) {
  using Geo = DqGeom<NB, F>;
  auto fn = expert_dq_kernel<MODE, NB, F>;
  cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)Geo::SMEM);
  launch_dependent(fn, a.grid, kDqThreads, Geo::SMEM, s, a);
}

template <int F>
static void launch_dq_fmt(int mode, int nb, const DqArgs &a, cudaStream_t s) {
  if (nb <= 64) {
    if (mode == MODE_GATEUP) launch_dq_one<MODE_GATEUP, 64, F>(a, s);
    else launch_dq_one<MODE_DOWN, 64, F>(a, s);
  } else {
    if (mode == MODE_GATEUP) launch_dq_one<MODE_GATEUP, 128, F>(a, s);
    else launch_dq_one<MODE_DOWN, 128, F>(a, s);
  }
}

void launch_expert_dq(int mode, int nb, const DqArgs &a, cudaStream_t s) {
  if (a.grid <= 0) return;
  if (a.wfmt == DQ_I4) launch_dq_fmt<DQ_I4>(mode, nb, a, s);
  else if (a.wfmt == DQ_F8) launch_dq_fmt<DQ_F8>(mode, nb, a, s);
  else launch_dq_fmt<DQ_NV>(mode, nb, a, s);
}

}  // namespace moe
