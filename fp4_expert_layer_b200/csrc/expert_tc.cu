// expert_tc.cu -- EXACT numerics for MXFP4 experts on the tcgen05 tensor core.
//
// The pages' engines decode E2M1 to BF16 in registers and multiply with
// mma.sync ("ro99/strata", description of the SM86 kernel).  On sm_100a the
// tensor core can take E2M1 weights with their E8M0 block scales directly
// (tcgen05.mma kind::mxf8f6f4, block32), but only against an 8-bit (or
// narrower) second operand.  A bf16 activation v is therefore written as two
// E4M3 "pieces" with their own UE8M0 block scales,
//     v = 2^e1 * q1 + 2^e2 * q2,
// q1 = RN_E4M3(v * 2^-e1) with e1 = floor(log2(max|v| of the 32-block)) - 7,
// q2 = RN_E4M3(r * 2^-e2) for the remainder r.  A bf16 value has 8
// significant bits and E4M3 holds 4, so q1 keeps the top four bits and the
// remainder (at most four bits) is exact in q2: the split is exact for every
// block element within 13 binades of the block maximum (smaller ones are
// rounded at 2^-9 of the piece scale).  Both pieces are rows of the B operand
// (N = 2 x tokens); the epilogue adds the two columns of each token, so one
// MMA pass over the weight tile computes the exact products accumulated in
// fp32.  The weights' own scales are the A scale factors, unchanged.
//
// The same split is applied to h = silu(a) * u (fp32) in the gate/up
// epilogue: there the two pieces keep about nine significant bits, the
// precision of a bf16 h.
//
// Kernels:
//  * tc_quant_x_kernel: gathers each tile's token rows of x (expert-sorted
//    order) and writes the two E4M3 pieces and their scale-factor blocks;
//  * expert_tc_kernel<GATEUP|DOWN, NBOX>: persistent, work items (tile, 256
//    weight rows), NBOX piece rows per tile;
//    a producer warp streams 128x128 weight tiles (TMA unpacks the E2M1 codes
//    to one byte per element), the matching 128-element slab of the tile's
//    activation pieces and both scale-factor blocks into a ring of stages;
//    two warps issue the MMAs (M = 128, N = 2 x tokens, K = 32 each) into
//    their own TMEM accumulator, one elected lane each; four warps read the
//    accumulators back.  Gate/up stages alternate
//    gate and up tiles of the same K slab (two accumulators) and the epilogue
//    computes SwiGLU and the pieces of h; down scales by the gate and writes
//    O' (the ordered combine into y is a separate kernel).
//  All mbarrier waits are bounded (error word, then the kernel runs out).
#include "checks.cuh"
#include "device_utils.cuh"
#include "moe_internal.h"
#include "launch.cuh"
#include "pieces.cuh"
#include "tcgen05.cuh"
#include "tma.cuh"

namespace moe {

namespace {

// warp 0: weight TMA (one lane: one 16 KB box per stage); warp 1: TMEM
// allocation and MMA issue (first accumulator); warps 2..5: epilogue; warp 6:
// activation pieces (16-row TMA boxes) and scale factors (bulk copies); warp
// 7: MMA issue (second accumulator).  The MMA and piece-copy loops run on
// whole warps with one elected lane issuing (from a one-lane loop behind a
// lane test each issue cost about twice as much); a per-lane cp.async copy of
// the pieces cost about a thousand cycles of issue per slab at prefill sizes
constexpr int kTcThreads = 256;
constexpr int kSched = 8;         // work items handed from the producer to the other roles in flight
constexpr int kSchedReaders = 7;  // arrivals that free a hand-over slot: 2 MMA lanes, the loader warp, 4 epilogue warps

// tile descriptor read from L2 (written by another kernel)
__device__ __forceinline__ TileInfo load_tile(const TileInfo *p) {
  const int4 v = __ldcg(reinterpret_cast<const int4 *>(p));
  return TileInfo{v.x, v.y, v.z, v.w};
}


}  // namespace

// ---------------------------------------------------------------------------
// x pieces: one warp per (tile, token of the tile); lane handles 32-blocks
// lane, lane + 32, ...
// ---------------------------------------------------------------------------
__global__ void __launch_bounds__(256) tc_quant_x_kernel(const TcQuantArgs q) {
  wait_prior_grid();
  if (threadIdx.x == 0) trigger_dependents();          // the expert pass may start its weight stream
  const int gw = blockIdx.x * 8 + (threadIdx.x >> 5);
  const int tile = gw / q.tile_tokens, j = gw % q.tile_tokens;
  if (tile >= q.max_tiles || tile >= *q.n_tiles) return;
  tc_quant_x_row(q, tile, j);
}

void launch_tc_quant_x(const TcQuantArgs &q, cudaStream_t s) {
  const long warps = (long)q.max_tiles * q.tile_tokens;
  const int blocks = (int)((warps + 7) / 8);
  if (blocks > 0) launch_dependent(tc_quant_x_kernel, blocks, 256, 0, s, q);
}

// ---------------------------------------------------------------------------
// Expert pass on the tensor core, persistent.  A work item is (tile, 256
// weight rows): gate/up = 128 gate rows + the same 128 up rows (one 4-D TMA
// box), down = 256 output rows (one 3-D box); each half has its own
// accumulator.  CTAs take items from the pass's counter in index order
// (concurrent CTAs then work on neighbouring items: tiles of one expert share
// its weights in L2; a CTA that starts early takes more); the stage ring runs
// across items, and the accumulators are double-buffered
// (8-token tiles with six stages, 56-token tiles with four: 2 x 2 x 112
// accumulator columns plus 12 scale columns per stage fill the 512 TMEM
// columns) so the epilogue of one item overlaps the main loop of the next.
// ---------------------------------------------------------------------------
namespace {
template <int NBOX>
struct TcGeom {
  static constexpr int STAGES = NBOX <= 16 ? 6 : (NBOX <= 32 ? 5 : 4);
  static constexpr int A_BYTES = 2 * 128 * 128;      // two 128 x 128 tiles, E2M1 unpacked to bytes
  static constexpr int A_TX = 2 * 128 * 128 / 2;     // bytes the TMA moves for them (packed)
  static constexpr int B_OFF = A_BYTES;
  static constexpr int B_BYTES = NBOX * 128;         // NBOX piece rows x 128 E4M3
  static constexpr int SF_OFF = B_OFF + B_BYTES;     // SFA half 0, SFA half 1, SFB: 512 B each
  static constexpr int STAGE = ((SF_OFF + 3 * 512) + 1023) / 1024 * 1024;
  // accumulator buffers: two whenever they fit in TMEM beside the scale columns
  // TMEM scale columns per stage: per MMA issuer its weight half's block and
  // its own copy of the activation block (4 columns each)
  static constexpr int SF_PER_STAGE = 16;
  static constexpr int NBUF = (2 * 2 * NBOX + SF_PER_STAGE * STAGES <= 512) ? 2 : 1;
  static constexpr int SF_COL0 = NBUF * 2 * NBOX;    // TMEM: accumulators first
  static constexpr int COLS_NEEDED = SF_COL0 + SF_PER_STAGE * STAGES;
  static constexpr int TMEM_COLS = COLS_NEEDED <= 128 ? 128 : (COLS_NEEDED <= 256 ? 256 : 512);
  static_assert(COLS_NEEDED <= 512, "TMEM budget");
  static constexpr size_t SMEM = (size_t)STAGES * STAGE + 1024;
};
}  // namespace

template <int MODE, int NBOX>
__global__ void __launch_bounds__(kTcThreads, 1) expert_tc_kernel(const __grid_constant__ TcArgs a) {
  using Geo = TcGeom<NBOX>;
  constexpr int S = Geo::STAGES;
  constexpr int NBUF = Geo::NBUF;
  extern __shared__ __align__(1024) uint8_t tc_smem_raw[];
  __shared__ __align__(8) uint64_t full_bar[S];    // weights landed (TMA)
  __shared__ __align__(8) uint64_t bfull_bar[S];   // activation pieces + scale factors landed (TMA, bulk)
  __shared__ __align__(8) uint64_t empty_bar[S];
  __shared__ __align__(8) uint64_t accf_bar[NBUF];
  __shared__ __align__(8) uint64_t acce_bar[NBUF];
  __shared__ __align__(8) uint64_t quiesce_bar;   // all MMAs of the CTA done (before TMEM is freed)
  __shared__ uint32_t tmem_base_s;
  // Work items are taken from the pass's counter (atomicAdd, in index order)
  // by the producer, which loads each item's tile descriptor and expert
  // location and hands all three to the other roles through this ring (-1 =
  // no more items).  A CTA that starts early or runs faster takes more items.
  __shared__ __align__(8) uint64_t sched_full[kSched];
  __shared__ __align__(8) uint64_t sched_empty[kSched];
  __shared__ int sched_item[kSched];
  __shared__ TileInfo sched_ti[kSched];
  __shared__ int sched_loc[kSched];
  // down epilogue: pair index and gate of each token of the current item
  __shared__ int tok_pair[NBOX / 2];
  __shared__ float tok_gate[NBOX / 2];
  // per epilogue warp: one chunk of its 32 rows (16 tokens), turned from one
  // row per lane into token rows so that the stores go out 16 bytes a lane
  // (gate/up: 32 piece rows x 32 bytes; down: 16 pairs x 32 fp32)
  __shared__ __align__(16) uint32_t epi_tile[4][16 * 32];

  uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(tc_smem_raw) + 1023) & ~uintptr_t(1023));
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int K = a.K;
  const int nslab = K / 128;
  const int nsf = K / 32;
  const int ipt = a.n_rowblocks;                      // items per tile
  const int region_map = (MODE == MODE_GATEUP) ? 0 : 1;

  if (threadIdx.x == 0) {
    for (int s = 0; s < S; ++s) {
      mbar_init(smem_u32(&full_bar[s]), 1);
      mbar_init(smem_u32(&bfull_bar[s]), 1);
      mbar_init(smem_u32(&empty_bar[s]), 2);           // both MMA issuers commit
    }
    for (int b = 0; b < NBUF; ++b) {
      mbar_init(smem_u32(&accf_bar[b]), 2);
      mbar_init(smem_u32(&acce_bar[b]), 4);           // one arrival per epilogue warp
    }
    for (int q = 0; q < kSched; ++q) {
      mbar_init(smem_u32(&sched_full[q]), 1);
      mbar_init(smem_u32(&sched_empty[q]), kSchedReaders);
    }
    mbar_init(smem_u32(&quiesce_bar), 2);
    mbar_fence_init();
  }
  if (warp == 1) {
    tmem_alloc(smem_u32(&tmem_base_s), Geo::TMEM_COLS);
    tmem_relinquish();
  }
  // Everything above overlaps the previous kernel.  With `early`, the tile
  // list, the expert locations and the item counter (written by the routing
  // step, which finished before the previous kernel let this one launch) are
  // read now and the producer streams weights at once; every other role waits
  // for the previous kernel below, before it reads activations.
  if (!a.early) wait_prior_grid();
  const int n_items = __ldcg(a.n_tiles) * ipt;
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  // (a down pass with per-tile hand-over never waits for the whole gate/up
  // grid: its loaders wait for each tile's count instead)
  const bool per_tile = MODE == MODE_DOWN && a.tile_done != nullptr;
  if (a.early && warp != 0 && !per_tile) wait_prior_grid();
  // the down pass (persistent, one CTA per SM: it lands on SMs as this grid's
  // CTAs exit) may start its own weight stream now; after the down pass the
  // combine kernel is launched as usual, when this grid exits (its many
  // waiting blocks would share the SMs with this pass)
  if (MODE == MODE_GATEUP && threadIdx.x == 64) trigger_dependents();   // after this thread's wait
  const uint32_t tmem = tmem_base_s;

  if (warp == 0) {
    // ---------------- producer
    if (lane == 0) {
      int s = 0, issued = 0;
      uint32_t ph = 0;
      int q = 0;
      uint32_t qph = 0;
      bool failed = false;
      int item = atomicAdd(a.work_ctr, 1);
      TileInfo ti{};
      int loc = kLocAbsent;
      if (item < n_items) {
        ti = load_tile(a.tiles + item / ipt);
        loc = load_loc(a.loc, ti.expert, a.db);
      }
      for (int j = 0; !failed; ++j) {
        // hand item j (or the end) to the other roles
        if (j >= kSched && !mbar_wait(smem_u32(&sched_empty[q]), qph ^ 1u, a.err, 38)) { failed = true; break; }
        const bool done = item >= n_items;
        sched_item[q] = done ? -1 : item;
        sched_ti[q] = ti;
        sched_loc[q] = loc;
        mbar_arrive(smem_u32(&sched_full[q]));               // release: the slot is written
        if (++q == kSched) { q = 0; qph ^= 1u; }
        if (done) break;
        // the next item's index is fetched at this item's first slab and its
        // descriptor loaded a few slabs later, both hidden behind the stream
        int nxt = -1;
        TileInfo nti{};
        int nloc = kLocAbsent;
        bool have_next = false;
        if (loc != kLocAbsent) {
          const int rb = item % ipt;
          const bool in_slot = loc >= 0;
          const int bidx = in_slot ? loc : (-2 - loc);
          const int region = in_slot ? 0 : 1;
          const CUtensorMap *wm = &a.maps.w[region][region_map];
          const int slab_meta = min(2, nslab - 1);
          for (int slab = 0; slab < nslab; ++slab) {
            if (issued >= S && !mbar_wait(smem_u32(&empty_bar[s]), ph ^ 1u, a.err, 32)) { failed = true; break; }
            const uint32_t bar = smem_u32(&full_bar[s]);
            const uint32_t st = smem_u32(smem + (size_t)s * Geo::STAGE);
            mbar_arrive_expect_tx(bar, (uint32_t)Geo::A_TX);
            tma_load_4d(st, wm, bar, 0, 0, rb * nslab + slab, bidx);   // one contiguous 16 KB chunk
            ++issued;
            if (++s == S) { s = 0; ph ^= 1u; }
            if (slab == 0) nxt = atomicAdd(a.work_ctr, 1);
            if (slab == slab_meta) {
              if (nxt < n_items) {
                nti = load_tile(a.tiles + nxt / ipt);
                nloc = load_loc(a.loc, nti.expert, a.db);
              }
              have_next = true;
            }
          }
        }
        if (failed) break;
        if (!have_next) {
          if (nxt < 0) nxt = atomicAdd(a.work_ctr, 1);
          if (nxt < n_items) {
            nti = load_tile(a.tiles + nxt / ipt);
            nloc = load_loc(a.loc, nti.expert, a.db);
          }
        }
        item = nxt;
        ti = nti;
        loc = nloc;
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
  } else if (warp == 1 || warp == 7) {
    // ---------------- MMA issuers: warp 1 the MMAs of the first accumulator
    // (gate, or the first 128 down rows), warp 7 those of the second.  Each
    // copies the scale blocks its MMAs read (its weight half, and its own copy
    // of the activation block: a tcgen05.cp is ordered only before the MMAs of
    // the thread that issued it).  The whole warp runs the loop (every wait
    // warp-uniform) and one elected lane issues, so that the descriptors,
    // advanced from ones computed up front, stay in uniform registers.
    const int h = warp == 1 ? 0 : 1;
    int s = 0, n = 0;
    uint32_t ph = 0;
    int q = 0;
    uint32_t qph = 0;
    bool failed = false;
    const uint32_t sbase = smem_u32(smem);
    const uint64_t adesc0 = umma_desc(sbase + h * 16384, 16, 1024, 2);
    const uint64_t bdesc0 = umma_desc(sbase + Geo::B_OFF, 16, 1024, 2);
    while (!failed) {
      if (!mbar_wait_warp(smem_u32(&sched_full[q]), qph, a.err, 39)) break;
      // broadcast from lane 0: values the compiler knows to be warp-uniform
      const int item = __shfl_sync(0xffffffffu, sched_item[q], 0);
      const int nrows = __shfl_sync(0xffffffffu, sched_ti[q].nrows, 0);
      const int loc = __shfl_sync(0xffffffffu, sched_loc[q], 0);
      if (lane == 0) mbar_arrive(smem_u32(&sched_empty[q]));
      if (++q == kSched) { q = 0; qph ^= 1u; }
      if (item < 0) break;
      if (loc == kLocAbsent) continue;
      const int N = max(16, (2 * nrows + 15) & ~15);         // piece rows rounded up to 16
      const int buf = n % NBUF;
      // the epilogue must have drained this accumulator buffer
      if (n >= NBUF && !mbar_wait_warp(smem_u32(&acce_bar[buf]), ((n / NBUF) - 1) & 1, a.err, 34)) break;
      tc_fence_after();
      const uint32_t acc = tmem + (uint32_t)(buf * 2 * NBOX + h * NBOX);
      uint32_t idesc[4];
#pragma unroll
      for (int kk = 0; kk < 4; ++kk)
        idesc[kk] = idesc_f8f6f4_block(128, N, kFmtE2M1_f8f6f4, kFmtE4M3, (uint32_t)kk, (uint32_t)kk);
      for (int slab = 0; slab < nslab; ++slab) {
        if (!mbar_wait_warp(smem_u32(&full_bar[s]), ph, a.err, 31) ||
            !mbar_wait_warp(smem_u32(&bfull_bar[s]), ph, a.err, 36)) {
          failed = true;
          break;
        }
        tc_fence_after();
        const uint32_t soff = (uint32_t)s * (uint32_t)Geo::STAGE;
        const uint32_t sf = tmem + (uint32_t)(Geo::SF_COL0 + Geo::SF_PER_STAGE * s + 8 * h);
        const uint64_t ad = adesc0 + (uint64_t)(soff >> 4), bd = bdesc0 + (uint64_t)(soff >> 4);
        if (elect_one()) {
          tc_cp_sf_block(sf, sbase + soff + Geo::SF_OFF + 512 * h);       // this half's weight scales
          tc_cp_sf_block(sf + 4, sbase + soff + Geo::SF_OFF + 1024);      // the activation rows' scales
#pragma unroll
          for (int kk = 0; kk < 4; ++kk)                  // K = 32 per MMA
            umma_mxf8f6f4(acc, ad + (uint64_t)(2 * kk), bd + (uint64_t)(2 * kk), idesc[kk], sf | ((uint32_t)kk << 30),
                          (sf + 4) | ((uint32_t)kk << 30), (slab > 0 || kk > 0) ? 1u : 0u);
          tc_commit(smem_u32(&empty_bar[s]));              // stage free once both issuers' MMAs finish
        }
        __syncwarp();
        if (++s == S) { s = 0; ph ^= 1u; }
      }
      if (failed) break;
      if (elect_one()) tc_commit(smem_u32(&accf_bar[buf]));   // this item's accumulators complete
      __syncwarp();
      ++n;
    }
    // every MMA issued above has completed before the CTA frees TMEM and
    // leaves (also after a wait gave up and the loop was left early)
    __syncwarp();
    if (elect_one()) tc_commit(smem_u32(&quiesce_bar));
    __syncwarp();
    mbar_drain(smem_u32(&quiesce_bar), 0);
  } else if (warp == 6) {
    // ---------------- loader (warp 6): per K slab, the tile's
    // activation-piece rows by TMA (16-row boxes, 128-byte swizzle as the MMA
    // descriptor reads them) and the three scale-factor blocks (the weight
    // chunk's two halves, the activation rows) by bulk copy
    if (warp == 6) {
      int s = 0, issued = 0;
      uint32_t ph = 0;
      int q = 0;
      uint32_t qph = 0;
      bool failed = false;
      while (!failed) {
        int okw = 1;
        if (lane == 0) okw = mbar_wait(smem_u32(&sched_full[q]), qph, a.err, 40) ? 1 : 0;
        okw = __shfl_sync(0xffffffffu, okw, 0);
        if (!okw) break;                                     // warp-uniform
        __syncwarp();
        const int item = sched_item[q];
        const TileInfo ti = sched_ti[q];
        const int loc = sched_loc[q];
        __syncwarp();
        if (lane == 0) mbar_arrive(smem_u32(&sched_empty[q]));
        if (++q == kSched) { q = 0; qph ^= 1u; }
        if (item < 0) break;
        if (loc == kLocAbsent) continue;
        const int tile = item / ipt, rb = item % ipt;
        const uint8_t *blob = (loc >= 0 ? a.slots : a.staging) + (size_t)(loc >= 0 ? loc : (-2 - loc)) * a.blob_bytes;
        const int act_row0 = tile * kTcSlotRows;
        // scale blocks of the chunk's two halves (1 KB per chunk), and of the activation rows
        const uint8_t *sfa = blob + a.L.scales[MODE == MODE_GATEUP ? 0 : 2] + (size_t)rb * nslab * kTcSfChunk;
        const uint8_t *sfb = a.bsf + sf_offset(nsf, act_row0, 0);
        const int nbox = max(16, (2 * ti.nrows + 15) & ~15) / 16;   // 16-row boxes of piece rows read
        const uint32_t tx = (uint32_t)(nbox * 16 * 128 + kTcSfChunk + 512);
        if (per_tile) {
          // this tile's h pieces are complete once every gate/up item of it is
          int okt = 1;
          if (lane == 0) okt = flag_wait(a.tile_done + tile, a.tile_target, a.err, 42) ? 1 : 0;
          okt = __shfl_sync(0xffffffffu, okt, 0);
          if (!okt) { failed = true; break; }                // warp-uniform
          // the h pieces were written by other CTAs' ordinary stores; the TMA
          // reads them through the async proxy
          asm volatile("fence.proxy.async.global;" ::: "memory");
        }
        // the whole warp runs the slab loop (warp-uniform waits) and one
        // elected lane issues the copies
        for (int slab = 0; slab < nslab; ++slab) {
          if (issued >= S && !mbar_wait_warp(smem_u32(&empty_bar[s]), ph ^ 1u, a.err, 35)) { failed = true; break; }
          const uint32_t st = smem_u32(smem + (size_t)s * Geo::STAGE);
          const uint32_t bar = smem_u32(&bfull_bar[s]);
          if (elect_one()) {
            mbar_arrive_expect_tx(bar, tx);
            for (int b = 0; b < nbox; ++b)
              tma_load_2d(st + Geo::B_OFF + b * 2048, &a.maps.act, bar, slab * 128, act_row0 + 16 * b);
            bulk_load(st + Geo::SF_OFF, sfa + (size_t)slab * kTcSfChunk, kTcSfChunk, bar);
            bulk_load(st + Geo::SF_OFF + kTcSfChunk, sfb + (size_t)slab * 512, 512, bar);
          }
          __syncwarp();
          ++issued;
          if (++s == S) { s = 0; ph ^= 1u; }
        }
      }
      // the last copies issued have landed before the CTA exits (also when a
      // wait gave up)
      if (lane == 0) {
        int s2 = 0;
        uint32_t ph2 = 0;
        for (int i = 0; i < issued; ++i) {
          if (i >= issued - S) mbar_drain(smem_u32(&bfull_bar[s2]), ph2);
          if (++s2 == S) { s2 = 0; ph2 ^= 1u; }
        }
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
      if (lane == 0) okw = mbar_wait(smem_u32(&sched_full[q]), qph, a.err, 41) ? 1 : 0;
      okw = __shfl_sync(0xffffffffu, okw, 0);
      __syncwarp();
      const int item = okw ? sched_item[q] : -1;
      const TileInfo ti = sched_ti[q];
      const int loc = sched_loc[q];
      __syncwarp();
      if (okw && lane == 0) mbar_arrive(smem_u32(&sched_empty[q]));
      if (++q == kSched) { q = 0; qph ^= 1u; }
      // the four warps stop together (each takes every named barrier below)
      if (!named_bar_and(1, 128, okw != 0 && item >= 0)) break;
      if (loc == kLocAbsent) continue;
      const int tile = item / ipt, rb = item % ipt;
      const int ntok = ti.nrows;
      const int act_row0 = tile * kTcSlotRows;
      const int buf = n % NBUF;
      const int et = threadIdx.x - 64;                       // 0..127 over warps 2..5
      // down: load the item's pair indices and gates while its MMAs run
      int my_pair = 0;
      float my_gate = 0.0f;
      if (MODE == MODE_DOWN && et < ntok) {
        my_pair = checked_index(__ldg(a.prow_pair + ti.prow0 + et), 0, a.db.n_pairs, 0, a.db.err, kChkPair);
        my_gate = __ldg(a.gates + my_pair);
      }
      ok = mbar_wait(smem_u32(&accf_bar[buf]), (n / NBUF) & 1, a.err, 33);
      if (MODE == MODE_DOWN && et < ntok) {
        tok_pair[et] = my_pair;
        tok_gate[et] = my_gate;
      }
      ok = named_bar_and(1, 128, ok);                        // one decision for all four warps
      tc_fence_after();
      const uint32_t acc = tmem + (uint32_t)(buf * 2 * NBOX) + ((uint32_t)(32 * quad) << 16);
      if constexpr (MODE == MODE_GATEUP) {
        const int I = a.rows, nsf_h = I / 32;
        const int r = rb * 128 + 32 * quad + lane;           // h column
        for (int c0 = 0; c0 < 2 * ntok; c0 += 32) {
          uint32_t g[32], u[32];
          tmem_ld32(acc + (uint32_t)c0, g);
          tmem_ld32(acc + (uint32_t)(NBOX + c0), u);
          tmem_ld_wait();
          if (!ok) continue;
          // 16 tokens at a time: the warp reductions of different tokens are
          // independent, so their shuffles overlap (columns past the tile's
          // tokens hold no data and are never stored)
          float w[16], am[16];
#pragma unroll
          for (int jj = 0; jj < 16; ++jj) {
            const float av = __uint_as_float(g[2 * jj]) + __uint_as_float(g[2 * jj + 1]);
            const float uv = __uint_as_float(u[2 * jj]) + __uint_as_float(u[2 * jj + 1]);
            w[jj] = silu_f(av) * uv;
            am[jj] = fabsf(w[jj]);
          }
#pragma unroll
          for (int o = 16; o > 0; o >>= 1)
#pragma unroll
            for (int jj = 0; jj < 16; ++jj) am[jj] = fmaxf(am[jj], __shfl_xor_sync(0xffffffffu, am[jj], o));
          int e1[16];
          uint32_t c1[16];
#pragma unroll
          for (int jj = 0; jj < 16; ++jj) {
            e1[jj] = split_e1(am[jj]);
            const float v = w[jj] * exp2_int(-e1[jj]);
            c1[jj] = e4m3x2(v, 0.0f) & 0xFFu;
            w[jj] = v - e4m3_value(c1[jj]);                   // remainder in units of 2^e1
            am[jj] = fabsf(w[jj]);
          }
#pragma unroll
          for (int o = 16; o > 0; o >>= 1)
#pragma unroll
            for (int jj = 0; jj < 16; ++jj) am[jj] = fmaxf(am[jj], __shfl_xor_sync(0xffffffffu, am[jj], o));
          int e2r[16];
          uint32_t c2[16];
#pragma unroll
          for (int jj = 0; jj < 16; ++jj) {
            e2r[jj] = split_e2rel(am[jj], e1[jj]);
            c2[jj] = e4m3x2(w[jj] * exp2_int(-e2r[jj]), 0.0f) & 0xFFu;
          }
          // piece row 2 jj + p of the tile holds this warp's 32 columns
          uint8_t *tile8 = reinterpret_cast<uint8_t *>(epi_tile[quad]);
#pragma unroll
          for (int jj = 0; jj < 16; ++jj) {
            tile8[(2 * jj) * 32 + lane] = (uint8_t)c1[jj];
            tile8[(2 * jj + 1) * 32 + lane] = (uint8_t)c2[jj];
          }
          __syncwarp();
          const int nj = min(16, ntok - c0 / 2);             // warp-uniform
#pragma unroll
          for (int i = 0; i < 2; ++i) {                      // 16 piece rows per pass, 2 lanes a row
            const int pr = (lane >> 1) + 16 * i;
            if (pr < 2 * nj)
              *reinterpret_cast<uint4 *>(a.hq + ((size_t)act_row0 + c0 + pr) * I + (r - lane) + 16 * (lane & 1)) =
                  *reinterpret_cast<const uint4 *>(tile8 + pr * 32 + 16 * (lane & 1));
          }
          if (lane == 0) {
#pragma unroll
            for (int jj = 0; jj < 16; ++jj) {
              if (jj >= nj) break;
              const int row = act_row0 + c0 + 2 * jj;
              a.hsf[sf_offset(nsf_h, row, r / 32)] = (uint8_t)(e1[jj] + 127);
              a.hsf[sf_offset(nsf_h, row + 1, r / 32)] = (uint8_t)(e1[jj] + e2r[jj] + 127);
            }
          }
          __syncwarp();                                      // the tile is rewritten by the next chunk
        }
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(smem_u32(&acce_bar[buf]));
        if (a.tile_done) {
          __threadfence();                                   // this thread's h pieces and scales are out
          named_bar_sync(1, 128);
          if (et == 0 && ok) atomicAdd(a.tile_done + tile, 1);
        }
      } else {
        const int H = a.rows;
        for (int hh = 0; hh < 2; ++hh) {
          const int r = rb * 256 + hh * 128 + 32 * quad + lane;   // output row
          for (int c0 = 0; c0 < 2 * ntok; c0 += 32) {
            uint32_t d[32];
            tmem_ld32(acc + (uint32_t)(hh * NBOX + c0), d);
            tmem_ld_wait();
            if (!ok) continue;
            // pair row jj of the tile holds this warp's 32 output values of
            // that pair (column index rotated by the row against bank conflicts)
            uint32_t *tile = epi_tile[quad];
#pragma unroll
            for (int jj = 0; jj < 16; ++jj)
              tile[jj * 32 + ((lane + jj) & 31)] = __float_as_uint(
                  (__uint_as_float(d[2 * jj]) + __uint_as_float(d[2 * jj + 1])) * tok_gate[c0 / 2 + jj]);
            __syncwarp();
            const int nj = min(16, ntok - c0 / 2);
#pragma unroll
            for (int i = 0; i < 4; ++i) {                    // 4 pair rows per pass, 8 lanes a row
              const int pr = (lane >> 3) + 4 * i;
              if (pr < nj) {
                const int c = 4 * (lane & 7);
                float4 v;
                v.x = __uint_as_float(tile[pr * 32 + ((c + 0 + pr) & 31)]);
                v.y = __uint_as_float(tile[pr * 32 + ((c + 1 + pr) & 31)]);
                v.z = __uint_as_float(tile[pr * 32 + ((c + 2 + pr) & 31)]);
                v.w = __uint_as_float(tile[pr * 32 + ((c + 3 + pr) & 31)]);
                *reinterpret_cast<float4 *>(a.o_out + (size_t)tok_pair[c0 / 2 + pr] * H + (r - lane) + c) = v;
              }
            }
            __syncwarp();                                    // the tile is rewritten by the next chunk
          }
        }
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(smem_u32(&acce_bar[buf]));
        named_bar_sync(1, 128);                              // tok_pair / tok_gate are rewritten next item
      }
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
static void launch_tc_one(const TcArgs &a, cudaStream_t s) {
  using Geo = TcGeom<NBOX>;
  auto fn = expert_tc_kernel<MODE, NBOX>;
  cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)Geo::SMEM);
  launch_dependent(fn, a.grid, kTcThreads, Geo::SMEM, s, a);
}

void launch_expert_tc(int mode, int nbox, const TcArgs &a, int grid_tiles, cudaStream_t s) {
  if (grid_tiles <= 0 || a.grid <= 0) return;
  if (nbox <= 16) {
    if (mode == MODE_GATEUP) launch_tc_one<MODE_GATEUP, 16>(a, s);
    else launch_tc_one<MODE_DOWN, 16>(a, s);
  } else if (nbox <= 32) {
    if (mode == MODE_GATEUP) launch_tc_one<MODE_GATEUP, 32>(a, s);
    else launch_tc_one<MODE_DOWN, 32>(a, s);
  } else {
    if (mode == MODE_GATEUP) launch_tc_one<MODE_GATEUP, 112>(a, s);
    else launch_tc_one<MODE_DOWN, 112>(a, s);
  }
}

}  // namespace moe
