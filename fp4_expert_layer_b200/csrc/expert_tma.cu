// expert_tma.cu -- routed NVFP4 expert FFN kernels fed by TMA, for decode-sized batches.
//
// Weights are the mma.sync A operand: E2M1 pairs are decoded to f16x2 in
// registers by the hardware conversion and multiplied by their group's E4M3
// scale in f16 (an E2M1 value times an E4M3 value is exact in f16); the
// per-tensor fp32 scale is applied after the K loop.  The tokens of one
// expert are the B operand, as f16 rows with one power-of-two multiplier per
// 128-element chunk, and the tensor core accumulates each chunk in fp32.
// The weight stream is decoupled from registers: one producer warp issues
// TMA tile loads of the code bytes (64 bytes x 128 or 256 rows per 128-element
// K chunk) and bulk copies of the matching 512-byte scale-factor blocks into a
// 4-stage shared-memory ring guarded by mbarriers; eight consumer warps decode
// from shared memory.  The weights are read from HBM exactly once per CTA and
// kept in flight by the copy engine, so the kernel is bound by HBM bandwidth
// rather than by per-thread load latency ("ro99/strata": a weight-stationary
// matmul is bound by reading the weights).
//
// Every mbarrier wait is bounded (kWaitLimit polls); on expiry the thread
// records an error code in a device-visible word and carries on without the
// data, so the kernel always terminates and the host reports the failure.
#include <cooperative_groups.h>

#include "checks.cuh"
#include "device_utils.cuh"
#include "moe_internal.h"
#include "tcgen05.cuh"
#include "tma.cuh"

namespace cg = cooperative_groups;

namespace moe {

namespace {

constexpr int kStages = 4;
constexpr int kConsumers = 8;                       // consumer warps
constexpr int kThreads = (kConsumers + 1) * 32;     // + producer warp
constexpr int kABytes = 16384;                      // code bytes per stage (256 rows x 64 B)

// Scale bytes per stage: two 128-row groups x two 512-byte E4M3 blocks (a
// 128-element K chunk holds 8 NVFP4 groups of 16).
struct StageGeom {
  static constexpr int kSfPerGroup = 1024;
  static constexpr int kSfBytes = 2 * kSfPerGroup;
  static constexpr int kStageBytes = kABytes + kSfBytes;
};

template <int I>
__device__ __forceinline__ uint32_t comp(const uint4 &v) {
  if constexpr (I == 0) return v.x;
  else if constexpr (I == 1) return v.y;
  else if constexpr (I == 2) return v.z;
  else return v.w;
}

}  // namespace

template <int MODE, int NT>
__global__ void __launch_bounds__(kThreads, NT == 1 ? 2 : 1) expert_tma_kernel(const __grid_constant__ TmaExpertArgs a) {
  using Geo = StageGeom;
  constexpr int RPW = (MODE == MODE_GATEUP) ? 16 : 32;
  constexpr int RPC = RPW * kConsumers;                     // 128 (gate/up) or 256 (down) rows
  extern __shared__ __align__(1024) uint8_t smem[];
  __shared__ __align__(8) uint64_t full_bar[kStages];
  __shared__ __align__(8) uint64_t empty_bar[kStages];
  __shared__ float amax_s[kConsumers][8 * NT];
  __shared__ int cexp_s[8 * NT];
  __shared__ int last_tok[8 * NT];

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int g = lane >> 2, q = lane & 3;
  const int CS = a.k_split;
  int rank = 0;
  if (CS > 1) rank = (int)cg::this_cluster().block_rank();
  const int cid = blockIdx.x / CS;
  const int rb = cid % a.n_rowblocks;
  const int tile = cid / a.n_rowblocks;
  const int K = a.K;
  const int nck = K / kChunk;

  // ---- task (uniform over the CTA and its cluster)
  if (tile >= *a.n_tiles) return;
  const TileInfo ti = a.tiles[tile];
  const int loc = load_loc(a.loc, ti.expert, a.db);
  if (loc == kLocAbsent) return;
  const int prow0 = ti.prow0, nrows = ti.nrows;
  const bool in_slot = loc >= 0;
  const int bidx = in_slot ? loc : (-2 - loc);
  const uint8_t *blob = (in_slot ? a.slots : a.staging) + (size_t)bidx * a.blob_bytes;
  const CUtensorMap *maps = in_slot ? a.maps.slot : a.maps.stage;

  const int c_begin = rank * nck / CS, c_end = (rank + 1) * nck / CS;
  const int n_iter = c_end - c_begin;

  if (threadIdx.x == 0) {
    for (int s = 0; s < kStages; ++s) {
      mbar_init(smem_u32(&full_bar[s]), 1);
      mbar_init(smem_u32(&empty_bar[s]), kConsumers);
    }
    mbar_fence_init();
  }
  __syncthreads();

  float acc[2][NT][4];
#pragma unroll
  for (int j = 0; j < 2; ++j)
#pragma unroll
    for (int nt = 0; nt < NT; ++nt)
#pragma unroll
      for (int x = 0; x < 4; ++x) acc[j][nt][x] = 0.0f;
  float rowf[2][2] = {{1.f, 1.f}, {1.f, 1.f}};
  int mrow[2][2] = {{0, 0}, {0, 0}};        // matrix row of (m-tile j, half i)

  if (warp == kConsumers) {
    // ================= producer: the whole warp runs the loop (warp-uniform
    // waits) and one elected lane issues the copies
    {
      const int nsf = K / 16;
      int issued = 0;
      for (int it = 0; it < n_iter; ++it) {
        const int s = it % kStages;
        if (it >= kStages && !mbar_wait_warp(smem_u32(&empty_bar[s]), ((it / kStages) - 1) & 1, a.err, 2)) break;
        issued = it + 1;
        const int c = c_begin + it;
        const uint32_t bar = smem_u32(&full_bar[s]);
        const uint32_t dst = smem_u32(smem + (size_t)s * Geo::kStageBytes);
        if (elect_one()) {
          mbar_arrive_expect_tx(bar, Geo::kStageBytes);
          // scale columns covered by this chunk: 8 (two 512-byte blocks)
          const int col0 = 8 * c;
          if constexpr (MODE == MODE_GATEUP) {
            tma_load_3d(dst, &maps[0], bar, c * 64, rb * 128, bidx);
            tma_load_3d(dst + 8192, &maps[1], bar, c * 64, rb * 128, bidx);
            for (int j = 0; j < 2; ++j)
              bulk_load(dst + kABytes + j * Geo::kSfPerGroup, blob + a.L.scales[j] + sf_offset(nsf, rb * 128, col0),
                        Geo::kSfPerGroup, bar);
          } else {
            tma_load_3d(dst, &maps[2], bar, c * 64, rb * 256, bidx);
            for (int j = 0; j < 2; ++j)
              bulk_load(dst + kABytes + j * Geo::kSfPerGroup,
                        blob + a.L.scales[2] + sf_offset(nsf, rb * 256 + 128 * j, col0), Geo::kSfPerGroup, bar);
          }
        }
        __syncwarp();
      }
      // the last copies issued have landed before the CTA exits: at once on a
      // normal run (the consumers waited for them), and also when a wait gave up
      if (lane == 0)
        for (int i = max(0, issued - kStages); i < issued; ++i)
          mbar_drain(smem_u32(&full_bar[i % kStages]), (i / kStages) & 1);
    }
  } else {
    // ================= consumers
#pragma unroll
    for (int j = 0; j < 2; ++j)
#pragma unroll
      for (int i = 0; i < 2; ++i) {
        const int m = (MODE == MODE_GATEUP) ? j : 2;
        const int local = (MODE == MODE_GATEUP) ? (warp * 16 + g + 8 * i) : (warp * 32 + 16 * j + g + 8 * i);
        mrow[j][i] = rb * RPC + local;
        rowf[j][i] = reinterpret_cast<const float *>(blob + a.L.glob)[m];   // per-tensor fp32 scale
      }

    // B rows (token rows of n-tile nt, row g) and C columns (2q, 2q+1)
    const uint16_t *bptr[NT];
    int crow[NT][2];
#pragma unroll
    for (int nt = 0; nt < NT; ++nt) {
      const int lb = nt * 8 + g;
      int arow = -1;
      if (lb < nrows)
        arow = (MODE == MODE_GATEUP)
                   ? checked_index(a.prow_token[prow0 + lb], 0, a.db.n_tokens, 0, a.db.err, kChkToken)
                   : prow0 + lb;
      bptr[nt] = (arow >= 0) ? a.act + (size_t)arow * K + q * 32 : nullptr;
#pragma unroll
      for (int cb = 0; cb < 2; ++cb) {
        const int lc = nt * 8 + 2 * q + cb;
        int r = -1;
        if (lc < nrows)
          r = (MODE == MODE_GATEUP)
                  ? checked_index(a.prow_token[prow0 + lc], 0, a.db.n_tokens, 0, a.db.err, kChkToken)
                  : prow0 + lc;
        crow[nt][cb] = r;
      }
    }

    // smem byte offsets of this thread's four 16-byte code reads and scale bytes
    uint32_t a_off[2][2], sf_off[2][2];
#pragma unroll
    for (int j = 0; j < 2; ++j)
#pragma unroll
      for (int i = 0; i < 2; ++i) {
        const int local = (MODE == MODE_GATEUP) ? (warp * 16 + g + 8 * i) : (warp * 32 + 16 * j + g + 8 * i);
        const int rowbuf = (MODE == MODE_GATEUP) ? (j * 128 + local) : local;     // row in the 256-row stage tile
        a_off[j][i] = rowbuf * 64 + q * 16;
        const int grp = (MODE == MODE_GATEUP) ? j : (local >> 7);                 // 128-row scale group
        const int rr = local & 127;
        const uint32_t base = grp * Geo::kSfPerGroup + 16 * (rr & 31) + 4 * (rr >> 5);
        sf_off[j][i] = kABytes + base + (q >> 1) * 512 + 2 * (q & 1);
      }

    // B operand of chunk c: 32 sixteen-bit values of token row g, physical 32q..32q+31.
    // Prefetched one chunk ahead when registers allow (NT <= 2).
    constexpr bool kPrefetchB = NT <= 2;
    uint4 bnext[kPrefetchB ? NT : 1][4];
    if constexpr (kPrefetchB) {
      if (n_iter > 0) {
#pragma unroll
        for (int nt = 0; nt < NT; ++nt)
#pragma unroll
          for (int u = 0; u < 4; ++u)
            bnext[nt][u] = bptr[nt] ? ldg_v4(bptr[nt] + (size_t)c_begin * kChunk + u * 8) : make_uint4(0, 0, 0, 0);
      }
    }

    for (int it = 0; it < n_iter; ++it) {
      const int s = it % kStages;
      const int c = c_begin + it;
      uint4 bv[NT][4];
      if constexpr (kPrefetchB) {
#pragma unroll
        for (int nt = 0; nt < NT; ++nt)
#pragma unroll
          for (int u = 0; u < 4; ++u) bv[nt][u] = bnext[nt][u];
        if (it + 1 < n_iter) {
#pragma unroll
          for (int nt = 0; nt < NT; ++nt)
#pragma unroll
            for (int u = 0; u < 4; ++u)
              bnext[nt][u] = bptr[nt] ? ldg_v4(bptr[nt] + (size_t)(c + 1) * kChunk + u * 8) : make_uint4(0, 0, 0, 0);
        }
      } else {
#pragma unroll
        for (int nt = 0; nt < NT; ++nt)
#pragma unroll
          for (int u = 0; u < 4; ++u)
            bv[nt][u] = bptr[nt] ? ldg_v4(bptr[nt] + (size_t)c * kChunk + u * 8) : make_uint4(0, 0, 0, 0);
      }

      mbar_wait(smem_u32(&full_bar[s]), (it / kStages) & 1, a.err, 1);
      const uint32_t st = smem_u32(smem + (size_t)s * Geo::kStageBytes);
      uint4 wv[2][2];
      uint32_t mul[2][2][2];
#pragma unroll
      for (int j = 0; j < 2; ++j)
#pragma unroll
        for (int i = 0; i < 2; ++i) {
          wv[j][i] = lds128(st + a_off[j][i]);
          const uint16_t s2 = *reinterpret_cast<const uint16_t *>(smem + (size_t)s * Geo::kStageBytes + sf_off[j][i]);
          const uint32_t h2 = e4m3x2_to_f16x2(s2);
          mul[j][i][0] = dup_lo16(h2);
          mul[j][i][1] = dup_hi16(h2);
        }
      __syncwarp();
      if (lane == 0) mbar_arrive(smem_u32(&empty_bar[s]));

      float tmp[2][NT][4];
#pragma unroll
      for (int j = 0; j < 2; ++j)
#pragma unroll
        for (int nt = 0; nt < NT; ++nt)
#pragma unroll
          for (int x = 0; x < 4; ++x) tmp[j][nt][x] = 0.0f;

#define MOE_TMA_WORD(W)                                                                 \
  {                                                                                     \
    uint32_t f[2][2][4];                                                                \
    _Pragma("unroll") for (int j = 0; j < 2; ++j) {                                     \
      e2m1x8_to_f16x2(comp<W>(wv[j][0]), f[j][0]);                                      \
      e2m1x8_to_f16x2(comp<W>(wv[j][1]), f[j][1]);                                      \
    }                                                                                   \
    _Pragma("unroll") for (int sub = 0; sub < 2; ++sub) {                               \
      constexpr int ms = (W >= 2) ? 1 : 0;                                              \
      uint32_t A[2][4];                                                                 \
      _Pragma("unroll") for (int j = 0; j < 2; ++j) {                                   \
        A[j][0] = hmul2_u32(f[j][0][2 * sub], mul[j][0][ms]);                           \
        A[j][1] = hmul2_u32(f[j][1][2 * sub], mul[j][1][ms]);                           \
        A[j][2] = hmul2_u32(f[j][0][2 * sub + 1], mul[j][0][ms]);                       \
        A[j][3] = hmul2_u32(f[j][1][2 * sub + 1], mul[j][1][ms]);                       \
      }                                                                                 \
      _Pragma("unroll") for (int nt = 0; nt < NT; ++nt) {                               \
        const uint4 &bq = bv[nt][W];                                                    \
        const uint32_t b0 = sub ? bq.z : bq.x;                                          \
        const uint32_t b1 = sub ? bq.w : bq.y;                                          \
        mma_f16(tmp[0][nt], A[0], b0, b1, tmp[0][nt]);                                  \
        mma_f16(tmp[1][nt], A[1], b0, b1, tmp[1][nt]);                                  \
      }                                                                                 \
    }                                                                                   \
  }
      MOE_TMA_WORD(0)
      MOE_TMA_WORD(1)
      MOE_TMA_WORD(2)
      MOE_TMA_WORD(3)
#undef MOE_TMA_WORD

#pragma unroll
      for (int nt = 0; nt < NT; ++nt) {
        const float m0 = crow[nt][0] >= 0 ? a.act_scale[(size_t)crow[nt][0] * nck + c] : 0.0f;
        const float m1 = crow[nt][1] >= 0 ? a.act_scale[(size_t)crow[nt][1] * nck + c] : 0.0f;
#pragma unroll
        for (int j = 0; j < 2; ++j) {
          acc[j][nt][0] = fmaf(tmp[j][nt][0], m0, acc[j][nt][0]);
          acc[j][nt][1] = fmaf(tmp[j][nt][1], m1, acc[j][nt][1]);
          acc[j][nt][2] = fmaf(tmp[j][nt][2], m0, acc[j][nt][2]);
          acc[j][nt][3] = fmaf(tmp[j][nt][3], m1, acc[j][nt][3]);
        }
      }
    }
  }

  // ---- K split across the cluster: rank 0 sums partials in rank order.  Every
  // thread (producer warp included) takes part in both cluster barriers.
  float *red = reinterpret_cast<float *>(smem + (size_t)kStages * Geo::kStageBytes);
  if (CS > 1) {
    const int ct = threadIdx.x;   // consumer threads are 0..255
    if (warp < kConsumers) {
#pragma unroll
      for (int j = 0; j < 2; ++j)
#pragma unroll
        for (int nt = 0; nt < NT; ++nt)
#pragma unroll
          for (int x = 0; x < 4; ++x) red[((j * NT + nt) * 4 + x) * 256 + ct] = acc[j][nt][x];
    }
    cg::cluster_group cluster = cg::this_cluster();
    cluster.sync();
    if (rank == 0 && warp < kConsumers) {
      for (int r = 1; r < CS; ++r) {
        const float *rem = cluster.map_shared_rank(red, r);
#pragma unroll
        for (int j = 0; j < 2; ++j)
#pragma unroll
          for (int nt = 0; nt < NT; ++nt)
#pragma unroll
            for (int x = 0; x < 4; ++x) acc[j][nt][x] += rem[((j * NT + nt) * 4 + x) * 256 + ct];
      }
    }
    cluster.sync();
    if (rank != 0) return;
  }
  if (warp == kConsumers) return;

  // ---- epilogues (consumer warps only; bar 1 counts 256 threads)
  if constexpr (MODE == MODE_GATEUP) {
    float hv[NT][4];
#pragma unroll
    for (int nt = 0; nt < NT; ++nt)
#pragma unroll
      for (int x = 0; x < 4; ++x) {
        const int i = x >> 1;
        hv[nt][x] = silu_f(acc[0][nt][x] * rowf[0][i]) * (acc[1][nt][x] * rowf[1][i]);
      }
#pragma unroll
    for (int nt = 0; nt < NT; ++nt)
#pragma unroll
      for (int cb = 0; cb < 2; ++cb) {
        float m = fmaxf(fabsf(hv[nt][cb]), fabsf(hv[nt][2 + cb]));
        m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, 4));
        m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, 8));
        m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, 16));
        if (g == 0) amax_s[warp][nt * 8 + 2 * q + cb] = m;
      }
    named_bar_sync(1, kConsumers * 32);
    if (threadIdx.x < 8 * NT) {
      float m = 0.0f;
#pragma unroll
      for (int w = 0; w < kConsumers; ++w) m = fmaxf(m, amax_s[w][threadIdx.x]);
      const int ce = chunk_exponent(m);
      cexp_s[threadIdx.x] = ce;
      if ((int)threadIdx.x < nrows) a.h_scale[(size_t)(prow0 + threadIdx.x) * a.n_rowblocks + rb] = pow2f(ce);
    }
    named_bar_sync(1, kConsumers * 32);
#pragma unroll
    for (int nt = 0; nt < NT; ++nt)
#pragma unroll
      for (int x = 0; x < 4; ++x) {
        const int col = nt * 8 + 2 * q + (x & 1);
        if (col < nrows)
          a.h_out[(size_t)(prow0 + col) * a.rows + mrow[0][x >> 1]] = f16_bits(hv[nt][x] * pow2f(-cexp_s[col]));
      }
  } else {
#pragma unroll
    for (int nt = 0; nt < NT; ++nt)
#pragma unroll
      for (int x = 0; x < 4; ++x) {
        const int col = nt * 8 + 2 * q + (x & 1);
        if (col >= nrows) continue;
        const int p = checked_index(a.prow_pair[prow0 + col], 0, a.db.n_pairs, 0, a.db.err, kChkPair);
        const float gp = a.gates[p];
#pragma unroll
        for (int j = 0; j < 2; ++j)
          a.o_out[(size_t)p * a.rows + mrow[j][x >> 1]] = acc[j][nt][x] * rowf[j][x >> 1] * gp;
      }
    // ordered combine by the last arrival of each token on this row block
    // (y null: the combine kernel runs after this pass instead)
    if (a.y == nullptr) return;
    __threadfence();
    named_bar_sync(1, kConsumers * 32);
    if (threadIdx.x < 8 * NT) {
      const int col = threadIdx.x;
      int t = -1;
      if (col < nrows) {
        const int p = checked_index(a.prow_pair[prow0 + col], 0, a.db.n_pairs, 0, a.db.err, kChkPair);
        const int tok = p / a.top_k;
        if (atomicAdd(&a.comb_cnt[(size_t)tok * a.n_rowblocks + rb], 1) == a.top_k - 1) t = tok;
      }
      last_tok[col] = t;
    }
    named_bar_sync(1, kConsumers * 32);
    __threadfence();
    const int r = rb * RPC + threadIdx.x;     // one output row per consumer thread (RPC == 256)
    for (int col = 0; col < 8 * NT; ++col) {
      const int t = last_tok[col];
      if (t < 0) continue;
      const float *o = a.o_out + (size_t)t * a.top_k * a.rows + r;
      float part[kMaxTopK];
#pragma unroll
      for (int j = 0; j < kMaxTopK; ++j) part[j] = j < a.top_k ? __ldcg(o + (size_t)j * a.rows) : 0.0f;
      float v = part[0];
#pragma unroll
      for (int j = 1; j < kMaxTopK; ++j)
        if (j < a.top_k) v += part[j];
      if (a.shared) v += __ldcg(a.shared + (size_t)t * a.rows + r);
      a.y[(size_t)t * a.rows + r] = v;
      if (threadIdx.x == 0) a.comb_cnt[(size_t)t * a.n_rowblocks + rb] = 0;
    }
  }
}

template <int MODE, int NT>
static void launch_tma_one(const TmaExpertArgs &a, int grid_tiles, cudaStream_t s) {
  using Geo = StageGeom;
  const int CS = a.k_split;
  const size_t red = CS > 1 ? (size_t)2 * NT * 4 * 256 * sizeof(float) : 0;
  const size_t smem = (size_t)kStages * Geo::kStageBytes + red + 1024;
  auto fn = expert_tma_kernel<MODE, NT>;
  cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((unsigned)(grid_tiles * a.n_rowblocks * CS));
  cfg.blockDim = dim3(kThreads);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = s;
  cudaLaunchAttribute attr[1];
  cfg.numAttrs = 0;
  if (CS > 1) {
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = CS;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
  }
  cudaLaunchKernelEx(&cfg, fn, a);
}

template <int MODE>
static void launch_tma_nt(int nt, const TmaExpertArgs &a, int grid_tiles, cudaStream_t s) {
  switch (nt) {
    case 1: launch_tma_one<MODE, 1>(a, grid_tiles, s); break;
    case 2: launch_tma_one<MODE, 2>(a, grid_tiles, s); break;
    default: launch_tma_one<MODE, 4>(a, grid_tiles, s); break;
  }
}

void launch_expert_tma(int wf, int mode, int nt, const TmaExpertArgs &a, int grid_tiles, cudaStream_t s) {
  if (grid_tiles <= 0) return;
  // NVFP4 experts only: MXFP4 experts in EXACT numerics run on the tensor core
  // (expert_tc.cu)
  if (wf != WF_NV) return;
  if (mode == MODE_GATEUP) launch_tma_nt<MODE_GATEUP>(nt, a, grid_tiles, s);
  else launch_tma_nt<MODE_DOWN>(nt, a, grid_tiles, s);
}

// Expert location table for one pass: start from the resident table (or all
// absent) and overwrite the listed experts.
__global__ void loc_update_kernel(const LocUpdate u, const int *resident, int *out) {
  for (int e = threadIdx.x; e < u.E; e += blockDim.x) out[e] = u.keep_resident ? resident[e] : kLocAbsent;
  if (u.work_ctr && (int)threadIdx.x < kWorkCtrs) u.work_ctr[threadIdx.x] = 0;
  __syncthreads();
  for (int i = threadIdx.x; i < u.n; i += blockDim.x) out[u.expert[i]] = u.loc[i];
}

void launch_loc_update(const LocUpdate &u, const int *resident, int *out, cudaStream_t s) {
  loc_update_kernel<<<1, 256, 0, s>>>(u, resident, out);
}

}  // namespace moe
