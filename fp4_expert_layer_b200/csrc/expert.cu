// expert.cu -- expert FFN kernels read straight from MXFP4 / NVFP4 bytes.
//
// Weight-stationary grouped GEMV/GEMM for decode-sized batches.  The weights
// are the mma A operand (16 rows per m16n8k16 tile), the tokens of one expert
// the B operand (8 per n-tile, NT n-tiles per CTA).  Each lane loads, per
// 128-element K chunk, 16 contiguous code bytes of a weight row (one 32-element
// group: one E8M0 scale, or two E4M3 scales) with a 128-bit load; E2M1 pairs are
// decoded to f16x2 in registers by the hardware conversion, multiplied by the
// group's scale folded into f16, and fed to the tensor core.  Only the code
// bytes cross HBM: nothing is widened in memory ("ro99/strata": the four-bit
// codes stay four bits in memory and are decoded into MMA operand registers;
// the kernel is bound by reading the weights).
//
// Numerics (EXACT mode): e2m1 * 2^(s - s_row) is exact in f16 whenever the
// row's scale spread is at most 24 binades (s_row = the row's largest E8M0
// code, applied in fp32 after the K loop); E2M1 * E4M3 is always exact in f16.
// Activations are f16 "chunk-scaled": every 128-element chunk of a row carries
// an fp32 power-of-two multiplier chosen so that its largest value lands in
// [2^14, 2^15); the tensor core accumulates each chunk in fp32 and the chunk's
// multiplier is applied to that partial sum.  Products are exact, accumulation
// is fp32.
//
// Logical-to-physical K map (the same for A and B, so the dot product is
// unchanged): in step s of a chunk, lane quad q supplies logical k {2q, 2q+1}
// from physical 32q + 4s + {0,1} and logical {2q+8, 2q+9} from 32q + 4s + {2,3}.
//
// K may be split across a cluster of CTAs; partial accumulators are summed by
// the cluster's rank-0 CTA through distributed shared memory in rank order,
// so results do not depend on timing (paged output == resident output).
#include <cooperative_groups.h>

#include "device_utils.cuh"
#include "moe_internal.h"

namespace cg = cooperative_groups;

namespace moe {

template <int I>
__device__ __forceinline__ uint32_t u4c(const uint4 &v) {
  if constexpr (I == 0) return v.x;
  else if constexpr (I == 1) return v.y;
  else if constexpr (I == 2) return v.z;
  else return v.w;
}

template <int WF, int MODE, int NT>
__global__ void __launch_bounds__(256) expert_kernel(const ExpertArgs a) {
  constexpr bool ROUTED = WF != WF_BF16;
  constexpr int RPW = (MODE == MODE_GATEUP) ? 16 : 32;     // rows per warp (per matrix)
  constexpr int RPC = RPW * kWarps;                         // rows per CTA
  extern __shared__ float red_smem[];
  __shared__ float amax_s[kWarps][8 * NT];
  __shared__ int cexp_s[8 * NT];

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

  int prow0, nrows, expert = 0;
  const uint8_t *blob = nullptr;
  if constexpr (ROUTED) {
    if (tile >= *a.n_tiles) return;
    const TileInfo ti = a.tiles[tile];
    expert = ti.expert;
    prow0 = ti.prow0;
    nrows = ti.nrows;
    blob = a.expert_ptr[expert];
    if (blob == nullptr) return;
  } else {
    prow0 = tile * a.tile_tokens;
    nrows = min(a.tile_tokens, a.T - prow0);
    if (nrows <= 0) return;
  }
  (void)expert;

  // ---- weight rows of this thread: m-tile j, half i -> row rbase[j] + g + 8i
  int mat[2], rbase[2];
  if constexpr (MODE == MODE_GATEUP) {
    mat[0] = 0; mat[1] = 1;
    rbase[0] = rbase[1] = rb * RPC + warp * RPW;
  } else {
    mat[0] = mat[1] = 2;
    rbase[0] = rb * RPC + warp * RPW;
    rbase[1] = rbase[0] + 16;
  }

  const uint8_t *wcode[2][2];     // FP4 code pointer (chunk 0, this lane's 16 bytes)
  const uint8_t *wscale[2][2];    // block-scale pointer (chunk 0)
  const uint16_t *wdense[2][2];   // bf16 weight pointer (chunk 0, this lane's 32 elements)
  int sref[2][2];
  float rowf[2][2];
#pragma unroll
  for (int j = 0; j < 2; ++j) {
#pragma unroll
    for (int i = 0; i < 2; ++i) {
      const int r = rbase[j] + g + 8 * i;
      if constexpr (ROUTED) {
        const int m = mat[j];
        wcode[j][i] = blob + a.L.codes[m] + (size_t)r * (K / 2) + q * 16;
        if constexpr (WF == WF_MX) {
          wscale[j][i] = blob + a.L.scales[m] + (size_t)r * (K / 32) + q;
          sref[j][i] = blob[a.L.sref[m] + r];
          rowf[j][i] = pow2f(sref[j][i] - 127);
        } else {
          wscale[j][i] = blob + a.L.scales[m] + (size_t)r * (K / 16) + 2 * q;
          sref[j][i] = 0;
          rowf[j][i] = reinterpret_cast<const float *>(blob + a.L.glob)[m];
        }
        wdense[j][i] = nullptr;
      } else {
        const uint16_t *base = (MODE == MODE_GATEUP && j == 1) ? a.dense_w1 : a.dense_w0;
        wdense[j][i] = base + (size_t)r * K + q * 32;
        wcode[j][i] = nullptr;
        wscale[j][i] = nullptr;
        sref[j][i] = 0;
        rowf[j][i] = 1.0f;
      }
    }
  }

  // ---- activation rows: B rows (n-tile row g) and C columns (2q, 2q+1)
  const uint16_t *bptr[NT];
  int crow[NT][2];
#pragma unroll
  for (int nt = 0; nt < NT; ++nt) {
    const int lb = nt * 8 + g;
    int arow = -1;
    if (lb < nrows) {
      if constexpr (ROUTED && MODE == MODE_GATEUP) arow = a.prow_token[prow0 + lb];
      else arow = prow0 + lb;
    }
    bptr[nt] = (arow >= 0) ? a.act + (size_t)arow * K + q * 32 : nullptr;
#pragma unroll
    for (int cb = 0; cb < 2; ++cb) {
      const int lc = nt * 8 + 2 * q + cb;
      int r = -1;
      if (lc < nrows) {
        if constexpr (ROUTED && MODE == MODE_GATEUP) r = a.prow_token[prow0 + lc];
        else r = prow0 + lc;
      }
      crow[nt][cb] = r;
    }
  }

  float acc[2][NT][4];
#pragma unroll
  for (int j = 0; j < 2; ++j)
#pragma unroll
    for (int nt = 0; nt < NT; ++nt)
#pragma unroll
      for (int x = 0; x < 4; ++x) acc[j][nt][x] = 0.0f;

  const int c_begin = rank * nck / CS, c_end = (rank + 1) * nck / CS;
  for (int c = c_begin; c < c_end; ++c) {
    // B operand: 32 sixteen-bit values of token row g (physical 32q .. 32q+31 of the chunk)
    uint4 bv[NT][4];
#pragma unroll
    for (int nt = 0; nt < NT; ++nt) {
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        bv[nt][u] = bptr[nt] ? ldg_v4(bptr[nt] + (size_t)c * kChunk + u * 8) : make_uint4(0, 0, 0, 0);
      }
    }
    if constexpr (ROUTED) {
      uint4 wv[2][2];
      uint32_t mul[2][2][2];
#pragma unroll
      for (int j = 0; j < 2; ++j) {
#pragma unroll
        for (int i = 0; i < 2; ++i) {
          wv[j][i] = ldg_nc_v4(wcode[j][i] + (size_t)c * 64);
          if constexpr (WF == WF_MX) {
            const int s = wscale[j][i][(size_t)c * 4];
            mul[j][i][0] = mul[j][i][1] = f16x2_pow2(s - sref[j][i]);
          } else {
            const uint16_t s2 = *reinterpret_cast<const uint16_t *>(wscale[j][i] + (size_t)c * 8);
            const uint32_t h2 = e4m3x2_to_f16x2(s2);
            mul[j][i][0] = dup_lo16(h2);
            mul[j][i][1] = dup_hi16(h2);
          }
        }
      }
      float tmp[2][NT][4];
#pragma unroll
      for (int j = 0; j < 2; ++j)
#pragma unroll
        for (int nt = 0; nt < NT; ++nt)
#pragma unroll
          for (int x = 0; x < 4; ++x) tmp[j][nt][x] = 0.0f;

#define MOE_WORD_STEP(W)                                                                    \
  {                                                                                         \
    uint32_t f[2][2][4];                                                                    \
    _Pragma("unroll") for (int j = 0; j < 2; ++j) {                                         \
      e2m1x8_to_f16x2(u4c<W>(wv[j][0]), f[j][0]);                                           \
      e2m1x8_to_f16x2(u4c<W>(wv[j][1]), f[j][1]);                                           \
    }                                                                                       \
    _Pragma("unroll") for (int sub = 0; sub < 2; ++sub) {                                   \
      constexpr int ms = (WF == WF_NV && W >= 2) ? 1 : 0;                                   \
      uint32_t A[2][4];                                                                     \
      _Pragma("unroll") for (int j = 0; j < 2; ++j) {                                       \
        A[j][0] = hmul2_u32(f[j][0][2 * sub], mul[j][0][ms]);                               \
        A[j][1] = hmul2_u32(f[j][1][2 * sub], mul[j][1][ms]);                               \
        A[j][2] = hmul2_u32(f[j][0][2 * sub + 1], mul[j][0][ms]);                           \
        A[j][3] = hmul2_u32(f[j][1][2 * sub + 1], mul[j][1][ms]);                           \
      }                                                                                     \
      _Pragma("unroll") for (int nt = 0; nt < NT; ++nt) {                                   \
        const uint4 &bq = bv[nt][W];                                                        \
        const uint32_t b0 = sub ? bq.z : bq.x;                                              \
        const uint32_t b1 = sub ? bq.w : bq.y;                                              \
        mma_f16(tmp[0][nt], A[0], b0, b1, tmp[0][nt]);                                      \
        mma_f16(tmp[1][nt], A[1], b0, b1, tmp[1][nt]);                                      \
      }                                                                                     \
    }                                                                                       \
  }
      MOE_WORD_STEP(0)
      MOE_WORD_STEP(1)
      MOE_WORD_STEP(2)
      MOE_WORD_STEP(3)
#undef MOE_WORD_STEP

      // chunk multipliers of the two C columns of each n-tile
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
    } else {
      // dense bf16 weights: 32 values per row per lane per chunk
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        uint4 wv[2][2];
#pragma unroll
        for (int j = 0; j < 2; ++j) {
          wv[j][0] = ldg_nc_v4(wdense[j][0] + (size_t)c * kChunk + u * 8);
          wv[j][1] = ldg_nc_v4(wdense[j][1] + (size_t)c * kChunk + u * 8);
        }
#pragma unroll
        for (int sub = 0; sub < 2; ++sub) {
          uint32_t A[2][4];
#pragma unroll
          for (int j = 0; j < 2; ++j) {
            A[j][0] = sub ? wv[j][0].z : wv[j][0].x;
            A[j][1] = sub ? wv[j][1].z : wv[j][1].x;
            A[j][2] = sub ? wv[j][0].w : wv[j][0].y;
            A[j][3] = sub ? wv[j][1].w : wv[j][1].y;
          }
#pragma unroll
          for (int nt = 0; nt < NT; ++nt) {
            const uint4 &bq = bv[nt][u];
            const uint32_t b0 = sub ? bq.z : bq.x;
            const uint32_t b1 = sub ? bq.w : bq.y;
            mma_bf16(acc[0][nt], A[0], b0, b1, acc[0][nt]);
            mma_bf16(acc[1][nt], A[1], b0, b1, acc[1][nt]);
          }
        }
      }
    }
  }

  // ---- K split across the cluster: rank 0 sums the partials in rank order
  if (CS > 1) {
    constexpr int NV_ = 2 * NT * 4;
#pragma unroll
    for (int j = 0; j < 2; ++j)
#pragma unroll
      for (int nt = 0; nt < NT; ++nt)
#pragma unroll
        for (int x = 0; x < 4; ++x) red_smem[((j * NT + nt) * 4 + x) * 256 + threadIdx.x] = acc[j][nt][x];
    cg::cluster_group cluster = cg::this_cluster();
    cluster.sync();
    if (rank == 0) {
      for (int r = 1; r < CS; ++r) {
        const float *rem = cluster.map_shared_rank(red_smem, r);
#pragma unroll
        for (int j = 0; j < 2; ++j)
#pragma unroll
          for (int nt = 0; nt < NT; ++nt)
#pragma unroll
            for (int x = 0; x < 4; ++x) acc[j][nt][x] += rem[((j * NT + nt) * 4 + x) * 256 + threadIdx.x];
      }
    }
    cluster.sync();
    (void)NV_;
    if (rank != 0) return;
  }

  // ---- epilogues
  if constexpr (MODE == MODE_GATEUP) {
    float hv[NT][4];
#pragma unroll
    for (int nt = 0; nt < NT; ++nt)
#pragma unroll
      for (int x = 0; x < 4; ++x) {
        const int i = x >> 1;
        const float av = acc[0][nt][x] * rowf[0][i];
        const float uv = acc[1][nt][x] * rowf[1][i];
        hv[nt][x] = silu_f(av) * uv;
      }
    const int rloc = warp * RPW + g;   // row within the CTA's 128-row chunk (+8 for i=1)
    if constexpr (ROUTED) {
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
      __syncthreads();
      if (threadIdx.x < 8 * NT) {
        float m = 0.0f;
#pragma unroll
        for (int w = 0; w < kWarps; ++w) m = fmaxf(m, amax_s[w][threadIdx.x]);
        const int ce = chunk_exponent(m);
        cexp_s[threadIdx.x] = ce;
        if ((int)threadIdx.x < nrows)
          a.h_scale[(size_t)(prow0 + threadIdx.x) * a.n_rowblocks + rb] = pow2f(ce);
      }
      __syncthreads();
#pragma unroll
      for (int nt = 0; nt < NT; ++nt)
#pragma unroll
        for (int x = 0; x < 4; ++x) {
          const int col = nt * 8 + 2 * q + (x & 1);
          if (col < nrows) {
            const int row = rb * RPC + rloc + 8 * (x >> 1);
            a.h_out[(size_t)(prow0 + col) * a.rows + row] = f16_bits(hv[nt][x] * pow2f(-cexp_s[col]));
          }
        }
    } else {
#pragma unroll
      for (int nt = 0; nt < NT; ++nt)
#pragma unroll
        for (int x = 0; x < 4; ++x) {
          const int col = nt * 8 + 2 * q + (x & 1);
          if (col < nrows) {
            const int row = rb * RPC + rloc + 8 * (x >> 1);
            a.h_out[(size_t)(prow0 + col) * a.rows + row] = bf16_bits(hv[nt][x]);
          }
        }
    }
  } else {
#pragma unroll
    for (int nt = 0; nt < NT; ++nt)
#pragma unroll
      for (int x = 0; x < 4; ++x) {
        const int col = nt * 8 + 2 * q + (x & 1);
        if (col >= nrows) continue;
#pragma unroll
        for (int j = 0; j < 2; ++j) {
          const int row = rbase[j] + g + 8 * (x >> 1);
          if constexpr (ROUTED) {
            const int p = a.prow_pair[prow0 + col];
            a.o_out[(size_t)p * a.rows + row] = acc[j][nt][x] * rowf[j][x >> 1] * a.gates[p];
          } else {
            a.o_out[(size_t)(prow0 + col) * a.rows + row] = acc[j][nt][x];
          }
        }
      }
  }
}

template <int WF, int MODE, int NT>
static cudaError_t launch_one(const ExpertArgs &a, int grid_tiles, cudaStream_t s) {
  const int CS = a.k_split;
  const size_t smem = CS > 1 ? (size_t)2 * NT * 4 * 256 * sizeof(float) : 0;
  auto fn = expert_kernel<WF, MODE, NT>;
  if (smem > 48 * 1024) {
    cudaError_t e = cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
  }
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((unsigned)(grid_tiles * a.n_rowblocks * CS));
  cfg.blockDim = dim3(256);
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
  return cudaLaunchKernelEx(&cfg, fn, a);
}

template <int WF, int MODE>
static cudaError_t launch_nt(int nt, const ExpertArgs &a, int grid_tiles, cudaStream_t s) {
  switch (nt) {
    case 1: return launch_one<WF, MODE, 1>(a, grid_tiles, s);
    case 2: return launch_one<WF, MODE, 2>(a, grid_tiles, s);
    default: return launch_one<WF, MODE, 4>(a, grid_tiles, s);
  }
}

// Only the dense bf16 (shared expert) path is instantiated here; routed FP4
// experts run in the TMA-fed kernels of expert_tma.cu.
void launch_expert(int wf, int mode, int nt, const ExpertArgs &a, int grid_tiles, cudaStream_t s) {
  if (grid_tiles <= 0 || wf != WF_BF16) return;
  if (mode == MODE_GATEUP) launch_nt<WF_BF16, MODE_GATEUP>(nt, a, grid_tiles, s);
  else launch_nt<WF_BF16, MODE_DOWN>(nt, a, grid_tiles, s);
}

}  // namespace moe
