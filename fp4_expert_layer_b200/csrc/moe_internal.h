// moe_internal.h -- internal interfaces of the sm_100a MoE layer library.
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <stddef.h>
#include <stdint.h>

#include "moe_layer.h"

namespace moe {

constexpr int kChunk = 128;        // K elements per activation-scale chunk / per mainloop step
constexpr int kWarps = 8;          // warps per expert-kernel CTA
constexpr int kMaxExperts = 1024;
constexpr int kMaxTopK = 32;
constexpr int kPermThreads = 512;
constexpr int kPtrListMax = 256;   // experts one location-table update launch can carry

// Device layout of one routed expert ("blob"): the checkpoint code bytes of the
// three matrices unchanged, the block scales rearranged into 512-byte blocks of
// 128 rows x 4 scale columns (the scale-factor block the sm_100 block-scaled MMA
// reads through tcgen05.cp; see sf_offset), plus, for MXFP4, one byte
// per row holding the row's largest E8M0 code (the row reference exponent the
// decode kernels fold out of the f16 operand), or, for NVFP4, the three fp32
// per-tensor scales.  Every piece starts on a 256-byte boundary.  The pinned
// host store holds all E experts in exactly this layout, so a miss is one
// contiguous host-to-device copy.
struct BlobLayout {
  size_t codes[3];
  size_t scales[3];
  size_t sref[3];     // MXFP4 only
  size_t glob;        // NVFP4 only: float[3]
  size_t bytes;
  int rows[3];
  int K[3];
  int G;              // block size along K: 32 (MXFP4) or 16 (NVFP4)
  int fmt;
  int tiled;          // 1: tile-major codes and scales (tensor-core EXACT layers);
                      // 2: gate and up interleaved per 64 rows (A4 layers); see below
};

// tiled = 0: codes in checkpoint order ([rows, K/2] per matrix), scales in
// 512-byte blocks (sf_offset).  tiled = 1 (MXFP4 layers on the tensor-core
// EXACT path): every 16 KB chunk of codes the kernels stream is contiguous --
//   gate/up, chunk rb * (H/128) + slab: gate rows rb*128 .. +127 then up rows
//     rb*128 .. +127, 64 bytes (128 elements, K slab `slab`) each;
//   down, chunk rb * (I/128) + slab: rows rb*256 .. +255, 64 bytes each;
// and the scale blocks of a chunk (gate, up / rows 0..127, 128..255 of the
// chunk) are one contiguous 1 KB at the same chunk index.  codes[0] / scales[0]
// start the gate/up regions, codes[2] / scales[2] the down regions.
// tiled = 2 (A4 layers): gate and up form one matrix of 2I rows from codes[0]
// / scales[0] (the two regions are adjacent), row c holding gate row
// (c / 128) * 64 + c % 64 when (c / 64) is even, else that up row; codes in
// checkpoint row format, scales in 512-byte blocks (sf_offset over the 2I
// rows); down as in tiled = 0.
BlobLayout blob_layout(int H, int I, int fmt, int tiled);
constexpr int kTcChunk = 16384;      // code bytes of one tiled chunk
constexpr int kTcSfChunk = 1024;     // scale bytes of one tiled chunk

// Byte offset of scale (row r, scale column col) inside a matrix's scale area
// with nsf scale columns per row: blocks of 128 rows x 4 columns (512 bytes),
// ordered row-block-major; inside a block, row r sits at 16*(r%32) + 4*((r%128)/32)
// and its 4 columns are consecutive bytes.
__host__ __device__ inline size_t sf_offset(int nsf, int r, int col) {
  return ((size_t)(r >> 7) * (size_t)(nsf >> 2) + (size_t)(col >> 2)) * 512u + 16u * (r & 31) +
         4u * ((r & 127) >> 5) + (col & 3);
}

// Where an expert's blob lives for one pass: >= 0 resident slot, <= -2 staging
// buffer (-2 - index), -1 not available in this pass.
constexpr int kLocAbsent = -1;
__host__ __device__ inline int loc_staging(int i) { return -2 - i; }

// One token tile of one expert: rows [prow0, prow0 + nrows) of the padded,
// expert-sorted activation order; each expert's rows start on a multiple of 8.
// Item counters of the tensor-core expert passes ([0] gate/up, [1] down): the
// CTAs take work items in index order by atomicAdd; the kernel that writes the
// tile list (or the staged wave's location update) zeroes them.
constexpr int kWorkCtrs = 2;

struct alignas(16) TileInfo {
  int expert;
  int prow0;
  int nrows;
  int sorted0;   // first row in the unpadded sorted order
};

// Ranges of the indices the kernels take from device data (a routing target,
// a location-table entry, a padded row's token or pair), for the device bounds
// checks of the checked build (checks.cuh); the normal build ignores them.
struct DevBounds {
  int n_experts;           // location-table entries (routed experts)
  int n_targets;           // routing targets (experts, then sinks)
  int n_slots, n_staging;  // blobs in the slot pool and in the staging ring
  int n_tokens, n_pairs;   // tokens of this forward, and T * k
  int *err;                // the layer's error word
};

// ------------------------------------------------------------------ routing
struct PermArgs {
  const int *ids;        // [T*k]
  int n_pairs, E, k, tile_tokens;   // E: routing targets (experts, then sinks)
  int n_real;            // experts with an FFN; targets >= n_real are sinks (no rows, no tiles)
  int *counts;           // [E]
  int *offsets;          // [E+1]
  int *perm;             // [n_pairs]
  int *inv;              // [n_pairs]
  TileInfo *tiles;       // [max tiles]
  int *n_tiles;          // [1]
  int *prow_token;       // [max prows]
  int *prow_pair;        // [max prows]
  int *active;           // [1] experts with >= 1 pair
  int pad;               // row padding granularity per expert (8 or 128)
  int *n_prows;          // [1] total padded rows (may be null)
  int *work_ctr;         // [kWorkCtrs] zeroed here (may be null): item counters of the expert passes
  int *tile_done;        // [tiles] zeroed here (may be null): gate/up items finished per tile
  DevBounds db;           // device bounds checks (checked build)
};
struct RouterArgs {
  const uint16_t *x;     // bf16 [T, H]
  int T, H, E, k;        // E: logit rows (targets, then the shared-expert gate row if any)
  int E_t;               // routing targets (experts, then sinks) among the E rows
  int scoring, renorm;   // 0 softmax / 1 sigmoid; 1: chosen scores renormalised
  const float *w;        // [E, H]
  const float *bias;     // [E] or null
  float *logits;         // [T, E]
  int *ids;              // [T, k]
  float *gates;          // [T, k]
  uint16_t *xf16;        // f16 [T, H], chunk-scaled
  float *xs;             // [T, H/128] chunk multipliers
  int *counter;          // [ceil(T/TT)] zero-initialised completion counters
  int fuse_perm;         // 1: the last token tile also runs the permutation
  int *tiles_done;       // [1] zero-initialised second-level counter
  PermArgs perm;         // permutation arguments (fuse_perm only)
};
void launch_router(const RouterArgs &a, cudaStream_t s);

void launch_permute(const PermArgs &a, cudaStream_t s);

// Prefill-sized batches: router logits by a register-tiled fp32 GEMM
// (x 16-byte aligned, H a multiple of 32), then top-k from the logits.
// splits > 1: partial logits of K ranges into parts [splits, T, E], assembled
// (in split order, + bias) by the top-k kernel.
int router_gemm_splits(int T, int H, int E, size_t part_floats);
void launch_router_gemm(const uint16_t *x, const float *w, const float *bias, int T, int H, int E, float *logits,
                        float *parts, int splits, cudaStream_t s);
// E: logit rows (row stride); E_t: routing targets among them (top-k runs over
// the first E_t); scoring / renorm as in RouterArgs.
void launch_topk(float *logits, const float *parts, int splits, const float *bias, int T, int E, int E_t, int k,
                 int scoring, int renorm, int *ids, float *gates, cudaStream_t s);

// ------------------------------------------------------------------ experts
enum WeightFmt { WF_MX = 0, WF_NV = 1 };
enum ExpertMode { MODE_GATEUP = 0, MODE_DOWN = 1 };

struct CombineArgs {
  const float *oprime;   // [T*k, H]
  const float *shared;   // [T, H] or null
  void *y;               // [T, H]: fp32, or bf16 when out_bf16
  int T, H, k;
  int out_bf16;
  // sink targets: slots whose id is >= n_real add nothing (their O' rows are
  // never written); ids may be null when the layer has no sinks
  const int *ids;        // [T*k]
  int n_real;
  // sigmoid-gated shared expert: s is scaled by sigmoid(logits[t * ld + sg_col])
  // (null: weight 1)
  const float *sg_logits;
  int ld, sg_col;
};
void launch_combine(const CombineArgs &a, cudaStream_t s);


// ------------------------------------------------------------------ TMA-fed routed experts
struct LocUpdate {
  int n;
  int keep_resident;
  int E;
  int *work_ctr;         // [kWorkCtrs] zeroed for the wave's expert passes (may be null)
  int expert[kPtrListMax];
  int loc[kPtrListMax];
};
void launch_loc_update(const LocUpdate &u, const int *resident, int *out, cudaStream_t s);

// Tensor maps over the code bytes of one matrix for every blob of a region
// (3-D: K/2 bytes, rows, blob index), box = 64 bytes x (128 or 256) rows.
struct CodeMaps {
  CUtensorMap slot[3];
  CUtensorMap stage[3];
};

struct TmaExpertArgs {
  CodeMaps maps;
  const int *loc;          // [E]
  const uint8_t *slots;    // slot pool base
  const uint8_t *staging;  // staging ring base
  size_t blob_bytes;
  BlobLayout L;
  int K, rows, n_rowblocks, k_split, tile_tokens;
  const TileInfo *tiles;
  const int *n_tiles;
  const int *prow_token;
  const int *prow_pair;
  const float *gates;
  const uint16_t *act;
  const float *act_scale;
  uint16_t *h_out;
  float *h_scale;
  float *o_out;
  int *err;                // device-visible error word (bounded waits)
  // fused ordered combine (down pass): the last of a token's k contributions to
  // a 256-row block writes y = sum_j O'[t*k + j] (j order) + shared[t]
  float *y;
  const float *shared;     // [T, H] or null
  int *comb_cnt;           // [max_tokens, H/256] zero-initialised arrival counters
  int top_k;
  DevBounds db;           // device bounds checks (checked build)
};
void launch_expert_tma(int wf, int mode, int nt, const TmaExpertArgs &a, int grid_tiles, cudaStream_t s);

// ------------------------------------------------------------------ A4 (activation FP4) path
// Quantise rows to the experts' 4-bit format: codes [rows, K/2], scale blocks
// laid out like the weights' (sf_offset over rows), NVFP4 per-row tensor scale.
struct QuantArgs {
  int max_rows;
  const int *n_rows;         // device: rows to produce (padded count)
  int K, fmt;
  const uint16_t *src_bf16;  // x [T, K] gathered by row_token (x path), or null
  const int *row_token;      // padded row -> token (-1 = pad)
  const float *src_f32;      // h [rows, K] (h path), or null
  const int *row_pair;       // padded row -> pair (-1 = pad), h path
  const int *loc;            // h path: only rows whose expert is present in this pass
  const int *ids;            // [T*k] pair -> expert
  uint8_t *codes;
  uint8_t *sf;
  float *G;                  // NVFP4: per-row tensor scale
  DevBounds db;           // device bounds checks (checked build)
};
void launch_quant(const QuantArgs &q, cudaStream_t s);

struct A4Maps {
  // [slot | staging][matrix]: code bytes, box 128 B x 128 rows, 128-byte
  // swizzle; matrix 0 is gate and up together (2I rows interleaved per 64,
  // blob layout tiled = 2), 1 is unused, 2 is down
  CUtensorMap w[2][3];
  CUtensorMap act[2];        // [x | h]: quantised activation rows, box 128 B x 128 rows, 128-byte swizzle
};

struct A4GemmArgs {
  A4Maps maps;
  int act_map;               // 0 = x (gate/up), 1 = h (down)
  const int *loc;
  const uint8_t *slots;
  const uint8_t *staging;
  size_t blob_bytes;
  BlobLayout L;
  int K, rows, n_rowblocks;
  const TileInfo *tiles;
  const int *n_tiles;
  const uint8_t *bsf;        // activation scale blocks
  const float *bG;           // NVFP4 activation per-row scale (null for MXFP4)
  float *h_out;              // gate/up: h fp32 [rows of activations, I]
  // gate/up, MXFP4 only (may be null): h quantised in the epilogue instead,
  // E2M1 codes [rows, I/2] and E8M0 block scales (sf_offset layout, I/32 per row)
  uint8_t *hq_out;
  uint8_t *hsf_out;
  float *o_out;              // down: O' [pairs, H]
  const int *prow_pair;
  const float *gates;
  int *err;
  int *work_ctr;             // item counter of this pass, zero at launch
  int grid;                  // persistent CTAs
  DevBounds db;           // device bounds checks (checked build)
};
// rows: h width I (gate/up; items cover 64 h columns each, n_rowblocks = I / 64)
// or H (down; n_rowblocks = H / 128).
void launch_gemm_a4(int wf, int mode, const A4GemmArgs &a, cudaStream_t s);

// ---------------------------------------------------------------------------
// EXACT numerics on the tensor core (MXFP4 experts): the weights stay E2M1
// with their E8M0 block scales; each activation row (x before gate/up, h
// before down) is written as two E4M3 rows ("pieces") with one UE8M0 scale per
// 32 elements each, v = s1 * q1 + s2 * q2, so that kind::mxf8f6f4 MMAs of the
// E2M1 weights against both pieces sum to the product with the activation.
// For a bf16 value the two pieces are exact; for the fp32 h they keep about
// nine significant bits.  Activation rows live in per-tile slots of
// kTcSlotRows rows: row kTcSlotRows * tile + 2 * j + piece for the tile's j-th
// pair, so that every tile starts a 128-row scale-factor block.
constexpr int kTcSlotRows = 128;

struct TcMaps {
  // [slot | staging][0 = gate and up together (4-D: K, rows, matrix, blob; box 128 x 128 x 2 x 1),
  //                  1 = down (3-D: K, rows, blob; box 128 x 256 x 1)]: E2M1 codes unpacked by the
  // TMA to one byte per element, 128-byte swizzle
  CUtensorMap w[2][2];
  // the pass's activation pieces [slot rows, K] E4M3 (x pieces for gate/up,
  // h pieces for down), box 128 bytes x 16 rows, 128-byte swizzle
  CUtensorMap act;
};

struct TcQuantArgs {
  const uint16_t *x;         // [T, H] bf16
  int H;
  const TileInfo *tiles;
  const int *n_tiles;
  int max_tiles, tile_tokens;
  const int *prow_token;
  uint8_t *xq;               // [max_tiles * kTcSlotRows, H] E4M3 pieces
  uint8_t *xsf;              // scale-factor blocks of xq (UE8M0, per 32)
  DevBounds db;           // device bounds checks (checked build)
};
void launch_tc_quant_x(const TcQuantArgs &q, cudaStream_t s);

// Shared expert (bf16) on the tensor core for prefill-sized batches.
struct DenseTcArgs {
  CUtensorMap wmap[2];       // gate/up: gate [I_s, H], up [I_s, H]; down: [H, I_s] (bf16, box 64 x 128)
  CUtensorMap xmap;          // activations bf16 [rows >= T, K], box 64 x 128
  int T, K, rows, n_rowblocks, grid;
  uint16_t *h_out;           // gate/up: bf16 [T, I_s]
  float *s_out;              // down: fp32 [T, H]
  int *err;
};
void launch_dense_tc(int mode, const DenseTcArgs &a, cudaStream_t s);
// Decode-sized batches (T <= 128): K split over a cluster of S CTAs per row
// block (xmap's box is 64 x NP rows, NP = T rounded up to 16, 32, 64 or 128).
// The cluster size S is chosen per launch: the largest (8, 4, 2) that keeps
// at least 4 K slabs per CTA and fits every row block's cluster on the device
// at once (cudaOccupancyMaxActiveClusters), else 1.
void launch_dense_splitk(int mode, const DenseTcArgs &a, cudaStream_t s);
inline int dense_splitk_rows(int T) { return T <= 16 ? 16 : (T <= 32 ? 32 : (T <= 64 ? 64 : 128)); }

struct TcArgs {
  TcMaps maps;
  const int *loc;
  const uint8_t *slots;
  const uint8_t *staging;
  size_t blob_bytes;
  BlobLayout L;
  int K, rows, n_rowblocks;  // reduction length, weight rows of the pass, rows / 128
  const TileInfo *tiles;
  const int *n_tiles;
  const uint8_t *act;        // activation pieces [slot rows, K] E4M3 (x for gate/up, h for down)
  const uint8_t *bsf;        // activation scale-factor blocks
  // gate/up: h pieces for the down pass
  uint8_t *hq, *hsf;
  // down: O'[pair, H] = gate * (W_down . h)
  const int *prow_pair;
  const float *gates;
  float *o_out;
  int *work_ctr;             // item counter of this pass, zero at launch (set two or more kernels back)
  // Per-tile hand-over from the gate/up pass to the down pass (decode, all
  // resident; null otherwise): gate/up adds 1 per finished item of a tile, the
  // down pass reads a tile's h once its count reaches tile_target (I / 128)
  // instead of waiting for the whole gate/up grid
  int *tile_done;
  int tile_target;
  int *err;
  int grid;                  // persistent CTAs
  // 1: the tile list and `loc` were written two or more kernels back on the
  // stream, so the weight stream may start before this kernel waits for its
  // predecessor (the resident path; not the staged waves, whose location
  // table is written by the kernel right before)
  int early;
  DevBounds db;           // device bounds checks (checked build)
};
// nbox: activation rows per tile (2 x tile tokens): 16 or 112.  The kernel is
// persistent: `a.grid` CTAs take the work items (tile, 256 weight rows) from
// `a.work_ctr` in index order.
void launch_expert_tc(int mode, int nbox, const TcArgs &a, int grid_tiles, cudaStream_t s);

// ---------------------------------------------------------------------------
// EXACT numerics for NVFP4 experts at prefill-sized batches (expert_dq.cu):
// each 64-element K slab of a weight tile is decoded once per token tile into
// shared memory as bf16 (E2M1 x E4M3 is exact in bf16) and multiplied with
// tcgen05 kind::f16 against bf16 activation rows; the per-tensor scale is
// applied in the epilogue.  h is written as bf16 in padded-row order.
struct DqMaps {
  // code bytes of matrix m of every blob in a region, 3-D (K/2 bytes, rows,
  // blob), box 32 bytes x (128 rows: gate / up | 256 rows: down) x 1
  CUtensorMap slot[3];
  CUtensorMap stage[3];
  // the pass's 16-bit activation rows in padded-row order (gate/up: x rows
  // gathered beforehand; down: h), 128-byte swizzle, box 64 x 64 rows
  CUtensorMap act;
};

// weight formats of the dequantise-to-shared kernels
enum DqFmt { DQ_NV = 0, DQ_I4 = 1, DQ_F8 = 2 };

struct DqArgs {
  DqMaps maps;
  int wfmt;                  // DqFmt
  const int *loc;
  const uint8_t *slots;
  const uint8_t *staging;
  size_t blob_bytes;
  BlobLayout L;
  int K, rows, n_rowblocks;  // reduction length, weight rows of the pass, items per tile
  const TileInfo *tiles;
  const int *n_tiles;
  const int *prow_token;     // gate/up: padded row -> token
  const int *prow_pair;      // down: padded row -> pair
  const float *gates;
  const uint16_t *act;       // gate/up: x rows in padded-row order [padded rows, H], bf16 (NVFP4: f16, see
                             // act_scale); down: h bf16 [padded rows, I]
  const float *act_scale;    // gate/up of NVFP4 layers: per padded row, the scale of its f16 x row (x = row * scale)
  uint16_t *h_out;           // gate/up: h bf16 [padded rows, I]
  float *o_out;              // down: O' [pairs, H]
  int *work_ctr;             // item counter of this pass, zero at launch
  int *err;
  int grid;                  // persistent CTAs
  DevBounds db;           // device bounds checks (checked build)
};
// nb: tokens per tile (64 or 128)
void launch_expert_dq(int mode, int nb, const DqArgs &a, cudaStream_t s);
// x rows into the padded expert order for the dequantising expert pass:
// bf16 copies, or (to_f16) f16 rows with a power-of-two scale per row (xs =
// its inverse); rows up to *n_rows, pad rows (token -1) left as they are
void launch_gather_rows(const uint16_t *x, int H, const int *prow_token, const int *n_rows, int max_rows,
                        int to_f16, uint16_t *xg, float *xs, const DevBounds &db, cudaStream_t s);

}  // namespace moe
