// route_common.cuh -- block-level pieces of the routing step shared by the
// router kernels: warp top-k with renormalised gates, and the stable
// token-to-expert permutation.
#pragma once

#include "checks.cuh"
#include "device_utils.cuh"
#include "moe_internal.h"

namespace moe {

template <bool IDS_GLOBAL>
__device__ __forceinline__ int load_id(const int *ids, int p) {
  if constexpr (IDS_GLOBAL) return __ldcg(ids + p);
  else return ids[p];
}

// Top-k of one token by one warp: lane holds the logits of targets lane,
// lane + 32, ... in lv (-inf past E; E counts experts and sink targets).  Ids
// in descending-logit order, lower index first on ties (both scorings are
// monotone in the logit).  Scores: softmax s_j = exp(l_j - l_max) / sum over
// all E targets, or sigmoid s_j = 1 / (1 + exp(-l_j)); gates = s_j / sum of
// the k chosen s (summed in j order) when renorm, else s_j.  Softmax with
// renormalisation is computed as exp(l_j - l_max) over the chosen k's sum.
// Writes ids / gates (k entries each) and, if ids_s is not null, the ids to
// shared memory too.
template <int KPER>
__device__ __forceinline__ void topk_warp(const float (&lv)[KPER], int E, int k, int *ids, float *gates,
                                          int *ids_s, int scoring = 0, int renorm = 1) {
  const int lane = threadIdx.x & 31;
  float lmax = 0.0f, den = 0.0f;
  float my_l = 0.0f;    // lane j keeps the logit of choice j
  int my_id = 0;
  // Each logit as an order-preserving 32-bit key (-0 taken as +0, so that
  // equal values tie as they compare), 0 for targets that are out of range or
  // taken: a round is one warp max of the keys and one warp min of the
  // indices that hold it (the lower index wins a tie).
  uint32_t key[KPER];
#pragma unroll
  for (int i = 0; i < KPER; ++i) {
    const float v = lv[i] == 0.0f ? 0.0f : lv[i];
    const uint32_t b = __float_as_uint(v);
    key[i] = (lane + 32 * i < E) ? ((b & 0x80000000u) ? ~b : (b | 0x80000000u)) : 0u;
  }
  for (int j = 0; j < k; ++j) {
    uint32_t kb = 0u;
#pragma unroll
    for (int i = 0; i < KPER; ++i) kb = max(kb, key[i]);
    const uint32_t kmax = __reduce_max_sync(0xffffffffu, kb);
    uint32_t ib = 0xffffffffu;
#pragma unroll
    for (int i = 0; i < KPER; ++i)
      if (key[i] == kmax && ib == 0xffffffffu) ib = (uint32_t)(lane + 32 * i);
    const int bi = (int)__reduce_min_sync(0xffffffffu, ib);
    const float bv = __uint_as_float((kmax & 0x80000000u) ? (kmax & 0x7fffffffu) : ~kmax);   // the winning logit
    if ((bi & 31) == lane) {
#pragma unroll
      for (int i = 0; i < KPER; ++i)
        if (i == (bi >> 5)) key[i] = 0u;                 // taken
    }
    if (j == 0) lmax = bv;
    if (lane == j) { my_l = bv; my_id = bi; }
  }
  float ex;
  if (scoring == 0) {
    ex = (lane < k) ? expf(my_l - lmax) : 0.0f;
    if (!renorm) {
      // softmax over every target: this lane's terms, then a butterfly sum
      float all = 0.0f;
#pragma unroll
      for (int i = 0; i < KPER; ++i)
        if (lane + 32 * i < E) all += expf(lv[i] - lmax);
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) all += __shfl_xor_sync(0xffffffffu, all, o);
      ex = ex / all;
    }
  } else {
    ex = (lane < k) ? 1.0f / (1.0f + expf(-my_l)) : 0.0f;
  }
  if (renorm) {
    // ordered sum over j = 0..k-1
    for (int j = 0; j < k; ++j) den += __shfl_sync(0xffffffffu, ex, j);
  }
  if (lane < k) {
    ids[lane] = my_id;
    gates[lane] = renorm ? ex / den : ex;
    if (ids_s) ids_s[lane] = my_id;
  }
}

// ---------------------------------------------------------------------------
// Permutation: stable counting sort of pair index p = t*k + j by expert, as a
// block-level routine (NTH threads, `sm` = shared scratch of
// (5E + 3 + (NTH/32)*E) ints).  Each warp owns one contiguous range of pairs:
// per-warp counts by shared-memory atomics, then per target the start of each
// warp's run (warp order), offsets / padded offsets / tile offsets by one
// block scan, and each warp places its range in order, 32 pairs at a time
// (ranks inside a group from warp match, a per-warp cursor per target across
// groups), so equal experts keep ascending p (stable).  The expert ids are
// read from global memory (IDS_GLOBAL, another CTA wrote them) or from this
// CTA's shared memory.
// ---------------------------------------------------------------------------
template <int NTH, bool IDS_GLOBAL>
__device__ void permute_block(const PermArgs &a, const int *ids, int *sm) {
  constexpr int W = NTH / 32;
  __shared__ int4 wsum[W];
  const int E = a.E;
  int *cnt = sm;                  // [E]
  int *cursor = cnt + E;          // [E]
  int *off = cursor + E;          // [E+1]
  int *poff = off + E + 1;        // [E+1] padded (multiple of 8) offsets
  int *toff = poff + E + 1;       // [E+1] tile offsets
  int *wcnt = toff + E + 1;       // [W][E]
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;

  (void)cursor;
  if (a.work_ctr && tid < kWorkCtrs) a.work_ctr[tid] = 0;
  for (int i = tid; i < W * E; i += NTH) wcnt[i] = 0;
  __syncthreads();
  // warp w owns pairs [p0, p1): its own count per target
  const int span = (a.n_pairs + W - 1) / W;
  const int p0 = min(a.n_pairs, warp * span), p1 = min(a.n_pairs, p0 + span);
  for (int p = p0 + lane; p < p1; p += 32) {
    const int e = load_id<IDS_GLOBAL>(ids, p);
    if (dcheck(e >= 0 && e < E, a.db.err, kChkTarget)) atomicAdd(&wcnt[warp * E + e], 1);
  }
  __syncthreads();
  // per target: its count, and each warp's count replaced by the start of
  // its run among the target's pairs (exclusive, in warp order)
  for (int e = tid; e < E; e += NTH) {
    int run = 0;
    for (int w = 0; w < W; ++w) {
      const int c = wcnt[w * E + e];
      wcnt[w * E + e] = run;
      run += c;
    }
    cnt[e] = run;
  }
  __syncthreads();

  // block exclusive scan of (count, padded count, tiles, active) over targets;
  // sink targets (e >= n_real) have counts and offsets but no rows or tiles
  const int per = (E + NTH - 1) / NTH;
  const int e0 = min(E, tid * per), e1 = min(E, e0 + per);
  int4 v = make_int4(0, 0, 0, 0);
  for (int e = e0; e < e1; ++e) {
    const int c = cnt[e];
    const int cr = e < a.n_real ? c : 0;
    v.x += c;
    v.y += (cr + a.pad - 1) / a.pad * a.pad;
    v.z += (cr + a.tile_tokens - 1) / a.tile_tokens;
    v.w += cr > 0;
  }
  int4 inc = v;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    int4 t;
    t.x = __shfl_up_sync(0xffffffffu, inc.x, o);
    t.y = __shfl_up_sync(0xffffffffu, inc.y, o);
    t.z = __shfl_up_sync(0xffffffffu, inc.z, o);
    t.w = __shfl_up_sync(0xffffffffu, inc.w, o);
    if (lane >= o) { inc.x += t.x; inc.y += t.y; inc.z += t.z; inc.w += t.w; }
  }
  if (lane == 31) wsum[warp] = inc;
  __syncthreads();
  if (warp == 0) {
    int4 w = lane < W ? wsum[lane] : make_int4(0, 0, 0, 0);
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      int4 t;
      t.x = __shfl_up_sync(0xffffffffu, w.x, o);
      t.y = __shfl_up_sync(0xffffffffu, w.y, o);
      t.z = __shfl_up_sync(0xffffffffu, w.z, o);
      t.w = __shfl_up_sync(0xffffffffu, w.w, o);
      if (lane >= o) { w.x += t.x; w.y += t.y; w.z += t.z; w.w += t.w; }
    }
    if (lane < W) wsum[lane] = w;
  }
  __syncthreads();
  {
    const int4 pre = warp > 0 ? wsum[warp - 1] : make_int4(0, 0, 0, 0);
    int o = pre.x + inc.x - v.x, po = pre.y + inc.y - v.y, to = pre.z + inc.z - v.z;
    for (int e = e0; e < e1; ++e) {
      const int c = cnt[e];
      const int cr = e < a.n_real ? c : 0;
      off[e] = o; poff[e] = po; toff[e] = to;
      o += c;
      po += (cr + a.pad - 1) / a.pad * a.pad;
      to += (cr + a.tile_tokens - 1) / a.tile_tokens;
    }
    if (tid == NTH - 1) {
      const int4 tot = wsum[W - 1];
      off[E] = tot.x; poff[E] = tot.y; toff[E] = tot.z;
      *a.n_tiles = tot.z;
      *a.active = tot.w;
      if (a.n_prows) *a.n_prows = tot.y;
    }
  }
  __syncthreads();
  if (a.tile_done)
    for (int t = tid; t < toff[E]; t += NTH) a.tile_done[t] = 0;
  for (int e = tid; e <= E; e += NTH) a.offsets[e] = off[e];
  for (int e = tid; e < E; e += NTH) {
    const int c = cnt[e];
    a.counts[e] = c;
    if (e >= a.n_real) continue;                   // a sink: no rows, no tiles
    const int nt = (c + a.tile_tokens - 1) / a.tile_tokens;
    for (int i = 0; i < nt; ++i) {
      TileInfo ti;
      ti.expert = e;
      ti.prow0 = poff[e] + i * a.tile_tokens;
      ti.nrows = min(a.tile_tokens, c - i * a.tile_tokens);
      ti.sorted0 = off[e] + i * a.tile_tokens;
      a.tiles[toff[e] + i] = ti;
    }
    for (int r = poff[e] + c; r < poff[e + 1]; ++r) { a.prow_token[r] = -1; a.prow_pair[r] = -1; }
  }

  const unsigned lt_mask = (1u << lane) - 1u;
  for (int base = p0; base < p1; base += 32) {
    const int p = base + lane;
    int e = p < p1 ? load_id<IDS_GLOBAL>(ids, p) : -1;
    if (kCheckedBuild && (e < 0 || e >= E)) e = -1;   // recorded by the count above
    const bool valid = e >= 0;
    const unsigned peers = __match_any_sync(0xffffffffu, e);
    const int rank = __popc(peers & lt_mask);
    const int local = valid ? wcnt[warp * E + e] + rank : 0;   // index among the target's pairs
    __syncwarp();
    if (valid && rank == 0) wcnt[warp * E + e] += __popc(peers);
    __syncwarp();
    if (valid) {
      const int pos = off[e] + local;
      a.perm[pos] = p;
      a.inv[p] = pos;
      if (e < a.n_real) {
        const int prow = poff[e] + local;
        a.prow_token[prow] = p / a.k;
        a.prow_pair[prow] = p;
      }
    }
  }
}

__host__ __device__ inline size_t perm_smem_ints(int E, int nth) { return (size_t)5 * E + 3 + (size_t)(nth / 32) * E; }

}  // namespace moe
