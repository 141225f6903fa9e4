// route.cu -- router GEMV/GEMM with fused softmax top-k, the token-to-expert
// permutation, expert pointer-table updates and the ordered combine.
//
// Routing semantics (which function, how many experts, top-k) are what the
// checkpoint declares and never change silently ("ro99/strata", rules list).
// This library implements softmax routing with the top-k gates renormalised to
// sum to one: ids are the k largest logits in descending order (lower expert
// index first on ties) and g_j = exp(l_j - l_max) / sum_i exp(l_i - l_max)
// over the chosen k, which equals softmax over all E renormalised to the k.
#include <cooperative_groups.h>

#include <algorithm>

#include "device_utils.cuh"
#include "moe_internal.h"
#include "launch.cuh"
#include "route_common.cuh"

namespace moe {

constexpr int kRouterTT = 4;      // tokens per router CTA
constexpr int kRouterEB = 8;      // experts per router CTA (one per warp)


// grid (ceil(T/TT), ceil(E/EB)), 256 threads.  Each CTA computes logits for
// its TT tokens x EB experts; the CTA with blockIdx.y == 0 also writes the
// chunk-scaled f16 copy of its tokens; the last CTA of a token tile to finish
// (completion counter) runs top-k for the tile; with fuse_perm, the last of
// those (second counter) runs the permutation for the whole batch.
// KPER = experts per lane in the top-k scan (E <= 32 * KPER).
template <int KPER>
__global__ void __launch_bounds__(256) router_kernel(const RouterArgs a) {
  extern __shared__ float xs_smem[];   // [TT][H], reused by the fused permutation
  __shared__ int is_last;
  const int H = a.H, E = a.E;
  const int t0 = blockIdx.x * kRouterTT;
  const int nt = min(kRouterTT, a.T - t0);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int e = blockIdx.y * kRouterEB + warp;
  const float *w = a.w + (size_t)min(e, E - 1) * H;
  // the first 8 weight vectors of this lane are in flight while x is staged
  float4 wv[8];
#pragma unroll
  for (int u = 0; u < 8; ++u) {
    const int h = lane * 4 + u * 128;
    wv[u] = h < H ? __ldg(reinterpret_cast<const float4 *>(w + h)) : make_float4(0.f, 0.f, 0.f, 0.f);
  }

  // x tile -> smem (fp32)
  for (int i = threadIdx.x; i < nt * H / 2; i += blockDim.x) {
    const int t = (2 * i) / H, h = (2 * i) % H;
    uint32_t v = *reinterpret_cast<const uint32_t *>(a.x + (size_t)(t0 + t) * H + h);
    xs_smem[t * H + h] = __uint_as_float(v << 16);
    xs_smem[t * H + h + 1] = __uint_as_float(v & 0xFFFF0000u);
  }
  __syncthreads();

  // logits: warp w -> expert e
  if (e < E) {
    float acc[kRouterTT];
#pragma unroll
    for (int t = 0; t < kRouterTT; ++t) acc[t] = 0.0f;
    // 8 independent 16-byte loads in flight per lane before any use
    for (int h0 = lane * 4; h0 < H; h0 += 128 * 8) {
      if (h0 != lane * 4) {
#pragma unroll
        for (int u = 0; u < 8; ++u) {
          const int h = h0 + u * 128;
          wv[u] = h < H ? __ldg(reinterpret_cast<const float4 *>(w + h)) : make_float4(0.f, 0.f, 0.f, 0.f);
        }
      }
#pragma unroll
      for (int u = 0; u < 8; ++u) {
        const int h = h0 + u * 128;
        if (h < H) {
#pragma unroll
          for (int t = 0; t < kRouterTT; ++t) {
            if (t < nt) {
              const float4 xv = *reinterpret_cast<const float4 *>(xs_smem + t * H + h);
              acc[t] = fmaf(wv[u].x, xv.x, acc[t]);
              acc[t] = fmaf(wv[u].y, xv.y, acc[t]);
              acc[t] = fmaf(wv[u].z, xv.z, acc[t]);
              acc[t] = fmaf(wv[u].w, xv.w, acc[t]);
            }
          }
        }
      }
    }
#pragma unroll
    for (int t = 0; t < kRouterTT; ++t) {
      float v = acc[t];
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
      if (lane == 0 && t < nt) a.logits[(size_t)(t0 + t) * E + e] = v + (a.bias ? a.bias[e] : 0.0f);
    }
  }

  // chunk-scaled f16 copy of x: warp per (token, 128-chunk)
  if (blockIdx.y == 0 && a.xf16) {
    const int nck = H / kChunk;
    for (int job = warp; job < nt * nck; job += kWarps) {
      const int t = job / nck, c = job % nck;
      const float4 v = *reinterpret_cast<const float4 *>(xs_smem + t * H + c * kChunk + lane * 4);
      float m = fmaxf(fmaxf(fabsf(v.x), fabsf(v.y)), fmaxf(fabsf(v.z), fabsf(v.w)));
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
      const int ce = chunk_exponent(m);
      const float inv = pow2f(-ce);
      uint2 out;
      __half2 p0 = __floats2half2_rn(v.x * inv, v.y * inv);
      __half2 p1 = __floats2half2_rn(v.z * inv, v.w * inv);
      out.x = *reinterpret_cast<uint32_t *>(&p0);
      out.y = *reinterpret_cast<uint32_t *>(&p1);
      *reinterpret_cast<uint2 *>(a.xf16 + (size_t)(t0 + t) * H + c * kChunk + lane * 4) = out;
      if (lane == 0) a.xs[(size_t)(t0 + t) * nck + c] = pow2f(ce);
    }
  }

  // completion: the last CTA of this token tile runs top-k
  __threadfence();
  __syncthreads();
  if (threadIdx.x == 0) {
    const int prev = atomicAdd(&a.counter[blockIdx.x], 1);
    is_last = (prev == (int)gridDim.y - 1);
  }
  __syncthreads();
  if (!is_last) return;
  __threadfence();
  if (threadIdx.x == 0) a.counter[blockIdx.x] = 0;

  // top-k: warp per token; lane holds experts lane, lane+32, ...
  if (warp < nt) {
    const int t = t0 + warp;
    float lv[KPER];
    const float *lrow = a.logits + (size_t)t * E;
#pragma unroll
    for (int i = 0; i < KPER; ++i) {
      const int ee = lane + 32 * i;
      lv[i] = (ee < a.E_t) ? __ldcg(lrow + ee) : -INFINITY;
    }
    topk_warp<KPER>(lv, a.E_t, a.k, a.ids + (size_t)t * a.k, a.gates + (size_t)t * a.k, nullptr, a.scoring,
                    a.renorm);
  }
  if (!a.fuse_perm) return;

  // the last token tile to finish top-k runs the permutation (with a single
  // token tile this CTA wrote every id itself: a block barrier suffices)
  if (gridDim.x > 1) {
    __threadfence();
    __syncthreads();
    if (threadIdx.x == 0) is_last = (atomicAdd(a.tiles_done, 1) == (int)gridDim.x - 1);
    __syncthreads();
    if (!is_last) return;
    __threadfence();
    if (threadIdx.x == 0) *a.tiles_done = 0;
  } else {
    __syncthreads();
  }
  permute_block<256, true>(a.perm, a.perm.ids, reinterpret_cast<int *>(xs_smem));
}

template <int KPER>
static void launch_router_k(const RouterArgs &a, cudaStream_t s) {
  dim3 grid((a.T + kRouterTT - 1) / kRouterTT, (a.E + kRouterEB - 1) / kRouterEB);
  size_t smem = (size_t)kRouterTT * a.H * sizeof(float);
  if (a.fuse_perm) smem = std::max(smem, perm_smem_ints(a.E, 256) * sizeof(int));
  if (smem > 48 * 1024) cudaFuncSetAttribute(router_kernel<KPER>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  router_kernel<KPER><<<grid, 256, smem, s>>>(a);
}

void launch_router(const RouterArgs &a, cudaStream_t s) {
  if (a.E_t <= 64) launch_router_k<2>(a, s);
  else if (a.E_t <= 128) launch_router_k<4>(a, s);
  else if (a.E_t <= 256) launch_router_k<8>(a, s);
  else if (a.E_t <= 512) launch_router_k<16>(a, s);
  else launch_router_k<32>(a, s);
}

__global__ void __launch_bounds__(kPermThreads) permute_kernel(const PermArgs a) {
  extern __shared__ int psm[];
  permute_block<kPermThreads, true>(a, a.ids, psm);
}

void launch_permute(const PermArgs &a, cudaStream_t s) {
  const size_t smem = sizeof(int) * perm_smem_ints(a.E, kPermThreads);
  if (smem > 48 * 1024) cudaFuncSetAttribute(permute_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  permute_kernel<<<1, kPermThreads, smem, s>>>(a);
}

// ---------------------------------------------------------------------------
// Ordered combine: y[t] = sum_{j<k, ids_j an expert} O'[t*k + j] (in j order)
// + gs[t] * s[t], gs = 1 or sigmoid(shared-gate logit); y fp32 or bf16 (RN).
// ---------------------------------------------------------------------------
__global__ void combine_kernel(const CombineArgs a) {
  wait_prior_grid();
  const int H4 = a.H / 4;
  const size_t n = (size_t)a.T * H4;
  for (size_t i = blockIdx.x * (size_t)blockDim.x + threadIdx.x; i < n;
       i += (size_t)gridDim.x * blockDim.x) {
    const size_t t = i / H4, c = i % H4;
    const float4 *o = reinterpret_cast<const float4 *>(a.oprime) + t * a.k * H4 + c;
    float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);       // 0 + v == v: the first term is exact
    for (int j = 0; j < a.k; ++j) {
      if (a.ids && __ldg(a.ids + t * a.k + j) >= a.n_real) continue;   // a sink: no FFN
      const float4 v = __ldcs(o + (size_t)j * H4);
      acc.x += v.x; acc.y += v.y; acc.z += v.z; acc.w += v.w;
    }
    if (a.shared) {
      float4 v = reinterpret_cast<const float4 *>(a.shared)[t * H4 + c];
      if (a.sg_logits) {
        const float gs = 1.0f / (1.0f + expf(-__ldg(a.sg_logits + t * a.ld + a.sg_col)));
        v.x *= gs; v.y *= gs; v.z *= gs; v.w *= gs;
      }
      acc.x += v.x; acc.y += v.y; acc.z += v.z; acc.w += v.w;
    }
    if (a.out_bf16) {
      uint2 b;
      b.x = (uint32_t)bf16_bits(acc.x) | ((uint32_t)bf16_bits(acc.y) << 16);
      b.y = (uint32_t)bf16_bits(acc.z) | ((uint32_t)bf16_bits(acc.w) << 16);
      reinterpret_cast<uint2 *>(a.y)[t * H4 + c] = b;
    } else {
      reinterpret_cast<float4 *>(a.y)[t * H4 + c] = acc;
    }
  }
}

// ---------------------------------------------------------------------------
// Router logits for prefill-sized batches: a register-tiled fp32 GEMM on the
// CUDA cores.  CTA tile 128 tokens x 16 JN experts, K in chunks of 32 staged
// in shared memory (x converted from bf16, both operands transposed to
// [k][.], double-buffered, the next chunk's global loads in flight during this
// one's 32 k steps), each thread 8 tokens x JN experts (tokens 4 ty .. +3 and
// 64 + 4 ty .. +3, experts 4 tx .. +3 and, for JN = 8, 64 + 4 tx .. +3, so that
// the 16-byte shared loads of a quarter warp fall in distinct banks).  Each
// chunk's 32 products are summed into a chunk partial that is then added to
// the running sum (two-level summation: the fp32 rounding of H = 4096
// sequential additions would otherwise approach the 1e-5 the logits are held
// to).  With few tiles (small T or E) the K range is split over gridDim.z
// CTAs that write partial logits to a workspace; the top-k kernel adds the
// parts in split order (deterministic, no atomics).
// ---------------------------------------------------------------------------
namespace {
constexpr int kRgT = 128, kRgK = 32;
template <int JN>
constexpr size_t router_gemm_smem() { return (size_t)2 * kRgK * (kRgT + 16 * JN) * sizeof(float); }
}

template <int JN>
__global__ void __launch_bounds__(256, 1) router_gemm_kernel(const uint16_t *__restrict__ x,
                                                             const float *__restrict__ w,
                                                             const float *__restrict__ bias, int T, int H, int E,
                                                             float *__restrict__ logits, float *__restrict__ parts) {
  constexpr int TE = 16 * JN;                           // experts per CTA
  constexpr int WPR = 256 / TE;                         // loader threads per expert row
  constexpr int WF4 = kRgK / WPR / 4;                   // float4 per loader thread
  extern __shared__ __align__(16) float rg_smem[];
  float (*xs)[kRgK][kRgT] = reinterpret_cast<float (*)[kRgK][kRgT]>(rg_smem);
  float (*ws)[kRgK][TE] = reinterpret_cast<float (*)[kRgK][TE]>(rg_smem + 2 * kRgK * kRgT);
  const int tid = threadIdx.x;
  const int tx = tid & 15, ty = tid >> 4;
  const int t0 = blockIdx.x * kRgT, e0 = blockIdx.y * TE;
  const int nsplit = gridDim.z;
  const int ck0 = (int)((long)(H / kRgK) * blockIdx.z / nsplit);
  const int ck1 = (int)((long)(H / kRgK) * (blockIdx.z + 1) / nsplit);
  const int nck = ck1 - ck0;
  // loader roles: x token tid/2, 16 elements from (tid%2)*16; w expert tid/WPR, 4 WF4 from (tid%WPR)*4 WF4
  const int lt = tid >> 1, lk = (tid & 1) * 16;
  const int le = tid / WPR, lkw = (tid % WPR) * 4 * WF4;
  const bool xok = t0 + lt < T, wok = e0 + le < E;
  const uint16_t *xrow = x + (size_t)(t0 + lt) * H + lk;
  const float *wrow = w + (size_t)(e0 + le) * H + lkw;
  uint4 xr0, xr1;
  float4 wr[WF4];
  auto fetch = [&](int c) {
    const int k0 = (ck0 + c) * kRgK;
    if (xok) {
      xr0 = __ldg(reinterpret_cast<const uint4 *>(xrow + k0));
      xr1 = __ldg(reinterpret_cast<const uint4 *>(xrow + k0 + 8));
    } else {
      xr0 = xr1 = make_uint4(0u, 0u, 0u, 0u);
    }
#pragma unroll
    for (int q = 0; q < WF4; ++q)
      wr[q] = wok ? __ldg(reinterpret_cast<const float4 *>(wrow + k0) + q) : make_float4(0.f, 0.f, 0.f, 0.f);
  };
  auto stash = [&](int b) {
    const uint32_t xv[8] = {xr0.x, xr0.y, xr0.z, xr0.w, xr1.x, xr1.y, xr1.z, xr1.w};
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      xs[b][lk + 2 * i][lt] = __uint_as_float(xv[i] << 16);
      xs[b][lk + 2 * i + 1][lt] = __uint_as_float(xv[i] & 0xFFFF0000u);
    }
#pragma unroll
    for (int q = 0; q < WF4; ++q) {
      ws[b][lkw + 4 * q + 0][le] = wr[q].x;
      ws[b][lkw + 4 * q + 1][le] = wr[q].y;
      ws[b][lkw + 4 * q + 2][le] = wr[q].z;
      ws[b][lkw + 4 * q + 3][le] = wr[q].w;
    }
  };
  float acc[8][JN];
#pragma unroll
  for (int i = 0; i < 8; ++i)
#pragma unroll
    for (int j = 0; j < JN; ++j) acc[i][j] = 0.0f;
  fetch(0);
  stash(0);
  __syncthreads();
  for (int c = 0; c < nck; ++c) {
    const int b = c & 1;
    if (c + 1 < nck) fetch(c + 1);
    // chunk partials as pairs of adjacent experts: one packed fp32 FMA
    // (two IEEE fmaf, the same per-element sequence) per pair
    float2 part[8][JN / 2];
#pragma unroll
    for (int i = 0; i < 8; ++i)
#pragma unroll
      for (int j = 0; j < JN / 2; ++j) part[i][j] = make_float2(0.0f, 0.0f);
#pragma unroll 4
    for (int k = 0; k < kRgK; ++k) {
      const float4 a0 = *reinterpret_cast<const float4 *>(&xs[b][k][ty * 4]);
      const float4 a1 = *reinterpret_cast<const float4 *>(&xs[b][k][64 + ty * 4]);
      const float av[8] = {a0.x, a0.y, a0.z, a0.w, a1.x, a1.y, a1.z, a1.w};
      float2 bv[JN / 2];
      const float4 b0 = *reinterpret_cast<const float4 *>(&ws[b][k][tx * 4]);
      bv[0] = make_float2(b0.x, b0.y);
      bv[1] = make_float2(b0.z, b0.w);
      if constexpr (JN == 8) {
        const float4 b1 = *reinterpret_cast<const float4 *>(&ws[b][k][64 + tx * 4]);
        bv[2] = make_float2(b1.x, b1.y);
        bv[3] = make_float2(b1.z, b1.w);
      }
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        const float2 ai = make_float2(av[i], av[i]);
#pragma unroll
        for (int j = 0; j < JN / 2; ++j) part[i][j] = __ffma2_rn(ai, bv[j], part[i][j]);
      }
    }
#pragma unroll
    for (int i = 0; i < 8; ++i)
#pragma unroll
      for (int j = 0; j < JN / 2; ++j) {
        acc[i][2 * j] += part[i][j].x;
        acc[i][2 * j + 1] += part[i][j].y;
      }
    if (c + 1 < nck) stash(b ^ 1);
    __syncthreads();
  }
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    const int t = t0 + ty * 4 + (i & 3) + 64 * (i >> 2);
    if (t >= T) continue;
#pragma unroll
    for (int j = 0; j < JN; ++j) {
      const int e = e0 + tx * 4 + (j & 3) + 64 * (j >> 2);
      if (e >= E) continue;
      if (nsplit == 1) logits[(size_t)t * E + e] = acc[i][j] + (bias ? bias[e] : 0.0f);
      else parts[((size_t)blockIdx.z * T + t) * E + e] = acc[i][j];
    }
  }
}

static int router_gemm_te(int E) { return E <= 64 ? 64 : 128; }

int router_gemm_splits(int T, int H, int E, size_t part_floats) {
  const int te = router_gemm_te(E);
  const int tiles = ((T + kRgT - 1) / kRgT) * ((E + te - 1) / te);
  int sp = 1;
  while (sp < 8 && tiles * sp < 2 * 148 && (H / kRgK) / (sp * 2) >= 4 &&
         (size_t)(sp * 2) * T * E <= part_floats)
    sp *= 2;
  return sp;
}

template <int JN>
static void launch_router_gemm_jn(const uint16_t *x, const float *w, const float *bias, int T, int H, int E,
                                  float *logits, float *parts, int splits, cudaStream_t s) {
  constexpr size_t smem = router_gemm_smem<JN>();
  cudaFuncSetAttribute(router_gemm_kernel<JN>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  dim3 grid((T + kRgT - 1) / kRgT, (E + 16 * JN - 1) / (16 * JN), splits);
  router_gemm_kernel<JN><<<grid, 256, smem, s>>>(x, w, bias, T, H, E, logits, parts);
}

void launch_router_gemm(const uint16_t *x, const float *w, const float *bias, int T, int H, int E, float *logits,
                        float *parts, int splits, cudaStream_t s) {
  if (router_gemm_te(E) == 64) launch_router_gemm_jn<4>(x, w, bias, T, H, E, logits, parts, splits, s);
  else launch_router_gemm_jn<8>(x, w, bias, T, H, E, logits, parts, splits, s);
}

// Top-k of tokens whose logits are in memory: warp per token.
// With splits > 1 the logits are first assembled from the K parts (in split
// order, plus the bias) and written out.
template <int KPER>
__global__ void __launch_bounds__(256) topk_kernel(float *logits, const float *parts, int splits,
                                                   const float *bias, int T, int E, int E_t, int k, int scoring,
                                                   int renorm, int *ids, float *gates) {
  wait_prior_grid();
  const int t = blockIdx.x * 8 + (threadIdx.x >> 5), lane = threadIdx.x & 31;
  if (t >= T) return;
  float *lrow = logits + (size_t)t * E;
  if (splits > 1) {
    // every logit row of the token (targets and a shared-expert gate row)
    for (int ee = lane; ee < E; ee += 32) {
      float v = __ldcg(parts + (size_t)t * E + ee);
      for (int sp = 1; sp < splits; ++sp) v += __ldcg(parts + ((size_t)sp * T + t) * E + ee);
      v += bias ? bias[ee] : 0.0f;
      lrow[ee] = v;
    }
    __syncwarp();
  }
  float lv[KPER];
#pragma unroll
  for (int i = 0; i < KPER; ++i) {
    const int ee = lane + 32 * i;
    lv[i] = ee < E_t ? __ldcg(lrow + ee) : -INFINITY;
  }
  topk_warp<KPER>(lv, E_t, k, ids + (size_t)t * k, gates + (size_t)t * k, nullptr, scoring, renorm);
}

void launch_topk(float *logits, const float *parts, int splits, const float *bias, int T, int E, int E_t, int k,
                 int scoring, int renorm, int *ids, float *gates, cudaStream_t s) {
  const int blocks = (T + 7) / 8;
#define MOE_TOPK_ARGS logits, parts, splits, bias, T, E, E_t, k, scoring, renorm, ids, gates
  if (E_t <= 64) launch_dependent(topk_kernel<2>, blocks, 256, 0, s, MOE_TOPK_ARGS);
  else if (E_t <= 128) launch_dependent(topk_kernel<4>, blocks, 256, 0, s, MOE_TOPK_ARGS);
  else if (E_t <= 256) launch_dependent(topk_kernel<8>, blocks, 256, 0, s, MOE_TOPK_ARGS);
  else if (E_t <= 512) launch_dependent(topk_kernel<16>, blocks, 256, 0, s, MOE_TOPK_ARGS);
  else launch_dependent(topk_kernel<32>, blocks, 256, 0, s, MOE_TOPK_ARGS);
#undef MOE_TOPK_ARGS
}

void launch_combine(const CombineArgs &a, cudaStream_t s) {
  const size_t n = (size_t)a.T * (a.H / 4);
  int blocks = (int)((n + 255) / 256);
  blocks = blocks > 148 * 8 ? 148 * 8 : blocks;
  if (blocks < 1) blocks = 1;
  launch_dependent(combine_kernel, blocks, 256, 0, s, a);
}

}  // namespace moe
