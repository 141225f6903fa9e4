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

  // x tile -> smem (fp32)
  for (int i = threadIdx.x; i < nt * H / 2; i += blockDim.x) {
    const int t = (2 * i) / H, h = (2 * i) % H;
    uint32_t v = *reinterpret_cast<const uint32_t *>(a.x + (size_t)(t0 + t) * H + h);
    xs_smem[t * H + h] = __uint_as_float(v << 16);
    xs_smem[t * H + h + 1] = __uint_as_float(v & 0xFFFF0000u);
  }
  __syncthreads();

  // logits: warp w -> expert e
  const int e = blockIdx.y * kRouterEB + warp;
  if (e < E) {
    float acc[kRouterTT];
#pragma unroll
    for (int t = 0; t < kRouterTT; ++t) acc[t] = 0.0f;
    const float *w = a.w + (size_t)e * H;
    // 8 independent 16-byte loads in flight per lane before any use
    for (int h0 = lane * 4; h0 < H; h0 += 128 * 8) {
      float4 wv[8];
#pragma unroll
      for (int u = 0; u < 8; ++u) {
        const int h = h0 + u * 128;
        wv[u] = h < H ? __ldg(reinterpret_cast<const float4 *>(w + h)) : make_float4(0.f, 0.f, 0.f, 0.f);
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
      lv[i] = (ee < E) ? __ldcg(lrow + ee) : -INFINITY;
    }
    topk_warp<KPER>(lv, E, a.k, a.ids + (size_t)t * a.k, a.gates + (size_t)t * a.k, nullptr);
  }
  if (!a.fuse_perm) return;

  // the last token tile to finish top-k runs the permutation
  __threadfence();
  __syncthreads();
  if (threadIdx.x == 0) is_last = (atomicAdd(a.tiles_done, 1) == (int)gridDim.x - 1);
  __syncthreads();
  if (!is_last) return;
  __threadfence();
  if (threadIdx.x == 0) *a.tiles_done = 0;
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
  if (a.E <= 64) launch_router_k<2>(a, s);
  else if (a.E <= 128) launch_router_k<4>(a, s);
  else if (a.E <= 256) launch_router_k<8>(a, s);
  else if (a.E <= 512) launch_router_k<16>(a, s);
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
// Expert pointer table for one pass: start from the resident table (or all
// null) and overwrite the listed experts.
// ---------------------------------------------------------------------------
__global__ void ptr_update_kernel(const PtrUpdate u, const uint8_t *const *resident,
                                  const uint8_t **out) {
  for (int e = threadIdx.x; e < u.E; e += blockDim.x) out[e] = u.keep_resident ? resident[e] : nullptr;
  __syncthreads();
  for (int i = threadIdx.x; i < u.n; i += blockDim.x) out[u.expert[i]] = u.ptr[i];
}

void launch_ptr_update(const PtrUpdate &u, const uint8_t *const *resident, const uint8_t **out,
                       cudaStream_t s) {
  ptr_update_kernel<<<1, 256, 0, s>>>(u, resident, out);
}

// ---------------------------------------------------------------------------
// Ordered combine: y[t] = sum_{j<k} O'[t*k + j] (in j order) + s[t].
// ---------------------------------------------------------------------------
__global__ void combine_kernel(const CombineArgs a) {
  wait_prior_grid();
  const int H4 = a.H / 4;
  const size_t n = (size_t)a.T * H4;
  for (size_t i = blockIdx.x * (size_t)blockDim.x + threadIdx.x; i < n;
       i += (size_t)gridDim.x * blockDim.x) {
    const size_t t = i / H4, c = i % H4;
    const float4 *o = reinterpret_cast<const float4 *>(a.oprime) + t * a.k * H4 + c;
    float4 acc = __ldcs(o);
    for (int j = 1; j < a.k; ++j) {
      const float4 v = __ldcs(o + (size_t)j * H4);
      acc.x += v.x; acc.y += v.y; acc.z += v.z; acc.w += v.w;
    }
    if (a.shared) {
      const float4 v = reinterpret_cast<const float4 *>(a.shared)[t * H4 + c];
      acc.x += v.x; acc.y += v.y; acc.z += v.z; acc.w += v.w;
    }
    reinterpret_cast<float4 *>(a.y)[t * H4 + c] = acc;
  }
}

void launch_combine(const CombineArgs &a, cudaStream_t s) {
  const size_t n = (size_t)a.T * (a.H / 4);
  int blocks = (int)((n + 255) / 256);
  blocks = blocks > 148 * 8 ? 148 * 8 : blocks;
  if (blocks < 1) blocks = 1;
  launch_dependent(combine_kernel, blocks, 256, 0, s, a);
}

}  // namespace moe
