// route_noalloc.cu -- router + softmax top-k for callers that cannot allocate.
//
// Some callers may not allocate device memory when they call in: a serving
// loop that plans every byte of HBM once at start-up and hands the library only
// its own buffers, or a latency-critical path that must not pay the device-wide
// synchronisation that cudaMalloc/cudaFree imply.  moe_route_topk_noalloc gives
// them the routing step (fp32 router logits, top-k ids in descending order with
// the lower index first on ties, renormalised softmax gates) with no allocation
// of any kind: the kernel's scratch (the logits and the per-tile completion
// counters) lives in one file-scope __device__ array of fixed size, which every
// GPU that loads this library holds until the process exits.
//
// Host code must not use the array's name as a device address (on the host it
// is only a stand-in symbol).  The address is fetched once per device, with the
// device current, by cudaGetSymbolAddress during the first call on that device;
// that first call should therefore come before any stream capture.
//
// All calls share the one array and it keeps the last call's contents: the
// counters are cleared at the start of every call, and calls whose work
// overlaps on the GPU (different streams, or different host threads on one
// device) race on the array and must be serialised by the caller.
#include <mutex>
#include <string>

#include "device_utils.cuh"
#include "moe_internal.h"
#include "route_common.cuh"

namespace moe {
const char *set_error_text(const std::string &s);   // defined in api.cu
}

namespace {

constexpr int kTT = 4;                    // tokens per CTA
constexpr int kEB = 8;                    // experts per CTA (one per warp)
constexpr size_t kMaxLogits = 1u << 20;   // T * E fp32 logits
constexpr int kMaxTokens = 65536;
constexpr size_t kCounterOff = kMaxLogits * sizeof(float);
constexpr size_t kScratchBytes = kCounterOff + (size_t)(kMaxTokens / kTT) * sizeof(int);

__device__ __align__(256) unsigned char g_route_scratch[kScratchBytes];

struct StaticRouteArgs {
  const uint16_t *x;
  const float *w;
  const float *bias;
  int T, H, E, k;
  float *logits;      // scratch
  int *counter;       // scratch, zero at launch
  int *ids;
  float *gates;
};

__global__ void __launch_bounds__(256) route_static_kernel(const StaticRouteArgs a) {
  extern __shared__ float xt[];   // [kTT][H]
  __shared__ int is_last;
  const int H = a.H, E = a.E;
  const int t0 = blockIdx.x * kTT;
  const int nt = min(kTT, a.T - t0);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  for (int i = threadIdx.x; i < nt * H; i += blockDim.x) {
    const int t = i / H, h = i % H;
    xt[i] = moe::bf16_bits_to_float(a.x[(size_t)(t0 + t) * H + h]);
  }
  __syncthreads();
  const int e = blockIdx.y * kEB + warp;
  if (e < E) {
    float acc[kTT] = {0.f, 0.f, 0.f, 0.f};
    const float *w = a.w + (size_t)e * H;
    for (int h = lane * 4; h < H; h += 128) {
      const float4 wv = *reinterpret_cast<const float4 *>(w + h);
#pragma unroll
      for (int t = 0; t < kTT; ++t) {
        if (t < nt) {
          const float4 xv = *reinterpret_cast<const float4 *>(xt + t * H + h);
          acc[t] = fmaf(wv.x, xv.x, acc[t]);
          acc[t] = fmaf(wv.y, xv.y, acc[t]);
          acc[t] = fmaf(wv.z, xv.z, acc[t]);
          acc[t] = fmaf(wv.w, xv.w, acc[t]);
        }
      }
    }
#pragma unroll
    for (int t = 0; t < kTT; ++t) {
      float v = acc[t];
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
      if (lane == 0 && t < nt) a.logits[(size_t)(t0 + t) * E + e] = v + (a.bias ? a.bias[e] : 0.0f);
    }
  }
  __threadfence();
  __syncthreads();
  if (threadIdx.x == 0) is_last = (atomicAdd(&a.counter[blockIdx.x], 1) == (int)gridDim.y - 1);
  __syncthreads();
  if (!is_last) return;
  __threadfence();
  if (warp >= nt) return;
  const int t = t0 + warp;
  constexpr int kPer = moe::kMaxExperts / 32;
  float lv[kPer];
#pragma unroll
  for (int i = 0; i < kPer; ++i) {
    const int ee = lane + 32 * i;
    lv[i] = (ee < E) ? __ldcg(a.logits + (size_t)t * E + ee) : -INFINITY;
  }
  // the same warp top-k and gate arithmetic as moe_forward's routing step
  moe::topk_warp<kPer>(lv, E, a.k, a.ids + (size_t)t * a.k, a.gates + (size_t)t * a.k, nullptr);
}

std::mutex g_setup_mu;
void *g_scratch_ptr[256] = {};   // per device ordinal

moe_status_t scratch_for_current_device(unsigned char **out) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess || dev < 0 || dev >= 256) {
    moe::set_error_text(std::string("cudaGetDevice failed: ") + cudaGetErrorString(e));
    return MOE_ERR_CUDA;
  }
  std::lock_guard<std::mutex> lock(g_setup_mu);
  if (!g_scratch_ptr[dev]) {
    void *p = nullptr;
    e = cudaGetSymbolAddress(&p, g_route_scratch);
    if (e != cudaSuccess || !p) {
      moe::set_error_text(std::string("cudaGetSymbolAddress(route scratch) failed: ") + cudaGetErrorString(e));
      return MOE_ERR_CUDA;
    }
    g_scratch_ptr[dev] = p;
  }
  *out = static_cast<unsigned char *>(g_scratch_ptr[dev]);
  return MOE_OK;
}

// Largest dynamic shared memory the routing kernel may use on the current
// device: the per-block opt-in limit less the kernel's static shared memory.
moe_status_t shared_limit_for_current_device(size_t *out) {
  int dev = 0, optin = 0;
  cudaFuncAttributes fa{};
  cudaError_t e = cudaGetDevice(&dev);
  if (e == cudaSuccess) e = cudaDeviceGetAttribute(&optin, cudaDevAttrMaxSharedMemoryPerBlockOptin, dev);
  if (e == cudaSuccess) e = cudaFuncGetAttributes(&fa, route_static_kernel);
  if (e != cudaSuccess) {
    moe::set_error_text(std::string("moe_route_topk_noalloc: ") + cudaGetErrorString(e));
    return MOE_ERR_CUDA;
  }
  *out = (size_t)optin > fa.sharedSizeBytes ? (size_t)optin - fa.sharedSizeBytes : 0;
  return MOE_OK;
}

}  // namespace

extern "C" moe_status_t moe_route_topk_noalloc(const void *x, int32_t T, int32_t H, const float *router_w,
                                               const float *router_bias, int32_t E, int32_t k, int32_t *ids,
                                               float *gates, float *logits, void *stream) {
  if (T < 0 || H <= 0 || H % 4 || E < 1 || E > moe::kMaxExperts || k < 1 || k > E || k > moe::kMaxTopK) {
    moe::set_error_text("moe_route_topk_noalloc: need T >= 0, H > 0 a multiple of 4, 1 <= E <= 1024, 1 <= k <= min(E, 32)");
    return MOE_ERR_INVALID_ARG;
  }
  if (T == 0) return MOE_OK;
  if (!x || !router_w || !ids || !gates) {
    moe::set_error_text("moe_route_topk_noalloc: x, router_w, ids and gates must be device pointers");
    return MOE_ERR_INVALID_ARG;
  }
  if (T > kMaxTokens || (size_t)T * (size_t)E > kMaxLogits) {
    moe::set_error_text("moe_route_topk_noalloc: T * E exceeds the fixed scratch of 2^20 logits (or T > 65536); "
                        "split the batch or use moe_forward");
    return MOE_ERR_INVALID_ARG;
  }
  if (reinterpret_cast<uintptr_t>(router_w) & 15u) {
    moe::set_error_text("moe_route_topk_noalloc: router_w must be 16-byte aligned (its rows are read as float4)");
    return MOE_ERR_INVALID_ARG;
  }
  unsigned char *scratch = nullptr;
  moe_status_t st = scratch_for_current_device(&scratch);
  if (st != MOE_OK) return st;
  // the kernel's token tile (kTT rows of x in fp32) plus its static shared
  // memory must fit the per-block limit of the device
  const size_t smem = (size_t)kTT * H * sizeof(float);
  size_t smem_limit = 0;
  st = shared_limit_for_current_device(&smem_limit);
  if (st != MOE_OK) return st;
  if (smem > smem_limit) {
    const size_t hmax = (smem_limit / (kTT * sizeof(float))) & ~(size_t)3;
    moe::set_error_text("moe_route_topk_noalloc: H too large for the shared-memory token tile (H <= " +
                        std::to_string(hmax) + " on this device)");
    return MOE_ERR_INVALID_ARG;
  }
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  const int tiles = (T + kTT - 1) / kTT;
  int *counter = reinterpret_cast<int *>(scratch + kCounterOff);
  cudaError_t e = cudaMemsetAsync(counter, 0, (size_t)tiles * sizeof(int), s);
  if (e == cudaSuccess && smem > 48 * 1024)
    e = cudaFuncSetAttribute(route_static_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) {
    moe::set_error_text(std::string("moe_route_topk_noalloc: ") + cudaGetErrorString(e));
    return MOE_ERR_CUDA;
  }
  StaticRouteArgs a;
  a.x = static_cast<const uint16_t *>(x);
  a.w = router_w;
  a.bias = router_bias;
  a.T = T; a.H = H; a.E = E; a.k = k;
  a.logits = reinterpret_cast<float *>(scratch);
  a.counter = counter;
  a.ids = ids;
  a.gates = gates;
  dim3 grid(tiles, (E + kEB - 1) / kEB);
  route_static_kernel<<<grid, 256, smem, s>>>(a);
  e = cudaGetLastError();
  if (e == cudaSuccess && logits)
    e = cudaMemcpyAsync(logits, a.logits, (size_t)T * E * sizeof(float), cudaMemcpyDeviceToDevice, s);
  if (e != cudaSuccess) {
    moe::set_error_text(std::string("moe_route_topk_noalloc: ") + cudaGetErrorString(e));
    return MOE_ERR_CUDA;
  }
  return MOE_OK;
}
