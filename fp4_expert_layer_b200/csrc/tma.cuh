// tma.cuh -- mbarrier, TMA and bulk-copy helpers (sm_100a inline PTX).
#pragma once

#include <stdint.h>

namespace moe {

// A wait gives up after this much GPU wall time (or at once when another wait
// has already recorded an error), records an error code and lets the kernel run
// to completion, so that no wait can run forever.
constexpr unsigned long long kWaitLimitNs = 2000000000ull;

// The error word the kernels share: a device-memory int that the bounded
// waits poll (a read of mapped host memory would cross PCIe at every check),
// followed by the address of the mapped host word that the host reads without
// synchronising.  A failure is recorded in both.
struct ErrWord {
  int code;
  int pad;
  int *host;
};
__device__ __forceinline__ void record_error(int *err, int code) {
  atomicExch(err, code);
  int *host = reinterpret_cast<ErrWord *>(err)->host;
  if (host) atomicExch(host, code);
}
// The same, keeping the first code recorded.
__device__ __forceinline__ void record_first_error(int *err, int code) {
  if (atomicCAS(err, 0, code) != 0) return;
  int *host = reinterpret_cast<ErrWord *>(err)->host;
  if (host) atomicCAS(host, 0, code);
}

__device__ __forceinline__ unsigned long long global_ns() {
  unsigned long long t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
  return t;
}

__device__ __forceinline__ uint32_t smem_u32(const void *p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ void mbar_init(uint32_t bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(bar), "r"(count) : "memory");
}

__device__ __forceinline__ void mbar_fence_init() {
  asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}

__device__ __forceinline__ void mbar_arrive_expect_tx(uint32_t bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(bar), "r"(bytes) : "memory");
}

__device__ __forceinline__ void mbar_arrive(uint32_t bar) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(bar) : "memory");
}

__device__ __forceinline__ bool mbar_try_wait(uint32_t bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(bar), "r"(parity)
      : "memory");
  return ok != 0;
}

// Bounded wait for phase `parity` of a barrier.  Returns false (and records
// `code` in *err) when the limit is reached or another wait already failed.
__device__ __forceinline__ bool mbar_wait(uint32_t bar, uint32_t parity, int *err, int code) {
  if (mbar_try_wait(bar, parity)) return true;
  const unsigned long long t0 = global_ns();
  for (uint32_t i = 1;; ++i) {
    if (mbar_try_wait(bar, parity)) return true;
    if ((i & 255u) == 0) {
      if (err && *(volatile int *)err != 0) return false;
      if (global_ns() - t0 > kWaitLimitNs) {
        if (err) record_error(err, code);
        return false;
      }
    }
  }
}

// The same wait by every lane of a warp, true only when it succeeded for all
// of them.  The result is warp-uniform, so the loop around it stays convergent:
// an MMA-issuing loop run by a whole warp, with one elected lane issuing,
// keeps its descriptors in uniform registers, and issues about twice as fast
// as the same loop run by one lane behind a lane test.
__device__ __forceinline__ bool mbar_wait_warp(uint32_t bar, uint32_t parity, int *err, int code) {
  return __all_sync(0xffffffffu, mbar_wait(bar, parity, err, code));
}

// Counters between kernels: the writer fences its data, then bumps the
// counter; the reader acquires it before reading the data.
__device__ __forceinline__ int flag_acquire(const int *f) {
  int v;
  asm volatile("ld.acquire.gpu.global.b32 %0, [%1];" : "=r"(v) : "l"(f) : "memory");
  return v;
}
// Bounded wait until *f == v; false (and `code` in *err) past the limit or
// once another wait has failed.
__device__ __forceinline__ bool flag_wait(const int *f, int v, int *err, int code) {
  if (flag_acquire(f) == v) return true;
  const unsigned long long t0 = global_ns();
  for (uint32_t i = 1;; ++i) {
    if (flag_acquire(f) == v) return true;
    if ((i & 63u) == 0) {
      if (err && *(volatile int *)err != 0) return false;
      if (global_ns() - t0 > kWaitLimitNs) {
        if (err) record_error(err, code);
        return false;
      }
    }
  }
}

// 3-D tiled TMA load of one box into this CTA's shared memory.
__device__ __forceinline__ void tma_load_3d(uint32_t dst, const void *tmap, uint32_t bar, int c0, int c1,
                                            int c2) {
  asm volatile(
      "cp.async.bulk.tensor.3d.shared::cluster.global.tile.mbarrier::complete_tx::bytes [%0], [%1, {%3, %4, "
      "%5}], [%2];" ::"r"(dst),
      "l"(reinterpret_cast<uint64_t>(tmap)), "r"(bar), "r"(c0), "r"(c1), "r"(c2)
      : "memory");
}

// 4-D tiled TMA load of one box into this CTA's shared memory.
__device__ __forceinline__ void tma_load_4d(uint32_t dst, const void *tmap, uint32_t bar, int c0, int c1, int c2,
                                            int c3) {
  asm volatile(
      "cp.async.bulk.tensor.4d.shared::cluster.global.tile.mbarrier::complete_tx::bytes [%0], [%1, {%3, %4, "
      "%5, %6}], [%2];" ::"r"(dst),
      "l"(reinterpret_cast<uint64_t>(tmap)), "r"(bar), "r"(c0), "r"(c1), "r"(c2), "r"(c3)
      : "memory");
}

// Fetch a tensor map into the descriptor cache ahead of its first use.
__device__ __forceinline__ void tmap_prefetch(const void *tmap) {
  asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(tmap)) : "memory");
}

// Contiguous bulk copy global -> this CTA's shared memory (16-byte aligned, size % 16 == 0).
__device__ __forceinline__ void bulk_load(uint32_t dst, const void *src, uint32_t bytes, uint32_t bar) {
  asm volatile("cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(dst),
               "l"(src), "r"(bytes), "r"(bar)
               : "memory");
}

// Wait for a barrier phase with a time limit only (drains copies in flight on
// an error path; ignores the error word).
__device__ __forceinline__ void mbar_drain(uint32_t bar, uint32_t parity) {
  const unsigned long long t0 = global_ns();
  while (!mbar_try_wait(bar, parity))
    if (global_ns() - t0 > kWaitLimitNs) return;
}

__device__ __forceinline__ void named_bar_sync(int id, int threads) {
  asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(threads) : "memory");
}

// Named barrier over `threads` threads that also ANDs a predicate across them.
__device__ __forceinline__ bool named_bar_and(int id, int threads, bool pred) {
  uint32_t r;
  asm volatile(
      "{\n\t.reg .pred p, q;\n\t"
      "setp.ne.u32 p, %1, 0;\n\t"
      "barrier.red.and.pred q, %2, %3, p;\n\t"
      "selp.u32 %0, 1, 0, q;\n\t}"
      : "=r"(r)
      : "r"((uint32_t)pred), "r"(id), "r"(threads)
      : "memory");
  return r != 0;
}

__device__ __forceinline__ void sts128(uint32_t addr, uint4 v) {
  asm volatile("st.shared.v4.u32 [%0], {%1,%2,%3,%4};" ::"r"(addr), "r"(v.x), "r"(v.y), "r"(v.z), "r"(v.w)
               : "memory");
}

__device__ __forceinline__ uint4 lds128(uint32_t addr) {
  uint4 v;
  asm volatile("ld.shared.v4.u32 {%0,%1,%2,%3}, [%4];" : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w) : "r"(addr)
               : "memory");
  return v;
}

}  // namespace moe
