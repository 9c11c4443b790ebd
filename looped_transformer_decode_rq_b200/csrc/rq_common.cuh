// rq_common.cuh -- device helpers shared by the sm_100a kernels: mbarrier and
// bulk/tensor-copy wrappers (inline PTX, no cluster multicast anywhere),
// bounded waits, bf16 unpacking and the status word.
#pragma once

#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "../../include/rq_api.h"

namespace rq {

constexpr int kD = RQ_HEAD_DIM;     // head_dim
constexpr int kPage = RQ_PAGE_TOKENS;

// ---------------------------------------------------------------------------
// status word
// ---------------------------------------------------------------------------
__device__ __forceinline__ void set_flag(int32_t* status, uint32_t bit) {
  if (status != nullptr) atomicOr(reinterpret_cast<unsigned int*>(status), bit);
}

// ---------------------------------------------------------------------------
// shared-memory addresses and mbarriers
// ---------------------------------------------------------------------------
__device__ __forceinline__ uint32_t smem_u32(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ void mbar_init(uint32_t bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(bar), "r"(count) : "memory");
}

// Programmatic dependent launch (sm_90 and later).  Each decode kernel lets the
// kernel that follows it on the stream (launched with programmatic stream
// serialization) be scheduled early; the follower does its input-only set-up,
// then waits in pdl_wait() until its predecessor has completed and its writes
// are visible.  This takes launches and set-up off the critical path.
__device__ __forceinline__ void pdl_launch_dependents() {
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}
__device__ __forceinline__ void pdl_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }

// Launches `kern` as a programmatic dependent of the previous kernel on
// stream `s`: it may be scheduled once that kernel has called
// pdl_launch_dependents() (or exited), and must call pdl_wait() before it
// touches memory the previous kernel writes or reads.
template <typename... Params, typename... Args>
inline cudaError_t launch_dependent(void (*kern)(Params...), unsigned grid, unsigned block, size_t smem,
                                    cudaStream_t s, Args&&... args) {
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(grid, 1, 1);
  cfg.blockDim = dim3(block, 1, 1);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = s;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  const cudaError_t e = cudaLaunchKernelEx(&cfg, kern, static_cast<Args&&>(args)...);
  return e != cudaSuccess ? e : cudaGetLastError();
}

__device__ __forceinline__ void fence_barrier_init() {
  asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}

__device__ __forceinline__ void fence_proxy_async_smem() {
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

__device__ __forceinline__ void mbar_arrive_expect_tx(uint32_t bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(bar), "r"(bytes)
               : "memory");
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

// Non-blocking test of a phase (never suspends the thread).
__device__ __forceinline__ bool mbar_test_wait(uint32_t bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.test_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(bar), "r"(parity)
      : "memory");
  return ok != 0;
}

__device__ __forceinline__ uint64_t global_timer_ns() {
  uint64_t t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
  return t;
}

// Every wait in these kernels is bounded: after kWaitLimitNs the caller gets
// `false`, records RQ_FLAG_PIPE_TIMEOUT and winds the CTA down.  A decode call
// takes well under a millisecond, so two seconds is never reached by a
// healthy pipeline.
constexpr uint64_t kWaitLimitNs = 2000000000ull;

// A try-wait that may suspend the thread for up to `hint_ns` while the phase
// is incomplete (it returns as soon as the phase completes), so that a waiting
// warp spends few issue slots polling.
__device__ __forceinline__ bool mbar_try_wait_hint(uint32_t bar, uint32_t parity, uint32_t hint_ns) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2, %3;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(bar), "r"(parity), "r"(hint_ns)
      : "memory");
  return ok != 0;
}

__device__ __forceinline__ bool mbar_wait_bounded(uint32_t bar, uint32_t parity) {
  if (mbar_try_wait(bar, parity)) return true;
  const uint64_t t0 = global_timer_ns();
  while (true) {
    if (mbar_try_wait_hint(bar, parity, 20000u)) return true;
    if (global_timer_ns() - t0 > kWaitLimitNs) return false;
  }
}

// ---------------------------------------------------------------------------
// bulk copies global -> shared, completion counted on an mbarrier.
// Non-multicast forms only.
// ---------------------------------------------------------------------------
__device__ __forceinline__ void bulk_g2s(uint32_t dst, const void* src, uint32_t bytes,
                                         uint32_t bar) {
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
          dst),
      "l"(src), "r"(bytes), "r"(bar)
      : "memory");
}

// 4-D tiled tensor copy (coordinates innermost first).
__device__ __forceinline__ void tma_load_4d(uint32_t dst, const CUtensorMap* map, int c0, int c1,
                                            int c2, int c3, uint32_t bar) {
  asm volatile(
      "cp.async.bulk.tensor.4d.shared::cluster.global.tile.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%2, %3, %4, %5}], [%6];" ::"r"(dst),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(c0), "r"(c1), "r"(c2), "r"(c3), "r"(bar)
      : "memory");
}

__device__ __forceinline__ void prefetch_tensormap(const CUtensorMap* map) {
  asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(map)) : "memory");
}

// named barrier among `count` threads (a multiple of 32)
__device__ __forceinline__ void named_bar_sync(int id, int count) {
  asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(count) : "memory");
}

// ---------------------------------------------------------------------------
// number formats
// ---------------------------------------------------------------------------
// two bf16 packed in a 32-bit word -> (low, high) as fp32 (exact)
__device__ __forceinline__ float2 bf16x2_to_f2(uint32_t w) {
  return make_float2(__uint_as_float(w << 16), __uint_as_float(w & 0xFFFF0000u));
}

__device__ __forceinline__ float bf16_bits_to_f(uint32_t lo16) { return __uint_as_float(lo16 << 16); }


// fp16 (scale, offset) pair packed in a 32-bit word
__device__ __forceinline__ float2 half2_bits_to_f2(uint32_t w) {
  __half2 h = *reinterpret_cast<__half2*>(&w);
  return __half22float2(h);
}

// ---------------------------------------------------------------------------
// page walk over the flattened (b, h, page) sequence (pages of any fixed size;
// nt[b] = pages of sequence b, pre[b] = pages of the sequences before b)
// ---------------------------------------------------------------------------
struct PageIter {
  int b, h, page;
  __device__ __forceinline__ void seek(int64_t x, const int* pre, const int* nt, int B, int Hkv) {
    int lo = 0, hi = B - 1;  // largest b with pre[b]*Hkv <= x
    while (lo < hi) {
      const int mid = (lo + hi + 1) >> 1;
      if (static_cast<int64_t>(pre[mid]) * Hkv <= x) lo = mid; else hi = mid - 1;
    }
    b = lo;
    const int64_t r = x - static_cast<int64_t>(pre[b]) * Hkv;
    h = static_cast<int>(r / nt[b]);
    page = static_cast<int>(r % nt[b]);
  }
  __device__ __forceinline__ void next(const int* nt, int B, int Hkv) {
    if (++page < nt[b]) return;
    page = 0;
    if (++h < Hkv) return;
    h = 0;
    do { ++b; } while (b < B && nt[b] == 0);
  }
};

}  // namespace rq
