// rq_static_scratch.cu -- decode attention for callers that cannot allocate.
//
// rq_decode_attention needs a caller-provided workspace for its split-K
// partials.  Some callers have no way to provide one: code hosted inside a
// framework that owns every device allocation and forbids raw cudaMalloc, or
// latency-critical serving loops that must not allocate once they are running
// (cudaMalloc/cudaFree can synchronise the device).  For them this file keeps
// the partials in a fixed-size array in the library's own device memory and
// forwards to rq_decode_attention, unchanged, with that array as workspace.
#include <cuda_runtime.h>

#include <cstdio>
#include <mutex>

#include "../../include/rq_api.h"
#include "rq_internal.h"

namespace {

// Every GPU that loads the library holds this array until the process exits.
constexpr size_t kStaticScratchBytes = RQ_STATIC_SCRATCH_BYTES;
static __device__ __align__(256) unsigned char g_scratch[kStaticScratchBytes];

constexpr int kMaxDevices = 64;
std::mutex g_mu;
void* g_scratch_ptr[kMaxDevices];  // device address of g_scratch, per device (null until set up)

}  // namespace

extern "C" RQ_API rq_status rq_decode_attention_static_scratch(
    const rq_cache* cache, int32_t loop, const void* q, const int32_t* ctx_len, const void* k_tail,
    const void* v_tail, int32_t n_tail, float softmax_scale, float* out, rq_stream_t stream) {
  if (cache == nullptr) return rq::set_last_error(RQ_ERR_INVALID_ARG, "cache is null");
  // the split-K partials of this loop's decode: the same rows per pass over
  // the cache as rq_decode_attention takes
  int64_t need = 0;
  rq_status st = rq::decode_scratch_need(cache, loop, 1, &need);
  if (st != RQ_OK) return st;
  if (need > static_cast<int64_t>(kStaticScratchBytes))
    return rq::set_last_error(RQ_ERR_WORKSPACE,
                              "this cache needs %lld bytes of split-K scratch but the static scratch "
                              "holds %zu; use rq_decode_attention with a caller workspace",
                              static_cast<long long>(need), kStaticScratchBytes);
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return rq::set_last_error(RQ_ERR_CUDA, "cudaGetDevice: %s", cudaGetErrorString(e));
  if (dev < 0 || dev >= kMaxDevices) return rq::set_last_error(RQ_ERR_UNSUPPORTED, "device ordinal %d", dev);
  // The array used is the current device's; the cache's planes must live there too.
  if (dev != rq::cache_device(cache))
    return rq::set_last_error(RQ_ERR_INVALID_ARG,
                              "current device %d is not the device %d the cache was created on", dev,
                              rq::cache_device(cache));
  void* scratch = nullptr;
  {
    // One-time set-up per device, done with that device current: in host code
    // g_scratch names a host-side stand-in, so the kernel must be given the
    // device address that the runtime reports for it.
    std::lock_guard<std::mutex> lock(g_mu);
    if (g_scratch_ptr[dev] == nullptr) {
      void* p = nullptr;
      e = cudaGetSymbolAddress(&p, g_scratch);
      if (e != cudaSuccess || p == nullptr)
        return rq::set_last_error(RQ_ERR_CUDA, "cudaGetSymbolAddress(static scratch): %s", cudaGetErrorString(e));
      g_scratch_ptr[dev] = p;
    }
    scratch = g_scratch_ptr[dev];
  }
  return rq_decode_attention(cache, loop, q, ctx_len, k_tail, v_tail, n_tail, softmax_scale, out, scratch,
                             static_cast<int64_t>(kStaticScratchBytes), stream);
}
