// rq_api.cpp -- host side of the C ABI declared in include/rq_api.h: argument
// validation, cache layout, tensor-map construction and kernel dispatch.  All
// device memory belongs to the caller; nothing here allocates on the device.
#include <cuda.h>
#include <cudaTypedefs.h>
#include <cuda_runtime.h>

#include <cstdarg>
#include <cstdio>
#include <cstring>
#include <mutex>
#include <new>
#include <string>

#include "../../include/rq_api.h"
#include "rq_internal.h"

struct rq_cache {
  rq_config cfg;
  rq_layout lay;
  uint8_t* base;
  int device;
  int num_ctas;
  int decode_kernel;                     // rq_decode_kernel
  int stall_page;                        // test hook (rq_cache_set_debug_stall)
  bool tmaps_ready[RQ_MAX_LOOPS];        // per bf16 anchor loop
  CUtensorMap tm_anchor[RQ_MAX_LOOPS][2];
};

namespace {

thread_local std::string g_msg;

rq_status fail(rq_status s, const char* fmt, ...) {
  char buf[512];
  va_list ap;
  va_start(ap, fmt);
  std::vsnprintf(buf, sizeof(buf), fmt, ap);
  va_end(ap);
  g_msg = buf;
  return s;
}

rq_status cuda_fail(cudaError_t e, const char* what) {
  return fail(RQ_ERR_CUDA, "%s: %s", what, cudaGetErrorString(e));
}

int64_t align_up(int64_t x, int64_t a) { return (x + a - 1) / a * a; }

bool aligned(const void* p, uintptr_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }

PFN_cuTensorMapEncodeTiled_v12000 tensor_map_encoder() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
  });
  return fn;
}

// bf16 plane [B][H][T][128] with element strides (sb, sh, st); tiles of
// 64 tokens x 64 dims with the 128-byte swizzle.
rq_status make_plane_map(CUtensorMap* map, const void* base, int B, int H, int64_t T, int64_t sb,
                         int64_t sh, int64_t st) {
  auto enc = tensor_map_encoder();
  if (enc == nullptr) return fail(RQ_ERR_CUDA, "cuTensorMapEncodeTiled unavailable");
  cuuint64_t dims[4] = {static_cast<cuuint64_t>(RQ_HEAD_DIM), static_cast<cuuint64_t>(T),
                        static_cast<cuuint64_t>(H), static_cast<cuuint64_t>(B)};
  cuuint64_t strides[3] = {static_cast<cuuint64_t>(st * 2), static_cast<cuuint64_t>(sh * 2),
                           static_cast<cuuint64_t>(sb * 2)};
  cuuint32_t box[4] = {64, static_cast<cuuint32_t>(RQ_PAGE_TOKENS), 1, 1};
  cuuint32_t estr[4] = {1, 1, 1, 1};
  CUresult r = enc(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, const_cast<void*>(base), dims, strides, box,
                   estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                   CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) return fail(RQ_ERR_INVALID_ARG, "tensor map rejected (CUresult %d)", static_cast<int>(r));
  return RQ_OK;
}

bool chained(const rq_config& c) {
  return c.anchor_policy == RQ_ANCHOR_PREVIOUS || c.anchor_policy == RQ_ANCHOR_NEXT;
}

// The loop whose (reconstructed) values loop l is stored against (l itself
// for an anchor).
int ref_of(const rq_config& c, int l) {
  const int L = c.num_loops;
  if (c.anchor_policy == RQ_ANCHOR_FIRST) return 0;
  if (c.anchor_policy == RQ_ANCHOR_PREVIOUS) return l > 0 ? l - 1 : 0;
  if (c.anchor_policy == RQ_ANCHOR_NEXT) return l < L - 1 ? l + 1 : L - 1;
  if (c.anchor_policy == RQ_ANCHOR_INTERVAL && c.anchor_interval >= 2) {
    const int n = c.anchor_interval;
    const int a = (l / n) * n + n - 1;
    return a < L - 1 ? a : L - 1;
  }
  return L - 1;
}

// The anchor at the end of loop l's reference chain (l itself for an anchor).
int anchor_of(const rq_config& c, int l) {
  for (int i = 0; i < RQ_MAX_LOOPS && ref_of(c, l) != l; ++i) l = ref_of(c, l);
  return l;
}

rq_status validate_config(const rq_config* c) {
  if (c == nullptr) return fail(RQ_ERR_INVALID_ARG, "config is null");
  if (c->num_loops < 2 || c->num_loops > RQ_MAX_LOOPS)
    return fail(RQ_ERR_INVALID_ARG, "num_loops %d outside [2, %d]", c->num_loops, RQ_MAX_LOOPS);
  if (c->batch < 1) return fail(RQ_ERR_INVALID_ARG, "batch %d < 1", c->batch);
  if (c->kv_heads < 1) return fail(RQ_ERR_INVALID_ARG, "kv_heads %d < 1", c->kv_heads);
  if (c->q_heads < 1 || c->q_heads % c->kv_heads != 0)
    return fail(RQ_ERR_INVALID_ARG, "q_heads %d not a multiple of kv_heads %d", c->q_heads, c->kv_heads);
  const int G = c->q_heads / c->kv_heads;
  if (G != 1 && G != 2 && G != 4 && G != 8)
    return fail(RQ_ERR_UNSUPPORTED, "q_heads / kv_heads = %d (supported: 1, 2, 4, 8)", G);
  if (c->head_dim != RQ_HEAD_DIM) return fail(RQ_ERR_UNSUPPORTED, "head_dim %d != 128", c->head_dim);
  if (c->capacity < 1) return fail(RQ_ERR_INVALID_ARG, "capacity %d < 1", c->capacity);
  if (c->anchor_policy < RQ_ANCHOR_LAST || c->anchor_policy > RQ_ANCHOR_NEXT)
    return fail(RQ_ERR_INVALID_ARG, "anchor_policy %d", c->anchor_policy);
  if (c->anchor_policy == RQ_ANCHOR_INTERVAL && (c->anchor_interval < 2 || c->anchor_interval > c->num_loops))
    return fail(RQ_ERR_INVALID_ARG, "anchor_interval %d outside [2, num_loops]", c->anchor_interval);
  for (int l = 0; l < c->num_loops; ++l) {
    if (anchor_of(*c, l) != l) continue;
    if (c->bits[l] != 16 && c->bits[l] != 4)
      return fail(RQ_ERR_UNSUPPORTED, "anchor loop %d bits %d (supported: 16, 4)", l, c->bits[l]);
    if (c->bits[l] == 4 && c->group[l] != 32)
      return fail(RQ_ERR_UNSUPPORTED, "INT4 anchor loop %d group %d (supported: 32)", l, c->group[l]);
  }
  for (int l = 0; l < c->num_loops; ++l) {
    if (anchor_of(*c, l) == l) continue;
    if (c->bits[l] != 2 && c->bits[l] != 4)
      return fail(RQ_ERR_UNSUPPORTED, "loop %d bits %d (supported: 2, 4)", l, c->bits[l]);
    if (c->group[l] != 16 && c->group[l] != 32)
      return fail(RQ_ERR_UNSUPPORTED, "loop %d group %d (supported: 16, 32)", l, c->group[l]);
    if (c->rotate[l] != 0 && c->rotate[l] != 1)
      return fail(RQ_ERR_INVALID_ARG, "loop %d rotate %d", l, c->rotate[l]);
    if (c->alpha_mode[l] < RQ_ALPHA_LS || c->alpha_mode[l] > RQ_ALPHA_NORM_RATIO)
      return fail(RQ_ERR_INVALID_ARG, "loop %d alpha_mode %d", l, c->alpha_mode[l]);
  }
  if (chained(*c)) {
    // the decode sums every link's rotated residual in one accumulator, so
    // the links share one format; the chain is at most RQ_MAX_CHAIN long
    if (c->num_loops > RQ_MAX_CHAIN + 1)
      return fail(RQ_ERR_UNSUPPORTED, "chained references with %d loops (at most %d)", c->num_loops,
                  RQ_MAX_CHAIN + 1);
    int first = -1;
    for (int l = 0; l < c->num_loops; ++l) {
      if (anchor_of(*c, l) == l) continue;
      if (c->alpha_mode[l] == RQ_ALPHA_ZERO)
        return fail(RQ_ERR_UNSUPPORTED, "chained references with alpha_mode ZERO (loop %d)", l);
      if (first < 0) {
        first = l;
      } else if (c->bits[l] != c->bits[first] || c->group[l] != c->group[first] || c->rotate[l] != c->rotate[first]) {
        return fail(RQ_ERR_UNSUPPORTED, "chained references need one residual format (loops %d and %d differ)",
                    first, l);
      }
    }
  }
  return RQ_OK;
}

// query rows per kv-head a decode call takes: 1, 2, 4, or blocks of 8
bool rows_supported(int rows) { return rows == 1 || rows == 2 || rows == 4 || (rows >= 8 && rows % 8 == 0); }

int ref_kind_for(const rq_config& c, int loop) {
  const int a = anchor_of(c, loop);
  if (loop != a && c.alpha_mode[loop] == RQ_ALPHA_ZERO) return rq::kRefNone;
  return c.bits[a] == 16 ? rq::kRefBf16 : rq::kRefInt4;
}

}  // namespace

namespace rq {
rq_status set_last_error(rq_status s, const char* fmt, ...) {
  char buf[512];
  va_list ap;
  va_start(ap, fmt);
  std::vsnprintf(buf, sizeof(buf), fmt, ap);
  va_end(ap);
  g_msg = buf;
  return s;
}
}  // namespace rq

extern "C" {

const char* rq_status_string(rq_status s) {
  switch (s) {
    case RQ_OK: return "RQ_OK";
    case RQ_ERR_INVALID_ARG: return "RQ_ERR_INVALID_ARG";
    case RQ_ERR_UNSUPPORTED: return "RQ_ERR_UNSUPPORTED";
    case RQ_ERR_CAPACITY: return "RQ_ERR_CAPACITY";
    case RQ_ERR_WORKSPACE: return "RQ_ERR_WORKSPACE";
    case RQ_ERR_CUDA: return "RQ_ERR_CUDA";
    case RQ_ERR_DEVICE_FLAG: return "RQ_ERR_DEVICE_FLAG";
  }
  return "RQ_UNKNOWN_STATUS";
}

const char* rq_last_error_message(void) { return g_msg.c_str(); }

rq_status rq_cache_layout(const rq_config* cfg, rq_layout* out) {
  if (out == nullptr) return fail(RQ_ERR_INVALID_ARG, "layout output is null");
  rq_status st = validate_config(cfg);
  if (st != RQ_OK) return st;
  rq_layout L;
  std::memset(&L, 0, sizeof(L));
  const int64_t cap_pad = align_up(cfg->capacity, RQ_PAGE_TOKENS);
  const int64_t recs = static_cast<int64_t>(cfg->batch) * cfg->kv_heads * cap_pad;
  int64_t off = 0;
  auto place = [&](int64_t bytes) {
    const int64_t o = off;
    off = align_up(off + bytes, 1024);
    return o;
  };
  L.capacity_padded = cap_pad;
  L.status_offset = place(256);
  for (int l = 0; l < RQ_MAX_LOOPS; ++l) {
    L.codes_offset[l][0] = L.codes_offset[l][1] = -1;
    L.meta_offset[l][0] = L.meta_offset[l][1] = -1;
    L.alpha_offset[l] = -1;
    L.anchor_of[l] = -1;
    L.ref_of[l] = -1;
  }
  for (int l = 0; l < cfg->num_loops; ++l) {
    const int a = anchor_of(*cfg, l);
    L.anchor_of[l] = a;
    L.ref_of[l] = ref_of(*cfg, l);
    if (a == l) {
      L.codes_record_bytes[l] = cfg->bits[l] == 16 ? 256 : 64;
      L.meta_record_bytes[l] = cfg->bits[l] == 16 ? 0 : 16;
    } else {
      L.codes_record_bytes[l] = cfg->bits[l] * RQ_HEAD_DIM / 8;
      L.meta_record_bytes[l] = 4 * (RQ_HEAD_DIM / cfg->group[l]);
    }
    for (int kv = 0; kv < 2; ++kv) L.codes_offset[l][kv] = place(recs * L.codes_record_bytes[l]);
    if (L.meta_record_bytes[l])
      for (int kv = 0; kv < 2; ++kv) L.meta_offset[l][kv] = place(recs * L.meta_record_bytes[l]);
    if (a != l) L.alpha_offset[l] = place(recs * 4);
  }
  L.total_bytes = off;
  *out = L;
  return RQ_OK;
}

rq_status rq_cache_create(const rq_config* cfg, void* device_buffer, int64_t buffer_bytes,
                          rq_cache** out) {
  if (out == nullptr) return fail(RQ_ERR_INVALID_ARG, "handle output is null");
  *out = nullptr;
  rq_layout L;
  rq_status st = rq_cache_layout(cfg, &L);
  if (st != RQ_OK) return st;
  if (device_buffer == nullptr) return fail(RQ_ERR_INVALID_ARG, "device buffer is null");
  if (!aligned(device_buffer, 1024)) return fail(RQ_ERR_INVALID_ARG, "device buffer not 1024-byte aligned");
  if (buffer_bytes < L.total_bytes)
    return fail(RQ_ERR_INVALID_ARG, "buffer has %lld bytes, layout needs %lld",
                static_cast<long long>(buffer_bytes), static_cast<long long>(L.total_bytes));
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return cuda_fail(e, "cudaGetDevice");
  e = cudaMemset(static_cast<uint8_t*>(device_buffer) + L.status_offset, 0, 256);
  if (e != cudaSuccess) return cuda_fail(e, "clearing the status word");
  rq_cache* c = new (std::nothrow) rq_cache;
  if (c == nullptr) return fail(RQ_ERR_INVALID_ARG, "out of host memory");
  c->cfg = *cfg;
  c->lay = L;
  c->base = static_cast<uint8_t*>(device_buffer);
  c->device = dev;
  c->num_ctas = rq::decode_grid_ctas(dev);
  c->decode_kernel = RQ_DECODE_KERNEL_AUTO;
  c->stall_page = -1;
  for (int l = 0; l < RQ_MAX_LOOPS; ++l) c->tmaps_ready[l] = false;
  *out = c;
  return RQ_OK;
}

void rq_cache_destroy(rq_cache* cache) { delete cache; }

rq_status rq_cache_set_decode_kernel(rq_cache* cache, int32_t kernel) {
  if (cache == nullptr) return fail(RQ_ERR_INVALID_ARG, "cache is null");
  if (kernel != RQ_DECODE_KERNEL_AUTO && kernel != RQ_DECODE_KERNEL_SIMT && kernel != RQ_DECODE_KERNEL_TENSOR)
    return fail(RQ_ERR_INVALID_ARG, "decode kernel %d", kernel);
  cache->decode_kernel = kernel;
  return RQ_OK;
}

rq_status rq_cache_set_debug_stall(rq_cache* cache, int32_t page) {
  if (cache == nullptr) return fail(RQ_ERR_INVALID_ARG, "cache is null");
  if (page < -1) return fail(RQ_ERR_INVALID_ARG, "stall page %d < -1", page);
  cache->stall_page = page;
  return RQ_OK;
}

rq_status rq_cache_info(const rq_cache* cache, rq_config* cfg_out, rq_layout* layout_out) {
  if (cache == nullptr) return fail(RQ_ERR_INVALID_ARG, "cache is null");
  if (cfg_out) *cfg_out = cache->cfg;
  if (layout_out) *layout_out = cache->lay;
  return RQ_OK;
}

namespace {

// Validates an encode request and fills its kernel parameters (n_tokens > 0).
rq_status build_encode(rq_cache* cache, const void* k, const void* v, const int64_t* strides, int32_t start_pos,
                       const int32_t* positions, int32_t n_tokens, rq::EncodeParams* out) {
  if (k == nullptr || v == nullptr || strides == nullptr) return fail(RQ_ERR_INVALID_ARG, "k, v or strides is null");
  if (!aligned(k, 16) || !aligned(v, 16)) return fail(RQ_ERR_INVALID_ARG, "k/v not 16-byte aligned");
  for (int i = 0; i < 4; ++i)
    if (strides[i] < 0 || strides[i] % 8 != 0)
      return fail(RQ_ERR_INVALID_ARG, "stride[%d] = %lld must be a non-negative multiple of 8", i,
                  static_cast<long long>(strides[i]));
  const rq_config& c = cache->cfg;
  if (positions == nullptr) {
    if (start_pos < 0) return fail(RQ_ERR_INVALID_ARG, "start_pos %d < 0", start_pos);
    if (static_cast<int64_t>(start_pos) + n_tokens > c.capacity)
      return fail(RQ_ERR_CAPACITY, "start_pos %d + n_tokens %d > capacity %d", start_pos, n_tokens, c.capacity);
  }
  if (static_cast<int64_t>(c.batch) * c.kv_heads * n_tokens > (int64_t(1) << 31) - 8)
    return fail(RQ_ERR_UNSUPPORTED, "too many vectors in one encode call");
  rq::EncodeParams& p = *out;
  std::memset(&p, 0, sizeof(p));
  p.L = c.num_loops;
  p.B = c.batch;
  p.Hkv = c.kv_heads;
  p.cap_pad = cache->lay.capacity_padded;
  p.capacity = c.capacity;
  p.n_tokens = n_tokens;
  p.start_pos = start_pos;
  p.positions = positions;
  p.k = static_cast<const uint16_t*>(k);
  p.v = static_cast<const uint16_t*>(v);
  p.s_l = strides[0];
  p.s_b = strides[1];
  p.s_h = strides[2];
  p.s_t = strides[3];
  const rq_layout& lay = cache->lay;
  for (int l = 0; l < c.num_loops; ++l) {
    for (int kv = 0; kv < 2; ++kv) {
      p.codes[l][kv] = cache->base + lay.codes_offset[l][kv];
      p.meta[l][kv] = lay.meta_offset[l][kv] >= 0 ? cache->base + lay.meta_offset[l][kv] : nullptr;
    }
    p.alpha[l] = lay.alpha_offset[l] >= 0 ? cache->base + lay.alpha_offset[l] : nullptr;
    p.bits[l] = c.bits[l];
    p.group[l] = c.group[l];
    p.rotate[l] = c.rotate[l];
    p.alpha_mode[l] = c.alpha_mode[l];
    p.anchor[l] = lay.anchor_of[l];
    p.ref[l] = lay.ref_of[l];
  }
  p.chained = chained(c) ? 1 : 0;
  p.status = reinterpret_cast<int32_t*>(cache->base + cache->lay.status_offset);
  return RQ_OK;
}

}  // namespace

rq_status rq_encode(rq_cache* cache, const void* k, const void* v, const int64_t* strides,
                    int32_t start_pos, const int32_t* positions, int32_t n_tokens,
                    rq_stream_t stream) {
  if (cache == nullptr) return fail(RQ_ERR_INVALID_ARG, "cache is null");
  if (n_tokens < 0) return fail(RQ_ERR_INVALID_ARG, "n_tokens %d < 0", n_tokens);
  if (n_tokens == 0) return RQ_OK;
  rq::EncodeParams p;
  const rq_status st = build_encode(cache, k, v, strides, start_pos, positions, n_tokens, &p);
  if (st != RQ_OK) return st;
  cudaError_t e = rq::launch_encode(p, static_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return cuda_fail(e, "encode launch");
  return RQ_OK;
}

rq_status rq_decode_workspace_size(const rq_cache* cache, int64_t* bytes_out) {
  if (cache == nullptr || bytes_out == nullptr) return fail(RQ_ERR_INVALID_ARG, "null argument");
  const int G = cache->cfg.q_heads / cache->cfg.kv_heads;
  *bytes_out = rq::decode_workspace_bytes(cache->cfg.batch, cache->cfg.kv_heads, G, cache->num_ctas);
  return RQ_OK;
}

rq_status rq_bf16_decode_workspace_size(int32_t batch, int32_t kv_heads, int32_t q_heads,
                                        int64_t* bytes_out) {
  if (bytes_out == nullptr) return fail(RQ_ERR_INVALID_ARG, "null argument");
  if (batch < 1 || kv_heads < 1 || q_heads < 1 || q_heads % kv_heads)
    return fail(RQ_ERR_INVALID_ARG, "bad sizes");
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return cuda_fail(e, "cudaGetDevice");
  *bytes_out = rq::decode_workspace_bytes(batch, kv_heads, q_heads / kv_heads, rq::decode_grid_ctas(dev));
  return RQ_OK;
}

namespace {

rq_status check_decode_common(int B, int Hkv, int Hq, const void* q, const int32_t* ctx_len,
                              const void* k_tail, const void* v_tail, int32_t n_tail, float scale,
                              const float* out, const void* ws, int64_t ws_bytes, int64_t need) {
  if (B > RQ_MAX_BATCH) return fail(RQ_ERR_UNSUPPORTED, "batch %d > %d", B, RQ_MAX_BATCH);
  if (q == nullptr || ctx_len == nullptr || out == nullptr) return fail(RQ_ERR_INVALID_ARG, "q, ctx_len or out is null");
  if (!aligned(q, 16) || !aligned(out, 16)) return fail(RQ_ERR_INVALID_ARG, "q/out not 16-byte aligned");
  if (n_tail < 0) return fail(RQ_ERR_INVALID_ARG, "n_tail %d < 0", n_tail);
  if (n_tail > 0 && (k_tail == nullptr || v_tail == nullptr)) return fail(RQ_ERR_INVALID_ARG, "tail is null");
  if (n_tail > 0 && (!aligned(k_tail, 8) || !aligned(v_tail, 8))) return fail(RQ_ERR_INVALID_ARG, "tail misaligned");
  if (!(scale > 0.f) || !(scale < 1e30f)) return fail(RQ_ERR_INVALID_ARG, "softmax_scale must be positive and finite");
  if (ws == nullptr || !aligned(ws, 256)) return fail(RQ_ERR_WORKSPACE, "workspace null or not 256-byte aligned");
  if (ws_bytes < need)
    return fail(RQ_ERR_WORKSPACE, "workspace %lld bytes < %lld needed", static_cast<long long>(ws_bytes),
                static_cast<long long>(need));
  (void)Hkv; (void)Hq;
  return RQ_OK;
}

}  // namespace

namespace {

// The loop's chain of residual links toward its anchor (one link unless the
// policy is chained); returns the number of links, or -1 if longer than
// RQ_MAX_CHAIN.
int loop_chain(const rq_cache* cache, int loop, int (&chain)[RQ_MAX_CHAIN]) {
  const rq_layout& lay = cache->lay;
  const int a = lay.anchor_of[loop];
  int n_chain = 0;
  for (int l = loop; l != a; l = lay.ref_of[l]) {
    if (n_chain == RQ_MAX_CHAIN) return -1;
    chain[n_chain++] = l;
  }
  return n_chain;
}

// Query rows per pass over the cache (G of the kernels) for a decode of `loop`
// with n_q query tokens per sequence: all rows up to 8; 16 rows (and each block
// of 16 of a multiple of 16) in one pass where the tensor-core kernel has a
// 16-row variant for the loop's format and is the kernel the call takes; else
// blocks of 8.  The CUDA-core kernel has no 8-row variant (its registers would
// spill, at about a tenth of the 4-row rate): 8 rows that land on the CUDA
// cores -- by the automatic choice or a forced one -- run as two passes of 4
// rows (each reads the cache once more).
rq_status block_rows(const rq_cache* cache, int loop, int n_q, int* G_out) {
  const rq_config& c = cache->cfg;
  if (loop < 0 || loop >= c.num_loops) return fail(RQ_ERR_INVALID_ARG, "loop %d outside [0, %d)", loop, c.num_loops);
  if (n_q < 1 || n_q > RQ_MAX_DRAFT) return fail(RQ_ERR_INVALID_ARG, "n_q %d outside [1, %d]", n_q, RQ_MAX_DRAFT);
  const int rows = n_q * (c.q_heads / c.kv_heads);
  if (!rows_supported(rows))
    return fail(RQ_ERR_UNSUPPORTED, "n_q * q_heads / kv_heads = %d (supported: 1, 2, 4, or a multiple of 8)", rows);
  int G = rows < 8 ? rows : 8;
  int chain[RQ_MAX_CHAIN];
  const int n_chain = loop_chain(cache, loop, chain);
  if (n_chain < 0) return fail(RQ_ERR_UNSUPPORTED, "reference chain longer than %d", RQ_MAX_CHAIN);
  const int a = cache->lay.anchor_of[loop];
  const int ref_kind = ref_kind_for(c, loop);
  const int res_bits = loop == a ? 0 : c.bits[loop];
  const int res_group = loop == a ? 32 : c.group[loop];
  const int nc = n_chain > 1 ? n_chain : 1;
  if (rows % 16 == 0 &&
      rq::decode_kernel_choice(ref_kind, res_bits, res_group, 16, cache->decode_kernel, nc) == rq::kKernelTensor &&
      rq::decode_variant_supported(ref_kind, res_bits, res_group, 16, rq::kKernelTensor, nc))
    G = 16;
  if (G == 8 && rq::decode_kernel_choice(ref_kind, res_bits, res_group, 8, cache->decode_kernel, nc) == rq::kKernelSimt)
    G = 4;
  *G_out = G;
  return RQ_OK;
}

}  // namespace

}  // extern "C"

namespace rq {
rq_status decode_scratch_need(const rq_cache* cache, int loop, int n_q, int64_t* bytes_out) {
  if (cache == nullptr || bytes_out == nullptr) return fail(RQ_ERR_INVALID_ARG, "null argument");
  int G = 0;
  const rq_status st = block_rows(cache, loop, n_q, &G);
  if (st != RQ_OK) return st;
  *bytes_out = decode_workspace_bytes(cache->cfg.batch, cache->cfg.kv_heads, G, cache->num_ctas);
  return RQ_OK;
}

int cache_device(const rq_cache* cache) { return cache->device; }
}  // namespace rq

extern "C" {

namespace {

// n_q > 1: a multi-query call (q and out [B][n_q][Hq][128]; the last n_q tail
// tokens are the draft tokens, each seen by itself and the later ones)
rq_status decode_impl(const rq_cache* cache_c, int32_t loop, const void* q, int32_t n_q, const int32_t* ctx_len,
                      const void* k_tail, const void* v_tail, int32_t n_tail, float softmax_scale, float* out,
                      void* workspace, int64_t workspace_bytes, rq_stream_t stream,
                      const rq::EncodeParams* append) {
  if (cache_c == nullptr) return fail(RQ_ERR_INVALID_ARG, "cache is null");
  rq_cache* cache = const_cast<rq_cache*>(cache_c);
  const rq_config& c = cache->cfg;
  const int gq = c.q_heads / c.kv_heads;
  int G = 0;  // rows per pass over the cache
  rq_status st = block_rows(cache, loop, n_q, &G);
  if (st != RQ_OK) return st;
  const int rows = n_q * gq;  // query rows per kv-head, decoded in blocks of G
  if (n_q > 1 && n_tail < n_q)
    return fail(RQ_ERR_INVALID_ARG, "n_tail %d < n_q %d (the draft tokens are the last n_q tail tokens)", n_tail, n_q);
  const int64_t need = rq::decode_workspace_bytes(c.batch, c.kv_heads, G, cache->num_ctas);
  st = check_decode_common(c.batch, c.kv_heads, c.q_heads, q, ctx_len, k_tail, v_tail, n_tail,
                                     softmax_scale, out, workspace, workspace_bytes, need);
  if (st != RQ_OK) return st;
  const rq_layout& lay = cache->lay;
  const int a = lay.anchor_of[loop];
  const int ref_kind = ref_kind_for(c, loop);
  const int res_bits = loop == a ? 0 : c.bits[loop];
  const int res_group = loop == a ? 32 : c.group[loop];
  // the loop's chain of residual links toward its anchor (one link unless chained)
  int chain[RQ_MAX_CHAIN];
  const int n_chain = loop_chain(cache, loop, chain);
  if (!rq::decode_variant_supported(ref_kind, res_bits, res_group, G, cache->decode_kernel, n_chain > 1 ? n_chain : 1))
    return fail(RQ_ERR_UNSUPPORTED, "no %s decode kernel for this loop format, G = %d and a chain of %d",
                cache->decode_kernel == RQ_DECODE_KERNEL_TENSOR ? "tensor-core" : "", G, n_chain);
  if (ref_kind == rq::kRefBf16 && !cache->tmaps_ready[a]) {
    const int64_t cp = lay.capacity_padded;
    for (int kv = 0; kv < 2; ++kv) {
      st = make_plane_map(&cache->tm_anchor[a][kv], cache->base + lay.codes_offset[a][kv], c.batch, c.kv_heads, cp,
                          static_cast<int64_t>(c.kv_heads) * cp * RQ_HEAD_DIM, cp * RQ_HEAD_DIM, RQ_HEAD_DIM);
      if (st != RQ_OK) return st;
    }
    cache->tmaps_ready[a] = true;
  }
  rq::DecodeParams p;
  std::memset(&p, 0, sizeof(p));
  p.B = c.batch;
  p.Hkv = c.kv_heads;
  p.G = G;
  p.gq = gq;
  p.n_q = n_q;
  p.row0 = 0;
  p.q_stride_i = static_cast<int64_t>(c.q_heads) * RQ_HEAD_DIM;
  p.q_stride_b = n_q * p.q_stride_i;
  p.capacity = c.capacity;
  p.plane_tokens = lay.capacity_padded;
  if (ref_kind == rq::kRefInt4) {
    for (int kv = 0; kv < 2; ++kv) {
      p.ref_codes[kv] = cache->base + lay.codes_offset[a][kv];
      p.ref_meta[kv] = cache->base + lay.meta_offset[a][kv];
    }
  }
  p.n_chain = 1;
  if (res_bits) {
    p.n_chain = n_chain;
    for (int i = 0; i < n_chain; ++i) {
      for (int kv = 0; kv < 2; ++kv) {
        p.res_codes[i][kv] = cache->base + lay.codes_offset[chain[i]][kv];
        p.res_meta[i][kv] = cache->base + lay.meta_offset[chain[i]][kv];
      }
      p.alpha[i] = cache->base + lay.alpha_offset[chain[i]];
    }
    p.rotate = c.rotate[loop];
  }
  p.q = static_cast<const uint16_t*>(q);
  p.ctx_len = ctx_len;
  p.k_tail = static_cast<const uint16_t*>(k_tail);
  p.v_tail = static_cast<const uint16_t*>(v_tail);
  p.n_tail = n_tail;
  p.scale_log2 = softmax_scale * 1.4426950408889634f;
  p.out = out;
  p.partials = static_cast<float*>(workspace);
  p.num_ctas = cache->num_ctas;
  p.status = reinterpret_cast<int32_t*>(cache->base + cache->lay.status_offset);
  p.tma_tokens = lay.capacity_padded;
  p.stall_page = cache->stall_page;
  // one pass over the cache per block of 8 rows (stream-ordered, so the blocks
  // reuse one workspace)
  for (int row0 = 0; row0 < rows; row0 += G) {
    p.row0 = row0;
    // the step's append rides with the last block's combine, after every block has read the cache
    const rq::EncodeParams* app = row0 + G >= rows ? append : nullptr;
    cudaError_t e = rq::launch_decode(p, ref_kind, res_bits, res_group, cache->decode_kernel, &cache->tm_anchor[a][0],
                                      &cache->tm_anchor[a][1], static_cast<cudaStream_t>(stream), app);
    if (e != cudaSuccess) return cuda_fail(e, "decode launch");
  }
  return RQ_OK;
}

}  // namespace

rq_status rq_decode_attention(const rq_cache* cache, int32_t loop, const void* q, const int32_t* ctx_len,
                              const void* k_tail, const void* v_tail, int32_t n_tail, float softmax_scale,
                              float* out, void* workspace, int64_t workspace_bytes, rq_stream_t stream) {
  return decode_impl(cache, loop, q, 1, ctx_len, k_tail, v_tail, n_tail, softmax_scale, out, workspace,
                     workspace_bytes, stream, nullptr);
}

rq_status rq_decode_plan(const rq_cache* cache, int32_t loop, int32_t n_q, int32_t* kernel_out,
                         int32_t* rows_per_pass_out) {
  if (cache == nullptr || kernel_out == nullptr || rows_per_pass_out == nullptr)
    return fail(RQ_ERR_INVALID_ARG, "null argument");
  int G = 0;
  const rq_status st = block_rows(cache, loop, n_q, &G);
  if (st != RQ_OK) return st;
  const rq_config& c = cache->cfg;
  int chain[RQ_MAX_CHAIN];
  const int n_chain = loop_chain(cache, loop, chain);
  const int a = cache->lay.anchor_of[loop];
  const int ref_kind = ref_kind_for(c, loop);
  const int res_bits = loop == a ? 0 : c.bits[loop];
  const int res_group = loop == a ? 32 : c.group[loop];
  const int nc = n_chain > 1 ? n_chain : 1;
  if (!rq::decode_variant_supported(ref_kind, res_bits, res_group, G, cache->decode_kernel, nc))
    return fail(RQ_ERR_UNSUPPORTED, "no decode kernel for this loop format, G = %d and a chain of %d", G, n_chain);
  const int k = rq::decode_kernel_choice(ref_kind, res_bits, res_group, G, cache->decode_kernel, nc);
  *kernel_out = k == rq::kKernelTensor ? RQ_DECODE_KERNEL_TENSOR : RQ_DECODE_KERNEL_SIMT;
  *rows_per_pass_out = G;
  return RQ_OK;
}

rq_status rq_decode_multi_workspace_size(const rq_cache* cache, int32_t n_q, int64_t* bytes_out) {
  if (cache == nullptr || bytes_out == nullptr) return fail(RQ_ERR_INVALID_ARG, "null argument");
  if (n_q < 1 || n_q > RQ_MAX_DRAFT) return fail(RQ_ERR_INVALID_ARG, "n_q %d outside [1, %d]", n_q, RQ_MAX_DRAFT);
  const int rows = n_q * (cache->cfg.q_heads / cache->cfg.kv_heads);
  // the most rows one pass may take (any loop of the cache)
  const int G = rows < 8 ? rows : (rows % 16 == 0 ? 16 : 8);
  *bytes_out = rq::decode_workspace_bytes(cache->cfg.batch, cache->cfg.kv_heads, G, cache->num_ctas);
  return RQ_OK;
}

rq_status rq_decode_attention_multi(const rq_cache* cache, int32_t loop, const void* q, int32_t n_q,
                                    const int32_t* ctx_len, const void* k_tail, const void* v_tail, int32_t n_tail,
                                    float softmax_scale, float* out, void* workspace, int64_t workspace_bytes,
                                    rq_stream_t stream) {
  return decode_impl(cache, loop, q, n_q, ctx_len, k_tail, v_tail, n_tail, softmax_scale, out, workspace,
                     workspace_bytes, stream, nullptr);
}

rq_status rq_decode_attention_append(rq_cache* cache, int32_t loop, const void* q, const int32_t* ctx_len,
                                     const void* k_tail, const void* v_tail, int32_t n_tail, float softmax_scale,
                                     float* out, void* workspace, int64_t workspace_bytes, const void* k_new,
                                     const void* v_new, const int64_t* strides, const int32_t* positions,
                                     int32_t n_new, rq_stream_t stream) {
  if (cache == nullptr) return fail(RQ_ERR_INVALID_ARG, "cache is null");
  if (positions == nullptr) return fail(RQ_ERR_INVALID_ARG, "positions is null (device int32 [batch] required)");
  if (n_new < 0) return fail(RQ_ERR_INVALID_ARG, "n_new %d < 0", n_new);
  rq::EncodeParams ep;
  if (n_new > 0) {
    const rq_status st = build_encode(cache, k_new, v_new, strides, 0, positions, n_new, &ep);
    if (st != RQ_OK) return st;
  }
  return decode_impl(cache, loop, q, 1, ctx_len, k_tail, v_tail, n_tail, softmax_scale, out, workspace,
                     workspace_bytes, stream, n_new > 0 ? &ep : nullptr);
}

rq_status rq_bf16_decode_attention(int32_t batch, int32_t kv_heads, int32_t q_heads,
                                   const void* k_cache, const void* v_cache,
                                   const int64_t* strides, int32_t capacity, const void* q,
                                   const int32_t* ctx_len, const void* k_tail, const void* v_tail,
                                   int32_t n_tail, float softmax_scale, float* out,
                                   void* workspace, int64_t workspace_bytes, int32_t* status_word,
                                   rq_stream_t stream) {
  if (batch < 1 || kv_heads < 1 || q_heads < 1 || q_heads % kv_heads)
    return fail(RQ_ERR_INVALID_ARG, "bad sizes");
  const int G = q_heads / kv_heads;
  if (G != 1 && G != 2 && G != 4 && G != 8) return fail(RQ_ERR_UNSUPPORTED, "q_heads / kv_heads = %d", G);
  if (k_cache == nullptr || v_cache == nullptr || strides == nullptr) return fail(RQ_ERR_INVALID_ARG, "cache is null");
  if (!aligned(k_cache, 16) || !aligned(v_cache, 16)) return fail(RQ_ERR_INVALID_ARG, "cache not 16-byte aligned");
  for (int i = 0; i < 3; ++i)
    if (strides[i] <= 0 || strides[i] % 8 != 0)
      return fail(RQ_ERR_INVALID_ARG, "stride[%d] must be a positive multiple of 8", i);
  if (capacity < 1) return fail(RQ_ERR_INVALID_ARG, "capacity %d < 1", capacity);
  int64_t need = 0;
  rq_status st = rq_bf16_decode_workspace_size(batch, kv_heads, q_heads, &need);
  if (st != RQ_OK) return st;
  st = check_decode_common(batch, kv_heads, q_heads, q, ctx_len, k_tail, v_tail, n_tail, softmax_scale, out,
                           workspace, workspace_bytes, need);
  if (st != RQ_OK) return st;
  CUtensorMap tk, tv;
  st = make_plane_map(&tk, k_cache, batch, kv_heads, capacity, strides[0], strides[1], strides[2]);
  if (st != RQ_OK) return st;
  st = make_plane_map(&tv, v_cache, batch, kv_heads, capacity, strides[0], strides[1], strides[2]);
  if (st != RQ_OK) return st;
  int dev = 0;
  cudaGetDevice(&dev);
  rq::DecodeParams p;
  std::memset(&p, 0, sizeof(p));
  p.B = batch;
  p.Hkv = kv_heads;
  p.G = G;
  p.gq = G;
  p.n_q = 1;
  p.q_stride_i = static_cast<int64_t>(q_heads) * RQ_HEAD_DIM;
  p.q_stride_b = p.q_stride_i;
  p.capacity = capacity;
  p.plane_tokens = 0;
  p.q = static_cast<const uint16_t*>(q);
  p.ctx_len = ctx_len;
  p.k_tail = static_cast<const uint16_t*>(k_tail);
  p.v_tail = static_cast<const uint16_t*>(v_tail);
  p.n_tail = n_tail;
  p.scale_log2 = softmax_scale * 1.4426950408889634f;
  p.out = out;
  p.partials = static_cast<float*>(workspace);
  p.num_ctas = rq::decode_grid_ctas(dev);
  p.status = status_word;
  p.tma_tokens = capacity;
  p.stall_page = -1;
  cudaError_t e = rq::launch_decode(p, rq::kRefBf16, 0, 32, rq::kKernelAuto, &tk, &tv,
                                    static_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return cuda_fail(e, "decode launch");
  return RQ_OK;
}

rq_status rq_reconstruct(const rq_cache* cache, int32_t loop, int32_t t0, int32_t n, float* k_out,
                         float* v_out, rq_stream_t stream) {
  if (cache == nullptr) return fail(RQ_ERR_INVALID_ARG, "cache is null");
  const rq_config& c = cache->cfg;
  if (loop < 0 || loop >= c.num_loops) return fail(RQ_ERR_INVALID_ARG, "loop %d outside [0, %d)", loop, c.num_loops);
  if (t0 < 0 || n < 0 || static_cast<int64_t>(t0) + n > c.capacity)
    return fail(RQ_ERR_INVALID_ARG, "token range [%d, %d) outside the capacity %d", t0, t0 + n, c.capacity);
  if (n == 0) return RQ_OK;
  if (k_out == nullptr || v_out == nullptr || !aligned(k_out, 16) || !aligned(v_out, 16))
    return fail(RQ_ERR_INVALID_ARG, "outputs null or not 16-byte aligned");
  const rq_layout& lay = cache->lay;
  const int a = lay.anchor_of[loop];
  // links from the anchor outward: the first reads the anchor planes, every
  // later one the previous link's reconstruction, in place in k_out / v_out
  int links[RQ_MAX_LOOPS];
  int n_links = 0;
  for (int l = loop; l != a && n_links < RQ_MAX_LOOPS; l = lay.ref_of[l]) links[n_links++] = l;
  for (int i = n_links - 1; i >= (n_links > 0 ? 0 : -1); --i) {
    const int l = i >= 0 ? links[i] : loop;
    rq::ReconstructParams p;
    std::memset(&p, 0, sizeof(p));
    p.B = c.batch;
    p.Hkv = c.kv_heads;
    p.cap_pad = lay.capacity_padded;
    p.t0 = t0;
    p.n = n;
    p.ref_bits = c.bits[a];
    for (int kv = 0; kv < 2; ++kv) {
      p.ref_plane[kv] = cache->base + lay.codes_offset[a][kv];
      p.ref_meta[kv] = lay.meta_offset[a][kv] >= 0 ? cache->base + lay.meta_offset[a][kv] : nullptr;
    }
    p.is_ref = l == a;
    p.ref_from_out = i >= 0 && i < n_links - 1;
    if (!p.is_ref) {
      for (int kv = 0; kv < 2; ++kv) {
        p.codes[kv] = cache->base + lay.codes_offset[l][kv];
        p.meta[kv] = cache->base + lay.meta_offset[l][kv];
      }
      p.alpha = cache->base + lay.alpha_offset[l];
      p.bits = c.bits[l];
      p.group = c.group[l];
      p.rotate = c.rotate[l];
    }
    p.out[0] = k_out;
    p.out[1] = v_out;
    cudaError_t e = rq::launch_reconstruct(p, static_cast<cudaStream_t>(stream));
    if (e != cudaSuccess) return cuda_fail(e, "reconstruct launch");
  }
  return RQ_OK;
}

rq_status rq_get_error(const rq_cache* cache, rq_stream_t stream, uint32_t* flags_out) {
  if (cache == nullptr) return fail(RQ_ERR_INVALID_ARG, "cache is null");
  cudaError_t e = cudaStreamSynchronize(static_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return cuda_fail(e, "stream synchronize");
  uint32_t w = 0;
  void* dev = cache->base + cache->lay.status_offset;
  e = cudaMemcpy(&w, dev, sizeof(w), cudaMemcpyDeviceToHost);
  if (e != cudaSuccess) return cuda_fail(e, "reading the status word");
  if (w != 0) {
    e = cudaMemset(dev, 0, sizeof(w));
    if (e != cudaSuccess) return cuda_fail(e, "clearing the status word");
  }
  if (flags_out) *flags_out = w;
  if (w != 0) return fail(RQ_ERR_DEVICE_FLAG, "device status word 0x%x", w);
  return RQ_OK;
}

}  // extern "C"
