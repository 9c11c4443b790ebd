// rq_internal.h -- kernel parameter blocks and launcher entry points shared by
// the host library (rq_api.cpp) and the CUDA translation units.  Not part of
// the public ABI.
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "../../include/rq_api.h"

namespace rq {

enum RefKind : int { kRefNone = 0, kRefBf16 = 1, kRefInt4 = 2 };

struct EncodeParams {
  int L, B, Hkv;
  int64_t cap_pad;
  int capacity;
  int n_tokens;
  int start_pos;
  const int32_t* positions;  // device [B] or null
  const uint16_t* k;         // bf16 bits
  const uint16_t* v;
  int64_t s_l, s_b, s_h, s_t;  // element strides
  // per loop: anchors (anchor[l] == l) store bf16 values or INT4 codes + meta
  // in codes/meta; the others store residual codes, meta and alpha
  uint8_t* codes[RQ_MAX_LOOPS][2];
  uint8_t* meta[RQ_MAX_LOOPS][2];
  uint8_t* alpha[RQ_MAX_LOOPS];
  int bits[RQ_MAX_LOOPS], group[RQ_MAX_LOOPS], rotate[RQ_MAX_LOOPS], alpha_mode[RQ_MAX_LOOPS];
  int anchor[RQ_MAX_LOOPS];
  int ref[RQ_MAX_LOOPS];  // the loop each loop is stored against (== anchor unless chained)
  int chained;            // 1: references are reconstructed neighbours (Previous-/Next-loop)
  int32_t* status;
};

struct ReconstructParams {
  int B, Hkv;
  int64_t cap_pad;
  int t0, n;
  int ref_bits;
  const uint8_t* ref_plane[2];
  const uint8_t* ref_meta[2];
  int is_ref;  // reconstruct the anchor loop itself
  int ref_from_out;  // take the reference from out[] (a chain's previous link), not the anchor
  const uint8_t* codes[2];
  const uint8_t* meta[2];
  const uint8_t* alpha;
  int bits, group, rotate;
  float* out[2];
};

// One decode call: either a residual loop of a cache, an anchor loop, or a
// plain bf16 cache.  Planes are indexed by record = (b*Hkv + h)*plane_tokens + t.
struct DecodeParams {
  int B, Hkv, G;         // G: query rows per kv-head (n_q * gq)
  int capacity;          // valid positions per sequence (ctx_len is clamped to it)
  int64_t plane_tokens;  // record stride between (b, h) slabs for byte planes
  // reference (bf16 via tensor maps; INT4 via byte planes)
  const uint8_t* ref_codes[2];
  const uint8_t* ref_meta[2];
  // residual: the loop's chain c_0 = loop, c_1 = its reference, ... (n_chain
  // links, 1 unless the policy is chained), all in one format
  const uint8_t* res_codes[RQ_MAX_CHAIN][2];
  const uint8_t* res_meta[RQ_MAX_CHAIN][2];
  const uint8_t* alpha[RQ_MAX_CHAIN];  // (alpha_K, alpha_V) fp16 pairs, or null (alpha = 1)
  int n_chain;
  int rotate;
  // query / lengths / tail / output.  Row gi of kv-head h is draft token
  // i = gi / gq, head h * gq + gi % gq (see q_row_offset); q and out are
  // [B][n_q][Hkv * gq][128], so one decode query per sequence is n_q = 1
  int gq, n_q;
  int row0;              // rows [row0, row0 + G) of the n_q * gq rows of a kv-head (blocks of 8 beyond 8 rows)
  int64_t q_stride_b, q_stride_i;  // elements between sequences / draft tokens
  const uint16_t* q;     // bf16
  const int32_t* ctx_len;
  const uint16_t* k_tail;  // bf16 [B][Hkv][n_tail][128]
  const uint16_t* v_tail;
  int n_tail;
  float scale_log2;      // softmax_scale * log2(e)
  float* out;            // fp32 [B][Hq][128]
  float* partials;       // workspace
  int num_ctas;          // persistent grid size P of the split kernel
  int32_t* status;
  int64_t tma_tokens;    // token extent of the bf16 tensor maps
  int page_tokens;       // split granularity (set by launch_decode for the chosen kernel)
  int stall_page;        // test hook: CTA-local page before which the producer waits out its limit (-1: none)
};

// Element offset of query row gi of kv-head h of sequence b in q and out.
__host__ __device__ inline int64_t q_row_offset(const DecodeParams& P, int b, int h, int gi) {
  const int r = P.row0 + gi;
  const int i = r / P.gq, g = r - i * P.gq;
  return static_cast<int64_t>(b) * P.q_stride_b + static_cast<int64_t>(i) * P.q_stride_i +
         static_cast<int64_t>(h * P.gq + g) * RQ_HEAD_DIM;
}

// Split-K partial record per (slot, head): m, l, pad, pad, acc_ref[128], acc_res[128]
constexpr int kPartialFloats = 4 + 2 * RQ_HEAD_DIM;

int64_t decode_workspace_bytes(int B, int Hkv, int G, int num_ctas);
int decode_grid_ctas(int device);  // persistent grid size for this device

cudaError_t launch_encode(const EncodeParams& p, cudaStream_t s);
cudaError_t launch_reconstruct(const ReconstructParams& p, cudaStream_t s);
// Decode kernels: the CUDA-core split kernels (64- or 128-token pages, G in
// {1, 2, 4}) and the tensor-core split kernels (128-token pages, G in {1, 2, 4,
// 8, 16}; chained INT4-anchor loops at G in {4, 8}).
enum DecodeKernel : int { kKernelAuto = RQ_DECODE_KERNEL_AUTO, kKernelSimt = RQ_DECODE_KERNEL_SIMT,
                          kKernelTensor = RQ_DECODE_KERNEL_TENSOR };

// ref_kind: RefKind; res_bits: 0 | 2 | 4; res_group: 16 | 32
// `append` (or null): tokens to encode into the cache in the same launch as
// the combine kernel (positions past every context of this decode).
// p.n_chain > 1 (a chained loop): the tensor cores for an INT4 anchor at G in
// {4, 8}, else the CUDA cores.
cudaError_t launch_decode(DecodeParams p, int ref_kind, int res_bits, int res_group, int kernel,
                          const CUtensorMap* tmap_k, const CUtensorMap* tmap_v, cudaStream_t s,
                          const EncodeParams* append = nullptr);
bool decode_variant_supported(int ref_kind, int res_bits, int res_group, int G, int kernel, int n_chain = 1);
// the kernel an automatic choice resolves to
int decode_kernel_choice(int ref_kind, int res_bits, int res_group, int G, int kernel, int n_chain = 1);

// CUDA-core split kernel for the loops of chained policies (rq_decode_chain.cu):
// the launcher for a chain of n_chain (2 or 3) links, or null
using SplitLaunchFn = cudaError_t (*)(DecodeParams&, const CUtensorMap*, const CUtensorMap*, cudaStream_t);
SplitLaunchFn pick_chain(int ref_kind, int res_bits, int res_group, int G, int n_chain);

// tensor-core split kernel (rq_decode_tc.cuh; dispatch in rq_decode_tc.cu)
bool tc_variant_supported(int ref_kind, int res_bits, int res_group, int G, int n_chain = 1);
cudaError_t launch_split_tc(const DecodeParams& p, int ref_kind, int res_bits, int res_group, int n_chain,
                            const CUtensorMap* tmap_k, const CUtensorMap* tmap_v, cudaStream_t s);
// chained loops (2 or 3 residual links, INT4 anchor) on the tensor cores
bool tc_chain_variant_supported(int ref_kind, int res_bits, int res_group, int G, int n_chain);
cudaError_t launch_split_tc_chain(const DecodeParams& p, int ref_kind, int res_bits, int res_group, int n_chain,
                                  const CUtensorMap* tmap_k, const CUtensorMap* tmap_v, cudaStream_t s);
constexpr int kTcPage = 128;
// tensor-core split kernel for the byte-plane formats at one query row per
// kv-head, two warpgroups on alternate pages (rq_decode_pp.cu)
bool pp_variant_supported(int ref_kind, int res_bits, int res_group);
cudaError_t launch_split_pp(const DecodeParams& p, int ref_kind, int res_bits, int res_group, cudaStream_t s);

// Split-K workspace bytes a decode of `loop` with n_q query tokens per
// sequence needs (the rows of one pass over the cache, as the decode entry
// points size it).
rq_status decode_scratch_need(const rq_cache* cache, int loop, int n_q, int64_t* bytes_out);
// The device the cache was created on (current when rq_cache_create ran).
int cache_device(const rq_cache* cache);

// Records the calling thread's rq_last_error_message() text and returns `s`.
rq_status set_last_error(rq_status s, const char* fmt, ...);

}  // namespace rq
