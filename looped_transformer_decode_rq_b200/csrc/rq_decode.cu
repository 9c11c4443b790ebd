// rq_decode.cu -- fused dequantise-and-reconstruct split-K decode attention
// for sm_100a.
//
// "ResidualQuant: KV Cache Quantization for Looped Transformers with 2-Bit
// Residuals" stores loop l's keys as K_l ~ alpha K_ref + H^T deq(R_l) (abstract,
// Figure 1, Figure 2 caption) and credits its decode speed-up to the reduced
// KV memory traffic (abstract).  Here each cached token is scored directly from
// the compact cache:
//     q . K_l,t = alpha_t (q . K_ref,t) + (H q) . deq(R_l,t)
// and the value side accumulates sum p_t alpha_V,t V_ref,t in the original
// domain and sum p_t deq(R^V_l,t) in the rotated domain; the rotated sum is
// brought back with a single inverse Hadamard per (sequence, q-head) in the
// combine kernel.  No bf16 copy of loop l is ever formed.
//
// This file holds the combine kernel and the dispatch; the CUDA-core split
// kernel is in rq_decode_split.cuh, the tensor-core one in rq_decode_tc.cuh.
// Combine kernel: one warp per (b, query row) merges the CTA partials with the
// max-rescale rule, adds the bf16 tail tokens (a draft token of a multi-query
// call sees the tail up to itself), applies the inverse rotation and
// normalises.  It is a programmatic dependent launch: scheduled while the split
// kernel runs, it reads its inputs, then waits for the split grid's completion.
// With an append it also encodes the step's new tokens into every loop.
#include <cstring>

#include "rq_common.cuh"
#include "rq_decode_bp.cuh"
#include "rq_encode_dev.cuh"
#include "rq_internal.h"

namespace rq {
namespace {

// ---------------------------------------------------------------------------
// combine kernel: one warp per (b, q-head)
// ---------------------------------------------------------------------------
// x * a + y * b with a fixed rounding order (the result must not depend on how
// the compiler contracts this kernel's instances)
__device__ __forceinline__ float mix(float x, float a, float y, float b) { return __fmaf_rn(x, a, __fmul_rn(y, b)); }

// With APPEND, the warps past the B * Hq combine warps encode the new tokens of
// `E` into every loop's planes instead (positions past every context the split
// kernel read, so the two never touch the same records).
template <bool APPEND>
__global__ void __launch_bounds__(128) decode_combine_kernel(const DecodeParams P, int G, int rotate_res,
                                                             const __grid_constant__ EncodeParams E) {
  const int lane = threadIdx.x & 31;
  const int wid = blockIdx.x * 4 + (threadIdx.x >> 5);
  const int Hq = P.Hkv * G;
  pdl_launch_dependents();  // the next call's split kernel may be scheduled (it waits for this grid)
  if (wid >= P.B * Hq) {
    if constexpr (APPEND) {
      pdl_wait();  // the split kernel reads the pages these positions are written into
      enc::encode_warp(E, wid - P.B * Hq, lane);
    }
    return;
  }
  const int b = wid / Hq, qh = wid % Hq, h = qh / G, gi = qh % G;
  auto clamp_len = [&](int len) { return len < 0 ? 0 : (len > P.capacity ? P.capacity : len); };
  // page offsets (same arithmetic as the split kernel that wrote the partials)
  const int pt = P.page_tokens;
  int64_t pre = 0, tot = 0;
  for (int b2 = lane; b2 < P.B; b2 += 32) {
    const int nt = (clamp_len(P.ctx_len[b2]) + pt - 1) / pt;
    tot += nt;
    if (b2 < b) pre += nt;
  }
#pragma unroll
  for (int o = 16; o >= 1; o >>= 1) {
    tot += __shfl_xor_sync(0xffffffffu, tot, o);
    pre += __shfl_xor_sync(0xffffffffu, pre, o);
  }
  const int nt_b = (clamp_len(P.ctx_len[b]) + pt - 1) / pt;
  const int64_t total = tot * P.Hkv;
  const int64_t P_eff = total < P.num_ctas ? total : P.num_ctas;
  // inputs the split kernel does not write: the query and the first tail token
  const int64_t row = q_row_offset(P, b, h, gi);
  const uint2 qraw = *reinterpret_cast<const uint2*>(P.q + row + 4 * lane);
  // draft token i of a multi-query call sees the tail up to itself
  const int n_vis = P.n_tail - P.n_q + (P.row0 + gi) / P.gq + 1;
  uint2 kr0 = make_uint2(0u, 0u), vr0 = kr0;
  if (n_vis > 0) {
    const int64_t off = (static_cast<int64_t>(b) * P.Hkv + h) * P.n_tail * kD + 4 * lane;
    kr0 = *reinterpret_cast<const uint2*>(P.k_tail + off);
    vr0 = *reinterpret_cast<const uint2*>(P.v_tail + off);
  }
  // CTA range [c0, c1] of the split kernel that covered this segment
  const int64_t ts = pre * P.Hkv + static_cast<int64_t>(h) * nt_b;
  const int64_t c0 = nt_b > 0 ? ((ts + 1) * P_eff - 1) / total : 0;
  const int64_t c1 = nt_b > 0 ? ((ts + nt_b) * P_eff - 1) / total : -1;
  const float* rec0 = P.partials + ((static_cast<int64_t>(b) * P.Hkv + h + c0) * G + gi) * kPartialFloats;
  pdl_wait();  // the split kernel's partials are complete and visible from here on

  // the first kPre partials are loaded together (one memory round trip), then
  // merged in CTA order like the rest
  constexpr int kPre = 4;
  const int64_t npart = c1 - c0 + 1;
  float4 pml[kPre], pr[kPre], ps[kPre];
#pragma unroll
  for (int u = 0; u < kPre; ++u) {
    if (u < npart) {
      const float* rec = rec0 + static_cast<int64_t>(u) * G * kPartialFloats;
      pml[u] = reinterpret_cast<const float4*>(rec)[0];
      pr[u] = reinterpret_cast<const float4*>(rec + 4)[lane];
      ps[u] = reinterpret_cast<const float4*>(rec + 4 + kD)[lane];
    }
  }
  float m = -INFINITY, l = 0.f;
  float4 ar = make_float4(0.f, 0.f, 0.f, 0.f), as = ar;
  auto merge = [&](const float4& ml, const float4& r, const float4& s) {
    const float mn = fmaxf(m, ml.x);
    const float a = exp2f(m - mn), bb = exp2f(ml.x - mn);
    l = mix(l, a, ml.y, bb);
    ar = make_float4(mix(ar.x, a, r.x, bb), mix(ar.y, a, r.y, bb), mix(ar.z, a, r.z, bb), mix(ar.w, a, r.w, bb));
    as = make_float4(mix(as.x, a, s.x, bb), mix(as.y, a, s.y, bb), mix(as.z, a, s.z, bb), mix(as.w, a, s.w, bb));
    m = mn;
  };
#pragma unroll
  for (int u = 0; u < kPre; ++u)
    if (u < npart) merge(pml[u], pr[u], ps[u]);
  for (int64_t u = kPre; u < npart; ++u) {
    const float* rec = rec0 + u * G * kPartialFloats;
    merge(reinterpret_cast<const float4*>(rec)[0], reinterpret_cast<const float4*>(rec + 4)[lane],
          reinterpret_cast<const float4*>(rec + 4 + kD)[lane]);
  }
  // current (tail) tokens in bf16
  if (n_vis > 0) {
    const float2 q01 = bf16x2_to_f2(qraw.x), q23 = bf16x2_to_f2(qraw.y);
    for (int j = 0; j < n_vis; ++j) {
      const int64_t off = ((static_cast<int64_t>(b) * P.Hkv + h) * P.n_tail + j) * kD + 4 * lane;
      const uint2 kr = j == 0 ? kr0 : *reinterpret_cast<const uint2*>(P.k_tail + off);
      const uint2 vr = j == 0 ? vr0 : *reinterpret_cast<const uint2*>(P.v_tail + off);
      const float2 k01 = bf16x2_to_f2(kr.x), k23 = bf16x2_to_f2(kr.y);
      float d = __fmaf_rn(q23.y, k23.y, __fmaf_rn(q23.x, k23.x, __fmaf_rn(q01.y, k01.y, __fmul_rn(q01.x, k01.x))));
#pragma unroll
      for (int o = 16; o >= 1; o >>= 1) d += __shfl_xor_sync(0xffffffffu, d, o);
      const float sc = d * P.scale_log2;
      const float mn = fmaxf(m, sc);
      const float a = exp2f(m - mn), p = exp2f(sc - mn);
      const float2 v01 = bf16x2_to_f2(vr.x), v23 = bf16x2_to_f2(vr.y);
      l = __fmaf_rn(l, a, p);
      ar = make_float4(mix(ar.x, a, p, v01.x), mix(ar.y, a, p, v01.y), mix(ar.z, a, p, v23.x), mix(ar.w, a, p, v23.y));
      as = make_float4(__fmul_rn(as.x, a), __fmul_rn(as.y, a), __fmul_rn(as.z, a), __fmul_rn(as.w, a));
      m = mn;
    }
  }
  if (rotate_res) {
    float x[4] = {as.x, as.y, as.z, as.w};
    float t0 = x[0] + x[1], t1 = x[0] - x[1], t2 = x[2] + x[3], t3 = x[2] - x[3];
    x[0] = t0 + t2; x[2] = t0 - t2; x[1] = t1 + t3; x[3] = t1 - t3;
#pragma unroll
    for (int mm = 1; mm < 32; mm <<= 1) {
      const bool up = (lane & mm) != 0;
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const float o = __shfl_xor_sync(0xffffffffu, x[e], mm);
        x[e] = up ? (o - x[e]) : (x[e] + o);
      }
    }
    const float c = 0.08838834764831845f;
    as = make_float4(x[0] * c, x[1] * c, x[2] * c, x[3] * c);
  }
  const float inv = l > 0.f ? 1.f / l : 0.f;
  float4 o = make_float4(__fmul_rn(__fadd_rn(ar.x, as.x), inv), __fmul_rn(__fadd_rn(ar.y, as.y), inv),
                         __fmul_rn(__fadd_rn(ar.z, as.z), inv), __fmul_rn(__fadd_rn(ar.w, as.w), inv));
  reinterpret_cast<float4*>(P.out + row)[lane] = o;
}


SplitFn pick(int ref_kind, int res_bits, int res_group, int G, int n_chain) {
  if (n_chain > 1) return pick_chain(ref_kind, res_bits, res_group, G, n_chain);
  if (ref_kind == kRefBf16) {
    if (res_bits == 0) return pick_g<kRefBf16, 0, 32, 1>(G);
    if (res_bits == 2) return res_group == 16 ? pick_g<kRefBf16, 2, 16, 1>(G) : pick_g<kRefBf16, 2, 32, 1>(G);
    if (res_bits == 4) return res_group == 16 ? pick_g<kRefBf16, 4, 16, 1>(G) : pick_g<kRefBf16, 4, 32, 1>(G);
  } else if (ref_kind == kRefInt4) {
    if (res_bits == 0) return pick_g<kRefInt4, 0, 32, 1>(G);
    if (res_bits == 2) return res_group == 16 ? pick_g<kRefInt4, 2, 16, 1>(G) : pick_g<kRefInt4, 2, 32, 1>(G);
    if (res_bits == 4) return res_group == 16 ? pick_g<kRefInt4, 4, 16, 1>(G) : pick_g<kRefInt4, 4, 32, 1>(G);
  } else if (ref_kind == kRefNone) {
    if (res_bits == 2) return res_group == 16 ? pick_g<kRefNone, 2, 16, 1>(G) : pick_g<kRefNone, 2, 32, 1>(G);
    if (res_bits == 4) return res_group == 16 ? pick_g<kRefNone, 4, 16, 1>(G) : pick_g<kRefNone, 4, 32, 1>(G);
  }
  return nullptr;
}

}  // namespace

namespace {
// one query row of a byte-plane format on the tensor cores: the ping-pong kernel
bool pp_case(int ref_kind, int res_bits, int res_group, int G, int n_chain) {
  return G == 1 && n_chain <= 1 && ref_kind != kRefBf16 && pp_variant_supported(ref_kind, res_bits, res_group);
}
}  // namespace

// The automatic choice: the tensor cores from 4 query rows per kv-head, the
// CUDA cores below (at one row the byte-plane CUDA-core kernel measured faster
// than the ping-pong tensor-core kernel: 4.3 against 3.3 TB/s on the INT4-anchor
// [2,2,4,4] residual loop).
int decode_kernel_choice(int ref_kind, int res_bits, int res_group, int G, int kernel, int n_chain) {
  if (kernel == kKernelAuto)
    return (G >= 4 && tc_variant_supported(ref_kind, res_bits, res_group, G, n_chain)) ? kKernelTensor
                                                                                              : kKernelSimt;
  return kernel;
}

bool decode_variant_supported(int ref_kind, int res_bits, int res_group, int G, int kernel, int n_chain) {
  if (res_bits != 0 && res_group != 16 && res_group != 32) return false;
  kernel = decode_kernel_choice(ref_kind, res_bits, res_group, G, kernel, n_chain);
  if (kernel == kKernelTensor)
    return pp_case(ref_kind, res_bits, res_group, G, n_chain) ||
           tc_variant_supported(ref_kind, res_bits, res_group, G, n_chain);
  if (kernel == kKernelSimt) return pick(ref_kind, res_bits, res_group, G, n_chain) != nullptr;
  return false;
}

int decode_grid_ctas(int device) {
  int sms = 0;
  if (cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, device) != cudaSuccess || sms <= 0) sms = 148;
  return sms;  // one persistent CTA per SM
}

int64_t decode_workspace_bytes(int B, int Hkv, int G, int num_ctas) {
  const int64_t slots = static_cast<int64_t>(B) * Hkv + num_ctas;
  return slots * G * kPartialFloats * static_cast<int64_t>(sizeof(float));
}

cudaError_t launch_decode(DecodeParams p, int ref_kind, int res_bits, int res_group, int kernel,
                          const CUtensorMap* tmap_k, const CUtensorMap* tmap_v, cudaStream_t s,
                          const EncodeParams* append) {
  const int n_chain = (res_bits != 0 && p.n_chain > 1) ? p.n_chain : 1;
  kernel = decode_kernel_choice(ref_kind, res_bits, res_group, p.G, kernel, n_chain);
  cudaError_t e;
  if (kernel == kKernelTensor) {
    p.page_tokens = kTcPage;
    if (pp_case(ref_kind, res_bits, res_group, p.G, n_chain))
      e = launch_split_pp(p, ref_kind, res_bits, res_group, s);
    else
      e = launch_split_tc(p, ref_kind, res_bits, res_group, n_chain, tmap_k, tmap_v, s);
  } else {
    SplitFn fn = pick(ref_kind, res_bits, res_group, p.G, n_chain);
    if (fn == nullptr) return cudaErrorInvalidValue;
    e = fn(p, tmap_k, tmap_v, s);  // sets p.page_tokens
  }
  if (e != cudaSuccess) return e;
  const int64_t warps = static_cast<int64_t>(p.B) * p.Hkv * p.G;
  const int64_t enc_warps = append ? static_cast<int64_t>(append->B) * append->Hkv * append->n_tokens : 0;
  const int rot = (res_bits != 0 && p.rotate) ? 1 : 0;
  // programmatic dependent launch: scheduled while the split kernel runs, the
  // combine kernel waits for it in pdl_wait()
  if (enc_warps > 0) {
    e = launch_dependent(decode_combine_kernel<true>, static_cast<unsigned>((warps + enc_warps + 3) / 4), 128, 0, s,
                         p, p.G, rot, *append);
  } else {
    EncodeParams none;
    memset(&none, 0, sizeof(none));
    e = launch_dependent(decode_combine_kernel<false>, static_cast<unsigned>((warps + 3) / 4), 128, 0, s, p, p.G,
                         rot, none);
  }
  if (e != cudaSuccess) return e;
  return cudaGetLastError();
}

}  // namespace rq
