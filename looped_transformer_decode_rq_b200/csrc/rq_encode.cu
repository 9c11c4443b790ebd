// rq_encode.cu -- ResidualQuant encode and (test-support) reconstruction on
// sm_100a.
//
// Encode follows "ResidualQuant: KV Cache Quantization for Looped Transformers
// with 2-Bit Residuals" (abstract; Figure 1 steps 2-5; Figure 2 caption): an
// anchor loop (the final loop by default; Table 1 and Table 8 for the First-
// loop and anchor-interval variants) is the reference, every other loop is
// stored as the scaled residual against its anchor (LS, or Table 9's norm
// ratio), rotated by the order-128 Hadamard, quantised per group to INT2 or
// INT4 with an fp16 scale and offset.
//
// One warp handles one (b, h, token) for all loops: lanes 0-15 the key,
// lanes 16-31 the value; lane j of a half owns elements 8j..8j+7 and loads
// them with one 16-byte access.  The arithmetic order is fixed so that codes,
// scales, offsets and alphas are reproducible bit for bit:
//   dot products: per lane, +0 then += x_e*r_e in element order (each product
//     and sum rounded separately, no FMA contraction), then a butterfly over
//     lane distances 8, 4, 2, 1;
//   rotation: butterflies at strides 1..64 in increasing order, then one
//     multiply by fl32(1/sqrt(128));
//   quantiser: min/max made unsigned-zero, s = (mx - mn)/(2^b - 1), fp16 RNE
//     scale and offset, code = clamp(rint((y - z)/s), 0, 2^b - 1), code 0 when
//     the fp16 scale is 0.
#include "rq_common.cuh"
#include "rq_internal.h"

#include "rq_encode_dev.cuh"

namespace rq {
namespace {

using enc::kFull;
using enc::inv_sqrt_d;

__global__ void __launch_bounds__(256) encode_kernel(const EncodeParams P) {
  enc::encode_warp(P, blockIdx.x * 8 + (threadIdx.x >> 5), threadIdx.x & 31);
}

// ---------------------------------------------------------------------------
// Reconstruction (test support): fp32 alpha*ref + H^T deq(codes); under a
// chained policy ref is the previous link's reconstruction, already in out[]
// ---------------------------------------------------------------------------
__device__ __forceinline__ void fwht128_fast(float (&x)[8], int j) {
#pragma unroll
  for (int h = 1; h < 8; h <<= 1)
#pragma unroll
    for (int e = 0; e < 8; ++e)
      if ((e & h) == 0) {
        const float a = x[e], b = x[e + h];
        x[e] = a + b;
        x[e + h] = a - b;
      }
#pragma unroll
  for (int m = 1; m < 16; m <<= 1) {
    const bool upper = (j & m) != 0;
#pragma unroll
    for (int e = 0; e < 8; ++e) {
      const float o = __shfl_xor_sync(kFull, x[e], m);
      x[e] = upper ? (o - x[e]) : (x[e] + o);
    }
  }
  const float c = inv_sqrt_d();
#pragma unroll
  for (int e = 0; e < 8; ++e) x[e] *= c;
}

__device__ __forceinline__ void dequant8(const uint8_t* codes, const uint8_t* meta, int bits,
                                         int g, int64_t rec, int j, float (&y)[8]) {
  const int lpg = g >> 3;
  const float2 sz = half2_bits_to_f2(
      *reinterpret_cast<const uint32_t*>(meta + rec * (4 * (kD / g)) + 4 * (j / lpg)));
  if (bits == 2) {
    const uint32_t w = *reinterpret_cast<const uint16_t*>(codes + rec * 32 + 2 * j);
#pragma unroll
    for (int e = 0; e < 8; ++e) y[e] = fmaf(static_cast<float>((w >> (2 * e)) & 3u), sz.x, sz.y);
  } else {
    const uint32_t w = *reinterpret_cast<const uint32_t*>(codes + rec * 64 + 4 * j);
#pragma unroll
    for (int e = 0; e < 8; ++e) y[e] = fmaf(static_cast<float>((w >> (4 * e)) & 15u), sz.x, sz.y);
  }
}

__global__ void __launch_bounds__(256) reconstruct_kernel(const ReconstructParams P) {
  const int warp = blockIdx.x * 8 + (threadIdx.x >> 5);
  const int total = P.B * P.Hkv * P.n;
  if (warp >= total) return;
  const int lane = threadIdx.x & 31;
  const int kv = lane >> 4, j = lane & 15;
  const int i = warp % P.n;
  const int bh = warp / P.n;
  const int64_t rec = static_cast<int64_t>(bh) * P.cap_pad + P.t0 + i;
  float* dst = P.out[kv] + (static_cast<int64_t>(bh) * P.n + i) * kD + 8 * j;
  float ref[8];
  if (P.ref_from_out) {  // the previous link of a chain, reconstructed in place
    const float4 a = reinterpret_cast<const float4*>(dst)[0], b = reinterpret_cast<const float4*>(dst)[1];
    ref[0] = a.x; ref[1] = a.y; ref[2] = a.z; ref[3] = a.w;
    ref[4] = b.x; ref[5] = b.y; ref[6] = b.z; ref[7] = b.w;
  } else if (P.ref_bits == 16) {
    const uint4 raw = *reinterpret_cast<const uint4*>(P.ref_plane[kv] + rec * 256 + 16 * j);
    const uint32_t w[4] = {raw.x, raw.y, raw.z, raw.w};
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      const float2 f = bf16x2_to_f2(w[e]);
      ref[2 * e] = f.x;
      ref[2 * e + 1] = f.y;
    }
  } else {
    dequant8(P.ref_plane[kv], P.ref_meta[kv], 4, 32, rec, j, ref);
  }
  float out[8];
  if (P.is_ref) {
#pragma unroll
    for (int e = 0; e < 8; ++e) out[e] = ref[e];
  } else {
    dequant8(P.codes[kv], P.meta[kv], P.bits, P.group, rec, j, out);
    if (P.rotate) fwht128_fast(out, j);
    const float a = __half2float(*reinterpret_cast<const __half*>(P.alpha + rec * 4 + 2 * kv));
#pragma unroll
    for (int e = 0; e < 8; ++e) out[e] = fmaf(a, ref[e], out[e]);
  }
  reinterpret_cast<float4*>(dst)[0] = make_float4(out[0], out[1], out[2], out[3]);
  reinterpret_cast<float4*>(dst)[1] = make_float4(out[4], out[5], out[6], out[7]);
}

}  // namespace

cudaError_t launch_encode(const EncodeParams& p, cudaStream_t s) {
  const int64_t warps = static_cast<int64_t>(p.B) * p.Hkv * p.n_tokens;
  if (warps == 0) return cudaSuccess;
  const int64_t blocks = (warps + 7) / 8;
  encode_kernel<<<static_cast<unsigned>(blocks), 256, 0, s>>>(p);
  return cudaGetLastError();
}

cudaError_t launch_reconstruct(const ReconstructParams& p, cudaStream_t s) {
  const int64_t warps = static_cast<int64_t>(p.B) * p.Hkv * p.n;
  if (warps == 0) return cudaSuccess;
  const int64_t blocks = (warps + 7) / 8;
  reconstruct_kernel<<<static_cast<unsigned>(blocks), 256, 0, s>>>(p);
  return cudaGetLastError();
}

}  // namespace rq
