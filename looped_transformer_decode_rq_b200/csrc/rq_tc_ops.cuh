// rq_tc_ops.cuh -- per-thread operations shared by the tensor-core decode
// kernels (rq_decode_tc.cuh, rq_decode_pp.cu): warp reductions, the expansion of
// packed 2/4-bit codes into int8 rows in the byte order the MMAs' other
// operands use, and the 24-bit byte-plane operands that carry queries and
// softmax weights to the int8 tensor cores.
#pragma once

#include "rq_common.cuh"

namespace rq {
namespace {

constexpr unsigned kFull = 0xffffffffu;
constexpr float kQ3 = 8323072.f;  // signed 24-bit range whose top byte stays in [-127, 127]
constexpr float kU3 = 16777215.f; // unsigned 24-bit range

__device__ __forceinline__ float fast_exp2(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

__device__ __forceinline__ float rcp_approx(float x) {
  float y;
  asm("rcp.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

__device__ __forceinline__ float warp_max(float v) {
  int i = __float_as_int(v);
  i ^= (i >> 31) & 0x7fffffff;
  i = __reduce_max_sync(kFull, i);
  i ^= (i >> 31) & 0x7fffffff;
  return __int_as_float(i);
}

// max of non-negative floats (their bit patterns order as integers)
__device__ __forceinline__ float warp_max_nonneg(float v) {
  return __int_as_float(__reduce_max_sync(kFull, __float_as_int(v)));
}

__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
  for (int o = 16; o >= 1; o >>= 1) v += __shfl_xor_sync(kFull, v, o);
  return v;
}

// ---------------------------------------------------------------------------
// code expansion order.  Within a 32-dim chunk, byte j of the expanded row
// holds dim e(j):
//   2-bit codes: j = 8k + 4w + b  <->  e = 16w + 4b + k   ((word_w >> 2k) & 0x03030303)
//   4-bit codes: j = 16k + 4w + b <->  e = 8w + 2b + k    ((word_w >> 4k) & 0x0F0F0F0F)
// ---------------------------------------------------------------------------
template <int BITS>
__device__ __forceinline__ int pos_dim(int j) {  // position in chunk -> dim in chunk
  return BITS == 2 ? 16 * ((j >> 2) & 1) + 4 * (j & 3) + (j >> 3) : 8 * ((j >> 2) & 3) + 2 * (j & 3) + (j >> 4);
}
template <int BITS>
__device__ __forceinline__ int dim_pos(int e) {  // dim in chunk -> position in chunk
  return BITS == 2 ? 8 * (e & 3) + 4 * (e >> 4) + ((e >> 2) & 3) : 16 * (e & 1) + 4 * (e >> 3) + ((e >> 1) & 3);
}

// Expand one token's packed codes (BITS * 16 bytes) into row r of a 128 x 128
// int8 tile with the 128-byte swizzle (16-byte chunk q of row r stored at
// chunk q ^ (r & 7)).
template <int BITS>
__device__ __forceinline__ void expand_row(const uint8_t* src, uint8_t* tile, int r) {
  uint8_t* row = tile + r * 128;
  const int sw = r & 7;
  constexpr int NW = BITS * 4;  // packed 32-bit words per token
  uint32_t w[NW];
#pragma unroll
  for (int i = 0; i < NW / 4; ++i) {
    const uint4 v = *reinterpret_cast<const uint4*>(src + 16 * i);
    w[4 * i] = v.x; w[4 * i + 1] = v.y; w[4 * i + 2] = v.z; w[4 * i + 3] = v.w;
  }
  constexpr int WPC = BITS == 2 ? 2 : 4;  // words per 32-dim chunk
#pragma unroll
  for (int c = 0; c < 4; ++c) {
    uint32_t o[8];
#pragma unroll
    for (int u = 0; u < 8; ++u) {
      const int k = u / WPC, ww = u % WPC;
      o[u] = BITS == 2 ? ((w[WPC * c + ww] >> (2 * k)) & 0x03030303u) : ((w[WPC * c + ww] >> (4 * k)) & 0x0F0F0F0Fu);
    }
    *reinterpret_cast<uint4*>(row + (((2 * c) ^ sw) << 4)) = make_uint4(o[0], o[1], o[2], o[3]);
    *reinterpret_cast<uint4*>(row + (((2 * c + 1) ^ sw) << 4)) = make_uint4(o[4], o[5], o[6], o[7]);
  }
}

// byte (n, j) of an N x 128 int8 K-major operand with the 128-byte swizzle
__device__ __forceinline__ int kmaj_byte(int n, int j) {
  return (n >> 3) * 1024 + (n & 7) * 128 + (((j >> 4) ^ (n & 7)) << 4) + (j & 15);
}

// signed bytes of a 24-bit-range integer: v = 65536 b2 + 256 b1 + b0
__device__ __forceinline__ void split24(int v, int& b2, int& b1, int& b0) {
  const int t = (v + 128) >> 8;
  b0 = v - (t << 8);
  b2 = (t + 128) >> 8;
  b1 = t - (b2 << 8);
}

constexpr int round16(int x) { return (x + 15) & ~15; }

// ---------------------------------------------------------------------------
// segment set-up (warp w < G: query head w of kv-head h): the B operands that
// carry the queries.  Rows of the int8 operands are (sub-group, head, hi/lo).
// ---------------------------------------------------------------------------
// x: dims 4 lane .. 4 lane + 3 of query head hq, quantised to 24-bit integers
// with one scale per head and written as three signed bytes into rows
// p * 3 GG + 3 hq + j.  With 16-dim groups p is the group's parity within its
// 32-dim chunk and the rows of the other parity are zero there; with 32-dim
// groups p = 0.
template <int BITS, int RGRP, int GG>
__device__ __forceinline__ void put_q_s24(uint8_t* tile, const float (&x)[4], int hq, int lane, float* scale_out,
                                          float* gsum_out, float scale_log2) {
  float m = fmaxf(fmaxf(fabsf(x[0]), fabsf(x[1])), fmaxf(fabsf(x[2]), fabsf(x[3])));
  m = warp_max_nonneg(m);
  const float inv = m > 0.f ? kQ3 / m : 0.f;
#pragma unroll
  for (int e = 0; e < 4; ++e) {
    const int d = 4 * lane + e;
    int qi = __float2int_rn(x[e] * inv);
    qi = max(-8323072, min(8323072, qi));
    int b[3];
    split24(qi, b[0], b[1], b[2]);
    const int j = 32 * (d >> 5) + dim_pos<BITS>(d & 31);
    const int par = RGRP == 16 ? ((d >> 4) & 1) : 0;
#pragma unroll
    for (int k = 0; k < 3; ++k) {
      tile[kmaj_byte(par * 3 * GG + 3 * hq + k, j)] = static_cast<uint8_t>(b[k]);
      if constexpr (RGRP == 16) tile[kmaj_byte((1 - par) * 3 * GG + 3 * hq + k, j)] = 0;
    }
  }
  float s = x[0] + x[1] + x[2] + x[3];
  constexpr int LPG = RGRP / 4;  // lanes per group
#pragma unroll
  for (int o = 1; o < LPG; o <<= 1) s += __shfl_xor_sync(kFull, s, o);
  if ((lane % LPG) == 0) gsum_out[lane / LPG] = s * scale_log2;
  if (lane == 0) *scale_out = m * (1.f / kQ3) * scale_log2;
}

// The same query quantisation, written for one MMA sequence over all 128 dims
// whose output columns are (group, byte plane): row 3 g + k holds byte k of the
// query's elements in group g (RGRP dims each) and zero at every other group's
// K positions, so that accumulating the four 32-dim chunks gives each group's
// dot product in columns 3 g .. 3 g + 2.
template <int BITS, int RGRP>
__device__ __forceinline__ void put_q_grouped(uint8_t* tile, const float (&x)[4], int lane, float* scale_out,
                                              float* gsum_out, float scale_log2) {
  constexpr int NGRP = 128 / RGRP;
  float m = fmaxf(fmaxf(fabsf(x[0]), fabsf(x[1])), fmaxf(fabsf(x[2]), fabsf(x[3])));
  m = warp_max_nonneg(m);
  const float inv = m > 0.f ? kQ3 / m : 0.f;
#pragma unroll
  for (int e = 0; e < 4; ++e) {
    const int d = 4 * lane + e;
    int qi = __float2int_rn(x[e] * inv);
    qi = max(-8323072, min(8323072, qi));
    int b[3];
    split24(qi, b[0], b[1], b[2]);
    const int j = 32 * (d >> 5) + dim_pos<BITS>(d & 31);
    const int g = d / RGRP;
#pragma unroll
    for (int gg = 0; gg < NGRP; ++gg)
#pragma unroll
      for (int k = 0; k < 3; ++k) tile[kmaj_byte(3 * gg + k, j)] = gg == g ? static_cast<uint8_t>(b[k]) : 0;
  }
  float s = x[0] + x[1] + x[2] + x[3];
  constexpr int LPG = RGRP / 4;  // lanes per group
#pragma unroll
  for (int o = 1; o < LPG; o <<= 1) s += __shfl_xor_sync(kFull, s, o);
  if ((lane % LPG) == 0) gsum_out[lane / LPG] = s * scale_log2;
  if (lane == 0) *scale_out = m * (1.f / kQ3) * scale_log2;
}

// Byte planes of NB 24-bit values v[] (byte 2 = top): out[j] holds byte 2 - j
// of every value, value m at byte m of the plane.
template <int NB>
__device__ __forceinline__ void byte_planes(const uint32_t (&v)[NB], uint32_t (&out)[3][NB / 4]) {
#pragma unroll
  for (int j = 0; j < 3; ++j) {
    const uint32_t sel = (2 - j) | ((6 - j) << 4);
#pragma unroll
    for (int w = 0; w < NB / 4; ++w) {
      const uint32_t lo = __byte_perm(v[4 * w], v[4 * w + 1], sel);
      const uint32_t hi = __byte_perm(v[4 * w + 2], v[4 * w + 3], sel);
      out[j][w] = __byte_perm(lo, hi, 0x5410);
    }
  }
}

// store NB bytes (4, 8, 16 or 32) of a byte plane at rows n0.. of an MN-major
// (no swizzle) int8 operand, token row offset `wrow`
template <int NB>
__device__ __forceinline__ void put_plane(uint8_t* tile, int n0, int wrow, const uint32_t (&w)[NB / 4]) {
  uint8_t* dst = tile + (n0 >> 4) * 2048 + wrow + (n0 & 15);
  if constexpr (NB == 4) {
    *reinterpret_cast<uint32_t*>(dst) = w[0];
  } else if constexpr (NB == 8) {
    *reinterpret_cast<uint2*>(dst) = make_uint2(w[0], w[1]);
  } else if constexpr (NB == 16) {
    *reinterpret_cast<uint4*>(dst) = make_uint4(w[0], w[1], w[2], w[3]);
  } else {
    static_assert(NB == 32, "byte plane width");
    *reinterpret_cast<uint4*>(dst) = make_uint4(w[0], w[1], w[2], w[3]);
    *reinterpret_cast<uint4*>(dst + 2048) = make_uint4(w[4], w[5], w[6], w[7]);
  }
}

// One token's packed codes widened to int8, in 32-bit words, chunk-major: word
// 8c + u holds bytes 4u .. 4u + 3 of 32-dim chunk c, in the order of
// pos_dim / dim_pos (the layout expand_row writes into a shared tile).
template <int BITS>
__device__ __forceinline__ void widen_codes(const uint8_t* src, uint32_t (&o)[32]) {
  constexpr int NW = BITS * 4;  // packed 32-bit words per token
  uint32_t w[NW];
#pragma unroll
  for (int i = 0; i < NW / 4; ++i) {
    const uint4 v = *reinterpret_cast<const uint4*>(src + 16 * i);
    w[4 * i] = v.x; w[4 * i + 1] = v.y; w[4 * i + 2] = v.z; w[4 * i + 3] = v.w;
  }
  constexpr int WPC = BITS == 2 ? 2 : 4;  // words per 32-dim chunk
#pragma unroll
  for (int c = 0; c < 4; ++c)
#pragma unroll
    for (int u = 0; u < 8; ++u) {
      const int k = u / WPC, ww = u % WPC;
      o[8 * c + u] = BITS == 2 ? ((w[WPC * c + ww] >> (2 * k)) & 0x03030303u) : ((w[WPC * c + ww] >> (4 * k)) & 0x0F0F0F0Fu);
    }
}

// 65536 b2 + 256 b1 + b0 of three int32 byte-products (as fp32)
__device__ __forceinline__ float comb24(uint32_t b2, uint32_t b1, uint32_t b0) {
  return fmaf(65536.f, static_cast<float>(static_cast<int>(b2)),
              fmaf(256.f, static_cast<float>(static_cast<int>(b1)), static_cast<float>(static_cast<int>(b0))));
}

}  // namespace
}  // namespace rq
