// rq_encode_dev.cuh -- the per-warp encode of one (sequence, kv-head, token)
// for every loop, shared by the encode kernel and the decode call that appends
// the new token ("ResidualQuant: KV Cache Quantization for Looped Transformers
// with 2-Bit Residuals", abstract; Figure 1 steps 2-5; Figure 2 caption; the
// arithmetic order is documented at the top of rq_encode.cu).
#pragma once

#include "rq_common.cuh"
#include "rq_internal.h"

namespace rq {
namespace enc {

constexpr unsigned kFull = 0xffffffffu;
// fl32(1/sqrt(128)) = 0x3DB504F3
static __device__ __forceinline__ float inv_sqrt_d() { return __int_as_float(0x3DB504F3); }

static __device__ __forceinline__ void load8_bf16(const uint16_t* src, float (&x)[8]) {
  const uint4 raw = __ldg(reinterpret_cast<const uint4*>(src));
  float2 a = bf16x2_to_f2(raw.x), b = bf16x2_to_f2(raw.y), c = bf16x2_to_f2(raw.z),
         d = bf16x2_to_f2(raw.w);
  x[0] = a.x; x[1] = a.y; x[2] = b.x; x[3] = b.y;
  x[4] = c.x; x[5] = c.y; x[6] = d.x; x[7] = d.y;
}

static __device__ __forceinline__ bool in_range8(const float (&x)[8]) {
  bool ok = true;
#pragma unroll
  for (int e = 0; e < 8; ++e) ok &= (fabsf(x[e]) <= 65504.f);  // false for NaN
  return ok;
}

// <a, b> over a half-warp's 128 elements in the fixed order.
static __device__ __forceinline__ float tree_dot(const float (&a)[8], const float (&b)[8]) {
  float p = 0.f;
#pragma unroll
  for (int e = 0; e < 8; ++e) p = __fadd_rn(p, __fmul_rn(a[e], b[e]));
#pragma unroll
  for (int o = 8; o >= 1; o >>= 1) p = __fadd_rn(p, __shfl_xor_sync(kFull, p, o));
  return p;
}

// In-place rotation of a half-warp's 128 elements (lane j holds 8j..8j+7).
static __device__ __forceinline__ void fwht128(float (&x)[8], int j) {
#pragma unroll
  for (int h = 1; h < 8; h <<= 1) {
#pragma unroll
    for (int e = 0; e < 8; ++e) {
      if ((e & h) == 0) {
        const float a = x[e], b = x[e + h];
        x[e] = __fadd_rn(a, b);
        x[e + h] = __fsub_rn(a, b);
      }
    }
  }
#pragma unroll
  for (int m = 1; m < 16; m <<= 1) {
    const bool upper = (j & m) != 0;
#pragma unroll
    for (int e = 0; e < 8; ++e) {
      const float o = __shfl_xor_sync(kFull, x[e], m);
      x[e] = upper ? __fsub_rn(o, x[e]) : __fadd_rn(x[e], o);
    }
  }
  const float c = inv_sqrt_d();
#pragma unroll
  for (int e = 0; e < 8; ++e) x[e] = __fmul_rn(x[e], c);
}

// Group min-max quantiser.  lanes_per_group = g / 8 (2 or 4).  Returns the
// 8 codes of this lane and the group's fp16 scale/offset.
static __device__ __forceinline__ void quantize8(const float (&y)[8], int bits, int lanes_per_group,
                                          uint32_t (&c)[8], __half& s_h, __half& z_h) {
  float mn = y[0], mx = y[0];
#pragma unroll
  for (int e = 1; e < 8; ++e) {
    mn = fminf(mn, y[e]);
    mx = fmaxf(mx, y[e]);
  }
  for (int o = 1; o < lanes_per_group; o <<= 1) {
    mn = fminf(mn, __shfl_xor_sync(kFull, mn, o));
    mx = fmaxf(mx, __shfl_xor_sync(kFull, mx, o));
  }
  mn = __fadd_rn(mn, 0.f);  // an exact zero becomes +0 in every lane
  mx = __fadd_rn(mx, 0.f);
  const float qmax = static_cast<float>((1 << bits) - 1);
  const float s = __fdiv_rn(__fsub_rn(mx, mn), qmax);
  s_h = __float2half_rn(s);
  z_h = __float2half_rn(mn);
  const float sf = __half2float(s_h), zf = __half2float(z_h);
#pragma unroll
  for (int e = 0; e < 8; ++e) {
    float u = 0.f;
    if (sf > 0.f) u = fminf(fmaxf(rintf(__fdiv_rn(__fsub_rn(y[e], zf), sf)), 0.f), qmax);
    c[e] = static_cast<uint32_t>(u);
  }
}

static __device__ __forceinline__ uint32_t half2_bits(__half s, __half z) {
  return static_cast<uint32_t>(__half_as_ushort(s)) |
         (static_cast<uint32_t>(__half_as_ushort(z)) << 16);
}

static __device__ __forceinline__ bool half_finite(__half h) {
  return (__half_as_ushort(h) & 0x7C00u) != 0x7C00u;
}

// Encode token `warp` (flattened (b, h, i) over the call's tokens) with the 32
// lanes of the calling warp: lanes 0-15 the key, 16-31 the value.
static __device__ __forceinline__ void encode_warp(const EncodeParams& P, int warp, int lane) {
  const int total = P.B * P.Hkv * P.n_tokens;
  if (warp >= total) return;
  const int kv = lane >> 4;  // 0: key, 1: value
  const int j = lane & 15;
  const int i = warp % P.n_tokens;
  const int bh = warp / P.n_tokens;
  const int h = bh % P.Hkv;
  const int b = bh / P.Hkv;
  const int pos = (P.positions ? P.positions[b] : P.start_pos) + i;
  if (pos < 0 || pos >= P.capacity) {  // warp-uniform
    if (lane == 0) set_flag(P.status, RQ_FLAG_POSITION);
    return;
  }
  const uint16_t* X = kv ? P.v : P.k;
  const int64_t src0 = b * P.s_b + h * P.s_h + static_cast<int64_t>(i) * P.s_t + 8 * j;
  const int64_t rec = static_cast<int64_t>(b * P.Hkv + h) * P.cap_pad + pos;
  bool bad = false, overflow = false;

  for (int a = 0; a < P.L; ++a) {  // every anchor, then the loops it anchors
    if (P.anchor[a] != a) continue;
    float ref[8];
    {
      const uint16_t* src = X + static_cast<int64_t>(a) * P.s_l + src0;
      load8_bf16(src, ref);
      bad |= !in_range8(ref);
      if (P.bits[a] == 16) {
        *reinterpret_cast<uint4*>(P.codes[a][kv] + rec * 256 + 16 * j) =
            __ldg(reinterpret_cast<const uint4*>(src));
      } else {
        uint32_t c[8];
        __half s_h, z_h;
        quantize8(ref, 4, 4, c, s_h, z_h);
        uint32_t w = 0;
#pragma unroll
        for (int e = 0; e < 8; ++e) w |= c[e] << (4 * e);
        *reinterpret_cast<uint32_t*>(P.codes[a][kv] + rec * 64 + 4 * j) = w;
        if ((j & 3) == 0)
          *reinterpret_cast<uint32_t*>(P.meta[a][kv] + rec * 16 + 4 * (j >> 2)) = half2_bits(s_h, z_h);
        overflow |= !(half_finite(s_h) && half_finite(z_h));
        const float sf = __half2float(s_h), zf = __half2float(z_h);
#pragma unroll
        for (int e = 0; e < 8; ++e) ref[e] = __fadd_rn(zf, __fmul_rn(static_cast<float>(c[e]), sf));
      }
    }
    float refref = 0.f;
    bool have_refref = false;

    // Loops stored against `cur` (the anchor first).  Under a chained policy
    // exactly one loop takes `cur` as its reference; its binary32
    // reconstruction then becomes `ref` and the walk moves one link outward.
    int cur = a;
    for (int link = 0; link < P.L; ++link) {
      int next = -1;
      for (int l = 0; l < P.L; ++l) {
        if (l == cur || P.ref[l] != cur) continue;
        float x[8];
        load8_bf16(X + static_cast<int64_t>(l) * P.s_l + src0, x);
        bad |= !in_range8(x);
        float al = 0.f;
        const int mode = P.alpha_mode[l];
        if (mode == RQ_ALPHA_LS || mode == RQ_ALPHA_NORM_RATIO) {
          if (!have_refref) {
            refref = tree_dot(ref, ref);
            have_refref = true;
          }
          if (mode == RQ_ALPHA_LS) {
            const float num = tree_dot(x, ref);
            al = (refref == 0.f) ? 0.f : __fdiv_rn(num, refref);
          } else {
            const float xx = tree_dot(x, x);
            al = (refref == 0.f) ? 0.f : __fdiv_rn(__fsqrt_rn(xx), __fsqrt_rn(refref));
          }
        } else if (mode == RQ_ALPHA_ONE) {
          al = 1.f;
        }
        const __half a_h = __float2half_rn(al);
        overflow |= !half_finite(a_h);
        if (j == 0)
          *reinterpret_cast<__half*>(P.alpha[l] + rec * 4 + 2 * kv) = a_h;
        const float af = __half2float(a_h);
#pragma unroll
        for (int e = 0; e < 8; ++e) x[e] = __fsub_rn(x[e], __fmul_rn(af, ref[e]));
        if (P.rotate[l]) fwht128(x, j);
        const int bits = P.bits[l], g = P.group[l];
        uint32_t c[8];
        __half s_h, z_h;
        quantize8(x, bits, g >> 3, c, s_h, z_h);
        overflow |= !(half_finite(s_h) && half_finite(z_h));
        if (bits == 2) {
          uint32_t w = 0;
#pragma unroll
          for (int e = 0; e < 8; ++e) w |= c[e] << (2 * e);
          *reinterpret_cast<uint16_t*>(P.codes[l][kv] + rec * 32 + 2 * j) = static_cast<uint16_t>(w);
        } else {
          uint32_t w = 0;
#pragma unroll
          for (int e = 0; e < 8; ++e) w |= c[e] << (4 * e);
          *reinterpret_cast<uint32_t*>(P.codes[l][kv] + rec * 64 + 4 * j) = w;
        }
        const int lpg = g >> 3;
        if ((j % lpg) == 0)
          *reinterpret_cast<uint32_t*>(P.meta[l][kv] + rec * (4 * (kD / g)) + 4 * (j / lpg)) =
              half2_bits(s_h, z_h);
        if (P.chained) {  // x_hat = (alpha_hat * ref) + H deq, deq = z_hat + (code * s_hat)
          const float sf = __half2float(s_h), zf = __half2float(z_h);
          float u[8];
#pragma unroll
          for (int e = 0; e < 8; ++e) u[e] = __fadd_rn(zf, __fmul_rn(static_cast<float>(c[e]), sf));
          if (P.rotate[l]) fwht128(u, j);
#pragma unroll
          for (int e = 0; e < 8; ++e) ref[e] = __fadd_rn(__fmul_rn(af, ref[e]), u[e]);
          have_refref = false;
          next = l;
          break;
        }
      }
      if (next < 0) break;
      cur = next;
    }
  }
  const unsigned any_bad = __ballot_sync(kFull, bad);
  const unsigned any_ovf = __ballot_sync(kFull, overflow);
  if (lane == 0) {
    if (any_bad) set_flag(P.status, RQ_FLAG_BAD_INPUT);
    if (any_ovf) set_flag(P.status, RQ_FLAG_META_OVERFLOW);
  }
}

}  // namespace enc
}  // namespace rq
