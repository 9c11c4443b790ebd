// rq_decode_split.cuh -- the CUDA-core split kernel of the fused decode
// attention (see rq_decode.cu for the method), as templates over the loop
// format: anchor kind, residual bits and group, query rows per kv-head G, page
// size, the number of residual links NCH (1, or 2-3 for the loops of a chained
// Previous-/Next-loop policy) and the number of consumer groups NG.  Included by
// rq_decode.cu (NCH = 1) and rq_decode_chain.cu (NCH = 2, 3), so that the two
// sets of instantiations compile in parallel.
//
// Persistent, one CTA per SM:
//   * the flattened sequence of pages (64 tokens with a bf16 anchor, 128 for
//     the byte-plane formats) over all (b, kv-head) pairs is cut into num_ctas
//     contiguous ranges of equal length, so ragged batches balance to within
//     one page; a CTA emits one partial (m, l, acc) per (b, kv-head) segment
//     it touches;
//   * two warps after the consumers are the producers: one lane of each
//     (the even stages, the odd stages) streams pages into a ring of
//     shared-memory stages through the Tensor Memory Accelerator -- tiled
//     tensor copies with the 128-byte swizzle for bf16 anchor tiles, bulk
//     copies for code, metadata and alpha records -- completing on mbarriers;
//   * the consumer warps form NG groups of four (2, or 3 for the byte-plane
//     formats at G = 1) that take pages in turn, each with its own online
//     softmax and group-local barriers, so that one group's barrier and
//     reduction latency overlaps the others' math.  Within a group a page is
//     processed in two phases: scores (4G lanes per token, dp4a on the packed
//     codes, shuffle reduction) and values (16 lanes per token row, 8 dims per
//     lane, softmax weights recomputed per lane).  The groups merge once per
//     segment, in a fixed order;
//   * packed codes become subnormal floats with one AND each (c * 2^(p-149),
//     code_sub), against weights pre-multiplied by 2^100; the remaining power
//     of two is folded into the accumulators once per flush; fp32 pairs use
//     FFMA2.
#pragma once

#include "rq_common.cuh"
#include "rq_internal.h"
#include "rq_tcgen05.cuh"

// Internal linkage: each including translation unit has its own copy.
namespace rq {
namespace {

// Consumer warps come in groups of four; a CTA has NG = 2 or 3 groups (8 or 12
// consumer warps) plus the producer warp.
constexpr int kGW = 4;         // warps per consumer group
constexpr int kGT = kGW * 32;  // threads per consumer group
constexpr int kConsumerBar = 1;  // all consumers
constexpr int kGroupBar0 = 2;    // group g uses kGroupBar0 + g (128 threads)
constexpr unsigned kFull = 0xffffffffu;
// Register split of the variants that need more than the 168 registers a
// thread of a 288-thread CTA gets (warps take registers in fours): the producer
// warp comes with three idle warps, a warpgroup that keeps kSplitRegsAux of the
// 168 registers a thread and gives the rest to the two consumer warpgroups:
//   384 x 168 = 128 x kSplitRegsAux + 256 x kSplitRegsConsumer.
constexpr int kSplitRegsAux = 56;
constexpr int kSplitRegsConsumer = 224;
static_assert(384 * 168 == 128 * kSplitRegsAux + 256 * kSplitRegsConsumer, "register split");

__device__ __forceinline__ float pow2i(int e) { return __int_as_float((127 + e) << 23); }

// 2^x on the special-function unit (inputs are <= 0 here: softmax weights and
// their rescale factors)
__device__ __forceinline__ float fast_exp2(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

// max over the warp with one integer reduction on an order-preserving key
__device__ __forceinline__ float warp_max(float v) {
  int i = __float_as_int(v);
  i ^= (i >> 31) & 0x7fffffff;
  i = __reduce_max_sync(kFull, i);
  i ^= (i >> 31) & 0x7fffffff;
  return __int_as_float(i);
}

// NCH: residual links per token (1; 2-3 for the loops of a chained policy,
// whose links share one format).  NG: consumer groups (pages k with k % NG == g
// go to group g).
template <int REF, int RB, int RG, int G, int TT, int NCH = 1, int NG = 2>
struct Cfg {
  static_assert(NCH >= 1 && NCH <= RQ_MAX_CHAIN && (NCH == 1 || (RB != 0 && REF != kRefNone)), "chain");
  static_assert(NG == 2 || NG == 3, "consumer groups");
  static constexpr int NCW = kGW * NG;   // consumer warps
  static constexpr int NCT = NCW * 32;   // consumer threads
  // four query rows with residual links hold more than 168 registers a
  // consumer thread: those variants take the register split
  static constexpr bool REGSPLIT = NG == 2 && G >= 4 && RB != 0 && REF != kRefNone;
  // + two producer warps (+ two idle warps with the register split)
  static constexpr int NT = NCT + (REGSPLIT ? 128 : 64);
  static_assert(G <= NCW, "one warp per query head in the segment set-up");
  static constexpr int PAGE = TT;  // tokens per page / stage
  // phase 1 (scores): 4G lanes per token, D1 = 32/G dims per lane
  static constexpr int TPT = 4 * G;
  static constexpr int D1 = 32 / G;
  static constexpr int EB = D1 >= 8 ? 8 : D1;   // elements per accumulation block
  static constexpr int NB = D1 / EB;
  static constexpr int TOK_PASS = kGT / TPT;    // tokens per pass of a group
  static constexpr int PASSES = TT / TOK_PASS;
  // phase 2 (values)
  static constexpr int D2 = (G >= 4) ? 4 : 8;   // dims per lane
  static constexpr int TPR2 = kD / D2;          // lanes per token row
  static constexpr int SLICES = kGT / TPR2;
  static constexpr int TOK2 = TT / SLICES;     // tokens per lane per page
  // per-record bytes
  static constexpr int REF_REC = REF == kRefBf16 ? 256 : (REF == kRefInt4 ? 64 : 0);
  static constexpr int REFM_REC = REF == kRefInt4 ? 16 : 0;
  static constexpr int CB = RB * 16;
  static constexpr int MB = RB ? 4 * (kD / RG) : 0;
  static constexpr bool HAS_ALPHA = (REF != kRefNone) && (RB != 0);
  static constexpr int AL_REC = HAS_ALPHA ? 4 : 0;
  // stage layout (each piece 1024-byte aligned)
  static constexpr int al(int x) { return (x + 1023) & ~1023; }
  static constexpr int O_REFK = 0;
  static constexpr int O_REFV = O_REFK + al(TT * REF_REC);
  static constexpr int O_REFMK = O_REFV + al(TT * REF_REC);
  static constexpr int O_REFMV = O_REFMK + al(TT * REFM_REC);
  // residual link i: key codes, value codes, key meta, value meta, alphas
  static constexpr int O_RES = O_REFMV + al(TT * REFM_REC);
  static constexpr int RES_BLK = 2 * al(TT * CB) + 2 * al(TT * MB) + al(TT * AL_REC);
  static constexpr int o_resk(int i) { return O_RES + i * RES_BLK; }
  static constexpr int o_resv(int i) { return o_resk(i) + al(TT * CB); }
  static constexpr int o_resmk(int i) { return o_resv(i) + al(TT * CB); }
  static constexpr int o_resmv(int i) { return o_resmk(i) + al(TT * MB); }
  static constexpr int o_al(int i) { return o_resmv(i) + al(TT * MB); }
  static constexpr int STAGE_BYTES = O_RES + NCH * RES_BLK;
  static constexpr int TX_BYTES = TT * (2 * REF_REC + 2 * REFM_REC + NCH * (2 * CB + 2 * MB + AL_REC));
  // non-stage shared memory
  static constexpr int O_S = 0;                           // scores [NG groups][2 parity][G][TT]
  static constexpr int O_WM = O_S + 4 * NG * 2 * G * TT;  // warp maxima [NG][2][G][kGW]
  static constexpr int O_ACC = O_WM + 4 * NG * 2 * G * kGW;  // [G][256]
  static constexpr int O_L = O_ACC + 4 * G * 2 * kD;      // [G] (padded to 8)
  static constexpr int O_MG = O_L + 4 * 8;                // [NG][G] (padded to 32)
  static constexpr int O_QS = O_MG + 4 * 32;              // [G][128]
  static constexpr int O_QT = O_QS + 4 * G * kD;          // [G][128]
  static constexpr int O_PRE = O_QT + 4 * G * kD;         // [RQ_MAX_BATCH + 1]
  static constexpr int O_NT = O_PRE + 4 * (RQ_MAX_BATCH + 1);
  static constexpr int O_MISC = O_NT + 4 * RQ_MAX_BATCH;  // abort flag
  static constexpr int O_BAR = (O_MISC + 16 + 7) & ~7;
  static constexpr int MISC_BYTES = O_BAR + 16 * 8;
  static constexpr int kSmemLimit = 227 * 1024;
  static constexpr int STAGES_MAX = (kSmemLimit - 1024 - MISC_BYTES) / STAGE_BYTES;
  // A multiple of NG stages keeps each stage with one group, so that a group
  // waiting on a stage's parity never sees a phase of another group's page.
  static constexpr int STAGES = STAGES_MAX >= 2 * NG ? 2 * NG : NG;
  static_assert(2 * STAGES < 15, "full and empty barriers below the stall barrier");
  static constexpr int SMEM_BYTES = 1024 + STAGES * STAGE_BYTES + MISC_BYTES;
  static_assert(PASSES * TOK_PASS == TT && TOK2 * SLICES == TT, "lane mapping");
  static_assert((O_ACC % 16) == 0 && (O_QS % 16) == 0 && (O_WM % 16) == 0, "alignment");
};

// ---------------------------------------------------------------------------
// code unpacking helpers
// ---------------------------------------------------------------------------
// Load `NB` bytes (1, 2, 4, 8 or 16) of packed codes into 32-bit words.
template <int NB>
__device__ __forceinline__ void load_codes(const uint8_t* p, uint32_t (&w)[(NB + 3) / 4]) {
  if constexpr (NB == 16) {
    const uint4 v = *reinterpret_cast<const uint4*>(p);
    w[0] = v.x; w[1] = v.y; w[2] = v.z; w[3] = v.w;
  } else if constexpr (NB == 8) {
    const uint2 v = *reinterpret_cast<const uint2*>(p);
    w[0] = v.x; w[1] = v.y;
  } else if constexpr (NB == 4) {
    w[0] = *reinterpret_cast<const uint32_t*>(p);
  } else if constexpr (NB == 2) {
    w[0] = *reinterpret_cast<const uint16_t*>(p);
  } else {
    w[0] = *p;
  }
}

template <int BITS>
__device__ __forceinline__ int code_pos(int e) { return (e * BITS) & 15; }

// Code e of a thread's unit as the subnormal float c * 2^(p_e - 149): one AND
// leaves the code's bits in the mantissa under a zero exponent, so nothing has
// to be subtracted.  The value weights are multiplied by kSubScale = 2^100
// first, which keeps every product w * c a normal number (the FMA forms it
// exactly), and an accumulator of code e is scaled by 2^(kSubExp - p_e) at the
// end.  (Subnormals are kept: the library is built without flush-to-zero.)
constexpr float kSubScale = 0x1p100f;
constexpr int kSubExp = 49;
template <int BITS>
__device__ __forceinline__ float code_sub(const uint32_t* w, int e) {
  const int bit = e * BITS;
  const uint32_t word = w[bit >> 5];
  const int b32 = bit & 31;
  const uint32_t src = (b32 >= 16) ? (word >> 16) : word;
  const int p = b32 & 15;
  return __uint_as_float(src & (((1u << BITS) - 1u) << p));
}

// Integer-dot-product operands for a lane's D query values against BITS-bit
// packed codes.  The values are quantised to int16 with one scale per lane
// (|q| <= 32767 * scale) and split into a signed high byte and an unsigned low
// byte, so that  sum_e q_e c_e = scale * (256 * dp4a(c, hi) + dp4a(c, lo))
// exactly in 32-bit integers.  Byte b of operand [w][k] pairs with the code
// that the unpacking of word w puts into byte b at step k:
//   BITS = 2: (w >> 2k) & 0x03030303 holds elements 16w + 4b + k   (k < 4)
//   BITS = 4: (w >> 4k) & 0x0F0F0F0F holds elements  8w + 2b + k   (k < 2)
template <int BITS, int D>
struct DotOperands {
  static constexpr int NW = (D * BITS + 31) / 32;
  static constexpr int KPW = BITS == 2 ? 4 : 2;
  uint32_t hi[NW][KPW];
  uint32_t lo[NW][KPW];
  float scale;

  __device__ __forceinline__ void build(const float* v) {
    float m = 0.f;
#pragma unroll
    for (int e = 0; e < D; ++e) m = fmaxf(m, fabsf(v[e]));
    scale = m * (1.f / 32767.f);
    const float inv = m > 0.f ? 32767.f / m : 0.f;
#pragma unroll
    for (int w = 0; w < NW; ++w)
#pragma unroll
      for (int k = 0; k < KPW; ++k) hi[w][k] = lo[w][k] = 0u;
#pragma unroll
    for (int e = 0; e < D; ++e) {
      int qi = __float2int_rn(v[e] * inv);
      qi = max(-32767, min(32767, qi));
      const int per = 32 / BITS, w = e / per, in = e % per;
      const int b = BITS == 2 ? in / 4 : in / 2, k = BITS == 2 ? in % 4 : in % 2;
      hi[w][k] |= (static_cast<uint32_t>(qi >> 8) & 0xFFu) << (8 * b);
      lo[w][k] |= (static_cast<uint32_t>(qi) & 0xFFu) << (8 * b);
    }
  }
};

template <int BITS>
__device__ __forceinline__ uint32_t unpack_bytes(uint32_t w, int k) {
  return BITS == 2 ? ((w >> (2 * k)) & 0x03030303u) : ((w >> (4 * k)) & 0x0F0F0F0Fu);
}

constexpr float kQ24 = 8323072.f;  // signed 24-bit range whose top byte stays in [-127, 127]

// signed bytes of a 24-bit-range integer: v = 65536 b2 + 256 b1 + b0
__device__ __forceinline__ void split24s(int v, int& b2, int& b1, int& b0) {
  const int t = (v + 128) >> 8;
  b0 = v - (t << 8);
  b2 = (t + 128) >> 8;
  b1 = t - (b2 << 8);
}

// Integer-dot-product operands for a lane's D query values against 4-bit
// packed codes (the INT4 anchor, which is not rotated), with 24 bits of
// precision: the values are quantised to signed 24-bit integers with one
// scale (|q| <= kQ24 * scale) and split into three signed bytes, so that
//     sum_e q_e c_e = scale * (65536 dp4a(c, b2) + 256 dp4a(c, b1) + dp4a(c, b0))
// exactly.  Byte b of operand [w][k] pairs with element 8w + 2b + k, the code
// that (word_w >> 4k) & 0x0F0F0F0F puts into byte b.  A query with a few large
// channels keeps the precision of the others (16 bits per lane would lose it).
template <int D>
struct DotOperands24 {
  static constexpr int NW = (D + 7) / 8;
  uint32_t b2[NW][2], b1[NW][2], b0[NW][2];
  float scale;

  __device__ __forceinline__ void build(const float* v) {
    float m = 0.f;
#pragma unroll
    for (int e = 0; e < D; ++e) m = fmaxf(m, fabsf(v[e]));
    scale = m * (1.f / kQ24);
    const float inv = m > 0.f ? kQ24 / m : 0.f;
#pragma unroll
    for (int w = 0; w < NW; ++w)
#pragma unroll
      for (int k = 0; k < 2; ++k) b2[w][k] = b1[w][k] = b0[w][k] = 0u;
#pragma unroll
    for (int e = 0; e < D; ++e) {
      int qi = __float2int_rn(v[e] * inv);
      qi = max(-8323072, min(8323072, qi));
      int x2, x1, x0;
      split24s(qi, x2, x1, x0);
      const int w = e / 8, b = (e % 8) / 2, k = e % 2;
      b2[w][k] |= (static_cast<uint32_t>(x2) & 0xFFu) << (8 * b);
      b1[w][k] |= (static_cast<uint32_t>(x1) & 0xFFu) << (8 * b);
      b0[w][k] |= (static_cast<uint32_t>(x0) & 0xFFu) << (8 * b);
    }
  }
};

// 65536 x2 + 256 x1 + x0 of three byte-plane dot products, as fp32: |x1|, |x0|
// <= 32 * 15 * 128, so 256 x1 + x0 is exact in fp32 and the sum rounds once.
__device__ __forceinline__ float comb24s(int x2, int x1, int x0) {
  return fmaf(65536.f, static_cast<float>(x2), static_cast<float>(x1 * 256 + x0));
}

// ---------------------------------------------------------------------------
// split kernel
// ---------------------------------------------------------------------------
template <int REF, int RB, int RG, int G, int TT, int NCH, int NG>
__device__ __forceinline__ void issue_page(const DecodeParams& P, const CUtensorMap* tmK, const CUtensorMap* tmV,
                                           uint8_t* st, uint32_t full, const PageIter& it, int Hkv) {
  using C = Cfg<REF, RB, RG, G, TT, NCH, NG>;
  const int t0 = it.page * TT;
  // byte planes hold plane_tokens (a multiple of 64) records per (b, h): a
  // 128-token page may find only 64 of them at the plane's end
  const int nrec = (TT > kPage && P.plane_tokens > 0 && t0 + TT > P.plane_tokens)
                       ? static_cast<int>(P.plane_tokens - t0) : TT;
  mbar_arrive_expect_tx(full, REF == kRefBf16 ? C::TX_BYTES : static_cast<uint32_t>(nrec) * (C::TX_BYTES / TT));
  const int64_t rec0 = static_cast<int64_t>(it.b * Hkv + it.h) * P.plane_tokens + t0;
  if constexpr (REF == kRefBf16) {
    static_assert(TT == kPage, "bf16 anchor pages are one 64-token tile");
    tma_load_4d(smem_u32(st + C::O_REFK), tmK, 0, t0, it.h, it.b, full);
    tma_load_4d(smem_u32(st + C::O_REFK + TT * 128), tmK, 64, t0, it.h, it.b, full);
    tma_load_4d(smem_u32(st + C::O_REFV), tmV, 0, t0, it.h, it.b, full);
    tma_load_4d(smem_u32(st + C::O_REFV + TT * 128), tmV, 64, t0, it.h, it.b, full);
  } else if constexpr (REF == kRefInt4) {
    bulk_g2s(smem_u32(st + C::O_REFK), P.ref_codes[0] + rec0 * 64, nrec * 64, full);
    bulk_g2s(smem_u32(st + C::O_REFV), P.ref_codes[1] + rec0 * 64, nrec * 64, full);
    bulk_g2s(smem_u32(st + C::O_REFMK), P.ref_meta[0] + rec0 * 16, nrec * 16, full);
    bulk_g2s(smem_u32(st + C::O_REFMV), P.ref_meta[1] + rec0 * 16, nrec * 16, full);
  }
#pragma unroll
  for (int i = 0; i < NCH; ++i) {
    if constexpr (RB != 0) {
      bulk_g2s(smem_u32(st + C::o_resk(i)), P.res_codes[i][0] + rec0 * C::CB, nrec * C::CB, full);
      bulk_g2s(smem_u32(st + C::o_resv(i)), P.res_codes[i][1] + rec0 * C::CB, nrec * C::CB, full);
      bulk_g2s(smem_u32(st + C::o_resmk(i)), P.res_meta[i][0] + rec0 * C::MB, nrec * C::MB, full);
      bulk_g2s(smem_u32(st + C::o_resmv(i)), P.res_meta[i][1] + rec0 * C::MB, nrec * C::MB, full);
    }
    if constexpr (C::HAS_ALPHA) bulk_g2s(smem_u32(st + C::o_al(i)), P.alpha[i] + rec0 * 4, nrec * 4, full);
  }
}

template <int REF, int RB, int RG, int G, int TT, int NCH, int NG>
__global__ void __launch_bounds__(Cfg<REF, RB, RG, G, TT, NCH, NG>::NT, 1)
    decode_split_kernel(const __grid_constant__ DecodeParams P,
                        const __grid_constant__ CUtensorMap tmK,
                        const __grid_constant__ CUtensorMap tmV) {
  using C = Cfg<REF, RB, RG, G, TT, NCH, NG>;
  constexpr int kNCW = C::NCW, kNCT = C::NCT, kNT = C::NT;
  extern __shared__ __align__(16) uint8_t smem_raw[];
  // align by offsetting the shared array itself so that every access below
  // stays a shared-memory access
  uint8_t* base = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
  uint8_t* stages = base;
  uint8_t* misc = base + C::STAGES * C::STAGE_BYTES;
  float* sS = reinterpret_cast<float*>(misc + C::O_S);
  float* sWM = reinterpret_cast<float*>(misc + C::O_WM);
  float* sACC = reinterpret_cast<float*>(misc + C::O_ACC);
  float* sL = reinterpret_cast<float*>(misc + C::O_L);
  float* sMG = reinterpret_cast<float*>(misc + C::O_MG);
  float* sQS = reinterpret_cast<float*>(misc + C::O_QS);
  float* sQT = reinterpret_cast<float*>(misc + C::O_QT);
  int* sPre = reinterpret_cast<int*>(misc + C::O_PRE);
  int* sNt = reinterpret_cast<int*>(misc + C::O_NT);
  volatile int* sAbort = reinterpret_cast<volatile int*>(misc + C::O_MISC);
  uint64_t* bars = reinterpret_cast<uint64_t*>(misc + C::O_BAR);

  const int tid = threadIdx.x;
  const int lane = tid & 31;
  const int warp = tid >> 5;
  const int B = P.B, Hkv = P.Hkv;
  // Launched as a programmatic dependent of the previous kernel on the stream
  // (typically the previous call's combine kernel, which reads the partials
  // this grid writes): everything above overlaps its tail; nothing global is
  // touched before it has completed.
  pdl_wait();

  // ---- page counts and their prefix over sequences
  for (int b = tid; b < B; b += kNT) {
    int len = P.ctx_len[b];
    if (len < 0 || len > P.capacity) {
      if (blockIdx.x == 0) set_flag(P.status, RQ_FLAG_CTX_LEN);
      len = len < 0 ? 0 : P.capacity;
    }
    sNt[b] = (len + TT - 1) / TT;
  }
  for (int i = tid; i < G * 2 * kD; i += kNT) sACC[i] = 0.f;
  if (tid < 8) sL[tid] = 0.f;
  if (tid == 0) *sAbort = 0;
  __syncthreads();
  if (warp == 0) {
    int carry = 0;
    for (int b0 = 0; b0 < B; b0 += 32) {
      const int b = b0 + lane;
      const int v = b < B ? sNt[b] : 0;
      int x = v;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const int y = __shfl_up_sync(kFull, x, o);
        if (lane >= o) x += y;
      }
      if (b < B) sPre[b] = carry + x - v;
      carry += __shfl_sync(kFull, x, 31);
    }
    if (lane == 0) sPre[B] = carry;
  }
  if (tid == 0) {
    for (int s = 0; s < C::STAGES; ++s) {
      mbar_init(smem_u32(&bars[s]), 1);               // full: the producer's expect_tx
      mbar_init(smem_u32(&bars[C::STAGES + s]), kGW);  // empty: the 4 warps of the page's group
    }
    mbar_init(smem_u32(&bars[15]), 1);  // never arrived at: the wait of the stall test hook
    fence_barrier_init();
  }
  __syncthreads();
  pdl_launch_dependents();  // the combine kernel may be scheduled (it waits for this grid's completion)

  const int64_t total = static_cast<int64_t>(sPre[B]) * Hkv;
  const int64_t P_eff = total < P.num_ctas ? total : P.num_ctas;
  if (static_cast<int64_t>(blockIdx.x) >= P_eff) return;
  const int64_t x0 = static_cast<int64_t>(blockIdx.x) * total / P_eff;
  const int64_t x1 = static_cast<int64_t>(blockIdx.x + 1) * total / P_eff;
  const int n_pages = static_cast<int>(x1 - x0);

  // ========================= producer warp =========================
  // Two producer threads: the first fills the even stages, the second the odd
  // ones (a stage is always filled by the same thread).  A page's copy
  // instructions keep a producer thread busy for most of a page's time.
  if (warp >= kNCW) {
    if constexpr (C::REGSPLIT) tc::setmaxnreg_dec<kSplitRegsAux>();
    const int pw = warp - kNCW;
    if (pw < 2 && lane == 0) {
      if constexpr (REF == kRefBf16) {
        prefetch_tensormap(&tmK);
        prefetch_tensormap(&tmV);
      }
      PageIter it;
      it.seek(x0, sPre, sNt, B, Hkv);
      int k = 0;
      for (; k < n_pages; ++k) {
        const int s = k % C::STAGES;
        if ((s & 1) == pw) {
          if (!mbar_wait_bounded(smem_u32(&bars[C::STAGES + s]), ((k / C::STAGES) & 1) ^ 1)) {
            set_flag(P.status, RQ_FLAG_PIPE_TIMEOUT);
            *sAbort = 1;
            break;
          }
          if (k == P.stall_page && !mbar_wait_bounded(smem_u32(&bars[15]), 0)) set_flag(P.status, RQ_FLAG_PIPE_TIMEOUT);
          if (*sAbort) break;
          issue_page<REF, RB, RG, G, TT, NCH, NG>(P, &tmK, &tmV, stages + s * C::STAGE_BYTES, smem_u32(&bars[s]), it,
                                                  Hkv);
        }
        it.next(sNt, B, Hkv);
      }
      // Drain: no copy this thread issued may still be landing when it exits
      // (each of its stages' last page: nothing later went into those stages).
      for (int kk = (k > C::STAGES ? k - C::STAGES : 0); kk < k; ++kk) {
        if (((kk % C::STAGES) & 1) != pw) continue;
        if (!mbar_wait_bounded(smem_u32(&bars[kk % C::STAGES]), (kk / C::STAGES) & 1)) {
          set_flag(P.status, RQ_FLAG_PIPE_TIMEOUT);
          break;
        }
      }
    }
    return;
  }
  if constexpr (C::REGSPLIT) tc::setmaxnreg_inc<kSplitRegsConsumer>();

  // ========================= consumer groups =========================
  const int grp = warp / kGW;        // pages k with k % NG == grp
  const int gw = warp % kGW;         // warp within the group
  const int gtid = tid % kGT;        // thread within the group
  // phase-1 mapping: token within a pass and dim slice.  For G <= 2 the lanes
  // of one shared-memory phase read rows whose swizzle phases differ, so the
  // 16-byte loads of the bf16 reference never share a bank.
  int tok1, j1;
  if constexpr (G <= 2) {
    const int jj = lane & (2 * G - 1);
    const int tsub = (lane >> (G == 1 ? 1 : 2)) & ((4 / G) - 1);
    const int box = (lane >> 3) & 1;
    const int thi = lane >> 4;
    tok1 = gw * (8 / G) + thi * (4 / G) + tsub;
    j1 = box * (2 * G) + jj;
  } else {
    tok1 = gw * (8 / G) + lane / C::TPT;
    j1 = lane % C::TPT;
  }
  const int d1 = C::D1 * j1;
  const int slice = gtid / C::TPR2;  // phase-2 mapping
  const int j2 = gtid % C::TPR2;
  const int d2 = C::D2 * j2;
  float* gS = sS + grp * 2 * G * TT;    // [2 parity][G][TT] of this group
  float* gWM = sWM + grp * 2 * G * kGW;

  PageIter it;
  it.seek(x0, sPre, sNt, B, Hkv);
  int k = 0;
  while (k < n_pages) {
    const int b = it.b, h = it.h;
    const int seg_pages = min(sNt[b] - it.page, n_pages - k);
    int len_b = P.ctx_len[b];
    len_b = len_b < 0 ? 0 : (len_b > P.capacity ? P.capacity : len_b);

    // ---- segment set-up: the G queries of (b, h) and their rotation
    if (warp < G) {
      const int qh = h * G + warp;
      const uint2 raw = *reinterpret_cast<const uint2*>(P.q + q_row_offset(P, b, h, warp) + 4 * lane);
      const float2 a01 = bf16x2_to_f2(raw.x), a23 = bf16x2_to_f2(raw.y);
      float x[4] = {a01.x, a01.y, a23.x, a23.y};
      *reinterpret_cast<float4*>(&sQS[warp * kD + 4 * lane]) = make_float4(x[0], x[1], x[2], x[3]);
      if (RB != 0 && P.rotate) {
        const float t0 = x[0] + x[1], t1 = x[0] - x[1], t2 = x[2] + x[3], t3 = x[2] - x[3];
        x[0] = t0 + t2; x[2] = t0 - t2; x[1] = t1 + t3; x[3] = t1 - t3;
#pragma unroll
        for (int m = 1; m < 32; m <<= 1) {
          const bool up = (lane & m) != 0;
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            const float o = __shfl_xor_sync(kFull, x[e], m);
            x[e] = up ? (o - x[e]) : (x[e] + o);
          }
        }
        const float c = 0.08838834764831845f;
#pragma unroll
        for (int e = 0; e < 4; ++e) x[e] *= c;
      }
      *reinterpret_cast<float4*>(&sQT[warp * kD + 4 * lane]) = make_float4(x[0], x[1], x[2], x[3]);
    }
    named_bar_sync(kConsumerBar, kNCT);

    // phase-1 registers: the bf16 reference side keeps the query slice in
    // fp32; code planes (INT4 anchor, residual) get int16 dp4a operands
    constexpr int NG1 = RB ? ((C::D1 >= RG) ? C::D1 / RG : 1) : 1;
    float2 qref[G][REF == kRefBf16 ? C::D1 / 2 : 1];
    DotOperands24<REF == kRefInt4 ? C::D1 : 1> oref[G];
    DotOperands<RB ? RB : 2, RB ? C::D1 : 1> ores[G];
    float qsum_res[G][NG1];
    float qsum_ref[G];
#pragma unroll
    for (int gi = 0; gi < G; ++gi) {
      float vr[C::D1], vt[C::D1];
      qsum_ref[gi] = 0.f;
#pragma unroll
      for (int n = 0; n < NG1; ++n) qsum_res[gi][n] = 0.f;
#pragma unroll
      for (int e = 0; e < C::D1; ++e) {
        vr[e] = sQS[gi * kD + d1 + e];
        vt[e] = RB ? sQT[gi * kD + d1 + e] : 0.f;
        qsum_ref[gi] += vr[e];
        qsum_res[gi][(C::D1 >= RG) ? e / RG : 0] += vt[e];
      }
      if constexpr (REF == kRefBf16) {
#pragma unroll
        for (int e = 0; e < C::D1; e += 2) qref[gi][e / 2] = make_float2(vr[e], vr[e + 1]);
      } else {
        qref[gi][0] = make_float2(0.f, 0.f);
      }
      if constexpr (REF == kRefInt4) oref[gi].build(vr);
      if constexpr (RB != 0) ores[gi].build(vt);
    }

    // group-local running softmax state and per-lane accumulators
    float m_run[G], l_thr[G];
    float2 acc_ref[G][C::D2 / 2], acc_res[G][C::D2 / 2];
    float z_ref[G], z_res[G];
#pragma unroll
    for (int gi = 0; gi < G; ++gi) {
      m_run[gi] = -INFINITY;
      l_thr[gi] = 0.f;
      z_ref[gi] = 0.f;
      z_res[gi] = 0.f;
#pragma unroll
      for (int e = 0; e < C::D2 / 2; ++e) acc_ref[gi][e] = acc_res[gi][e] = make_float2(0.f, 0.f);
    }

    // this group's pages of the segment: every NG-th, from the first with
    // (k + sp) % NG == grp
    for (int sp = (grp - k % NG + NG) % NG; sp < seg_pages; sp += NG) {
      const int kp = k + sp;  // the CTA's page index
      const int s = kp % C::STAGES;
      const uint8_t* st = stages + s * C::STAGE_BYTES;
      if (!*sAbort) {
        if (!mbar_wait_bounded(smem_u32(&bars[s]), (kp / C::STAGES) & 1)) {
          set_flag(P.status, RQ_FLAG_PIPE_TIMEOUT);
          *sAbort = 1;
        }
      }
      const int n_valid = min(TT, len_b - (it.page + sp) * TT);
      const int par = (kp / NG) & 1;
      float* pS = gS + par * G * TT;
      float* pWM = gWM + par * G * kGW;

      // ---------------- phase 1: scores of the page's 64 tokens
      float wmax[G];
#pragma unroll
      for (int gi = 0; gi < G; ++gi) wmax[gi] = -INFINITY;
#pragma unroll
      for (int ps = 0; ps < C::PASSES; ++ps) {
        const int t = ps * C::TOK_PASS + tok1;
        float part[G];
#pragma unroll
        for (int gi = 0; gi < G; ++gi) part[gi] = 0.f;
        if constexpr (REF == kRefBf16) {
          float2 acc2[G][C::NB];
#pragma unroll
          for (int gi = 0; gi < G; ++gi)
#pragma unroll
            for (int c = 0; c < C::NB; ++c) acc2[gi][c] = make_float2(0.f, 0.f);
          const uint8_t* rowK = st + C::O_REFK + (d1 >> 6) * (TT * 128) + t * 128;
          if constexpr (C::D1 >= 8) {
#pragma unroll
            for (int c = 0; c < C::NB; ++c) {
              const int chunk = ((d1 & 63) >> 3) + c;
              const uint4 v = *reinterpret_cast<const uint4*>(rowK + ((chunk ^ (t & 7)) << 4));
              const uint32_t w4[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
              for (int u = 0; u < 4; ++u) {
                const float2 kv2 = bf16x2_to_f2(w4[u]);
#pragma unroll
                for (int gi = 0; gi < G; ++gi) acc2[gi][c] = __ffma2_rn(qref[gi][c * 4 + u], kv2, acc2[gi][c]);
              }
            }
          } else {
            const int chunk = (d1 & 63) >> 3;
            const uint2 v = *reinterpret_cast<const uint2*>(rowK + ((chunk ^ (t & 7)) << 4) + ((d1 & 7) << 1));
            const float2 k01 = bf16x2_to_f2(v.x), k23 = bf16x2_to_f2(v.y);
#pragma unroll
            for (int gi = 0; gi < G; ++gi) {
              acc2[gi][0] = __ffma2_rn(qref[gi][0], k01, acc2[gi][0]);
              acc2[gi][0] = __ffma2_rn(qref[gi][1], k23, acc2[gi][0]);
            }
          }
#pragma unroll
          for (int gi = 0; gi < G; ++gi) {
            float sum = 0.f;
#pragma unroll
            for (int c = 0; c < C::NB; ++c) sum += acc2[gi][c].x + acc2[gi][c].y;
            part[gi] = sum;
          }
        } else if constexpr (REF == kRefInt4) {
          using Ops = DotOperands24<C::D1>;
          uint32_t cw[Ops::NW];
          load_codes<C::D1 / 2>(st + C::O_REFK + t * 64 + (d1 >> 1), cw);
          const float2 sz = half2_bits_to_f2(*reinterpret_cast<const uint32_t*>(st + C::O_REFMK + t * 16 + 4 * (d1 >> 5)));
          int x2[G], x1[G], x0[G];
#pragma unroll
          for (int gi = 0; gi < G; ++gi) x2[gi] = x1[gi] = x0[gi] = 0;
#pragma unroll
          for (int w = 0; w < Ops::NW; ++w)
#pragma unroll
            for (int kk = 0; kk < 2; ++kk) {
              const int x = static_cast<int>(unpack_bytes<4>(cw[w], kk));
#pragma unroll
              for (int gi = 0; gi < G; ++gi) {
                x2[gi] = __dp4a(x, static_cast<int>(oref[gi].b2[w][kk]), x2[gi]);
                x1[gi] = __dp4a(x, static_cast<int>(oref[gi].b1[w][kk]), x1[gi]);
                x0[gi] = __dp4a(x, static_cast<int>(oref[gi].b0[w][kk]), x0[gi]);
              }
            }
#pragma unroll
          for (int gi = 0; gi < G; ++gi) {
            const float dot = comb24s(x2[gi], x1[gi], x0[gi]) * oref[gi].scale;
            part[gi] = fmaf(sz.x, dot, sz.y * qsum_ref[gi]);
          }
        }
        // links from the anchor outward (Horner): part = alpha_K,i * part + res_i
#pragma unroll
        for (int ci = NCH - 1; ci >= 0; --ci) {
          if constexpr (C::HAS_ALPHA) {
            const float aK = __half2float(*reinterpret_cast<const __half*>(st + C::o_al(ci) + t * 4));
#pragma unroll
            for (int gi = 0; gi < G; ++gi) part[gi] *= aK;
          }
          if constexpr (RB != 0) {
            using Ops = DotOperands<RB, C::D1>;
            constexpr int NBYTES = C::D1 * RB / 8;
            constexpr int WPG = (RG * RB) / 32;  // 32-bit code words per group
            uint32_t cw[Ops::NW];
            load_codes<NBYTES>(st + C::o_resk(ci) + t * C::CB + (d1 * RB >> 3), cw);
            int dhi[G][NG1];
            unsigned dlo[G][NG1];
#pragma unroll
            for (int gi = 0; gi < G; ++gi)
#pragma unroll
              for (int n = 0; n < NG1; ++n) { dhi[gi][n] = 0; dlo[gi][n] = 0u; }
#pragma unroll
            for (int w = 0; w < Ops::NW; ++w) {
              const int n = (NG1 > 1) ? w / WPG : 0;
#pragma unroll
              for (int kk = 0; kk < Ops::KPW; ++kk) {
                const uint32_t x = unpack_bytes<RB>(cw[w], kk);
#pragma unroll
                for (int gi = 0; gi < G; ++gi) {
                  dhi[gi][n] = __dp4a(static_cast<int>(x), static_cast<int>(ores[gi].hi[w][kk]), dhi[gi][n]);
                  dlo[gi][n] = __dp4a(x, ores[gi].lo[w][kk], dlo[gi][n]);
                }
              }
            }
#pragma unroll
            for (int n = 0; n < NG1; ++n) {
              const float2 sz = half2_bits_to_f2(*reinterpret_cast<const uint32_t*>(
                  st + C::o_resmk(ci) + t * C::MB + 4 * (d1 / RG + n)));
#pragma unroll
              for (int gi = 0; gi < G; ++gi) {
                const float dot = static_cast<float>(dhi[gi][n] * 256 + static_cast<int>(dlo[gi][n])) * ores[gi].scale;
                part[gi] += fmaf(sz.x, dot, sz.y * qsum_res[gi][n]);
              }
            }
          }
        }
        // reduce over the TPT lanes of this token
#pragma unroll
        for (int gi = 0; gi < G; ++gi) {
          float v = part[gi];
          if constexpr (G <= 2) {
#pragma unroll
            for (int o = 1; o < 2 * G; o <<= 1) v += __shfl_xor_sync(kFull, v, o);
            v += __shfl_xor_sync(kFull, v, 8);
          } else {
#pragma unroll
            for (int o = 1; o < C::TPT; o <<= 1) v += __shfl_xor_sync(kFull, v, o);
          }
          const float sc = (t < n_valid) ? v * P.scale_log2 : -INFINITY;
          wmax[gi] = fmaxf(wmax[gi], sc);
          if (j1 == 0) pS[gi * TT + t] = sc;
        }
      }
#pragma unroll
      for (int gi = 0; gi < G; ++gi) {
        const float v = warp_max(wmax[gi]);
        if (lane == 0) pWM[gi * kGW + gw] = v;
      }
      named_bar_sync(kGroupBar0 + grp, kGT);

      // ---------------- softmax bookkeeping (group-uniform values)
      float corr[G];
#pragma unroll
      for (int gi = 0; gi < G; ++gi) {
        const float4 a = *reinterpret_cast<const float4*>(&pWM[gi * kGW]);
        const float mt = fmaxf(fmaxf(a.x, a.y), fmaxf(a.z, a.w));
        const float mn = fmaxf(m_run[gi], mt);
        corr[gi] = fast_exp2(m_run[gi] - mn);
        m_run[gi] = mn;
        l_thr[gi] *= corr[gi];
        const float2 c2 = make_float2(corr[gi], corr[gi]);
#pragma unroll
        for (int e = 0; e < C::D2 / 2; ++e) {
          acc_ref[gi][e] = __fmul2_rn(acc_ref[gi][e], c2);
          acc_res[gi][e] = __fmul2_rn(acc_res[gi][e], c2);
        }
        z_ref[gi] *= corr[gi];
        z_res[gi] *= corr[gi];
      }

      // ---------------- phase 2: values (weights recomputed per lane)
      auto value_token = [&](int t) {
        // pw[i]: weight of link i = p times alpha_V of the links before it;
        // pa: the anchor's weight, p times every link's alpha_V
        float pw[NCH][G], pa[G];
#pragma unroll
        for (int gi = 0; gi < G; ++gi) {
          pw[0][gi] = fast_exp2(pS[gi * TT + t] - m_run[gi]);
          if (j2 == 0) l_thr[gi] += pw[0][gi];
        }
#pragma unroll
        for (int ci = 0; ci < NCH; ++ci) {
          float aV = 1.f;
          if constexpr (C::HAS_ALPHA) aV = __half2float(*reinterpret_cast<const __half*>(st + C::o_al(ci) + t * 4 + 2));
#pragma unroll
          for (int gi = 0; gi < G; ++gi) {
            const float w = pw[ci][gi] * aV;
            if (ci + 1 < NCH) pw[ci + 1 < NCH ? ci + 1 : 0][gi] = w;
            else pa[gi] = w;
          }
        }
        if constexpr (REF == kRefBf16) {
          const uint8_t* rowV = st + C::O_REFV + (d2 >> 6) * (TT * 128) + t * 128;
          const int chunk = (d2 & 63) >> 3;
          if constexpr (C::D2 == 8) {
            const uint4 v = *reinterpret_cast<const uint4*>(rowV + ((chunk ^ (t & 7)) << 4));
            const uint32_t w4[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
            for (int u = 0; u < 4; ++u) {
              const float2 vv = bf16x2_to_f2(w4[u]);
#pragma unroll
              for (int gi = 0; gi < G; ++gi) acc_ref[gi][u] = __ffma2_rn(make_float2(pa[gi], pa[gi]), vv, acc_ref[gi][u]);
            }
          } else {
            const uint2 v = *reinterpret_cast<const uint2*>(rowV + ((chunk ^ (t & 7)) << 4) + ((d2 & 7) << 1));
            const float2 v01 = bf16x2_to_f2(v.x), v23 = bf16x2_to_f2(v.y);
#pragma unroll
            for (int gi = 0; gi < G; ++gi) {
              acc_ref[gi][0] = __ffma2_rn(make_float2(pa[gi], pa[gi]), v01, acc_ref[gi][0]);
              acc_ref[gi][1] = __ffma2_rn(make_float2(pa[gi], pa[gi]), v23, acc_ref[gi][1]);
            }
          }
        } else if constexpr (REF == kRefInt4) {
          uint32_t cw[1];
          load_codes<C::D2 / 2>(st + C::O_REFV + t * 64 + (d2 >> 1), cw);
          const float2 sz = half2_bits_to_f2(*reinterpret_cast<const uint32_t*>(st + C::O_REFMV + t * 16 + 4 * (d2 >> 5)));
          const float sxs = sz.x * kSubScale;
#pragma unroll
          for (int e = 0; e < C::D2; e += 2) {
            const float2 f = make_float2(code_sub<4>(cw, e), code_sub<4>(cw, e + 1));
#pragma unroll
            for (int gi = 0; gi < G; ++gi) {
              const float w = pa[gi] * sxs;
              acc_ref[gi][e / 2] = __ffma2_rn(make_float2(w, w), f, acc_ref[gi][e / 2]);
            }
          }
#pragma unroll
          for (int gi = 0; gi < G; ++gi) z_ref[gi] = fmaf(pa[gi], sz.y, z_ref[gi]);
        }
        if constexpr (RB != 0) {
#pragma unroll
          for (int ci = 0; ci < NCH; ++ci) {
            uint32_t cw[1];
            load_codes<C::D2 * RB / 8>(st + C::o_resv(ci) + t * C::CB + (d2 * RB >> 3), cw);
            const float2 sz =
                half2_bits_to_f2(*reinterpret_cast<const uint32_t*>(st + C::o_resmv(ci) + t * C::MB + 4 * (d2 / RG)));
            const float sxs = sz.x * kSubScale;
#pragma unroll
            for (int e = 0; e < C::D2; e += 2) {
              const float2 f = make_float2(code_sub<RB>(cw, e), code_sub<RB>(cw, e + 1));
#pragma unroll
              for (int gi = 0; gi < G; ++gi) {
                const float w = pw[ci][gi] * sxs;
                acc_res[gi][e / 2] = __ffma2_rn(make_float2(w, w), f, acc_res[gi][e / 2]);
              }
            }
#pragma unroll
            for (int gi = 0; gi < G; ++gi) z_res[gi] = fmaf(pw[ci][gi], sz.y, z_res[gi]);
          }
        }
      };
      if (n_valid == TT) {
#pragma unroll 4
        for (int i = 0; i < C::TOK2; ++i) value_token(slice + i * C::SLICES);
      } else {
        for (int i = 0; i < C::TOK2; ++i) {
          const int t = slice + i * C::SLICES;
          if (t < n_valid) value_token(t);
        }
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(smem_u32(&bars[C::STAGES + s]));
    }
    // past the segment: the next (b, h) (the loop ends when the CTA's pages do)
    k += seg_pages;
    it.page += seg_pages - 1;
    it.next(sNt, B, Hkv);

    // ---- flush this (b, h) segment: merge the two groups, write one partial
    if (gtid == 0) {
#pragma unroll
      for (int gi = 0; gi < G; ++gi) sMG[grp * G + gi] = m_run[gi];
    }
    named_bar_sync(kConsumerBar, kNCT);
    // Sum the slices' contributions in a fixed order (warp by warp, and within a
    // warp its two slices by one shuffle), so that a decode is reproducible bit
    // for bit from run to run.
    constexpr int SPW = 32 / C::TPR2;  // token slices per warp (1 or 2)
    float cref[G][C::D2], cres[G][C::D2], cl[G];
#pragma unroll
    for (int gi = 0; gi < G; ++gi) {
      float M = fmaxf(sMG[gi], sMG[G + gi]);
      if constexpr (NG == 3) M = fmaxf(M, sMG[2 * G + gi]);
      const float f = (m_run[gi] == -INFINITY) ? 0.f : fast_exp2(m_run[gi] - M);
#pragma unroll
      for (int e = 0; e < C::D2; ++e) {
        const float2 ar = acc_ref[gi][e >> 1];
        float vr = (e & 1) ? ar.y : ar.x;
        if constexpr (REF == kRefInt4) vr = fmaf(vr, pow2i(kSubExp - code_pos<4>(e)), z_ref[gi]);
        cref[gi][e] = __fmul_rn(vr, f);
        float vs = 0.f;
        if constexpr (RB != 0) {
          const float2 as = acc_res[gi][e >> 1];
          vs = fmaf((e & 1) ? as.y : as.x, pow2i(kSubExp - code_pos<RB>(e)), z_res[gi]);
        }
        cres[gi][e] = __fmul_rn(vs, f);
        if constexpr (SPW == 2) {
          cref[gi][e] = __fadd_rn(cref[gi][e], __shfl_xor_sync(kFull, cref[gi][e], 16));
          cres[gi][e] = __fadd_rn(cres[gi][e], __shfl_xor_sync(kFull, cres[gi][e], 16));
        }
      }
      cl[gi] = __fmul_rn(l_thr[gi], f);
      if constexpr (SPW == 2) cl[gi] = __fadd_rn(cl[gi], __shfl_xor_sync(kFull, cl[gi], 16));
    }
    for (int w = 0; w < kNCW; ++w) {
      if (warp == w && lane < 32 / SPW) {
#pragma unroll
        for (int gi = 0; gi < G; ++gi) {
#pragma unroll
          for (int e = 0; e < C::D2; ++e) {
            if constexpr (REF != kRefNone) sACC[gi * 2 * kD + d2 + e] = __fadd_rn(sACC[gi * 2 * kD + d2 + e], cref[gi][e]);
            if constexpr (RB != 0) sACC[gi * 2 * kD + kD + d2 + e] = __fadd_rn(sACC[gi * 2 * kD + kD + d2 + e], cres[gi][e]);
          }
          if (j2 == 0) sL[gi] = __fadd_rn(sL[gi], cl[gi]);
        }
      }
      named_bar_sync(kConsumerBar, kNCT);
    }
    {
      const int pair = b * Hkv + h;
      float* rec = P.partials + static_cast<int64_t>(pair + blockIdx.x) * G * kPartialFloats;
      for (int i = tid; i < G * (2 * kD / 4); i += kNCT) {
        const int gi = i / (2 * kD / 4), f4 = i % (2 * kD / 4);
        float4* src = reinterpret_cast<float4*>(&sACC[gi * 2 * kD]) + f4;
        reinterpret_cast<float4*>(rec + gi * kPartialFloats + 4)[f4] = *src;
        *src = make_float4(0.f, 0.f, 0.f, 0.f);
      }
      if (tid < G) {
        float M = fmaxf(sMG[tid], sMG[G + tid]);
        if constexpr (NG == 3) M = fmaxf(M, sMG[2 * G + tid]);
        reinterpret_cast<float4*>(rec + tid * kPartialFloats)[0] = make_float4(M, sL[tid], 0.f, 0.f);
        sL[tid] = 0.f;
      }
    }
  }
}

// ---------------------------------------------------------------------------
// dispatch
// ---------------------------------------------------------------------------
// Pages of 64 tokens for a bf16 anchor (one tensor-copy tile); 128 for the
// byte-plane formats, whose 64-token pages are too small to amortise the
// per-page synchronisation, when four stages still fit.
// Three consumer groups (12 warps) for the byte-plane formats at G = 1, which
// are bound by instruction latency with two; two elsewhere (the bf16-anchor
// formats are bound by HBM, and larger G or chains need the registers: at
// G = 2 two groups run as fast as three, 2.70 against 2.71 TB/s on the
// INT4-anchor [2,2,4,4] loop, without the spills of the 128-register limit).
template <int REF, int RB, int RG, int G, int NCH>
constexpr int groups_of() {
  return (REF != kRefBf16 && G == 1) ? 3 : 2;
}

template <int REF, int RB, int RG, int G, int NCH>
constexpr int page_tokens_of() {
  constexpr int NG = groups_of<REF, RB, RG, G, NCH>();
  if constexpr (REF == kRefBf16) return kPage;
  else return Cfg<REF, RB, RG, G, 2 * kPage, NCH, NG>::STAGES_MAX >= (NG == 3 ? 3 : 4) ? 2 * kPage : kPage;
}

template <int REF, int RB, int RG, int G, int NCH>
cudaError_t launch_split(DecodeParams& p, const CUtensorMap* tk, const CUtensorMap* tv, cudaStream_t s) {
  constexpr int TT = page_tokens_of<REF, RB, RG, G, NCH>();
  constexpr int NG = groups_of<REF, RB, RG, G, NCH>();
  using C = Cfg<REF, RB, RG, G, TT, NCH, NG>;
  static_assert(C::STAGES_MAX >= NG, "stage ring does not fit in shared memory");
  auto kern = decode_split_kernel<REF, RB, RG, G, TT, NCH, NG>;
  p.page_tokens = TT;
  static bool attr_done = false;  // per instantiation; set once per process
  if (!attr_done) {
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, C::SMEM_BYTES);
    if (e != cudaSuccess) return e;
    attr_done = true;
  }
  return launch_dependent(kern, p.num_ctas, C::NT, C::SMEM_BYTES, s, p, *tk, *tv);
}

using SplitFn = cudaError_t (*)(DecodeParams&, const CUtensorMap*, const CUtensorMap*, cudaStream_t);

}  // namespace
}  // namespace rq
