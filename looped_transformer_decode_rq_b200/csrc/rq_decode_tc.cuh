// rq_decode_tc.cuh -- split-K decode attention on the fifth-generation tensor
// cores (tcgen05) of sm_100a, for kv-heads shared by G in {1, 2, 4, 8, 16} query rows.
//
// It computes what the CUDA-core split kernel in rq_decode.cu computes and
// writes the same partial records (so the same combine kernel finishes the
// call): "ResidualQuant: KV Cache Quantization for Looped Transformers with
// 2-Bit Residuals" keeps loop l's keys and values as alpha * anchor + H^T deq(R_l)
// (abstract, Figure 1, Figure 2 caption), and every cached token is scored and
// summed straight from that compact form:
//     q . K_l,t = alpha_K,t (q . K_anchor,t) + (H q) . deq(R^K_l,t)
//     o ~ sum_t p_t alpha_V,t V_anchor,t + H^T sum_t p_t deq(R^V_l,t).
// With G query heads per kv-head the score and value sums are small matrix
// products, and this kernel runs them on the tensor cores:
//
//  * a page is 128 tokens of one (sequence, kv-head).  A producer warp streams
//    pages into a ring of shared-memory stages: bf16 anchor tiles by tiled
//    tensor copies with the 128-byte swizzle, code / metadata / alpha records by
//    bulk copies, completing on mbarriers;
//  * two consumer warpgroups expand the packed 2/4-bit codes into int8 tiles
//    (one token per thread, rows of 128 bytes in the 128-byte swizzle); the
//    bytes of a 32-dim chunk are kept in the order the shift-and-mask expansion
//    produces them, and every operand that meets them uses the same order;
//  * one thread issues the score MMAs into tensor memory (M = 128 tokens):
//      bf16 anchor:  K_anchor (bf16) x q (bf16, one column per query head)
//      INT4 anchor:  codes (int8) x q (int16 as signed hi/lo bytes), per group
//      residual:     codes (int8) x H q (int16 as signed hi/lo bytes), per group
//    so that per group  (H q)_g . c_g = s_q (256 D_hi + D_lo)  exactly in int32;
//  * thread t reads token t's row, applies the per-token scale, offset and
//    alpha, and each warpgroup -- one per half of the query heads -- takes the
//    page maximum.  The page's softmax weights become the B operands of the
//    value MMAs (M = 128 dims): a bf16 hi + lo pair per weight against the bf16
//    anchor values, and per group an int16 (hi/lo bytes) weight relative to the
//    page's largest scale against the code tiles; the per-group offsets are
//    accumulated per thread;
//  * thread d then reads dim d's row of the page's value sums and merges it
//    into fp32 accumulators with the online-softmax rescale.
#pragma once

#include "rq_common.cuh"
#include "rq_internal.h"
#include "rq_tc_ops.cuh"
#include "rq_tcgen05.cuh"

namespace rq {
namespace {

constexpr int kTP = kTcPage;   // tokens per page
constexpr int kNCW = 8;        // consumer warps (two warpgroups)
constexpr int kNCT = kNCW * 32;
constexpr int kProducerWarp = kNCW;
constexpr int kMmaWarp = kNCW + 1;
constexpr int kNT = kNCT + 64; // + producer warp + MMA-issuing warp
// Register split of the variants that need more than 168 registers per
// consumer thread: a third warpgroup (producer, MMA issuer, two spare warps)
// launched with the others at 168 registers a thread gives up all but kRegsAux,
// and the two consumer warpgroups take them:
//   384 threads x 168 = 128 x kRegsAux + 256 x kRegsConsumer.
constexpr int kLaunchRegs = 168;
constexpr int kRegsAux = 56;
constexpr int kRegsConsumer = 224;
static_assert(384 * kLaunchRegs == 128 * kRegsAux + 256 * kRegsConsumer, "register split");
constexpr int kBarAll = 1;     // the 256 consumer threads
constexpr int kBarWG = 2;      // warpgroup w uses kBarWG + w
constexpr int kSmemLimit = 227 * 1024;

template <int REF, int RB, int RG, int G, int NCH = 1>
struct TcCfg {
  static constexpr int GH = G == 1 ? 1 : G / 2;          // query heads per warpgroup
  static constexpr int NGR = RB ? kD / RG : 0;            // residual groups
  static constexpr int NPAR = RG == 16 ? 2 : 1;           // residual groups per 32-dim chunk
  static constexpr int NGA = REF == kRefInt4 ? 4 : 0;     // INT4 anchor groups
  static constexpr bool HAS_ALPHA = (REF != kRefNone) && (RB != 0);
  // per-token record bytes
  static constexpr int REF_REC = REF == kRefBf16 ? 256 : (REF == kRefInt4 ? 64 : 0);
  static constexpr int REFM_REC = REF == kRefInt4 ? 16 : 0;
  static constexpr int CB = RB * 16;
  static constexpr int MB = RB ? 4 * NGR : 0;
  static constexpr int AL_REC = HAS_ALPHA ? 4 : 0;
  // MMA widths (N).  Query and weight operands carry 24-bit integers as three
  // bytes (j = 0: top, 1: middle, 2: bottom), one B row per byte; signed except
  // the residual value weights, which are non-negative.
  //   score rows per 32-dim chunk: (parity, head, byte)   n = p * 3G + 3 h + j
  //   value rows: (byte, warpgroup, group, head in it)    n = j * NG * G + wg * NG * GH + g * GH + i
  // so that a thread writes each byte plane of its warpgroup as one vector
  static constexpr int N_SA = round16(3 * G);                          // INT4 anchor score columns per chunk
  static constexpr int N_SR = round16(3 * G * NPAR);                   // residual score columns per chunk
  static constexpr int N_VA = round16(3 * 4 * G);                      // INT4 anchor value columns
  static constexpr int N_VR = round16(3 * NGR * G);                    // residual value columns
  static constexpr int N_VB = round16(2 * G);                          // bf16 anchor value columns (hi, lo)
  // With 16 query rows, or a chain of residual links, the integer key codes are
  // widened into tensor memory (the score MMAs' A operand) instead of shared
  // tiles, which the larger query and weight operands (or the links' value
  // tiles) need.
  static constexpr bool KTM = G == 16 || NCH > 1;
  // Chained links (NCH > 1: an INT4 anchor and NCH residual links in one
  // format): every link's value sums go into the one residual accumulator,
  // with signed weights (a link's weight carries the alpha_V of the links
  // before it, which may be negative), relative to a scale shared by the links.
  static constexpr bool SIGNED_RES = NCH > 1;
  static_assert(NCH >= 1 && NCH <= RQ_MAX_CHAIN && (NCH == 1 || (REF == kRefInt4 && RB != 0)), "chain");
  // tensor-memory columns: scores, then value sums (separate, so that the next
  // page's scores can be computed while this page's value sums are read), then
  // the key codes of the 16-row variants.  Where that exceeds the 512 columns
  // (16 rows with an INT4 anchor and residual links) the value sums overlay the
  // scores, and the next page's score MMAs wait until this page's sums are read.
  static constexpr int S_REF = 0;
  static constexpr int S_REF_COLS = REF == kRefBf16 ? 16 : (REF == kRefInt4 ? 4 * N_SA : 0);
  static constexpr int S_RES = S_REF + S_REF_COLS;
  static constexpr int S_COLS = S_RES + (RB ? NCH * 4 * N_SR : 0);  // link ci at S_RES + ci * 4 N_SR
  static constexpr int O_REF_COLS = REF == kRefBf16 ? N_VB : (REF == kRefInt4 ? N_VA : 0);
  static constexpr int O_SIZE = O_REF_COLS + (RB ? N_VR : 0);
  static constexpr int KT_COLS = KTM ? (REF == kRefInt4 ? 32 : 0) + (RB ? 32 * NCH : 0) : 0;
  static constexpr bool ALIAS = KTM && S_COLS + O_SIZE + KT_COLS > 512;
  static constexpr int O_REF = ALIAS ? 0 : S_COLS;
  static constexpr int O_RES = O_REF + O_REF_COLS;
  static constexpr int O_COLS = O_RES + (RB ? N_VR : 0);
  static constexpr int TK_REF = S_COLS > O_COLS ? S_COLS : O_COLS;   // INT4 anchor key codes (KTM)
  static constexpr int TK_RES = TK_REF + (REF == kRefInt4 ? 32 : 0);  // residual key codes (KTM), 32 per link
  static constexpr int COLS = TK_REF + KT_COLS;
  static constexpr int TMEM_COLS = COLS <= 32 ? 32 : COLS <= 64 ? 64 : COLS <= 128 ? 128 : COLS <= 256 ? 256 : 512;
  // stage layout (pieces 1024-byte aligned)
  static constexpr int al(int x) { return (x + 1023) & ~1023; }
  static constexpr int O_REFK = 0;
  static constexpr int O_REFV = O_REFK + al(kTP * REF_REC);
  static constexpr int O_REFMK = O_REFV + al(kTP * REF_REC);
  static constexpr int O_REFMV = O_REFMK + al(kTP * REFM_REC);
  // link ci's records: codes K, codes V, meta K, meta V, alpha
  static constexpr int O_RES0 = O_REFMV + al(kTP * REFM_REC);
  static constexpr int LINK = 2 * al(kTP * CB) + 2 * al(kTP * MB) + al(kTP * AL_REC);
  static constexpr int o_resk(int ci) { return O_RES0 + ci * LINK; }
  static constexpr int o_resv(int ci) { return o_resk(ci) + al(kTP * CB); }
  static constexpr int o_resmk(int ci) { return o_resv(ci) + al(kTP * CB); }
  static constexpr int o_resmv(int ci) { return o_resmk(ci) + al(kTP * MB); }
  static constexpr int o_al(int ci) { return o_resmv(ci) + al(kTP * MB); }
  static constexpr int O_RESK = o_resk(0);
  static constexpr int O_RESV = o_resv(0);
  static constexpr int O_RESMK = o_resmk(0);
  static constexpr int O_RESMV = o_resmv(0);
  static constexpr int O_AL = o_al(0);
  static constexpr int STAGE_BYTES = O_RES0 + NCH * LINK;
  // operand tiles (after the stages)
  static constexpr int F_UK = 0;                                   // residual K codes, int8 [128 tok][128]
  static constexpr int F_UV = F_UK + (RB && !KTM ? 16384 : 0);     // residual V codes (one tile per link)
  static constexpr int F_URK = F_UV + (RB ? 16384 * NCH : 0);      // INT4 anchor K codes
  static constexpr int F_URV = F_URK + (REF == kRefInt4 && !KTM ? 16384 : 0);
  static constexpr int F_QB = F_URV + (REF == kRefInt4 ? 16384 : 0);  // bf16 q [16][128], K-major sw128
  static constexpr int F_QA = F_QB + (REF == kRefBf16 ? 4096 : 0);    // int8 q bytes [N_SA][128]
  static constexpr int F_HQ = F_QA + (REF == kRefInt4 ? al(N_SA * 128) : 0);  // int8 H q bytes [N_SR][128]
  static constexpr int F_WB = F_HQ + (RB ? al(N_SR * 128) : 0);       // bf16 weights, MN-major [N_VB x 128 tok]
  static constexpr int F_WA = F_WB + (REF == kRefBf16 ? N_VB * 256 : 0);  // int8 weights [N_VA x 128 tok]
  static constexpr int F_WR = F_WA + (REF == kRefInt4 ? al(N_VA * 128) : 0);
  static constexpr int WR_BYTES = al(N_VR * 128);                   // one link's residual weights
  static constexpr int F_END = F_WR + (RB ? NCH * WR_BYTES : 0);
  // small state (after the tiles; 4-byte words)
  static constexpr int NRED = 1 + 8 + 4;                 // l, residual offsets, anchor offsets
  static constexpr int GS = G > 8 ? G : 8;               // head slots of the small arrays
  static constexpr int GHS = GH > 4 ? GH : 4;            // head slots per warpgroup
  static constexpr int W_CS = 0;                         // [GS] residual q scale * scale_log2
  static constexpr int W_QS = W_CS + GS;                 // [GS][8] residual group sums of H q
  static constexpr int W_CA = W_QS + 8 * GS;             // [GS] anchor q scale * scale_log2
  static constexpr int W_QA = W_CA + GS;                 // [GS][4] anchor group sums of q
  static constexpr int W_WM = W_QA + 4 * GS;             // [2][4 warps][GHS] warp maxima of scores
  static constexpr int W_SIG = W_WM + 8 * GHS;           // [2][4 warps][12] warp maxima of scales
  static constexpr int W_RED = W_SIG + 96;               // [4 warps][GS heads][NRED] flush sums
  static constexpr int W_PRE = W_RED + 4 * GS * NRED;    // [RQ_MAX_BATCH + 1] page prefix
  static constexpr int W_MISC = W_PRE + RQ_MAX_BATCH + 1;  // abort flag, tensor-memory base
  static constexpr int W_BAR = (W_MISC + 2 + 1) & ~1;    // 8-byte aligned mbarriers
  // Key and value halves of a stage on separate barriers (bf16 anchor, key
  // codes in shared memory): the producer refills a stage's key half as soon
  // as the page's score MMAs are done and its key metadata read, and its value
  // half once the value MMAs are done, so the next pages' keys are in flight
  // while this page's softmax and value sums run.
  // (measured: 2-3% faster at 8 rows, 1.5% slower at 4)
  static constexpr bool KVSPLIT = REF == kRefBf16 && !KTM && G >= 8;
  static constexpr int NBARS = 2 * 4 + 8 + 2 * 4;
  static constexpr int SMALL_BYTES = 4 * W_BAR + 8 * NBARS;
  static constexpr int FIXED = 1024 + F_END + SMALL_BYTES;
  static constexpr int STAGES_FIT = (kSmemLimit - FIXED) / STAGE_BYTES;
  static constexpr int STAGES = STAGES_FIT >= 4 ? 4 : (STAGES_FIT >= 2 ? STAGES_FIT : 2);
  // An INT4 anchor with residual links keeps both offset sums of its heads per
  // thread: from 2 rows on those variants take the register split
  static constexpr bool REGSPLIT = REF == kRefInt4 && RB != 0 && G >= 2;
  static constexpr int NT = REGSPLIT ? kNCT + 128 : kNT;
  static constexpr bool FITS = STAGES_FIT >= 2 && COLS <= 512 && N_VA <= 256 && N_VR <= 256 && N_SR <= 256;
  static constexpr int SMEM_BYTES = FIXED + STAGES * STAGE_BYTES;
  // instruction descriptors
  static constexpr uint32_t ID_SB = tc::instr_desc(tc::kAccF32, tc::kFmtBf16, tc::kFmtBf16, 0, 0, 128, 16);
  static constexpr uint32_t ID_SA = tc::instr_desc(tc::kAccS32, tc::kFmtS8, tc::kFmtS8, 0, 0, 128, N_SA);
  static constexpr uint32_t ID_SR = tc::instr_desc(tc::kAccS32, tc::kFmtS8, tc::kFmtS8, 0, 0, 128, N_SR);
  static constexpr uint32_t ID_VB = tc::instr_desc(tc::kAccF32, tc::kFmtBf16, tc::kFmtBf16, 1, 1, 128, N_VB);
  static constexpr uint32_t ID_VA = tc::instr_desc(tc::kAccS32, tc::kFmtS8, tc::kFmtS8, 1, 1, 128, N_VA);
  static constexpr uint32_t ID_VR = SIGNED_RES ? tc::instr_desc(tc::kAccS32, tc::kFmtS8, tc::kFmtS8, 1, 1, 128, N_VR)
                                               : tc::instr_desc(tc::kAccS32, 0, 0, 1, 1, 128, N_VR);  // unsigned bytes
  static_assert(G == 1 || G == 2 || G == 4 || G == 8 || G == 16, "query heads per kv-head");
};

// ---------------------------------------------------------------------------
// producer: one page into stage `st`
// ---------------------------------------------------------------------------
// PART: 0 the key half (bf16 anchor keys, key codes and metadata), 1 the value
// half (the rest), 2 the whole page
template <int REF, int RB, int RG, int G, int NCH, int PART = 2>
__device__ __forceinline__ void tc_issue_page(const DecodeParams& P, const CUtensorMap* tmK, const CUtensorMap* tmV,
                                              uint8_t* st, uint32_t full, const PageIter& it, int Hkv) {
  using C = TcCfg<REF, RB, RG, G, NCH>;
  static_assert(PART == 2 || REF == kRefBf16, "key / value halves: bf16 anchor");
  constexpr bool KH = PART != 1, VH = PART != 0;
  const int t0 = it.page * kTP;
  // byte planes hold plane_tokens (a multiple of 64) records per (b, h)
  const int nrec = (P.plane_tokens > 0 && t0 + kTP > P.plane_tokens) ? static_cast<int>(P.plane_tokens - t0) : kTP;
  const int halves = (REF == kRefBf16) ? ((t0 + 64 < P.tma_tokens) ? 2 : 1) : 0;
  const uint32_t bytes =
      PART == 2 ? halves * 4 * 8192 +
                      nrec * (2 * (REF == kRefInt4 ? 64 + 16 : 0) + NCH * (2 * C::CB + 2 * C::MB + C::AL_REC))
                : halves * 2 * 8192 + nrec * NCH * (C::CB + C::MB + (PART == 1 ? C::AL_REC : 0));
  mbar_arrive_expect_tx(full, bytes);
  const int64_t rec0 = static_cast<int64_t>(it.b * Hkv + it.h) * P.plane_tokens + t0;
  if constexpr (REF == kRefBf16) {
    for (int th = 0; th < halves; ++th) {
#pragma unroll
      for (int dh = 0; dh < 2; ++dh) {
        if (KH) tma_load_4d(smem_u32(st + C::O_REFK + dh * 16384 + th * 8192), tmK, 64 * dh, t0 + 64 * th, it.h, it.b, full);
        if (VH) tma_load_4d(smem_u32(st + C::O_REFV + dh * 16384 + th * 8192), tmV, 64 * dh, t0 + 64 * th, it.h, it.b, full);
      }
    }
  } else if constexpr (REF == kRefInt4) {
    bulk_g2s(smem_u32(st + C::O_REFK), P.ref_codes[0] + rec0 * 64, nrec * 64, full);
    bulk_g2s(smem_u32(st + C::O_REFV), P.ref_codes[1] + rec0 * 64, nrec * 64, full);
    bulk_g2s(smem_u32(st + C::O_REFMK), P.ref_meta[0] + rec0 * 16, nrec * 16, full);
    bulk_g2s(smem_u32(st + C::O_REFMV), P.ref_meta[1] + rec0 * 16, nrec * 16, full);
  }
#pragma unroll
  for (int ci = 0; ci < NCH; ++ci) {
    if constexpr (RB != 0) {
      if (KH) bulk_g2s(smem_u32(st + C::o_resk(ci)), P.res_codes[ci][0] + rec0 * C::CB, nrec * C::CB, full);
      if (VH) bulk_g2s(smem_u32(st + C::o_resv(ci)), P.res_codes[ci][1] + rec0 * C::CB, nrec * C::CB, full);
      if (KH) bulk_g2s(smem_u32(st + C::o_resmk(ci)), P.res_meta[ci][0] + rec0 * C::MB, nrec * C::MB, full);
      if (VH) bulk_g2s(smem_u32(st + C::o_resmv(ci)), P.res_meta[ci][1] + rec0 * C::MB, nrec * C::MB, full);
    }
    if constexpr (C::HAS_ALPHA) {
      if (VH) bulk_g2s(smem_u32(st + C::o_al(ci)), P.alpha[ci] + rec0 * 4, nrec * 4, full);
    }
  }
}

// one token's (scale, offset) pairs of NG groups (fp16 pairs), zero past the context
template <int NG>
__device__ __forceinline__ void token_meta(const uint8_t* rec, bool valid, float (&sc)[NG], float (&zo)[NG]) {
#pragma unroll
  for (int g = 0; g < NG; g += 4) {
    const uint4 m4 = *reinterpret_cast<const uint4*>(rec + 4 * g);
    const uint32_t w4[4] = {m4.x, m4.y, m4.z, m4.w};
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      const float2 a = half2_bits_to_f2(w4[u]);
      sc[g + u] = valid ? a.x : 0.f;
      zo[g + u] = valid ? a.y : 0.f;
    }
  }
}

// ---------------------------------------------------------------------------
// split kernel
// ---------------------------------------------------------------------------
template <int REF, int RB, int RG, int G, int NCH>
__global__ void __launch_bounds__(TcCfg<REF, RB, RG, G, NCH>::NT, 1)
    decode_tc_kernel(const __grid_constant__ DecodeParams P, const __grid_constant__ CUtensorMap tmK,
                     const __grid_constant__ CUtensorMap tmV) {
  using C = TcCfg<REF, RB, RG, G, NCH>;
  constexpr int GH = C::GH;
  constexpr int NGR = C::NGR;
  constexpr int NGA = C::NGA;
  extern __shared__ __align__(16) uint8_t smem_raw[];
  uint8_t* base = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
  uint8_t* stages = base;
  uint8_t* fx = base + C::STAGES * C::STAGE_BYTES;
  float* sw = reinterpret_cast<float*>(fx + C::F_END);
  float* sCS = sw + C::W_CS;
  float* sQS = sw + C::W_QS;
  float* sCA = sw + C::W_CA;
  float* sQA = sw + C::W_QA;
  float* sWM = sw + C::W_WM;
  float* sSig = sw + C::W_SIG;
  float* sRed = sw + C::W_RED;
  int* sPre = reinterpret_cast<int*>(sw + C::W_PRE);
  volatile int* sAbort = reinterpret_cast<volatile int*>(sw + C::W_MISC);
  uint32_t* sTmem = reinterpret_cast<uint32_t*>(sw + C::W_MISC + 1);
  uint64_t* bars = reinterpret_cast<uint64_t*>(sw + C::W_BAR);
  uint64_t* full = bars;       // [stage] the page's copies landed (KVSPLIT: its key half)
  uint64_t* empty = bars + 4;  // [stage] the page's value MMAs completed (KVSPLIT: its key half is free)
  uint64_t* sbar = bars + 8;   // score MMAs completed
  uint64_t* obar = bars + 9;   // value MMAs completed
  uint64_t* sfree = bars + 10;   // the page's query operands are written, the previous scores read
  uint64_t* kready = bars + 11;  // key code tiles written
  uint64_t* v1ready = bars + 12; // anchor value weights (and cleared anchor rows) written
  uint64_t* v2ready = bars + 13; // residual value weights (and value code tiles) written
  uint64_t* done = bars + 14;    // every MMA of the CTA completed
  uint64_t* never = bars + 15;   // never arrived at: the wait of the stall test hook
  uint64_t* fullV = bars + 16;   // [stage] KVSPLIT: the page's value half landed
  uint64_t* emptyV = bars + 20;  // [stage] KVSPLIT: the page's value MMAs completed

  const int tid = threadIdx.x;
  const int lane = tid & 31;
  const int warp = tid >> 5;
  const int B = P.B, Hkv = P.Hkv;
  pdl_wait();  // programmatic dependent of the previous kernel: no global access before it completed

  // ---- pages per sequence and their prefix (pre[b+1] - pre[b] = pages of b)
  if (warp == 0) {
    int carry = 0;
    for (int b0 = 0; b0 < B; b0 += 32) {
      const int b = b0 + lane;
      int v = 0;
      if (b < B) {
        int len = P.ctx_len[b];
        if (len < 0 || len > P.capacity) {
          if (blockIdx.x == 0) set_flag(P.status, RQ_FLAG_CTX_LEN);
          len = len < 0 ? 0 : P.capacity;
        }
        v = (len + kTP - 1) / kTP;
      }
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
    *sAbort = 0;
    for (int s = 0; s < C::STAGES; ++s) {
      mbar_init(smem_u32(&full[s]), 1);   // the producer's expect_tx
      // the commit after the page's value MMAs; KVSPLIT: the commit after its
      // score MMAs and every consumer warp once it has read the key metadata
      mbar_init(smem_u32(&empty[s]), C::KVSPLIT ? 1 + kNCW : 1);
      if constexpr (C::KVSPLIT) {
        mbar_init(smem_u32(&fullV[s]), 1);
        mbar_init(smem_u32(&emptyV[s]), 1);
      }
    }
    mbar_init(smem_u32(sbar), 1);
    mbar_init(smem_u32(obar), 1);
    mbar_init(smem_u32(sfree), kNCW);
    mbar_init(smem_u32(kready), 4);
    mbar_init(smem_u32(v1ready), kNCW);
    mbar_init(smem_u32(v2ready), kNCW);
    mbar_init(smem_u32(done), 1);
    mbar_init(smem_u32(never), 1);
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

  // page counts as a view of the prefix
  auto nt_of = [&](int b) { return sPre[b + 1] - sPre[b]; };
  auto seek = [&](PageIter& it, int64_t x) {
    int lo = 0, hi = B - 1;
    while (lo < hi) {
      const int mid = (lo + hi + 1) >> 1;
      if (static_cast<int64_t>(sPre[mid]) * Hkv <= x) lo = mid; else hi = mid - 1;
    }
    it.b = lo;
    const int64_t r = x - static_cast<int64_t>(sPre[lo]) * Hkv;
    const int nt = nt_of(lo);
    it.h = static_cast<int>(r / nt);
    it.page = static_cast<int>(r % nt);
  };
  auto advance = [&](PageIter& it) {
    if (++it.page < nt_of(it.b)) return;
    it.page = 0;
    if (++it.h < Hkv) return;
    it.h = 0;
    do { ++it.b; } while (it.b < B && nt_of(it.b) == 0);
  };

  // A wait that timed out marks the CTA aborted; later waits then return at once
  // so that every thread still walks the same barrier sequence to the end.
  auto wait_or_abort = [&](uint64_t* bar, uint32_t parity) -> bool {
    if (*sAbort) return false;
    if (mbar_wait_bounded(smem_u32(bar), parity)) return true;
    set_flag(P.status, RQ_FLAG_PIPE_TIMEOUT);
    *sAbort = 1;
    return false;
  };
  constexpr bool NEED_KREADY = (RB != 0) || (REF == kRefInt4);
  constexpr bool HAS_V1 = REF != kRefNone;
  constexpr bool HAS_V2 = RB != 0;

  // ---- tensor memory for the page's score and value sums
  if (warp == 0) {
    tc::tmem_alloc(smem_u32(sTmem), C::TMEM_COLS);
    tc::tmem_relinquish();
  }
  tc::fence_before_sync();
  __syncthreads();
  tc::fence_after_sync();
  const uint32_t tbase = *sTmem;

  // the producer warpgroup: producer warp, MMA-issuing warp (and, with the
  // register split, two spare warps); no path out of it reaches the consumers'
  // code, so each side is compiled for its own register budget
  if (warp >= kNCW) {
  if constexpr (C::REGSPLIT) tc::setmaxnreg_dec<kRegsAux>();

  // ========================= producer warp =========================
  if (warp == kProducerWarp) {
    if (lane == 0) {
      if constexpr (REF == kRefBf16) {
        prefetch_tensormap(&tmK);
        prefetch_tensormap(&tmV);
      }
      PageIter it;
      seek(it, x0);
      int k = 0;
      bool vissued = true;  // the last page's value half was issued
      for (; k < n_pages; ++k) {
        const int s = k % C::STAGES;
        if (!mbar_wait_bounded(smem_u32(&empty[s]), ((k / C::STAGES) & 1) ^ 1)) {
          set_flag(P.status, RQ_FLAG_PIPE_TIMEOUT);
          break;
        }
        if (k == P.stall_page && !mbar_wait_bounded(smem_u32(never), 0)) set_flag(P.status, RQ_FLAG_PIPE_TIMEOUT);
        if constexpr (C::KVSPLIT) {
          tc_issue_page<REF, RB, RG, G, NCH, 0>(P, &tmK, &tmV, stages + s * C::STAGE_BYTES, smem_u32(&full[s]), it,
                                                Hkv);
          if (!mbar_wait_bounded(smem_u32(&emptyV[s]), ((k / C::STAGES) & 1) ^ 1)) {
            set_flag(P.status, RQ_FLAG_PIPE_TIMEOUT);
            ++k;  // its key half is in flight: drained below
            vissued = false;
            break;
          }
          tc_issue_page<REF, RB, RG, G, NCH, 1>(P, &tmK, &tmV, stages + s * C::STAGE_BYTES, smem_u32(&fullV[s]), it,
                                                Hkv);
        } else {
          tc_issue_page<REF, RB, RG, G, NCH>(P, &tmK, &tmV, stages + s * C::STAGE_BYTES, smem_u32(&full[s]), it, Hkv);
        }
        advance(it);
      }
      // no copy this CTA issued may still be landing when it exits (a wait
      // that gave up stops the drain: the others would give up too)
      bool drained = true;
      for (int kk = (k > C::STAGES ? k - C::STAGES : 0); kk < k && drained; ++kk) {
        drained = mbar_wait_bounded(smem_u32(&full[kk % C::STAGES]), (kk / C::STAGES) & 1);
        if (C::KVSPLIT && drained && (kk + 1 < k || vissued))
          drained = mbar_wait_bounded(smem_u32(&fullV[kk % C::STAGES]), (kk / C::STAGES) & 1);
      }
      if (!drained) set_flag(P.status, RQ_FLAG_PIPE_TIMEOUT);
    }
    return;
  }

  // ========================= MMA-issuing warp =========================
  // One thread issues every tcgen05 MMA of the CTA, page by page, as soon as
  // its operands are ready: the bf16 anchor score MMAs when the page lands,
  // the integer score MMAs when the key code tiles are written, and the value
  // MMAs in two groups as their weight operands are written.
  if (warp == kMmaWarp) {
    if (lane == 0) {
      for (int k = 0; k < n_pages; ++k) {
        // with the register split this warp has few registers: the operand
        // descriptors are recomputed every page rather than kept
        uint8_t* fxk = fx;
        if constexpr (C::REGSPLIT) asm volatile("" : "+l"(fxk));
        uint8_t* UKm = fxk + C::F_UK;
        uint8_t* UVm = fxk + C::F_UV;
        uint8_t* URKm = fxk + C::F_URK;
        uint8_t* URVm = fxk + C::F_URV;
        uint8_t* QBm = fxk + C::F_QB;
        uint8_t* QAm = fxk + C::F_QA;
        uint8_t* HQm = fxk + C::F_HQ;
        uint8_t* WBm = fxk + C::F_WB;
        uint8_t* WAm = fxk + C::F_WA;
        uint8_t* WRm = fxk + C::F_WR;
        const int s = k % C::STAGES;
        uint8_t* st = stages + s * C::STAGE_BYTES;
        const uint32_t ph = k & 1;
        wait_or_abort(sfree, ph);
        wait_or_abort(&full[s], (k / C::STAGES) & 1);
        tc::fence_after_sync();
        if constexpr (REF == kRefBf16) {
#pragma unroll
          for (int ks = 0; ks < 8; ++ks)
            tc::mma_bf16(tbase + C::S_REF, tc::desc_k_sw128(smem_u32(st + C::O_REFK + (ks >> 2) * 16384 + (ks & 3) * 32)),
                         tc::desc_k_sw128(smem_u32(QBm + (ks >> 2) * 2048 + (ks & 3) * 32)), C::ID_SB, ks > 0);
        }
        if constexpr (NEED_KREADY) {
          wait_or_abort(kready, ph);
          tc::fence_after_sync();
          if constexpr (REF == kRefInt4) {
#pragma unroll
            for (int c = 0; c < 4; ++c) {
              if constexpr (C::KTM)
                tc::mma_s8_ta(tbase + C::S_REF + C::N_SA * c, tbase + C::TK_REF + 8 * c,
                              tc::desc_k_sw128(smem_u32(QAm + 32 * c)), C::ID_SA, 0);
              else
                tc::mma_s8(tbase + C::S_REF + C::N_SA * c, tc::desc_k_sw128(smem_u32(URKm + 32 * c)),
                           tc::desc_k_sw128(smem_u32(QAm + 32 * c)), C::ID_SA, 0);
            }
          }
          if constexpr (RB != 0) {
#pragma unroll
            for (int ci = 0; ci < NCH; ++ci) {  // every link against the one rotated query
#pragma unroll
              for (int c = 0; c < 4; ++c) {
                const uint32_t d = tbase + C::S_RES + 4 * C::N_SR * ci + C::N_SR * c;
                if constexpr (C::KTM)
                  tc::mma_s8_ta(d, tbase + C::TK_RES + 32 * ci + 8 * c, tc::desc_k_sw128(smem_u32(HQm + 32 * c)),
                                C::ID_SR, 0);
                else
                  tc::mma_s8(d, tc::desc_k_sw128(smem_u32(UKm + 32 * c)), tc::desc_k_sw128(smem_u32(HQm + 32 * c)),
                             C::ID_SR, 0);
              }
            }
          }
        }
        tc::commit(smem_u32(sbar));
        if constexpr (C::KVSPLIT) {
          tc::commit(smem_u32(&empty[s]));  // the key half's part: the score MMAs have read it
          wait_or_abort(&fullV[s], (k / C::STAGES) & 1);
        }
        if constexpr (HAS_V1) {
          wait_or_abort(v1ready, ph);
          tc::fence_after_sync();
          if constexpr (REF == kRefBf16) {
#pragma unroll
            for (int ks = 0; ks < 8; ++ks)
              tc::mma_bf16(tbase + C::O_REF, tc::desc_mn_sw128(smem_u32(st + C::O_REFV + ks * 2048), 16384),
                           tc::desc_mn_plain(smem_u32(WBm + ks * 256), 128, 2048), C::ID_VB, ks > 0);
          } else {
#pragma unroll
            for (int ks = 0; ks < 4; ++ks)
              tc::mma_s8(tbase + C::O_REF, tc::desc_mn_sw128(smem_u32(URVm + ks * 4096), 16384),
                         tc::desc_mn_plain(smem_u32(WAm + ks * 512), 128, 2048), C::ID_VA, ks > 0);
          }
        }
        if constexpr (HAS_V2) {
          wait_or_abort(v2ready, ph);
          tc::fence_after_sync();
#pragma unroll
          for (int ci = 0; ci < NCH; ++ci)  // every link into the one rotated accumulator
#pragma unroll
            for (int ks = 0; ks < 4; ++ks)
              tc::mma_s8(tbase + C::O_RES, tc::desc_mn_sw128(smem_u32(UVm + 16384 * ci + ks * 4096), 16384),
                         tc::desc_mn_plain(smem_u32(WRm + C::WR_BYTES * ci + ks * 512), 128, 2048), C::ID_VR,
                         ks > 0 || ci > 0);
        }
        tc::commit(smem_u32(obar));
        tc::commit(smem_u32(C::KVSPLIT ? &emptyV[s] : &empty[s]));
      }
      tc::commit(smem_u32(done));
    }
    return;
  }
  return;  // spare warps
  }
  if constexpr (C::REGSPLIT) tc::setmaxnreg_inc<kRegsConsumer>();

  // ========================= consumer warpgroups =========================
  // G >= 2: warpgroup wg scores and sums query heads [wg GH, wg GH + GH).
  // G == 1: both warpgroups score the one head; warpgroup 0 owns the anchor
  // value sums and the denominator, warpgroup 1 the residual value sums.
  // Pages are software-pipelined by one: while page k's value MMAs run, the
  // next page's key codes are expanded and its score MMAs issued.
  constexpr bool SPLIT = (G == 1);
  const int wg = warp >> 2;
  const int r = tid & 127;                   // tensor-memory lane: token, then dim position
  const uint32_t tl = tbase + (static_cast<uint32_t>(32 * (warp & 3)) << 16);
  const int chunk = warp & 3;                // 32-dim chunk of this thread's position
  const int hb = SPLIT ? 0 : wg * GH;        // first query head of this warpgroup
  const int wgo = SPLIT ? 0 : wg;            // warpgroup slot in operand rows / columns
  const bool own_ref = !SPLIT || wg == 0;    // anchor value sums, maximum and denominator
  const bool own_res = !SPLIT || wg == 1;    // residual value sums
  uint8_t* UK = fx + C::F_UK;
  uint8_t* UV = fx + C::F_UV;
  uint8_t* URK = fx + C::F_URK;
  uint8_t* URV = fx + C::F_URV;
  uint8_t* QB = fx + C::F_QB;
  uint8_t* QA = fx + C::F_QA;
  uint8_t* HQ = fx + C::F_HQ;
  uint8_t* WB = fx + C::F_WB;
  uint8_t* WA = fx + C::F_WA;
  uint8_t* WR = fx + C::F_WR;
  // residual group of this thread's dim position (and its parity for 16-groups)
  const int par_r = RB == 2 ? ((r >> 2) & 1) : ((r >> 3) & 1);
  const int g_res = RG == 16 ? 2 * chunk + par_r : chunk;

  auto seq_len = [&](int b) {
    const int len = P.ctx_len[b];
    return len < 0 ? 0 : (len > P.capacity ? P.capacity : len);
  };

  // query operands of the G heads of (b, h), for the score MMAs
  auto setup = [&](int b, int h) {
    for (int hq = warp; hq < G; hq += kNCW) {
      const uint2 raw = *reinterpret_cast<const uint2*>(P.q + q_row_offset(P, b, h, hq) + 4 * lane);
      const int d = 4 * lane;
      if constexpr (REF == kRefBf16) {
        *reinterpret_cast<uint2*>(QB + (d >> 6) * 2048 + (hq >> 3) * 1024 + (hq & 7) * 128 +
                                  ((((d & 63) >> 3) ^ (hq & 7)) << 4) + (d & 7) * 2) = raw;
      }
      const float2 a01 = bf16x2_to_f2(raw.x), a23 = bf16x2_to_f2(raw.y);
      float x[4] = {a01.x, a01.y, a23.x, a23.y};
      if constexpr (REF == kRefInt4) put_q_s24<4, 32, G>(QA, x, hq, lane, &sCA[hq], &sQA[hq * 4], P.scale_log2);
      if constexpr (RB != 0) {
        if (P.rotate) {
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
        put_q_s24<RB, RG, G>(HQ, x, hq, lane, &sCS[hq], &sQS[hq * 8], P.scale_log2);
      }
    }
    fence_proxy_async_smem();
    named_bar_sync(kBarAll, kNCT);
  };
  // "page k may be scored": its query operands are written and the previous
  // page's scores have been read out of tensor memory
  auto release_scores = [&]() {
    tc::fence_before_sync();
    __syncwarp();
    if (lane == 0) mbar_arrive(smem_u32(sfree));
  };
  // warpgroup 0: key-side code tiles of the page in stage `st`
  auto expand_keys = [&](const uint8_t* st) {
    if constexpr (C::KTM) {
      // token r's codes into tensor-memory lane r (its warp's quarter)
      if constexpr (REF == kRefInt4) {
        uint32_t o[32];
        widen_codes<4>(st + C::O_REFK + r * 64, o);
        tc::tmem_st_x32(tl + C::TK_REF, o);
      }
      if constexpr (RB != 0) {
#pragma unroll
        for (int ci = 0; ci < NCH; ++ci) {
          uint32_t o[32];
          widen_codes<RB>(st + C::o_resk(ci) + r * C::CB, o);
          tc::tmem_st_x32(tl + C::TK_RES + 32 * ci, o);
        }
      }
      tc::tmem_wait_st();
      tc::fence_before_sync();
    } else {
      if constexpr (RB != 0) expand_row<RB>(st + C::O_RESK + r * C::CB, UK, r);
      if constexpr (REF == kRefInt4) expand_row<4>(st + C::O_REFK + r * 64, URK, r);
      fence_proxy_async_smem();
    }
    if constexpr (NEED_KREADY) {
      __syncwarp();
      if (lane == 0) mbar_arrive(smem_u32(kready));
    }
  };
  // warpgroup 1: value-side code tiles (published by its later weight arrivals)
  auto expand_values = [&](const uint8_t* st) {
    if constexpr (RB != 0) {
#pragma unroll
      for (int ci = 0; ci < NCH; ++ci) expand_row<RB>(st + C::o_resv(ci) + r * C::CB, UV + 16384 * ci, r);
    }
    if constexpr (REF == kRefInt4) expand_row<4>(st + C::O_REFV + r * 64, URV, r);
    fence_proxy_async_smem();
  };

  // per-segment running state (query heads hb + i)
  float m_run[GH], l_thr[GH], acc_ref[GH], acc_res[GH];
  float zr[GH][NGR > 0 ? NGR : 1], za[GH][NGA > 0 ? NGA : 1];
  auto reset_state = [&]() {
#pragma unroll
    for (int i = 0; i < GH; ++i) {
      m_run[i] = -INFINITY;
      l_thr[i] = acc_ref[i] = acc_res[i] = 0.f;
#pragma unroll
      for (int g = 0; g < (NGR > 0 ? NGR : 1); ++g) zr[i][g] = 0.f;
#pragma unroll
      for (int g = 0; g < (NGA > 0 ? NGA : 1); ++g) za[i][g] = 0.f;
    }
  };

  // ---- prologue: operands of page 0
  PageIter cur;
  seek(cur, x0);
  int len_cur = seq_len(cur.b);  // cached per segment: no global load on a page's path
  reset_state();
  setup(cur.b, cur.h);
  release_scores();
  wait_or_abort(&full[0], 0);
  if constexpr (C::KVSPLIT) wait_or_abort(&fullV[0], 0);
  if (wg == 0) expand_keys(stages);
  else expand_values(stages);

  for (int k = 0; k < n_pages; ++k) {
    const int s = k % C::STAGES;
    uint8_t* st = stages + s * C::STAGE_BYTES;
    const uint32_t ph = k & 1;
    const int n_valid = min(kTP, len_cur - cur.page * kTP);
    const bool last = k + 1 == n_pages;
    PageIter nxt = cur;
    if (!last) advance(nxt);
    const bool seg_end = last || nxt.b != cur.b || nxt.h != cur.h;
    const int s1 = (k + 1) % C::STAGES;
    uint8_t* st1 = stages + s1 * C::STAGE_BYTES;

    // ---- per-token metadata (thread = token r), zero past the context
    if constexpr (C::KVSPLIT) {  // each warpgroup has waited for one half of this page only
      wait_or_abort(&full[s], (k / C::STAGES) & 1);
      wait_or_abort(&fullV[s], (k / C::STAGES) & 1);
    }
    const bool valid = r < n_valid;
    // alpha of every link (link 0 is the loop itself); a chained loop's value
    // weights carry the alpha_V of the links before each: bR[ci] for link ci,
    // bA (all of them) for the anchor
    float aKc[NCH], aVc[NCH];
#pragma unroll
    for (int ci = 0; ci < NCH; ++ci) {
      aKc[ci] = aVc[ci] = 1.f;
      if constexpr (C::HAS_ALPHA) {
        const float2 a = half2_bits_to_f2(*reinterpret_cast<const uint32_t*>(st + C::o_al(ci) + r * 4));
        aKc[ci] = a.x;
        aVc[ci] = a.y;
      }
      if (!valid) aKc[ci] = aVc[ci] = 0.f;
    }
    const float aK = aKc[0], aV = aVc[0];
    float bR[NCH];
    bR[0] = 1.f;
#pragma unroll
    for (int ci = 1; ci < NCH; ++ci) bR[ci] = bR[ci - 1] * aVc[ci - 1];
    const float bA = NCH == 1 ? aV : bR[NCH - 1] * aVc[NCH - 1];
    // with 16 rows the value-side metadata is read after the scores (the stage
    // stays until the page's value MMAs complete), so that fewer registers are
    // live across the score reads
    constexpr int NGR1 = NGR > 0 ? NGR : 1;
    float sK[NCH][NGR1], zK[NCH][NGR1], sV[NCH][NGR1], zV[NCH][NGR1];  // [link][group]
    float sAk[4], zAk[4], sAv[4], zAv[4];
    if constexpr (C::KTM) {
      if constexpr (RB != 0) {
#pragma unroll
        for (int ci = 0; ci < NCH; ++ci) token_meta(st + C::o_resmk(ci) + r * C::MB, valid, sK[ci], zK[ci]);
      }
      if constexpr (REF == kRefInt4) token_meta(st + C::O_REFMK + r * 16, valid, sAk, zAk);
    } else {
      if constexpr (RB != 0) {
#pragma unroll
        for (int g = 0; g < NGR; g += 4) {
          const uint4 mk = *reinterpret_cast<const uint4*>(st + C::O_RESMK + r * C::MB + 4 * g);
          const uint4 mv = *reinterpret_cast<const uint4*>(st + C::O_RESMV + r * C::MB + 4 * g);
          const uint32_t wk[4] = {mk.x, mk.y, mk.z, mk.w}, wv[4] = {mv.x, mv.y, mv.z, mv.w};
#pragma unroll
          for (int u = 0; u < 4; ++u) {
            const float2 a = half2_bits_to_f2(wk[u]), c2 = half2_bits_to_f2(wv[u]);
            sK[0][g + u] = valid ? a.x : 0.f;
            zK[0][g + u] = valid ? a.y : 0.f;
            sV[0][g + u] = valid ? c2.x : 0.f;
            zV[0][g + u] = valid ? c2.y : 0.f;
          }
        }
      }
      if constexpr (REF == kRefInt4) {
        const uint4 mk = *reinterpret_cast<const uint4*>(st + C::O_REFMK + r * 16);
        const uint4 mv = *reinterpret_cast<const uint4*>(st + C::O_REFMV + r * 16);
        const uint32_t wk[4] = {mk.x, mk.y, mk.z, mk.w}, wv[4] = {mv.x, mv.y, mv.z, mv.w};
#pragma unroll
        for (int u = 0; u < 4; ++u) {
          const float2 a = half2_bits_to_f2(wk[u]), c2 = half2_bits_to_f2(wv[u]);
          sAk[u] = valid ? a.x : 0.f;
          zAk[u] = valid ? a.y : 0.f;
          sAv[u] = valid ? c2.x : 0.f;
          zAv[u] = valid ? c2.y : 0.f;
        }
      }
    }

    if constexpr (C::KVSPLIT) {  // the key metadata is in registers: the key half may be refilled
      __syncwarp();
      if (lane == 0) mbar_arrive(smem_u32(&empty[s]));
    }

    wait_or_abort(sbar, ph);
    tc::fence_after_sync();

    // ---- scores of token r for this warpgroup's heads
    float S[GH];
#pragma unroll
    for (int i = 0; i < GH; ++i) S[i] = 0.f;
    // the bf16 anchor's scores are read with the first chunk of the integer
    // ones (one wait for both)
    uint32_t vb[REF == kRefBf16 ? GH : 1];
    if constexpr (REF == kRefBf16) tc::tmem_ld_n<GH>(tl + C::S_REF + hb, vb);
    auto anchor_scores = [&]() {
      if constexpr (REF == kRefBf16) {
        tc::reg_fence(vb);
        const float ak = aK * P.scale_log2;
#pragma unroll
        for (int i = 0; i < GH; ++i) S[i] = __uint_as_float(vb[i]) * ak;
      }
    };
    if constexpr (REF == kRefInt4 || RB != 0) {
      constexpr int HB = GH > 4 ? 4 : GH;  // heads per tensor-memory read
      // 32-dim chunks read per wait: as many as 24 registers hold
      constexpr int RPC = (REF == kRefInt4 ? 3 * HB : 0) + (RB != 0 ? NCH * C::NPAR * 3 * HB : 0);
      constexpr int CPW = HB < GH ? 1 : (4 * RPC <= 24 ? 4 : (2 * RPC <= 24 ? 2 : 1));
      float dotA[GH], offA[GH], dotR[NCH][GH], offR[NCH][GH];  // residual terms per link
#pragma unroll
      for (int i = 0; i < GH; ++i) {
        dotA[i] = offA[i] = 0.f;
#pragma unroll
        for (int ci = 0; ci < NCH; ++ci) dotR[ci][i] = offR[ci][i] = 0.f;
      }
#pragma unroll
      for (int c0 = 0; c0 < 4; c0 += CPW) {
#pragma unroll
        for (int h0 = 0; h0 < GH; h0 += HB) {
          uint32_t va[CPW][3 * HB], vr[CPW][NCH][C::NPAR][3 * HB];
#pragma unroll
          for (int cc = 0; cc < CPW; ++cc) {
            const int c = c0 + cc;
            if constexpr (REF == kRefInt4)
              tc::tmem_ld_n<3 * HB>(tl + C::S_REF + C::N_SA * c + 3 * (hb + h0), va[cc]);
            if constexpr (RB != 0) {
#pragma unroll
              for (int ci = 0; ci < NCH; ++ci)
#pragma unroll
                for (int p = 0; p < C::NPAR; ++p)
                  tc::tmem_ld_n<3 * HB>(tl + C::S_RES + 4 * C::N_SR * ci + C::N_SR * c + p * 3 * G + 3 * (hb + h0),
                                        vr[cc][ci][p]);
            }
          }
          tc::tmem_wait_ld();
#pragma unroll
          for (int cc = 0; cc < CPW; ++cc) {
            if constexpr (REF == kRefInt4) tc::reg_fence(va[cc]);
            if constexpr (RB != 0) {
#pragma unroll
              for (int ci = 0; ci < NCH; ++ci)
#pragma unroll
                for (int p = 0; p < C::NPAR; ++p) tc::reg_fence(vr[cc][ci][p]);
            }
          }
          if (c0 == 0 && h0 == 0) anchor_scores();
#pragma unroll
          for (int cc = 0; cc < CPW; ++cc) {
          const int c = c0 + cc;
#pragma unroll
          for (int i = 0; i < HB; ++i) {
            const int hi = h0 + i, hq = hb + hi;
            // (16 rows: the offsets are summed after the chunks, in the same order)
            if constexpr (REF == kRefInt4) {
              dotA[hi] = fmaf(sAk[c], comb24(va[cc][3 * i], va[cc][3 * i + 1], va[cc][3 * i + 2]), dotA[hi]);
              if constexpr (!C::KTM) offA[hi] = fmaf(zAk[c], sQA[hq * 4 + c], offA[hi]);
            }
            if constexpr (RB != 0) {
#pragma unroll
              for (int ci = 0; ci < NCH; ++ci)
#pragma unroll
                for (int p = 0; p < C::NPAR; ++p) {
                  const uint32_t* w = vr[cc][ci][p];
                  const int g = c * C::NPAR + p;
                  dotR[ci][hi] = fmaf(sK[ci][g], comb24(w[3 * i], w[3 * i + 1], w[3 * i + 2]), dotR[ci][hi]);
                  if constexpr (!C::KTM) offR[ci][hi] = fmaf(zK[ci][g], sQS[hq * 8 + g], offR[ci][hi]);
                }
            }
          }
          }
        }
      }
#pragma unroll
      for (int i = 0; i < GH; ++i) {
        const int hq = hb + i;
        if constexpr (C::KTM) {
          if constexpr (REF == kRefInt4) {
#pragma unroll
            for (int c = 0; c < 4; ++c) offA[i] = fmaf(zAk[c], sQA[hq * 4 + c], offA[i]);
          }
          if constexpr (RB != 0) {
#pragma unroll
            for (int ci = 0; ci < NCH; ++ci)
#pragma unroll
              for (int g = 0; g < NGR; ++g) offR[ci][i] = fmaf(zK[ci][g], sQS[hq * 8 + g], offR[ci][i]);
          }
        }
        if constexpr (NCH == 1) {
          if constexpr (REF == kRefInt4) S[i] = aK * fmaf(dotA[i], sCA[hq], offA[i]);
          if constexpr (RB != 0) S[i] += fmaf(dotR[0][i], sCS[hq], offR[0][i]);
        } else {
          // links from the anchor outward (Horner): part = alpha_K,ci part + link ci's term
          float part = fmaf(dotA[i], sCA[hq], offA[i]);
#pragma unroll
          for (int ci = NCH - 1; ci >= 0; --ci) part = fmaf(aKc[ci], part, fmaf(dotR[ci][i], sCS[hq], offR[ci][i]));
          S[i] = part;
        }
      }
    } else {
      tc::tmem_wait_ld();
      anchor_scores();
    }
    if constexpr (C::KTM) {
      if constexpr (RB != 0) {
#pragma unroll
        for (int ci = 0; ci < NCH; ++ci) token_meta(st + C::o_resmv(ci) + r * C::MB, valid, sV[ci], zV[ci]);
      }
      if constexpr (REF == kRefInt4) token_meta(st + C::O_REFMV + r * 16, valid, sAv, zAv);
    }
#pragma unroll
    for (int i = 0; i < GH; ++i) S[i] = valid ? S[i] : -INFINITY;

    // ---- page maxima of the scores (per head) and of the value scales (per group)
#pragma unroll
    for (int i = 0; i < GH; ++i) {
      const float v = warp_max(S[i]);
      if (lane == 0) sWM[(wg * 4 + (warp & 3)) * C::GHS + i] = v;
    }
    if constexpr (RB != 0) {
#pragma unroll
      for (int g = 0; g < NGR; ++g) {
        // the links' weights share one scale per group: the page's largest |beta s|
        float x = sV[0][g];
#pragma unroll
        for (int ci = 1; ci < NCH; ++ci) x = fmaxf(x, fabsf(bR[ci] * sV[ci][g]));
        const float v = warp_max_nonneg(x);
        if (lane == 0) sSig[(wg * 4 + (warp & 3)) * 12 + g] = v;
      }
    }
    if constexpr (REF == kRefInt4) {
#pragma unroll
      for (int g = 0; g < 4; ++g) {
        const float v = warp_max_nonneg(fabsf(bA * sAv[g]));
        if (lane == 0) sSig[(wg * 4 + (warp & 3)) * 12 + 8 + g] = v;
      }
    }
    named_bar_sync(kBarWG + wg, 128);
    float pm[GH], crun[GH], prel[GH];
#pragma unroll
    for (int i = 0; i < GH; ++i) {
      const float* wm = sWM + wg * (4 * C::GHS) + i;
      const float mp = fmaxf(fmaxf(wm[0], wm[C::GHS]), fmaxf(wm[2 * C::GHS], wm[3 * C::GHS]));
      const float mn = fmaxf(m_run[i], mp);
      crun[i] = fast_exp2(m_run[i] - mn);
      pm[i] = fast_exp2(mp - mn);
      m_run[i] = mn;
      prel[i] = fast_exp2(S[i] - mp);
    }
    float sig[NGR > 0 ? NGR : 1], siga[4];
    if constexpr (RB != 0) {
#pragma unroll
      for (int g = 0; g < NGR; ++g) {
        const float* sg = sSig + wg * 48 + g;
        sig[g] = fmaxf(fmaxf(sg[0], sg[12]), fmaxf(sg[24], sg[36]));
      }
    }
    if constexpr (REF == kRefInt4) {
#pragma unroll
      for (int g = 0; g < 4; ++g) {
        const float* sg = sSig + wg * 48 + 8 + g;
        siga[g] = fmaxf(fmaxf(sg[0], sg[12]), fmaxf(sg[24], sg[36]));
      }
    }

    // ---- B operands of the value MMAs: column t = token r
    const int wrow = (r >> 3) * 128 + (r & 7) * 16;  // MN-major core-matrix row of token r
    if constexpr (REF == kRefBf16) {
      if (own_ref) {
        uint32_t pk[GH];
#pragma unroll
        for (int i = 0; i < GH; ++i) {
          const float w = prel[i] * aV;
          const __nv_bfloat16 hi = __float2bfloat16_rn(w);
          const __nv_bfloat16 lo = __float2bfloat16_rn(w - __bfloat162float(hi));
          pk[i] = static_cast<uint32_t>(__bfloat16_as_ushort(hi)) |
                  (static_cast<uint32_t>(__bfloat16_as_ushort(lo)) << 16);
        }
        const int n0 = wgo * G;  // rows n = 2 * head + (0: hi, 1: lo)
        uint8_t* dst = WB + (n0 >> 3) * 2048 + wrow + (n0 & 7) * 2;
        if constexpr (GH == 8) {
          *reinterpret_cast<uint4*>(dst) = make_uint4(pk[0], pk[1], pk[2], pk[3]);
          *reinterpret_cast<uint4*>(dst + 2048) = make_uint4(pk[4], pk[5], pk[6], pk[7]);
        } else if constexpr (GH == 4) *reinterpret_cast<uint4*>(dst) = make_uint4(pk[0], pk[1], pk[2], pk[3]);
        else if constexpr (GH == 2) *reinterpret_cast<uint2*>(dst) = make_uint2(pk[0], pk[1]);
        else *reinterpret_cast<uint32_t*>(dst) = pk[0];
      }
      // bf16 anchor rows past the context may hold anything: clear them so
      // that their zero weights give exact zeros
      if (!valid && (!SPLIT || wg == 0)) {
#pragma unroll
        for (int half = 0; half < (SPLIT ? 2 : 1); ++half) {
          uint4* row = reinterpret_cast<uint4*>(st + C::O_REFV + (SPLIT ? half : wg) * 16384 + r * 128);
#pragma unroll
          for (int q = 0; q < 8; ++q) row[q] = make_uint4(0u, 0u, 0u, 0u);
        }
      }
    }
    if constexpr (REF == kRefInt4) {
      if (own_ref) {
        // signed weights (alpha may be negative): three signed bytes each;
        // with 8 heads a warpgroup writes them in two halves of the groups
        constexpr int NB = 4 * GH;
        constexpr int NH = NB > 16 ? 2 : 1;
        constexpr int GPH = 4 / NH;
#pragma unroll
        for (int hh = 0; hh < NH; ++hh) {
          uint32_t v[NB / NH];
#pragma unroll
          for (int gg = 0; gg < GPH; ++gg) {
            const int g = hh * GPH + gg;
            const float t = siga[g] > 0.f ? bA * sAv[g] * rcp_approx(siga[g]) * kQ3 : 0.f;
#pragma unroll
            for (int i = 0; i < GH; ++i) {
              int qi = __float2int_rn(prel[i] * t);
              qi = max(-8323072, min(8323072, qi));
              int b2, b1, b0;
              split24(qi, b2, b1, b0);
              v[gg * GH + i] = (static_cast<uint32_t>(b0) & 0xFFu) | ((static_cast<uint32_t>(b1) & 0xFFu) << 8) |
                               ((static_cast<uint32_t>(b2) & 0xFFu) << 16);
            }
          }
          uint32_t planes[3][NB / NH / 4];
          byte_planes<NB / NH>(v, planes);
#pragma unroll
          for (int j = 0; j < 3; ++j) put_plane<NB / NH>(WA, j * 4 * G + wgo * NB + hh * (NB / NH), wrow, planes[j]);
        }
      }
    }
    // the scores are in registers: the value sums may now be written
    tc::fence_before_sync();
    if constexpr (HAS_V1) {
      fence_proxy_async_smem();
      __syncwarp();
      if (lane == 0) mbar_arrive(smem_u32(v1ready));
    }
    if constexpr (RB != 0 && C::SIGNED_RES) {
      if (own_res) {
        // chained links: link ci's weights p * beta_ci * s_ci,g relative to the
        // page's largest |beta s| of the group, as signed 24-bit integers
        constexpr int NB = NGR * GH;
#pragma unroll
        for (int ci = 0; ci < NCH; ++ci) {
          uint32_t v[NB];
#pragma unroll
          for (int g = 0; g < NGR; ++g) {
            const float t = sig[g] > 0.f ? bR[ci] * sV[ci][g] * rcp_approx(sig[g]) * kQ3 : 0.f;
#pragma unroll
            for (int i = 0; i < GH; ++i) {
              int qi = __float2int_rn(prel[i] * t);
              qi = max(-8323072, min(8323072, qi));
              int b2, b1, b0;
              split24(qi, b2, b1, b0);
              v[g * GH + i] = (static_cast<uint32_t>(b0) & 0xFFu) | ((static_cast<uint32_t>(b1) & 0xFFu) << 8) |
                              ((static_cast<uint32_t>(b2) & 0xFFu) << 16);
            }
          }
          uint32_t planes[3][NB / 4];
          byte_planes<NB>(v, planes);
#pragma unroll
          for (int j = 0; j < 3; ++j) put_plane<NB>(WR + C::WR_BYTES * ci, j * NGR * G + wgo * NB, wrow, planes[j]);
        }
      }
    }
    if constexpr (RB != 0 && !C::SIGNED_RES) {
      if (own_res) {
        // non-negative weights p * s_g / max_page(s_g) as unsigned 24-bit integers
        constexpr int NB = NGR * GH;
        constexpr int NH = (NB > 16 && GH == 8 && C::REGSPLIT) ? 2 : 1;  // halves, as for the anchor
        constexpr int GPH = NGR / NH;
#pragma unroll
        for (int hh = 0; hh < NH; ++hh) {
          uint32_t v[NB / NH];
#pragma unroll
          for (int gg = 0; gg < GPH; ++gg) {
            const int g = hh * GPH + gg;
            const float t = sig[g] > 0.f ? sV[0][g] * rcp_approx(sig[g]) * kU3 : 0.f;
#pragma unroll
            for (int i = 0; i < GH; ++i) v[gg * GH + i] = min(__float2uint_rn(prel[i] * t), 16777215u);
          }
          uint32_t planes[3][NB / NH / 4];
          byte_planes<NB / NH>(v, planes);
#pragma unroll
          for (int j = 0; j < 3; ++j) put_plane<NB / NH>(WR, j * NGR * G + wgo * NB + hh * (NB / NH), wrow, planes[j]);
        }
      }
    }
    if constexpr (HAS_V2) {
      fence_proxy_async_smem();
      __syncwarp();
      if (lane == 0) mbar_arrive(smem_u32(v2ready));
    }

    // ---- running denominators and offset sums (thread = token r)
#pragma unroll
    for (int i = 0; i < GH; ++i) {
      const float pr = prel[i] * pm[i];
      if (own_ref) l_thr[i] = fmaf(l_thr[i], crun[i], pr);
      if constexpr (RB != 0) {
        if (own_res) {
#pragma unroll
          for (int g = 0; g < NGR; ++g) {
            float zsum = zV[0][g];
#pragma unroll
            for (int ci = 1; ci < NCH; ++ci) zsum = fmaf(bR[ci], zV[ci][g], zsum);
            zr[i][g] = fmaf(zr[i][g], crun[i], pr * zsum);
          }
        }
      }
      if constexpr (REF == kRefInt4) {
        if (own_ref) {
#pragma unroll
          for (int g = 0; g < 4; ++g) za[i][g] = fmaf(za[i][g], crun[i], pr * bA * zAv[g]);
        }
      }
    }

    // ---- run ahead: operands of page k + 1 (query operands of a new
    // segment, then its key code tiles) while page k's value MMAs run
    int len_nxt = len_cur;
    if (!last) {
      if (seg_end) {
        len_nxt = seq_len(nxt.b);
        setup(nxt.b, nxt.h);
      }
      if constexpr (!C::ALIAS) release_scores();
      if (wg == 0) {
        wait_or_abort(&full[s1], ((k + 1) / C::STAGES) & 1);
        expand_keys(st1);
      }
    }

    wait_or_abort(obar, ph);
    tc::fence_after_sync();

    // ---- merge the page's value sums (thread = dim position r); the bf16
    // anchor's sums are read with the residual ones (one wait for both)
    uint32_t vO[REF == kRefBf16 ? 2 * GH : 1];
    if constexpr (REF == kRefBf16) {
      if (own_ref) tc::tmem_ld_n<2 * GH>(tl + C::O_REF + wgo * G, vO);
    } else if constexpr (REF == kRefInt4) {
      if (own_ref) {
        uint32_t v[3][GH];
#pragma unroll
        for (int j = 0; j < 3; ++j) tc::tmem_ld_n<GH>(tl + C::O_REF + j * 4 * G + wgo * 4 * GH + chunk * GH, v[j]);
        tc::tmem_wait_ld();
#pragma unroll
        for (int j = 0; j < 3; ++j) tc::reg_fence(v[j]);
        float sg = siga[0];
#pragma unroll
        for (int g = 1; g < 4; ++g) sg = (chunk == g) ? siga[g] : sg;
        const float f = sg * (1.f / kQ3);
#pragma unroll
        for (int i = 0; i < GH; ++i) acc_ref[i] = fmaf(acc_ref[i], crun[i], pm[i] * f * comb24(v[0][i], v[1][i], v[2][i]));
      }
    }
    if constexpr (RB != 0) {
      if (own_res) {
        uint32_t v[C::NPAR][3][GH];
#pragma unroll
        for (int p = 0; p < C::NPAR; ++p)
#pragma unroll
          for (int j = 0; j < 3; ++j)
            tc::tmem_ld_n<GH>(tl + C::O_RES + j * NGR * G + wgo * NGR * GH + (chunk * C::NPAR + p) * GH, v[p][j]);
        tc::tmem_wait_ld();
#pragma unroll
        for (int p = 0; p < C::NPAR; ++p)
#pragma unroll
          for (int j = 0; j < 3; ++j) tc::reg_fence(v[p][j]);
        float sg = sig[0];
#pragma unroll
        for (int g = 1; g < NGR; ++g) sg = (g_res == g) ? sig[g] : sg;
        const float f = sg * (1.f / (C::SIGNED_RES ? kQ3 : kU3));
#pragma unroll
        for (int i = 0; i < GH; ++i) {
          uint32_t b2 = v[0][0][i], b1 = v[0][1][i], b0 = v[0][2][i];
          if constexpr (C::NPAR == 2) {
            b2 = par_r ? v[1][0][i] : b2;
            b1 = par_r ? v[1][1][i] : b1;
            b0 = par_r ? v[1][2][i] : b0;
          }
          acc_res[i] = fmaf(acc_res[i], crun[i], pm[i] * f * comb24(b2, b1, b0));
        }
      }
    }
    if constexpr (REF == kRefBf16) {
      if (own_ref) {
        if (!(RB != 0 && own_res)) tc::tmem_wait_ld();
        tc::reg_fence(vO);
#pragma unroll
        for (int i = 0; i < GH; ++i)
          acc_ref[i] = fmaf(acc_ref[i], crun[i], pm[i] * (__uint_as_float(vO[2 * i]) + __uint_as_float(vO[2 * i + 1])));
      }
    }

    // the value sums overlay the scores: page k + 1 may be scored once they are read
    if constexpr (C::ALIAS) {
      if (!last) release_scores();
    }

    // ---- flush a finished (b, h) segment: one partial record per query head
    if (seg_end) {
      // per-warp sums into their own slots, added in a fixed order below, so
      // that a decode is reproducible bit for bit from run to run
      float* myred = sRed + (warp & 3) * C::GS * C::NRED;
#pragma unroll
      for (int i = 0; i < GH; ++i) {
        const int hq = hb + i;
        if (own_ref) {
          const float lsum = warp_sum(l_thr[i]);
          if (lane == 0) myred[hq * C::NRED] = lsum;
        }
        if constexpr (RB != 0) {
          if (own_res) {
#pragma unroll
            for (int g = 0; g < NGR; ++g) {
              const float z = warp_sum(zr[i][g]);
              if (lane == 0) myred[hq * C::NRED + 1 + g] = z;
            }
          }
        }
        if constexpr (REF == kRefInt4) {
          if (own_ref) {
#pragma unroll
            for (int g = 0; g < 4; ++g) {
              const float z = warp_sum(za[i][g]);
              if (lane == 0) myred[hq * C::NRED + 9 + g] = z;
            }
          }
        }
      }
      named_bar_sync(kBarAll, kNCT);  // both warpgroups' sums (G == 1 splits them)
      auto red = [&](int hq, int slot) {
        const float* p = sRed + hq * C::NRED + slot;
        constexpr int WS = C::GS * C::NRED;  // one warp's slots
        return __fadd_rn(__fadd_rn(p[0], p[WS]), __fadd_rn(p[2 * WS], p[3 * WS]));
      };
      const int pair = cur.b * Hkv + cur.h;
      const int d_ref = REF == kRefInt4 ? 32 * chunk + pos_dim<4>(r & 31) : r;
      const int d_res = RB ? 32 * chunk + pos_dim<RB ? RB : 2>(r & 31) : r;
#pragma unroll
      for (int i = 0; i < GH; ++i) {
        const int hq = hb + i;
        float* rec = P.partials + (static_cast<int64_t>(pair + blockIdx.x) * G + hq) * kPartialFloats;
        if (own_ref) {
          float vref = 0.f;
          if constexpr (REF != kRefNone) vref = acc_ref[i];
          if constexpr (REF == kRefInt4) vref += red(hq, 9 + chunk);
          rec[4 + d_ref] = vref;
          if (r == 0) {
            rec[0] = m_run[i];
            rec[1] = red(hq, 0);
          }
        }
        if (own_res) {
          float vres = 0.f;
          if constexpr (RB != 0) vres = acc_res[i] + red(hq, 1 + g_res);
          rec[4 + kD + d_res] = vres;
        }
      }
      named_bar_sync(kBarAll, kNCT);
      reset_state();
    }

    // ---- run ahead: value code tiles of page k + 1 (page k's value MMAs are done)
    if (!last && wg == 1) {
      wait_or_abort(C::KVSPLIT ? &fullV[s1] : &full[s1], ((k + 1) / C::STAGES) & 1);
      expand_values(st1);
    }
    cur = nxt;
    len_cur = len_nxt;
  }

  // ---- release the tensor memory once every MMA and every consumer is done with it
  tc::fence_before_sync();
  named_bar_sync(kBarAll, kNCT);
  if (warp == 0) {
    if (!mbar_wait_bounded(smem_u32(done), 0)) set_flag(P.status, RQ_FLAG_PIPE_TIMEOUT);
    tc::fence_after_sync();
    tc::tmem_dealloc(tbase, C::TMEM_COLS);
  }
}

// ---------------------------------------------------------------------------
// dispatch
// ---------------------------------------------------------------------------
template <int REF, int RB, int RG, int G, int NCH>
cudaError_t launch_tc(const DecodeParams& p, const CUtensorMap* tk, const CUtensorMap* tv, cudaStream_t s) {
  using C = TcCfg<REF, RB, RG, G, NCH>;
  if constexpr (!C::FITS) {
    return cudaErrorInvalidValue;
  } else {
    auto kern = decode_tc_kernel<REF, RB, RG, G, NCH>;
    static bool attr_done = false;  // per instantiation; set once per process
    if (!attr_done) {
      cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, C::SMEM_BYTES);
      if (e != cudaSuccess) return e;
      attr_done = true;
    }
    return launch_dependent(kern, p.num_ctas, C::NT, C::SMEM_BYTES, s, p, *tk, *tv);
  }
}

using TcFn = cudaError_t (*)(const DecodeParams&, const CUtensorMap*, const CUtensorMap*, cudaStream_t);

template <int REF, int RB, int RG, int G, int NCH>
TcFn tc_if_fits() {
  if constexpr (TcCfg<REF, RB, RG, G, NCH>::FITS) return launch_tc<REF, RB, RG, G, NCH>;
  else return nullptr;
}

}  // namespace
}  // namespace rq
