// rq_decode_pp.cu -- split-K decode attention on the tensor cores for the
// byte-plane formats (an INT4 anchor, or no anchor term) at one query row per
// kv-head, with two warpgroups working on alternate pages ("ping-pong").
//
// Same method and the same partial records as the other split kernels:
// "ResidualQuant: KV Cache Quantization for Looped Transformers with 2-Bit
// Residuals" keeps loop l as alpha * anchor + H^T deq(R_l) (abstract, Figure 1,
// Figure 2 caption), and every cached token is scored and summed from that
// compact form.  On the CUDA cores these formats are bound by the per-token
// arithmetic (turning codes into floats); on the tensor cores the codes only
// have to be widened to int8, and the scores and value sums are integer MMAs:
//
//   * a page is 128 tokens of one (sequence, kv-head); a producer warp streams
//     pages into a ring of shared-memory stages by bulk copies (no multicast);
//     stage s always serves warpgroup s % 2 (the ring has an even number of
//     stages), and pages alternate between the warpgroups;
//   * a warpgroup takes its page from start to end, thread = token: it widens
//     the key codes into its own tensor-memory columns (the score MMAs' A
//     operand) and the value codes into its own shared tiles, reads the
//     page's metadata and then releases the stage; it reads the scores, takes
//     the page maximum, writes the softmax weights as 24-bit byte planes,
//     and merges the page's value sums into its running state (thread = dim);
//   * one thread issues every MMA, for whichever warpgroup is ready: the two
//     pipelines overlap, so that one warpgroup's arithmetic hides the other's
//     MMA latency;
//   * at the end of a (b, kv-head) segment the two warpgroups' states are
//     added in a fixed order into the CTA's partial record.
//
// Numerics are those of the tensor-core kernel in rq_decode_tc.cuh: queries and
// weights as 24-bit integers in byte planes, exact int32 sums.
#include "rq_common.cuh"
#include "rq_internal.h"
#include "rq_tc_ops.cuh"
#include "rq_tcgen05.cuh"

namespace rq {
namespace {

constexpr int kPP = kTcPage;        // tokens per page
constexpr int kPpNCT = 256;         // two consumer warpgroups
constexpr int kPpProducer = 8;      // producer warp
constexpr int kPpMma = 9;           // MMA-issuing warps: kPpMma + w serves warpgroup w
constexpr int kPpNT = kPpNCT + 96;
constexpr int kPpBarAll = 1;        // the 256 consumer threads
constexpr int kPpBarWG = 2;         // warpgroup w uses kPpBarWG + w
constexpr int kPpSmemLimit = 227 * 1024;

template <int REF, int RB, int RG>
struct PpCfg {
  static constexpr bool ANCH = REF == kRefInt4;
  static constexpr int NGR = RB ? kD / RG : 0;    // residual groups
  static constexpr int NGR1 = NGR > 0 ? NGR : 1;
  static constexpr int NPAR = RG == 16 ? 2 : 1;   // residual groups per 32-dim chunk
  static constexpr bool HAS_ALPHA = ANCH && RB != 0;
  static constexpr int REF_REC = ANCH ? 64 : 0;
  static constexpr int REFM_REC = ANCH ? 16 : 0;
  static constexpr int CB = RB * 16;
  static constexpr int MB = RB ? 4 * NGR : 0;
  static constexpr int AL_REC = HAS_ALPHA ? 4 : 0;
  // MMA widths (one query head): score columns are (group, byte plane) of the
  // query, value columns (byte plane, group) of the weights
  static constexpr int N_SA = 16;                 // 4 groups x 3
  static constexpr int N_SR = round16(3 * NGR1);  // 12 or 24
  static constexpr int N_VA = 16;
  static constexpr int N_VR = round16(3 * NGR1);
  // tensor-memory columns of one warpgroup
  static constexpr int T_KA = 0;                          // anchor key codes, int8 [128 tok][128]: 32 columns
  static constexpr int T_KR = T_KA + (ANCH ? 32 : 0);     // residual key codes
  static constexpr int T_SA = T_KR + (RB ? 32 : 0);       // anchor scores
  static constexpr int T_SR = T_SA + (ANCH ? N_SA : 0);   // residual scores
  static constexpr int T_OA = T_SR + (RB ? N_SR : 0);     // anchor value sums
  static constexpr int T_OR = T_OA + (ANCH ? N_VA : 0);   // residual value sums
  static constexpr int T_WG = T_OR + (RB ? N_VR : 0);
  static constexpr int TMEM_COLS = 2 * T_WG <= 128 ? 128 : (2 * T_WG <= 256 ? 256 : 512);
  // stage layout (pieces 1024-byte aligned)
  static constexpr int al(int x) { return (x + 1023) & ~1023; }
  static constexpr int O_REFK = 0;
  static constexpr int O_REFV = O_REFK + al(kPP * REF_REC);
  static constexpr int O_REFMK = O_REFV + al(kPP * REF_REC);
  static constexpr int O_REFMV = O_REFMK + al(kPP * REFM_REC);
  static constexpr int O_RESK = O_REFMV + al(kPP * REFM_REC);
  static constexpr int O_RESV = O_RESK + al(kPP * CB);
  static constexpr int O_RESMK = O_RESV + al(kPP * CB);
  static constexpr int O_RESMV = O_RESMK + al(kPP * MB);
  static constexpr int O_AL = O_RESMV + al(kPP * MB);
  static constexpr int STAGE_BYTES = O_AL + al(kPP * AL_REC);
  static constexpr int TX_REC = 2 * REF_REC + 2 * REFM_REC + 2 * CB + 2 * MB + AL_REC;  // bytes per token
  // shared tiles of one warpgroup
  static constexpr int F_URV = 0;                                  // anchor value codes, int8, sw128
  static constexpr int F_UV = F_URV + (ANCH ? 16384 : 0);          // residual value codes
  static constexpr int F_QA = F_UV + (RB ? 16384 : 0);             // anchor query bytes [N_SA][128], K-major sw128
  static constexpr int F_HQ = F_QA + (ANCH ? al(N_SA * 128) : 0);  // H q bytes [N_SR][128]
  static constexpr int F_WA = F_HQ + (RB ? al(N_SR * 128) : 0);    // anchor value weights [N_VA x 128 tok]
  static constexpr int F_WR = F_WA + (ANCH ? al(N_VA * 128) : 0);  // residual value weights [N_VR x 128 tok]
  static constexpr int F_WG = F_WR + (RB ? al(N_VR * 128) : 0);
  // small state, 4-byte words
  static constexpr int W_Q = 0;                         // [2][16]: anchor scale, residual scale, anchor sums[4], residual sums[8]
  static constexpr int W_WM = W_Q + 32;                 // [2][4 warps] warp maxima of the scores
  static constexpr int W_SIG = W_WM + 8;                // [2][4 warps][12] warp maxima of the value scales
  static constexpr int W_SLOT = W_SIG + 96;             // [2][4 + 2 * 128] flush slots
  static constexpr int SLOT = 4 + 2 * kD;
  static constexpr int W_RED = W_SLOT + 2 * SLOT;       // [2][4 warps][16] l and offset sums
  static constexpr int W_PRE = W_RED + 2 * 4 * 16;      // [RQ_MAX_BATCH + 1] page prefix
  static constexpr int W_MISC = W_PRE + RQ_MAX_BATCH + 1;  // abort flag, tensor-memory base
  static constexpr int W_BAR = (W_MISC + 2 + 1) & ~1;
  static constexpr int NBARS = 32;
  static constexpr int SMALL = 4 * W_BAR + 8 * NBARS;
  static constexpr int FIXED = 1024 + 2 * F_WG + SMALL;
  static constexpr int STAGES_FIT = (kPpSmemLimit - FIXED) / STAGE_BYTES;
  // an even number of stages: stage s always serves warpgroup s % 2
  static constexpr int STAGES = STAGES_FIT >= 6 ? 6 : (STAGES_FIT >= 4 ? 4 : 2);
  static constexpr bool FITS = STAGES_FIT >= 2 && 2 * T_WG <= 512;
  static constexpr int SMEM_BYTES = FIXED + STAGES * STAGE_BYTES;
  // instruction descriptors (M = 128)
  static constexpr uint32_t ID_SA = tc::instr_desc(tc::kAccS32, tc::kFmtS8, tc::kFmtS8, 0, 0, 128, N_SA);
  static constexpr uint32_t ID_SR = tc::instr_desc(tc::kAccS32, tc::kFmtS8, tc::kFmtS8, 0, 0, 128, N_SR);
  static constexpr uint32_t ID_VA = tc::instr_desc(tc::kAccS32, tc::kFmtS8, tc::kFmtS8, 1, 1, 128, N_VA);
  static constexpr uint32_t ID_VR = tc::instr_desc(tc::kAccS32, 0, 0, 1, 1, 128, N_VR);  // unsigned bytes
  static_assert(REF != kRefBf16, "byte-plane formats only");
  static_assert(STAGES <= 6, "barrier slots");
};

template <int REF, int RB, int RG>
__device__ __forceinline__ void pp_issue_page(const DecodeParams& P, uint8_t* st, uint32_t full, const PageIter& it,
                                              int Hkv) {
  using C = PpCfg<REF, RB, RG>;
  const int t0 = it.page * kPP;
  // byte planes hold plane_tokens (a multiple of 64) records per (b, h)
  const int nrec = (t0 + kPP > P.plane_tokens) ? static_cast<int>(P.plane_tokens - t0) : kPP;
  mbar_arrive_expect_tx(full, static_cast<uint32_t>(nrec) * C::TX_REC);
  const int64_t rec0 = static_cast<int64_t>(it.b * Hkv + it.h) * P.plane_tokens + t0;
  if constexpr (C::ANCH) {
    bulk_g2s(smem_u32(st + C::O_REFK), P.ref_codes[0] + rec0 * 64, nrec * 64, full);
    bulk_g2s(smem_u32(st + C::O_REFV), P.ref_codes[1] + rec0 * 64, nrec * 64, full);
    bulk_g2s(smem_u32(st + C::O_REFMK), P.ref_meta[0] + rec0 * 16, nrec * 16, full);
    bulk_g2s(smem_u32(st + C::O_REFMV), P.ref_meta[1] + rec0 * 16, nrec * 16, full);
  }
  if constexpr (RB != 0) {
    bulk_g2s(smem_u32(st + C::O_RESK), P.res_codes[0][0] + rec0 * C::CB, nrec * C::CB, full);
    bulk_g2s(smem_u32(st + C::O_RESV), P.res_codes[0][1] + rec0 * C::CB, nrec * C::CB, full);
    bulk_g2s(smem_u32(st + C::O_RESMK), P.res_meta[0][0] + rec0 * C::MB, nrec * C::MB, full);
    bulk_g2s(smem_u32(st + C::O_RESMV), P.res_meta[0][1] + rec0 * C::MB, nrec * C::MB, full);
  }
  if constexpr (C::HAS_ALPHA) bulk_g2s(smem_u32(st + C::O_AL), P.alpha[0] + rec0 * 4, nrec * 4, full);
}

template <int REF, int RB, int RG>
__global__ void __launch_bounds__(kPpNT, 1) decode_pp_kernel(const __grid_constant__ DecodeParams P) {
  using C = PpCfg<REF, RB, RG>;
  constexpr bool ANCH = C::ANCH;
  constexpr int NGR = C::NGR, NGR1 = C::NGR1;
  extern __shared__ __align__(16) uint8_t smem_raw[];
  uint8_t* base = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
  uint8_t* stages = base;
  uint8_t* fx = base + C::STAGES * C::STAGE_BYTES;  // two warpgroups' tiles, F_WG bytes apart
  float* sw = reinterpret_cast<float*>(fx + 2 * C::F_WG);
  float* sQ = sw + C::W_Q;
  float* sWM = sw + C::W_WM;
  float* sSig = sw + C::W_SIG;
  float* sSlot = sw + C::W_SLOT;
  float* sRed = sw + C::W_RED;
  int* sPre = reinterpret_cast<int*>(sw + C::W_PRE);
  volatile int* sAbort = reinterpret_cast<volatile int*>(sw + C::W_MISC);
  uint32_t* sTmem = reinterpret_cast<uint32_t*>(sw + C::W_MISC + 1);
  uint64_t* bars = reinterpret_cast<uint64_t*>(sw + C::W_BAR);
  uint64_t* full = bars;          // [stage] the page's copies landed
  uint64_t* empty = bars + 6;     // [stage] the page's warpgroup is done with the stage
  uint64_t* kready = bars + 12;   // [wg] the page's key codes (and the segment's query operands) written
  uint64_t* sbar = bars + 14;     // [wg] the page's score MMAs completed
  uint64_t* vready = bars + 16;   // [wg] the page's value codes and weights written
  uint64_t* obar = bars + 18;     // [wg] the page's value MMAs completed
  uint64_t* done = bars + 20;     // every MMA of the CTA completed
  uint64_t* never = bars + 21;    // never arrived at: the wait of the stall test hook

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
        v = (len + kPP - 1) / kPP;
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
      mbar_init(smem_u32(&empty[s]), 4);  // the four warps of the page's warpgroup
    }
    for (int w = 0; w < 2; ++w) {
      mbar_init(smem_u32(&kready[w]), 4);
      mbar_init(smem_u32(&sbar[w]), 1);
      mbar_init(smem_u32(&vready[w]), 4);
      mbar_init(smem_u32(&obar[w]), 1);
    }
    mbar_init(smem_u32(done), 2);  // both MMA-issuing warps
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
  // A wait that timed out marks the CTA aborted; later waits then return at once.
  auto wait_or_abort = [&](uint64_t* bar, uint32_t parity) -> bool {
    if (*sAbort) return false;
    if (mbar_wait_bounded(smem_u32(bar), parity)) return true;
    set_flag(P.status, RQ_FLAG_PIPE_TIMEOUT);
    *sAbort = 1;
    return false;
  };

  // ---- tensor memory: both warpgroups' key tiles, scores and value sums
  if (warp == 0) {
    tc::tmem_alloc(smem_u32(sTmem), C::TMEM_COLS);
    tc::tmem_relinquish();
  }
  tc::fence_before_sync();
  __syncthreads();
  tc::fence_after_sync();
  const uint32_t tbase = *sTmem;

  // ========================= producer warp =========================
  if (warp == kPpProducer) {
    if (lane == 0) {
      PageIter it;
      seek(it, x0);
      int k = 0;
      for (; k < n_pages; ++k) {
        const int s = k % C::STAGES;
        if (!mbar_wait_bounded(smem_u32(&empty[s]), ((k / C::STAGES) & 1) ^ 1)) {
          set_flag(P.status, RQ_FLAG_PIPE_TIMEOUT);
          *sAbort = 1;
          break;
        }
        if (k == P.stall_page && !mbar_wait_bounded(smem_u32(never), 0)) set_flag(P.status, RQ_FLAG_PIPE_TIMEOUT);
        if (*sAbort) break;
        pp_issue_page<REF, RB, RG>(P, stages + s * C::STAGE_BYTES, smem_u32(&full[s]), it, Hkv);
        advance(it);
      }
      // no copy this CTA issued may still be landing when it exits
      for (int kk = (k > C::STAGES ? k - C::STAGES : 0); kk < k; ++kk) {
        if (!mbar_wait_bounded(smem_u32(&full[kk % C::STAGES]), (kk / C::STAGES) & 1)) {
          set_flag(P.status, RQ_FLAG_PIPE_TIMEOUT);
          break;
        }
      }
    }
    return;
  }

  // ========================= MMA-issuing warps =========================
  // Warp kPpMma + w issues the MMAs of warpgroup w, whose pages are k = w,
  // w + 2, ...: for each, the score MMAs once its key codes are in tensor
  // memory, then the value MMAs once its weights are written.  The two warps
  // wait on their own warpgroup's barriers, so each reacts at once.
  if (warp == kPpMma || warp == kPpMma + 1) {
    if (lane == 0) {
      const int w = warp - kPpMma;
      const int todo = n_pages > w ? (n_pages - w + 1) / 2 : 0;
      uint8_t* fw = fx + w * C::F_WG;
      const uint32_t tw = tbase + w * C::T_WG;
      for (int cnt = 0; cnt < todo; ++cnt) {
        const uint32_t ph = cnt & 1;
        if (!wait_or_abort(&kready[w], ph)) break;
        tc::fence_after_sync();
        if constexpr (ANCH) {
#pragma unroll
          for (int c = 0; c < 4; ++c)
            tc::mma_s8_ta(tw + C::T_SA, tw + C::T_KA + 8 * c, tc::desc_k_sw128(smem_u32(fw + C::F_QA + 32 * c)),
                          C::ID_SA, c > 0);
        }
        if constexpr (RB != 0) {
#pragma unroll
          for (int c = 0; c < 4; ++c)
            tc::mma_s8_ta(tw + C::T_SR, tw + C::T_KR + 8 * c, tc::desc_k_sw128(smem_u32(fw + C::F_HQ + 32 * c)),
                          C::ID_SR, c > 0);
        }
        tc::commit(smem_u32(&sbar[w]));
        if (!wait_or_abort(&vready[w], ph)) break;
        tc::fence_after_sync();
        if constexpr (ANCH) {
#pragma unroll
          for (int ks = 0; ks < 4; ++ks)
            tc::mma_s8(tw + C::T_OA, tc::desc_mn_sw128(smem_u32(fw + C::F_URV + ks * 4096), 16384),
                       tc::desc_mn_plain(smem_u32(fw + C::F_WA + ks * 512), 128, 2048), C::ID_VA, ks > 0);
        }
        if constexpr (RB != 0) {
#pragma unroll
          for (int ks = 0; ks < 4; ++ks)
            tc::mma_s8(tw + C::T_OR, tc::desc_mn_sw128(smem_u32(fw + C::F_UV + ks * 4096), 16384),
                       tc::desc_mn_plain(smem_u32(fw + C::F_WR + ks * 512), 128, 2048), C::ID_VR, ks > 0);
        }
        tc::commit(smem_u32(&obar[w]));
      }
      tc::commit(smem_u32(done));
    }
    return;
  }

  // ========================= consumer warpgroups =========================
  const int wg = warp >> 2;                  // pages k with k % 2 == wg
  const int r = tid & 127;                   // tensor-memory lane: token, then dim position
  const int chunk = warp & 3;                // 32-dim chunk of this thread's dim position
  const uint32_t tl = tbase + wg * C::T_WG + (static_cast<uint32_t>(32 * chunk) << 16);
  uint8_t* fw = fx + wg * C::F_WG;
  float* q_sc = sQ + 16 * wg;                // [0] anchor scale, [1] residual scale, [2..6) anchor sums, [6..14) residual sums
  const int par_r = RB == 2 ? ((r >> 2) & 1) : ((r >> 3) & 1);
  const int g_res = RG == 16 ? 2 * chunk + par_r : chunk;

  auto seq_len = [&](int b) {
    const int len = P.ctx_len[b];
    return len < 0 ? 0 : (len > P.capacity ? P.capacity : len);
  };

  // query operands of (b, h) for this warpgroup's score MMAs (its first warp)
  auto setup = [&](int b, int h) {
    if ((warp & 3) == 0) {
      const uint2 raw = *reinterpret_cast<const uint2*>(P.q + q_row_offset(P, b, h, 0) + 4 * lane);
      const float2 a01 = bf16x2_to_f2(raw.x), a23 = bf16x2_to_f2(raw.y);
      float x[4] = {a01.x, a01.y, a23.x, a23.y};
      if constexpr (ANCH) put_q_grouped<4, 32>(fw + C::F_QA, x, lane, &q_sc[0], &q_sc[2], P.scale_log2);
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
        put_q_grouped<RB, RG>(fw + C::F_HQ, x, lane, &q_sc[1], &q_sc[6], P.scale_log2);
      }
    }
    fence_proxy_async_smem();
    named_bar_sync(kPpBarWG + wg, 128);
  };

  // per-segment running state of this warpgroup
  float m_run, l_thr, acc_ref, acc_res;
  float za[4], zr[NGR1];
  auto reset_state = [&]() {
    m_run = -INFINITY;
    l_thr = acc_ref = acc_res = 0.f;
#pragma unroll
    for (int g = 0; g < 4; ++g) za[g] = 0.f;
#pragma unroll
    for (int g = 0; g < NGR1; ++g) zr[g] = 0.f;
  };

  // A page's value sums are merged at the warpgroup's next page (after its key
  // codes and metadata), so that the value MMAs run behind that work; these
  // hold the pending page's rescale factors (thread = dim position).
  bool pend = false;
  float p_crun = 1.f, p_pm = 0.f, p_fa = 0.f, p_fr = 0.f;

  PageIter it;
  seek(it, x0);
  int k = 0;
  int n_w = 0;  // pages this warpgroup has taken (phase of its per-warpgroup barriers)

  auto merge_pending = [&]() {
    wait_or_abort(&obar[wg], (n_w - 1) & 1);
    tc::fence_after_sync();
    if constexpr (ANCH) {
      uint32_t v[3];
#pragma unroll
      for (int j = 0; j < 3; ++j)
        tc::tmem_ld_n<1>(tl + C::T_OA + j * 4 + chunk, *reinterpret_cast<uint32_t(*)[1]>(&v[j]));
      tc::tmem_wait_ld();
      tc::reg_fence(v);
      acc_ref = fmaf(acc_ref, p_crun, p_pm * p_fa * comb24(v[0], v[1], v[2]));
    }
    if constexpr (RB != 0) {
      // a tensor-memory load takes one address for the whole warp: both
      // parities' columns of 16-dim groups are loaded, then selected per thread
      uint32_t v[C::NPAR][3];
#pragma unroll
      for (int p = 0; p < C::NPAR; ++p)
#pragma unroll
        for (int j = 0; j < 3; ++j)
          tc::tmem_ld_n<1>(tl + C::T_OR + j * NGR + chunk * C::NPAR + p, *reinterpret_cast<uint32_t(*)[1]>(&v[p][j]));
      tc::tmem_wait_ld();
#pragma unroll
      for (int p = 0; p < C::NPAR; ++p) tc::reg_fence(v[p]);
      uint32_t b2 = v[0][0], b1 = v[0][1], b0 = v[0][2];
      if constexpr (C::NPAR == 2) {
        b2 = par_r ? v[1][0] : b2;
        b1 = par_r ? v[1][1] : b1;
        b0 = par_r ? v[1][2] : b0;
      }
      acc_res = fmaf(acc_res, p_crun, p_pm * p_fr * comb24(b2, b1, b0));
    }
    // the value sums are read: the next value MMAs may write them
    tc::fence_before_sync();
    pend = false;
  };
  while (k < n_pages) {
    const int b = it.b, h = it.h;
    const int seg_pages = min(nt_of(b) - it.page, n_pages - k);
    const int len_b = seq_len(b);
    reset_state();
    setup(b, h);

    for (int sp = 0; sp < seg_pages; ++sp, ++k) {
      if ((k & 1) != wg) {  // the other warpgroup's page
        advance(it);
        continue;
      }
      const int s = k % C::STAGES;
      const uint8_t* st = stages + s * C::STAGE_BYTES;
      const uint32_t ph = n_w & 1;
      wait_or_abort(&full[s], (k / C::STAGES) & 1);
      const int n_valid = min(kPP, len_b - it.page * kPP);
      const bool valid = r < n_valid;

      // ---- key codes of token r into this warpgroup's tensor memory (the
      // score MMAs of its previous page have completed: it read their scores)
      if constexpr (ANCH) {
        uint32_t o[32];
        widen_codes<4>(st + C::O_REFK + r * 64, o);
        tc::tmem_st_x32(tl + C::T_KA, o);
      }
      if constexpr (RB != 0) {
        uint32_t o[32];
        widen_codes<RB>(st + C::O_RESK + r * C::CB, o);
        tc::tmem_st_x32(tl + C::T_KR, o);
      }
      tc::tmem_wait_st();
      tc::fence_before_sync();
      __syncwarp();
      if (lane == 0) mbar_arrive(smem_u32(&kready[wg]));

      // ---- per-token metadata, zero past the context
      float aK = 1.f, aV = 1.f;
      if constexpr (C::HAS_ALPHA) {
        const float2 a = half2_bits_to_f2(*reinterpret_cast<const uint32_t*>(st + C::O_AL + r * 4));
        aK = a.x;
        aV = a.y;
      }
      if (!valid) aK = aV = 0.f;
      float sK[NGR1], zK[NGR1], sV[NGR1], zV[NGR1];
      if constexpr (RB != 0) {
#pragma unroll
        for (int g = 0; g < NGR; g += 4) {
          const uint4 mk = *reinterpret_cast<const uint4*>(st + C::O_RESMK + r * C::MB + 4 * g);
          const uint4 mv = *reinterpret_cast<const uint4*>(st + C::O_RESMV + r * C::MB + 4 * g);
          const uint32_t wk[4] = {mk.x, mk.y, mk.z, mk.w}, wv[4] = {mv.x, mv.y, mv.z, mv.w};
#pragma unroll
          for (int u = 0; u < 4; ++u) {
            const float2 a = half2_bits_to_f2(wk[u]), c2 = half2_bits_to_f2(wv[u]);
            sK[g + u] = valid ? a.x : 0.f;
            zK[g + u] = valid ? a.y : 0.f;
            sV[g + u] = valid ? c2.x : 0.f;
            zV[g + u] = valid ? c2.y : 0.f;
          }
        }
      }
      float sAk[4], zAk[4], sAv[4], zAv[4];
      if constexpr (ANCH) {
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
      // ---- the previous page's value sums (its MMAs have run meanwhile)
      if (pend) merge_pending();
      // ---- value codes into this warpgroup's shared tiles (the previous page's
      // value MMAs have completed: its sums are merged); then the stage is free
      if constexpr (ANCH) expand_row<4>(st + C::O_REFV + r * 64, fw + C::F_URV, r);
      if constexpr (RB != 0) expand_row<RB>(st + C::O_RESV + r * C::CB, fw + C::F_UV, r);
      __syncwarp();
      if (lane == 0) mbar_arrive(smem_u32(&empty[s]));

      // ---- scores of token r
      wait_or_abort(&sbar[wg], ph);
      tc::fence_after_sync();
      float S = 0.f;
      {
        // columns 3 g + k: byte plane k of group g (the residual's last four
        // 16-dim groups are read after the first ones are folded)
        uint32_t va[12], vr[12];
        if constexpr (ANCH) tc::tmem_ld_n<12>(tl + C::T_SA, va);
        if constexpr (RB != 0) tc::tmem_ld_n<12>(tl + C::T_SR, vr);
        tc::tmem_wait_ld();
        if constexpr (ANCH) {
          tc::reg_fence(va);
          float dotA = 0.f, offA = 0.f;
#pragma unroll
          for (int g = 0; g < 4; ++g) {
            dotA = fmaf(sAk[g], comb24(va[3 * g], va[3 * g + 1], va[3 * g + 2]), dotA);
            offA = fmaf(zAk[g], q_sc[2 + g], offA);
          }
          S = aK * fmaf(dotA, q_sc[0], offA);
        }
        if constexpr (RB != 0) {
          tc::reg_fence(vr);
          float dotR = 0.f, offR = 0.f;
#pragma unroll
          for (int g = 0; g < 4; ++g) {
            dotR = fmaf(sK[g], comb24(vr[3 * g], vr[3 * g + 1], vr[3 * g + 2]), dotR);
            offR = fmaf(zK[g], q_sc[6 + g], offR);
          }
          if constexpr (NGR == 8) {
            tc::tmem_ld_n<12>(tl + C::T_SR + 12, vr);
            tc::tmem_wait_ld();
            tc::reg_fence(vr);
#pragma unroll
            for (int g = 0; g < 4; ++g) {
              dotR = fmaf(sK[4 + g], comb24(vr[3 * g], vr[3 * g + 1], vr[3 * g + 2]), dotR);
              offR = fmaf(zK[4 + g], q_sc[10 + g], offR);
            }
          }
          S += fmaf(dotR, q_sc[1], offR);
        }
      }
      S = valid ? S : -INFINITY;

      // ---- page maxima of the scores and of the value scales (per group)
      {
        const float v = warp_max(S);
        if (lane == 0) sWM[wg * 4 + chunk] = v;
      }
      if constexpr (RB != 0) {
#pragma unroll
        for (int g = 0; g < NGR; ++g) {
          const float v = warp_max_nonneg(sV[g]);
          if (lane == 0) sSig[(wg * 4 + chunk) * 12 + g] = v;
        }
      }
      if constexpr (ANCH) {
#pragma unroll
        for (int g = 0; g < 4; ++g) {
          const float v = warp_max_nonneg(fabsf(aV * sAv[g]));
          if (lane == 0) sSig[(wg * 4 + chunk) * 12 + 8 + g] = v;
        }
      }
      named_bar_sync(kPpBarWG + wg, 128);
      const float* wm = sWM + wg * 4;
      const float mp = fmaxf(fmaxf(wm[0], wm[1]), fmaxf(wm[2], wm[3]));
      const float mn = fmaxf(m_run, mp);
      const float crun = fast_exp2(m_run - mn);
      const float pm = fast_exp2(mp - mn);
      m_run = mn;
      const float prel = fast_exp2(S - mp);
      float sig[NGR1], siga[4];
      if constexpr (RB != 0) {
#pragma unroll
        for (int g = 0; g < NGR; ++g) {
          const float* sg = sSig + wg * 48 + g;
          sig[g] = fmaxf(fmaxf(sg[0], sg[12]), fmaxf(sg[24], sg[36]));
        }
      }
      if constexpr (ANCH) {
#pragma unroll
        for (int g = 0; g < 4; ++g) {
          const float* sg = sSig + wg * 48 + 8 + g;
          siga[g] = fmaxf(fmaxf(sg[0], sg[12]), fmaxf(sg[24], sg[36]));
        }
      }

      // ---- B operands of the value MMAs: column t = token r
      const int wrow = (r >> 3) * 128 + (r & 7) * 16;  // MN-major core-matrix row of token r
      if constexpr (ANCH) {
        // signed weights (alpha may be negative): three signed bytes each
        uint32_t v[4];
#pragma unroll
        for (int g = 0; g < 4; ++g) {
          const float t = siga[g] > 0.f ? aV * sAv[g] * rcp_approx(siga[g]) * kQ3 : 0.f;
          int qi = __float2int_rn(prel * t);
          qi = max(-8323072, min(8323072, qi));
          int b2, b1, b0;
          split24(qi, b2, b1, b0);
          v[g] = (static_cast<uint32_t>(b0) & 0xFFu) | ((static_cast<uint32_t>(b1) & 0xFFu) << 8) |
                 ((static_cast<uint32_t>(b2) & 0xFFu) << 16);
        }
        uint32_t planes[3][1];
        byte_planes<4>(v, planes);
#pragma unroll
        for (int j = 0; j < 3; ++j) put_plane<4>(fw + C::F_WA, j * 4, wrow, planes[j]);
      }
      if constexpr (RB != 0) {
        // non-negative weights p * s_g / max_page(s_g) as unsigned 24-bit integers
        uint32_t v[NGR];
#pragma unroll
        for (int g = 0; g < NGR; ++g) {
          const float t = sig[g] > 0.f ? sV[g] * rcp_approx(sig[g]) * kU3 : 0.f;
          v[g] = min(__float2uint_rn(prel * t), 16777215u);
        }
        uint32_t planes[3][NGR / 4];
        byte_planes<NGR>(v, planes);
#pragma unroll
        for (int j = 0; j < 3; ++j) put_plane<NGR>(fw + C::F_WR, j * NGR, wrow, planes[j]);
      }
      // the value codes (written above) and the weights are complete
      tc::fence_before_sync();
      fence_proxy_async_smem();
      __syncwarp();
      if (lane == 0) mbar_arrive(smem_u32(&vready[wg]));

      // ---- running denominator and offset sums (thread = token r)
      {
        const float pr = prel * pm;
        l_thr = fmaf(l_thr, crun, pr);
        if constexpr (RB != 0) {
#pragma unroll
          for (int g = 0; g < NGR; ++g) zr[g] = fmaf(zr[g], crun, pr * zV[g]);
        }
        if constexpr (ANCH) {
#pragma unroll
          for (int g = 0; g < 4; ++g) za[g] = fmaf(za[g], crun, pr * aV * zAv[g]);
        }
      }

      // ---- this page's value sums are merged at the next page (or the flush)
      p_crun = crun;
      p_pm = pm;
      if constexpr (ANCH) {
        float sg = siga[0];
#pragma unroll
        for (int g = 1; g < 4; ++g) sg = (chunk == g) ? siga[g] : sg;
        p_fa = sg * (1.f / kQ3);
      }
      if constexpr (RB != 0) {
        float sg = sig[0];
#pragma unroll
        for (int g = 1; g < NGR; ++g) sg = (g_res == g) ? sig[g] : sg;
        p_fr = sg * (1.f / kU3);
      }
      pend = true;
      ++n_w;
      advance(it);
    }

    if (pend) merge_pending();
    // ---- flush this (b, h) segment: both warpgroups' states into their slots,
    // then added in a fixed order into the CTA's partial record
    {
      float* myred = sRed + (wg * 4 + chunk) * 16;
      const float lsum = warp_sum(l_thr);
      if (lane == 0) myred[0] = lsum;
      if constexpr (RB != 0) {
#pragma unroll
        for (int g = 0; g < NGR; ++g) {
          const float z = warp_sum(zr[g]);
          if (lane == 0) myred[1 + g] = z;
        }
      }
      if constexpr (ANCH) {
#pragma unroll
        for (int g = 0; g < 4; ++g) {
          const float z = warp_sum(za[g]);
          if (lane == 0) myred[9 + g] = z;
        }
      }
      named_bar_sync(kPpBarWG + wg, 128);
      auto red = [&](int slot) {
        const float* p = sRed + wg * 4 * 16 + slot;
        return __fadd_rn(__fadd_rn(p[0], p[16]), __fadd_rn(p[32], p[48]));
      };
      float* slot = sSlot + wg * C::SLOT;
      const int d_ref = ANCH ? 32 * chunk + pos_dim<4>(r & 31) : r;
      const int d_res = RB ? 32 * chunk + pos_dim<RB ? RB : 2>(r & 31) : r;
      slot[4 + d_ref] = ANCH ? acc_ref + red(9 + chunk) : 0.f;
      slot[4 + kD + d_res] = RB ? acc_res + red(1 + g_res) : 0.f;
      if (r == 0) {
        slot[0] = m_run;
        slot[1] = red(0);
      }
    }
    named_bar_sync(kPpBarAll, kPpNCT);
    {
      const float m0 = sSlot[0], m1 = sSlot[C::SLOT];
      const float M = fmaxf(m0, m1);
      const float f0 = m0 == -INFINITY ? 0.f : fast_exp2(m0 - M);
      const float f1 = m1 == -INFINITY ? 0.f : fast_exp2(m1 - M);
      const int pair = b * Hkv + h;
      float* rec = P.partials + static_cast<int64_t>(pair + blockIdx.x) * kPartialFloats;
      const int d = tid;  // 256 consumer threads: acc_ref[128], acc_res[128]
      rec[4 + d] = __fmaf_rn(sSlot[C::SLOT + 4 + d], f1, __fmul_rn(sSlot[4 + d], f0));
      if (tid == 0)
        reinterpret_cast<float4*>(rec)[0] =
            make_float4(M, __fmaf_rn(sSlot[C::SLOT + 1], f1, __fmul_rn(sSlot[1], f0)), 0.f, 0.f);
    }
    named_bar_sync(kPpBarAll, kPpNCT);  // the slots are read before either warpgroup writes them again
  }

  // ---- release the tensor memory once every MMA and every consumer is done with it
  tc::fence_before_sync();
  named_bar_sync(kPpBarAll, kPpNCT);
  if (warp == 0) {
    if (!mbar_wait_bounded(smem_u32(done), 0)) set_flag(P.status, RQ_FLAG_PIPE_TIMEOUT);
    tc::fence_after_sync();
    tc::tmem_dealloc(tbase, C::TMEM_COLS);
  }
}

template <int REF, int RB, int RG>
cudaError_t launch_pp(const DecodeParams& p, cudaStream_t s) {
  using C = PpCfg<REF, RB, RG>;
  if constexpr (!C::FITS) {
    return cudaErrorInvalidValue;
  } else {
    auto kern = decode_pp_kernel<REF, RB, RG>;
    static bool attr_done = false;  // per instantiation; set once per process
    if (!attr_done) {
      cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, C::SMEM_BYTES);
      if (e != cudaSuccess) return e;
      attr_done = true;
    }
    return launch_dependent(kern, p.num_ctas, kPpNT, C::SMEM_BYTES, s, p);
  }
}

using PpFn = cudaError_t (*)(const DecodeParams&, cudaStream_t);

template <int REF, int RB, int RG>
PpFn pp_if_fits() {
  if constexpr (PpCfg<REF, RB, RG>::FITS) return launch_pp<REF, RB, RG>;
  else return nullptr;
}

PpFn pp_pick(int ref_kind, int res_bits, int res_group) {
  if (res_bits != 0 && res_group != 16 && res_group != 32) return nullptr;
  const bool g16 = res_group == 16;
  if (ref_kind == kRefInt4) {
    if (res_bits == 0) return pp_if_fits<kRefInt4, 0, 32>();
    // INT2 with 16-dim groups needs more registers than the kernel's 168 a
    // thread: that format's one-row tensor-core decode is decode_tc_kernel's
    if (res_bits == 2) return g16 ? nullptr : pp_if_fits<kRefInt4, 2, 32>();
    if (res_bits == 4) return g16 ? pp_if_fits<kRefInt4, 4, 16>() : pp_if_fits<kRefInt4, 4, 32>();
  } else if (ref_kind == kRefNone) {
    if (res_bits == 2) return g16 ? pp_if_fits<kRefNone, 2, 16>() : pp_if_fits<kRefNone, 2, 32>();
    if (res_bits == 4) return g16 ? pp_if_fits<kRefNone, 4, 16>() : pp_if_fits<kRefNone, 4, 32>();
  }
  return nullptr;
}

}  // namespace

bool pp_variant_supported(int ref_kind, int res_bits, int res_group) {
  return pp_pick(ref_kind, res_bits, res_group) != nullptr;
}

cudaError_t launch_split_pp(const DecodeParams& p, int ref_kind, int res_bits, int res_group, cudaStream_t s) {
  PpFn fn = pp_pick(ref_kind, res_bits, res_group);
  if (fn == nullptr) return cudaErrorInvalidValue;
  return fn(p, s);
}

}  // namespace rq
