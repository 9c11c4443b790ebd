// rq_decode_bp.cuh -- the CUDA-core split kernel for the byte-plane formats (an
// INT4 anchor, or no anchor term) at one query row per kv-head.
//
// Same method and the same partial records as decode_split_kernel
// (rq_decode_split.cuh); "ResidualQuant: KV Cache Quantization for Looped
// Transformers with 2-Bit Residuals" stores loop l as alpha * anchor +
// H^T deq(R_l) (abstract, Figure 1, Figure 2 caption), and every cached token
// is scored and summed from that compact form.  These formats move so few
// bytes per token (160-460 B against 612 B with a bf16 anchor) that the
// per-token arithmetic, not HBM, sets the pace; this kernel is organised to
// spend as few instructions per token as it can:
//   * pages of 128 tokens stream into a shared ring exactly as for the other
//     kernel (TMA producer warps -- three, each filling its own stages, or one
//     with three links -- three groups of four consumer warps, a
//     page per group in turn), but each warp owns a 32-token quarter of its
//     group's pages and keeps its own online softmax: no barrier is taken per
//     page, only the stage's release counts the four warps;
//   * scores: four lanes per token, 32 dims per lane, integer dot products on
//     the packed codes (dp4a).  The INT4 anchor's query is carried as a signed
//     24-bit integer in three byte planes (one scale per lane), so that a query
//     with a few large channels keeps the precision of the others; the
//     residual's rotated query H q, whose channels the rotation evens out, as
//     a 16-bit integer in two planes;
//   * per-token weights once: after the warp's page maximum, lane t takes
//     token t -- its softmax weight p, the products of the links' alpha_V,
//     the weight of every (link, group) and the group offsets' sums -- and
//     leaves the weights in shared memory;
//   * values: 16 lanes per token, 8 dims per lane, one AND per code into a
//     subnormal float (code_sub), fp32 pair FMAs;
//   * at the end of a (b, kv-head) segment every warp leaves its state in a
//     slot and the CTA adds the twelve slots in a fixed order into its partial
//     record, so a decode is reproducible bit for bit.
#pragma once

#include "rq_decode_split.cuh"

namespace rq {
namespace {

__device__ __forceinline__ float bp_warp_sum(float v) {
#pragma unroll
  for (int o = 16; o >= 1; o >>= 1) v += __shfl_xor_sync(kFull, v, o);
  return v;
}

template <int REF, int RB, int RG, int NCH, int NG_>
struct BpCfgN {
  static constexpr int TT = 2 * kPage;  // tokens per page (stage)
  static constexpr int NG = NG_;        // consumer groups of kGW warps
  using S = Cfg<REF, RB, RG, 1, TT, NCH, NG>;  // stage layout, record sizes, copy bytes
  static constexpr int NCW = S::NCW, NCT = S::NCT;
  // Three links in three groups hold more than the 128 registers a thread of
  // 416 gets (warps take registers in fours): launched as four warpgroups of
  // 128 registers a thread, the producer's (the producer warp and three idle
  // warps) keeps kSplitRegsAux and the three consumer warpgroups take the rest.
  static constexpr bool REGSPLIT = NCH == 3 && NG == 3;
  static constexpr int REGS_CONSUMER = (512 * 128 - 128 * kSplitRegsAux) / NCT;
  static_assert(!REGSPLIT || (REGS_CONSUMER % 8 == 0 && 128 * kSplitRegsAux + NCT * REGS_CONSUMER == 512 * 128),
                "register split");
  // three producer warps (see the kernel) for up to two links (two measured
  // 1.3% slower on the [2,2,4,4] step, one 7.5%); the three-link variant keeps
  // one (two measured 10% slower there)
  static constexpr int NPROD = NCH <= 2 ? 3 : 1;
  static constexpr int NT = REGSPLIT ? NCT + 128 : NCT + 32 * NPROD;
  static constexpr int TW = TT / kGW;   // tokens of a warp's quarter of a page
  static_assert(TW == 32, "phase 1.5 takes one token per lane");
  static constexpr bool ANCH = REF == kRefInt4;
  static constexpr int NGR = RB ? kD / RG : 0;     // residual groups
  static constexpr int NGW = RB ? NGR : 4;         // weight groups (residual's, or the anchor's)
  static constexpr int P1 = (ANCH ? 1 : 0) + (RB ? NCH : 0);  // weights per (token, weight group)
  static constexpr int P1P = P1 == 3 ? 4 : P1;
  static constexpr int WS = NGW * P1P;
  // floats per token row (a row of 32 words would put every token on the same banks)
  static constexpr int WSTRIDE = (WS % 32 == 0) ? WS + 4 : WS;
  static constexpr int SLOT = 4 + 2 * kD;                       // m, l, -, -, acc_ref[128], acc_res[128]
  // shared memory after the stages, in 4-byte words
  static constexpr int W_W = 0;                                 // [NCW][TW][WSTRIDE]; flush slots alias it
  static constexpr int W_WORDS = NCW * TW * WSTRIDE > NCW * SLOT ? NCW * TW * WSTRIDE : NCW * SLOT;
  static constexpr int W_SC = W_W + W_WORDS;                    // [NCW][TW] scores
  static constexpr int W_QS = W_SC + NCW * TW;                  // [128] q
  static constexpr int W_QT = W_QS + kD;                        // [128] H q
  static constexpr int W_PRE = W_QT + kD;                       // [RQ_MAX_BATCH + 1]
  static constexpr int W_NT = W_PRE + RQ_MAX_BATCH + 1;         // [RQ_MAX_BATCH]
  static constexpr int W_MISC = W_NT + RQ_MAX_BATCH;            // abort flag
  static constexpr int W_BAR = (W_MISC + 2 + 1) & ~1;           // 8-byte aligned mbarriers
  static constexpr int NBARS = 20;                              // full[9], empty[9], -, never
  static constexpr int BAR_NEVER = NBARS - 1;
  static constexpr int MISC_BYTES = 4 * W_BAR + NBARS * 8;
  static constexpr int STAGES_MAX = (S::kSmemLimit - 1024 - MISC_BYTES) / S::STAGE_BYTES;
  // a multiple of NG stages, so that each stage always serves the same group:
  // up to three per group, as many as fit (small records keep more pages in
  // flight per SM)
  static constexpr int PER_GROUP = STAGES_MAX / NG >= 3 ? 3 : (STAGES_MAX / NG >= 2 ? 2 : 1);
  static constexpr int STAGES = NG * PER_GROUP;
  static_assert(2 * 9 < BAR_NEVER + 1, "barrier slots");
  static constexpr bool FITS = STAGES_MAX >= NG;
  static constexpr int SMEM_BYTES = 1024 + STAGES * S::STAGE_BYTES + MISC_BYTES;
  static_assert((W_QS % 4) == 0 && (W_QT % 4) == 0 && (WSTRIDE % P1P) == 0, "alignment");
};

// Three consumer groups where two stages per group fit (six stages), else two
// groups where two stages each fit (a group with a single stage cannot have
// its next page in flight while it works on one), else three groups of one.
template <int REF, int RB, int RG, int NCH>
constexpr int bp_groups() {
  return BpCfgN<REF, RB, RG, NCH, 3>::STAGES_MAX >= 6 ? 3 : (BpCfgN<REF, RB, RG, NCH, 2>::STAGES_MAX >= 4 ? 2 : 3);
}
template <int REF, int RB, int RG, int NCH>
using BpCfg = BpCfgN<REF, RB, RG, NCH, bp_groups<REF, RB, RG, NCH>()>;

template <int REF, int RB, int RG, int NCH>
__global__ void __launch_bounds__(BpCfg<REF, RB, RG, NCH>::NT, 1)
    decode_bp_kernel(const __grid_constant__ DecodeParams P, const __grid_constant__ CUtensorMap tmK,
                     const __grid_constant__ CUtensorMap tmV) {
  using C = BpCfg<REF, RB, RG, NCH>;
  using S = typename C::S;
  constexpr int TT = C::TT, NG = C::NG, NCW = C::NCW, NCT = C::NCT, NT = C::NT, TW = C::TW;
  constexpr bool ANCH = C::ANCH;
  constexpr int NGR = C::NGR;
  constexpr int NGR1 = NGR > 0 ? NGR : 1;
  static_assert(REF != kRefBf16, "byte-plane formats only");
  static_assert(NCH == 1 || (RB != 0 && ANCH), "chains need residual links and an anchor");
  extern __shared__ __align__(16) uint8_t smem_raw[];
  uint8_t* base = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
  uint8_t* stages = base;
  float* mw = reinterpret_cast<float*>(base + C::STAGES * S::STAGE_BYTES);
  float* sW = mw + C::W_W;
  float* sSC = mw + C::W_SC;
  float* sQS = mw + C::W_QS;
  float* sQT = mw + C::W_QT;
  int* sPre = reinterpret_cast<int*>(mw + C::W_PRE);
  int* sNt = reinterpret_cast<int*>(mw + C::W_NT);
  volatile int* sAbort = reinterpret_cast<volatile int*>(mw + C::W_MISC);
  uint64_t* bars = reinterpret_cast<uint64_t*>(mw + C::W_BAR);

  const int tid = threadIdx.x;
  const int lane = tid & 31;
  const int warp = tid >> 5;
  const int B = P.B, Hkv = P.Hkv;
  // a programmatic dependent of the previous kernel: nothing global is
  // touched before it has completed
  pdl_wait();

  // ---- page counts and their prefix over sequences
  for (int b = tid; b < B; b += NT) {
    int len = P.ctx_len[b];
    if (len < 0 || len > P.capacity) {
      if (blockIdx.x == 0) set_flag(P.status, RQ_FLAG_CTX_LEN);
      len = len < 0 ? 0 : P.capacity;
    }
    sNt[b] = (len + TT - 1) / TT;
  }
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
      mbar_init(smem_u32(&bars[s]), 1);                // full: the producer's expect_tx
      mbar_init(smem_u32(&bars[C::STAGES + s]), kGW);  // empty: the page's four warps
    }
    mbar_init(smem_u32(&bars[C::BAR_NEVER]), 1);  // never arrived at: the wait of the stall test hook
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

  // ========================= producer warps =========================
  // NPROD producer threads: producer p fills the stages s with s % NPROD == p,
  // so that a stage is always filled by the same thread.  A page's copy
  // instructions take a producer thread long enough that one thread alone held
  // the consumers back on these small-record formats.
  if (warp >= NCW) {
    if constexpr (C::REGSPLIT) tc::setmaxnreg_dec<kSplitRegsAux>();
    const int pw = warp - NCW;
    if (pw < C::NPROD && lane == 0) {
      PageIter it;
      it.seek(x0, sPre, sNt, B, Hkv);
      int k = 0;
      for (; k < n_pages; ++k) {
        const int s = k % C::STAGES;
        if (s % C::NPROD == pw) {
          if (!mbar_wait_bounded(smem_u32(&bars[C::STAGES + s]), ((k / C::STAGES) & 1) ^ 1)) {
            set_flag(P.status, RQ_FLAG_PIPE_TIMEOUT);
            *sAbort = 1;
            break;
          }
          if (k == P.stall_page && !mbar_wait_bounded(smem_u32(&bars[C::BAR_NEVER]), 0))
            set_flag(P.status, RQ_FLAG_PIPE_TIMEOUT);
          if (*sAbort) break;
          issue_page<REF, RB, RG, 1, TT, NCH, NG>(P, &tmK, &tmV, stages + s * S::STAGE_BYTES, smem_u32(&bars[s]), it,
                                                  Hkv);
        }
        it.next(sNt, B, Hkv);
      }
      // drain: no copy this thread issued may still be landing when it exits
      // (each of its stages' last page: nothing later went into those stages)
      for (int kk = (k > C::STAGES ? k - C::STAGES : 0); kk < k; ++kk) {
        if ((kk % C::STAGES) % C::NPROD != pw) continue;
        if (!mbar_wait_bounded(smem_u32(&bars[kk % C::STAGES]), (kk / C::STAGES) & 1)) {
          set_flag(P.status, RQ_FLAG_PIPE_TIMEOUT);
          break;
        }
      }
    }
    return;
  }
  if constexpr (C::REGSPLIT) tc::setmaxnreg_inc<C::REGS_CONSUMER>();

  // ========================= consumer warps =========================
  const int grp = warp / kGW;   // pages k with k % NG == grp
  const int gw = warp % kGW;    // quarter of the page: tokens [TW gw, TW gw + TW)
  const int j1 = lane & 3;      // phase 1: dims [32 j1, 32 j1 + 32) ...
  const int tq1 = lane >> 2;    // ... of token 8 ps + tq1 of the quarter
  // phase 2: VD value dims per lane, VL lanes per token, TPS tokens per step
  // (16 dims per lane halves the per-token loads but measured slower: 4.81
  // against 5.01 TB/s on the INT4-anchor INT2 loop)
  constexpr int VD = 8;
  constexpr int VL = kD / VD, TPS = 32 / VL;
  const int tph = lane / VL;    // phase 2: token phase ...
  const int j2 = lane % VL;     // ... and dims [VD j2, VD j2 + VD)
  const int gwl = RB ? (VD * j2) / RG : (VD * j2) / 32;  // weight group of the phase-2 lane
  float* wbuf = sW + warp * TW * C::WSTRIDE;
  float* scb = sSC + warp * TW;
  constexpr int NG1 = RB ? (32 >= RG ? 32 / RG : 1) : 1;  // residual groups in a phase-1 lane's dims

  PageIter it;
  it.seek(x0, sPre, sNt, B, Hkv);
  int k = 0;
  while (k < n_pages) {
    const int b = it.b, h = it.h;
    const int seg_pages = min(sNt[b] - it.page, n_pages - k);
    int len_b = P.ctx_len[b];
    len_b = len_b < 0 ? 0 : (len_b > P.capacity ? P.capacity : len_b);

    // ---- segment set-up: the query of (b, h) and its rotation (warp 0)
    if (warp == 0) {
      const uint2 raw = *reinterpret_cast<const uint2*>(P.q + q_row_offset(P, b, h, 0) + 4 * lane);
      const float2 a01 = bf16x2_to_f2(raw.x), a23 = bf16x2_to_f2(raw.y);
      float x[4] = {a01.x, a01.y, a23.x, a23.y};
      *reinterpret_cast<float4*>(&sQS[4 * lane]) = make_float4(x[0], x[1], x[2], x[3]);
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
      *reinterpret_cast<float4*>(&sQT[4 * lane]) = make_float4(x[0], x[1], x[2], x[3]);
    }
    // also orders the previous segment's flush (slots alias the weight buffers)
    named_bar_sync(kConsumerBar, NCT);

    // phase-1 operands of the lane's 32 dims, the softmax scale folded in
    DotOperands24<ANCH ? 32 : 8> oa;
    DotOperands<RB ? RB : 2, RB ? 32 : 1> orr;
    float qsa = 0.f, sca = 0.f, scr = 0.f;
    float qsr[NG1];
    {
      float v[32];
      if constexpr (ANCH) {
#pragma unroll
        for (int e = 0; e < 32; ++e) {
          v[e] = sQS[32 * j1 + e];
          qsa += v[e];
        }
        oa.build(v);
        sca = oa.scale * P.scale_log2;
        qsa *= P.scale_log2;
      }
      if constexpr (RB != 0) {
#pragma unroll
        for (int n = 0; n < NG1; ++n) qsr[n] = 0.f;
#pragma unroll
        for (int e = 0; e < 32; ++e) {
          v[e] = sQT[32 * j1 + e];
          qsr[(32 >= RG) ? e / RG : 0] += v[e];
        }
        orr.build(v);
        scr = orr.scale * P.scale_log2;
#pragma unroll
        for (int n = 0; n < NG1; ++n) qsr[n] *= P.scale_log2;
      }
    }

    // per-warp running state
    float m_run = -INFINITY, l_lane = 0.f;
    float2 acc_a[VD / 2], acc_r[VD / 2];
    float za[4], zr[NGR1];
#pragma unroll
    for (int e = 0; e < VD / 2; ++e) acc_a[e] = acc_r[e] = make_float2(0.f, 0.f);
#pragma unroll
    for (int g = 0; g < 4; ++g) za[g] = 0.f;
#pragma unroll
    for (int g = 0; g < NGR1; ++g) zr[g] = 0.f;

    // this group's pages of the segment: every NG-th, from the first with
    // (k + sp) % NG == grp
    for (int sp = (grp - k % NG + NG) % NG; sp < seg_pages; sp += NG) {
      const int kp = k + sp;  // the CTA's page index
      const int s = kp % C::STAGES;
      const uint8_t* st = stages + s * S::STAGE_BYTES;
      if (!*sAbort) {
        if (!mbar_wait_bounded(smem_u32(&bars[s]), (kp / C::STAGES) & 1)) {
          set_flag(P.status, RQ_FLAG_PIPE_TIMEOUT);
          *sAbort = 1;
        }
      }
      const int t0 = TW * gw;                                   // first stage row of this warp's quarter
      const int nv = min(TT, len_b - (it.page + sp) * TT) - t0;  // its valid tokens (warp-uniform; may be <= 0)
      if (nv > 0) {
        // ---------------- phase 1: scores of the quarter's 32 tokens
        float wmax = -INFINITY;
#pragma unroll
        for (int ps = 0; ps < TW / 8; ++ps) {
          const int tq = 8 * ps + tq1;
          const int t = t0 + tq;
          float part = 0.f;
          if constexpr (ANCH) {
            const uint4 cv = *reinterpret_cast<const uint4*>(st + S::O_REFK + t * 64 + 16 * j1);
            const uint32_t cw[4] = {cv.x, cv.y, cv.z, cv.w};
            int d2 = 0, d1 = 0, d0 = 0;
#pragma unroll
            for (int w = 0; w < 4; ++w)
#pragma unroll
              for (int kk = 0; kk < 2; ++kk) {
                const int x = static_cast<int>(unpack_bytes<4>(cw[w], kk));
                d2 = __dp4a(x, static_cast<int>(oa.b2[w][kk]), d2);
                d1 = __dp4a(x, static_cast<int>(oa.b1[w][kk]), d1);
                d0 = __dp4a(x, static_cast<int>(oa.b0[w][kk]), d0);
              }
            const float2 sz = half2_bits_to_f2(*reinterpret_cast<const uint32_t*>(st + S::O_REFMK + t * 16 + 4 * j1));
            part = fmaf(sz.x * sca, comb24s(d2, d1, d0), sz.y * qsa);
          }
          // links from the anchor outward (Horner): part = alpha_K,i part + res_i
#pragma unroll
          for (int ci = NCH - 1; ci >= 0; --ci) {
            if constexpr (S::HAS_ALPHA) {
              const float aK = __half2float(*reinterpret_cast<const __half*>(st + S::o_al(ci) + t * 4));
              part *= aK;
            }
            if constexpr (RB != 0) {
              using Ops = DotOperands<RB, 32>;
              constexpr int WPG = (RG * RB) / 32 > 0 ? (RG * RB) / 32 : 1;  // code words per group
              uint32_t cw[Ops::NW];
              load_codes<32 * RB / 8>(st + S::o_resk(ci) + t * S::CB + 4 * RB * j1, cw);
              int dhi[NG1];
              unsigned dlo[NG1];
#pragma unroll
              for (int n = 0; n < NG1; ++n) {
                dhi[n] = 0;
                dlo[n] = 0u;
              }
#pragma unroll
              for (int w = 0; w < Ops::NW; ++w) {
                const int n = (NG1 > 1) ? w / WPG : 0;
#pragma unroll
                for (int kk = 0; kk < Ops::KPW; ++kk) {
                  const uint32_t x = unpack_bytes<RB>(cw[w], kk);
                  dhi[n] = __dp4a(static_cast<int>(x), static_cast<int>(orr.hi[w][kk]), dhi[n]);
                  dlo[n] = __dp4a(x, orr.lo[w][kk], dlo[n]);
                }
              }
#pragma unroll
              for (int n = 0; n < NG1; ++n) {
                const float2 sz = half2_bits_to_f2(
                    *reinterpret_cast<const uint32_t*>(st + S::o_resmk(ci) + t * S::MB + 4 * ((32 * j1) / RG + n)));
                const float dot = static_cast<float>(dhi[n] * 256 + static_cast<int>(dlo[n]));
                part += fmaf(sz.x * scr, dot, sz.y * qsr[n]);
              }
            }
          }
          part += __shfl_xor_sync(kFull, part, 1);
          part += __shfl_xor_sync(kFull, part, 2);
          const float sc = (tq < nv) ? part : -INFINITY;
          wmax = fmaxf(wmax, sc);
          if (j1 == 0) scb[tq] = sc;
        }
        // ---------------- online softmax (warp-local)
        const float mp = warp_max(wmax);
        if (mp > m_run) {  // warp-uniform
          const float corr = fast_exp2(m_run - mp);
          const float2 c2 = make_float2(corr, corr);
#pragma unroll
          for (int e = 0; e < VD / 2; ++e) {
            acc_a[e] = __fmul2_rn(acc_a[e], c2);
            acc_r[e] = __fmul2_rn(acc_r[e], c2);
          }
#pragma unroll
          for (int g = 0; g < 4; ++g) za[g] *= corr;
#pragma unroll
          for (int g = 0; g < NGR1; ++g) zr[g] *= corr;
          l_lane *= corr;
          m_run = mp;
        }
        __syncwarp();
        // ---------------- phase 1.5: lane = token; weights and offset sums
        if (lane < nv) {
          const int t = t0 + lane;
          const float p = fast_exp2(scb[lane] - m_run);
          l_lane += p;
          float wl[NCH];  // p times the alpha_V of the links before link i
          float pa = p;   // the anchor's weight: p times every link's alpha_V
#pragma unroll
          for (int ci = 0; ci < NCH; ++ci) {
            wl[ci] = pa;
            if constexpr (S::HAS_ALPHA) pa *= __half2float(*reinterpret_cast<const __half*>(st + S::o_al(ci) + t * 4 + 2));
          }
          float wa[4];
          if constexpr (ANCH) {
            const uint4 mv = *reinterpret_cast<const uint4*>(st + S::O_REFMV + t * 16);
            const uint32_t m4[4] = {mv.x, mv.y, mv.z, mv.w};
            const float pas = pa * kSubScale;  // value weights carry the code scale (code_sub)
#pragma unroll
            for (int g = 0; g < 4; ++g) {
              const float2 sz = half2_bits_to_f2(m4[g]);
              wa[g] = pas * sz.x;
              za[g] = fmaf(pa, sz.y, za[g]);
            }
          }
          float wr[NCH][NGR1];
          if constexpr (RB != 0) {
#pragma unroll
            for (int ci = 0; ci < NCH; ++ci) {
#pragma unroll
              for (int g4 = 0; g4 < NGR; g4 += 4) {
                const uint4 mv = *reinterpret_cast<const uint4*>(st + S::o_resmv(ci) + t * S::MB + 4 * g4);
                const uint32_t m4[4] = {mv.x, mv.y, mv.z, mv.w};
#pragma unroll
                for (int u = 0; u < 4; ++u) {
                  const float2 sz = half2_bits_to_f2(m4[u]);
                  wr[ci][g4 + u] = (wl[ci] * kSubScale) * sz.x;
                  zr[g4 + u] = fmaf(wl[ci], sz.y, zr[g4 + u]);
                }
              }
            }
          }
          // row of token `lane`: per weight group, [anchor, link 0, link 1, ...]
          float* row = wbuf + lane * C::WSTRIDE;
#pragma unroll
          for (int g = 0; g < C::NGW; ++g) {
            float v[4] = {0.f, 0.f, 0.f, 0.f};
            int n = 0;
            if constexpr (ANCH) v[n++] = wa[RB ? (g * RG) / 32 : g];
            if constexpr (RB != 0) {
#pragma unroll
              for (int ci = 0; ci < NCH; ++ci) v[n++] = wr[ci][g];
            }
            if constexpr (C::P1P == 4) *reinterpret_cast<float4*>(row + 4 * g) = make_float4(v[0], v[1], v[2], v[3]);
            else if constexpr (C::P1P == 2) *reinterpret_cast<float2*>(row + 2 * g) = make_float2(v[0], v[1]);
            else row[g] = v[0];
          }
        } else {
          // past the context: zero weights (the stage rows there hold stale
          // records, so none of their metadata is read)
          float* row = wbuf + lane * C::WSTRIDE;
#pragma unroll
          for (int i = 0; i < C::WS; ++i) row[i] = 0.f;
        }
        __syncwarp();
        // ---------------- phase 2: values, TPS tokens per step (token phase `tph`)
        auto value_token = [&](int tq) {
          const int t = t0 + tq;
          const float* wrow = wbuf + tq * C::WSTRIDE + gwl * C::P1P;
          float w[4];
          if constexpr (C::P1P == 4) {
            const float4 x = *reinterpret_cast<const float4*>(wrow);
            w[0] = x.x; w[1] = x.y; w[2] = x.z; w[3] = x.w;
          } else if constexpr (C::P1P == 2) {
            const float2 x = *reinterpret_cast<const float2*>(wrow);
            w[0] = x.x; w[1] = x.y;
          } else {
            w[0] = wrow[0];
          }
          int n = 0;
          if constexpr (ANCH) {
            uint32_t cw[VD / 8];
            load_codes<VD / 2>(st + S::O_REFV + t * 64 + (VD / 2) * j2, cw);
            const float2 ww = make_float2(w[0], w[0]);
#pragma unroll
            for (int e = 0; e < VD; e += 2) {
              const float2 f = make_float2(code_sub<4>(cw, e), code_sub<4>(cw, e + 1));
              acc_a[e / 2] = __ffma2_rn(ww, f, acc_a[e / 2]);
            }
            ++n;
          }
          if constexpr (RB != 0) {
            constexpr int NBV = RB * VD / 8;  // code bytes of the lane's dims
#pragma unroll
            for (int ci = 0; ci < NCH; ++ci) {
              uint32_t cw[NBV >= 4 ? NBV / 4 : 1];
              load_codes<NBV>(st + S::o_resv(ci) + t * S::CB + NBV * j2, cw);
              const float wv = w[n + ci];
              const float2 ww = make_float2(wv, wv);
#pragma unroll
              for (int e = 0; e < VD; e += 2) {
                const float2 f = make_float2(code_sub<RB>(cw, e), code_sub<RB>(cw, e + 1));
                acc_r[e / 2] = __ffma2_rn(ww, f, acc_r[e / 2]);
              }
            }
          }
        };
        if (nv >= TW) {
          // fully unrolled with one link (constant offsets, no loop
          // arithmetic); chained links keep the register budget of unroll 4
          constexpr int UNROLL = NCH == 1 ? TW / TPS : 4;
#pragma unroll UNROLL
          for (int i = 0; i < TW / TPS; ++i) value_token(TPS * i + tph);
        } else {
          // a partial quarter: tokens past the context have zero weights, so
          // only the steps with a valid token are taken
          for (int i = 0; TPS * i < nv; ++i) value_token(TPS * i + tph);
        }
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(smem_u32(&bars[C::STAGES + s]));
    }
    // past the segment: the next (b, h) (the loop ends when the CTA's pages do)
    k += seg_pages;
    it.page += seg_pages - 1;
    it.next(sNt, B, Hkv);

    // ---- flush this (b, h) segment: every warp's state into its slot, then the
    // slots added in a fixed order into the CTA's partial record
    named_bar_sync(kConsumerBar, NCT);  // every warp is past its pages: the weight buffers are free
    {
      float* slot = sW + warp * C::SLOT;
      const float lsum = bp_warp_sum(l_lane);
#pragma unroll
      for (int g = 0; g < 4; ++g) za[g] = bp_warp_sum(za[g]);
#pragma unroll
      for (int g = 0; g < NGR1; ++g) zr[g] = bp_warp_sum(zr[g]);
      float zav = za[0], zrv = zr[0];
#pragma unroll
      for (int g = 1; g < 4; ++g) zav = (VD * j2) / 32 == g ? za[g] : zav;  // the lane's anchor group
#pragma unroll
      for (int g = 1; g < NGR1; ++g) zrv = gwl == g ? zr[g] : zrv;
#pragma unroll
      for (int e = 0; e < VD; ++e) {
        const float2 aa = acc_a[e >> 1], ar = acc_r[e >> 1];
        float va = (e & 1) ? aa.y : aa.x;
        float vr = (e & 1) ? ar.y : ar.x;
#pragma unroll
        for (int o = VL; o < 32; o <<= 1) {  // the token phases, in a fixed order
          va = __fadd_rn(va, __shfl_xor_sync(kFull, va, o));
          vr = __fadd_rn(vr, __shfl_xor_sync(kFull, vr, o));
        }
        if (lane < VL) {
          slot[4 + VD * j2 + e] = ANCH ? fmaf(va, pow2i(kSubExp - code_pos<4>(e)), zav) : 0.f;
          slot[4 + kD + VD * j2 + e] = RB ? fmaf(vr, pow2i(kSubExp - code_pos<RB ? RB : 2>(e)), zrv) : 0.f;
        }
      }
      if (lane == 0) {
        slot[0] = m_run;
        slot[1] = lsum;
      }
    }
    named_bar_sync(kConsumerBar, NCT);
    {
      float M = -INFINITY;
#pragma unroll
      for (int w = 0; w < NCW; ++w) M = fmaxf(M, sW[w * C::SLOT]);
      float f[NCW];
#pragma unroll
      for (int w = 0; w < NCW; ++w) {
        const float mw = sW[w * C::SLOT];
        f[w] = mw == -INFINITY ? 0.f : fast_exp2(mw - M);
      }
      const int pair = b * Hkv + h;
      float* rec = P.partials + static_cast<int64_t>(pair + blockIdx.x) * kPartialFloats;
      for (int d = tid; d < 2 * kD; d += NCT) {
        float acc = 0.f;
#pragma unroll
        for (int w = 0; w < NCW; ++w) acc = __fmaf_rn(sW[w * C::SLOT + 4 + d], f[w], acc);
        rec[4 + d] = acc;
      }
      if (tid == 0) {
        float L = 0.f;
#pragma unroll
        for (int w = 0; w < NCW; ++w) L = __fmaf_rn(sW[w * C::SLOT + 1], f[w], L);
        reinterpret_cast<float4*>(rec)[0] = make_float4(M, L, 0.f, 0.f);
      }
    }
  }
}

template <int REF, int RB, int RG, int NCH>
cudaError_t launch_bp(DecodeParams& p, const CUtensorMap* tk, const CUtensorMap* tv, cudaStream_t s) {
  using C = BpCfg<REF, RB, RG, NCH>;
  auto kern = decode_bp_kernel<REF, RB, RG, NCH>;
  p.page_tokens = C::TT;
  static bool attr_done = false;  // per instantiation; set once per process
  if (!attr_done) {
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, C::SMEM_BYTES);
    if (e != cudaSuccess) return e;
    attr_done = true;
  }
  return launch_dependent(kern, p.num_ctas, C::NT, C::SMEM_BYTES, s, p, *tk, *tv);
}

// The kernel a G = 1 decode of a byte-plane format takes: this one where its
// stages fit, else decode_split_kernel.
template <int REF, int RB, int RG, int NCH>
SplitFn pick_g1() {
  if constexpr (REF != kRefBf16) {
    if constexpr (BpCfg<REF, RB, RG, NCH>::FITS) return launch_bp<REF, RB, RG, NCH>;
    else return launch_split<REF, RB, RG, 1, NCH>;
  } else {
    return launch_split<REF, RB, RG, 1, NCH>;
  }
}

template <int REF, int RB, int RG, int NCH>
SplitFn pick_g(int G) {
  switch (G) {
    case 1: return pick_g1<REF, RB, RG, NCH>();
    case 2: return launch_split<REF, RB, RG, 2, NCH>;
    case 4: return launch_split<REF, RB, RG, 4, NCH>;
    default: return nullptr;  // 8 rows run as two passes of 4 (rq_api.cpp)
  }
}

}  // namespace
}  // namespace rq
