// rq_decode_tc.cu -- the tensor-core split kernel's instantiations for loops
// one link from their anchor (and anchor loops), and the tensor-core dispatch.
// The kernel is in rq_decode_tc.cuh; chained loops' instantiations are in
// rq_decode_tc_chain.cu.
#include "rq_decode_tc.cuh"

namespace rq {
namespace {

template <int REF, int RB, int RG>
TcFn tc_pick_g(int G) {
  switch (G) {
    case 1: return tc_if_fits<REF, RB, RG, 1, 1>();
    case 2: return tc_if_fits<REF, RB, RG, 2, 1>();
    case 4: return tc_if_fits<REF, RB, RG, 4, 1>();
    case 8: return tc_if_fits<REF, RB, RG, 8, 1>();
    case 16: return tc_if_fits<REF, RB, RG, 16, 1>();
    default: return nullptr;
  }
}

TcFn tc_pick(int ref_kind, int res_bits, int res_group, int G) {
  if (res_bits != 0 && res_group != 16 && res_group != 32) return nullptr;
  const bool g16 = res_group == 16;
  if (ref_kind == kRefBf16) {
    if (res_bits == 0) return tc_pick_g<kRefBf16, 0, 32>(G);
    if (res_bits == 2) return g16 ? tc_pick_g<kRefBf16, 2, 16>(G) : tc_pick_g<kRefBf16, 2, 32>(G);
    if (res_bits == 4) return g16 ? tc_pick_g<kRefBf16, 4, 16>(G) : tc_pick_g<kRefBf16, 4, 32>(G);
  } else if (ref_kind == kRefInt4) {
    if (res_bits == 0) return tc_pick_g<kRefInt4, 0, 32>(G);
    if (res_bits == 2) return g16 ? tc_pick_g<kRefInt4, 2, 16>(G) : tc_pick_g<kRefInt4, 2, 32>(G);
    if (res_bits == 4) return g16 ? tc_pick_g<kRefInt4, 4, 16>(G) : tc_pick_g<kRefInt4, 4, 32>(G);
  } else if (ref_kind == kRefNone) {
    if (res_bits == 2) return g16 ? tc_pick_g<kRefNone, 2, 16>(G) : tc_pick_g<kRefNone, 2, 32>(G);
    if (res_bits == 4) return g16 ? tc_pick_g<kRefNone, 4, 16>(G) : tc_pick_g<kRefNone, 4, 32>(G);
  }
  return nullptr;
}

}  // namespace

bool tc_variant_supported(int ref_kind, int res_bits, int res_group, int G, int n_chain) {
  if (n_chain > 1) return tc_chain_variant_supported(ref_kind, res_bits, res_group, G, n_chain);
  return tc_pick(ref_kind, res_bits, res_group, G) != nullptr;
}

cudaError_t launch_split_tc(const DecodeParams& p, int ref_kind, int res_bits, int res_group, int n_chain,
                            const CUtensorMap* tmap_k, const CUtensorMap* tmap_v, cudaStream_t s) {
  if (n_chain > 1) return launch_split_tc_chain(p, ref_kind, res_bits, res_group, n_chain, tmap_k, tmap_v, s);
  TcFn fn = tc_pick(ref_kind, res_bits, res_group, p.G);
  if (fn == nullptr) return cudaErrorInvalidValue;
  return fn(p, tmap_k, tmap_v, s);
}

}  // namespace rq
