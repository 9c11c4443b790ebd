// rq_decode_tc_chain.cu -- the tensor-core split kernel's instantiations for
// loops of a chained (Previous-/Next-loop) policy with an INT4 anchor: 2 or 3
// residual links, G in {4, 8} where they fit (the kernel: rq_decode_tc.cuh).
// Two rows stay on the CUDA cores: there some of these variants would need more
// than the 224 registers a consumer thread has.
#include "rq_decode_tc.cuh"

namespace rq {
namespace {

template <int RB, int RG, int NCH>
TcFn tc_chain_pick_g(int G) {
  switch (G) {
    case 4: return tc_if_fits<kRefInt4, RB, RG, 4, NCH>();
    case 8: return tc_if_fits<kRefInt4, RB, RG, 8, NCH>();
    default: return nullptr;
  }
}

template <int RB, int RG>
TcFn tc_chain_pick_n(int G, int n_chain) {
  if (n_chain == 2) return tc_chain_pick_g<RB, RG, 2>(G);
  if (n_chain == 3) return tc_chain_pick_g<RB, RG, 3>(G);
  return nullptr;
}

TcFn tc_chain_pick(int ref_kind, int res_bits, int res_group, int G, int n_chain) {
  if (ref_kind != kRefInt4 || (res_group != 16 && res_group != 32)) return nullptr;
  const bool g16 = res_group == 16;
  if (res_bits == 2) return g16 ? tc_chain_pick_n<2, 16>(G, n_chain) : tc_chain_pick_n<2, 32>(G, n_chain);
  if (res_bits == 4) return g16 ? tc_chain_pick_n<4, 16>(G, n_chain) : tc_chain_pick_n<4, 32>(G, n_chain);
  return nullptr;
}

}  // namespace

bool tc_chain_variant_supported(int ref_kind, int res_bits, int res_group, int G, int n_chain) {
  return tc_chain_pick(ref_kind, res_bits, res_group, G, n_chain) != nullptr;
}

cudaError_t launch_split_tc_chain(const DecodeParams& p, int ref_kind, int res_bits, int res_group, int n_chain,
                                  const CUtensorMap* tmap_k, const CUtensorMap* tmap_v, cudaStream_t s) {
  TcFn fn = tc_chain_pick(ref_kind, res_bits, res_group, p.G, n_chain);
  if (fn == nullptr) return cudaErrorInvalidValue;
  return fn(p, tmap_k, tmap_v, s);
}

}  // namespace rq
