// rq_decode_chain.cu -- the CUDA-core split kernel instantiated for the loops
// of the chained reference policies ("ResidualQuant: KV Cache Quantization for
// Looped Transformers with 2-Bit Residuals", Table 9 and Figure 3 caption: the
// Previous-loop and Next-loop reference family).  A loop two or three links
// from its anchor is decoded from the codes of every link:
//     q . x_hat_l = beta_n (q . ref) + sum_i beta_i (H q) . deq(codes of link i)
// with beta_0 = 1 and beta_(i+1) = beta_i alpha_i per token.  The kernel
// evaluates the score by Horner's rule from the anchor outward and gives link
// i's value codes the weight p_t beta_i; all links share one rotated
// accumulator, since they share one format and rotation.  Separate from
// rq_decode.cu so that the two sets of instantiations compile in parallel.
#include "rq_decode_bp.cuh"

namespace rq {
namespace {

template <int REF, int NCH>
SplitFn pick_format(int res_bits, int res_group, int G) {
  if (res_bits == 2) return res_group == 16 ? pick_g<REF, 2, 16, NCH>(G) : pick_g<REF, 2, 32, NCH>(G);
  if (res_bits == 4) return res_group == 16 ? pick_g<REF, 4, 16, NCH>(G) : pick_g<REF, 4, 32, NCH>(G);
  return nullptr;
}

template <int NCH>
SplitFn pick_ref(int ref_kind, int res_bits, int res_group, int G) {
  if (ref_kind == kRefBf16) return pick_format<kRefBf16, NCH>(res_bits, res_group, G);
  if (ref_kind == kRefInt4) return pick_format<kRefInt4, NCH>(res_bits, res_group, G);
  return nullptr;
}

}  // namespace

SplitLaunchFn pick_chain(int ref_kind, int res_bits, int res_group, int G, int n_chain) {
  if (res_group != 16 && res_group != 32) return nullptr;
  if (n_chain == 2) return pick_ref<2>(ref_kind, res_bits, res_group, G);
  if (n_chain == 3) return pick_ref<3>(ref_kind, res_bits, res_group, G);
  return nullptr;
}

}  // namespace rq
