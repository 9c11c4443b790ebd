"""Plant plausible mistakes in the oracle (on the CPU) and check that the pins
in ``test_oracle_pins.py`` catch every one of them."""
import numpy as np
import pytest

import oracle.rq_oracle as O
import tests.test_oracle_pins as P


def _fwht_wrong_sign(x):
    y = np.asarray(x, dtype=np.float32).copy()
    lead = y.shape[:-1]
    h = 1
    while h < 128:
        y = y.reshape(lead + (128 // (2 * h), 2, h))
        a, b = y[..., 0, :], y[..., 1, :]
        y = np.stack([a + b, b - a], axis=-2).reshape(lead + (128,))
        h *= 2
    return (y * O.INV_SQRT_D_F32).astype(np.float32)


def _alpha_swapped(x, ref, mode=O.ALPHA_LS):
    if mode != O.ALPHA_LS:
        return ORIG["ls_alpha_fp32"](x, ref, mode)
    num = O.lane_tree_dot_fp32(ref, ref)
    den = O.lane_tree_dot_fp32(x, ref)
    with np.errstate(all="ignore"):
        return np.where(den == 0, 0, num / np.where(den == 0, 1, den)).astype(np.float16)


def _reconstruct_no_alpha(enc, loop):
    if enc.cfg.is_anchor(loop):
        return ORIG["reconstruct_f64"](enc, loop)
    a = enc.cfg.anchor_of(loop)
    return tuple(O.reference_f64(enc, n, a) + O.residual_f64(enc.loops[loop][n]) for n in ("k", "v"))


def _residual_unnormalised(p):
    y = O.dequant_f64(p.codes, p.scale, p.zero, p.group)
    return y @ O.hadamard_pm1(128) if p.rotate else y


def _quant_floor(y, bits, g):
    q = ORIG["quantize_groups_fp32"](y, bits, g)
    lead = np.asarray(y).shape[:-1]
    yg = np.asarray(y, np.float32).reshape(lead + (128 // g, g))
    sf = q.scale.astype(np.float32)[..., None]
    zf = q.zero.astype(np.float32)[..., None]
    with np.errstate(all="ignore"):
        u = (yg - zf) / np.where(sf > 0, sf, 1)
    c = np.where(sf > 0, np.clip(np.floor(u), 0, (1 << bits) - 1), 0).astype(np.uint8)
    q.codes = c.reshape(lead + (128,))
    return q


def _dequant_strided_groups(codes, scale, zero, g):
    lead = codes.shape[:-1]
    c = codes.reshape(lead + (g, 128 // g)).swapaxes(-1, -2).astype(np.float64)
    v = zero.astype(np.float64)[..., None] + c * scale.astype(np.float64)[..., None]
    return v.swapaxes(-1, -2).reshape(lead + (128,))


def _decode_drop_value_alpha(enc, loop, q, ctx_len, k_tail=None, v_tail=None, scale=1 / np.sqrt(128)):
    if enc.cfg.is_anchor(loop):
        return ORIG["decode_attention_f64"](enc, loop, q, ctx_len, k_tail, v_tail, scale)
    saved = enc.loops[loop]["v"].alpha
    enc.loops[loop]["v"].alpha = np.ones_like(saved)
    try:
        return ORIG["decode_attention_f64"](enc, loop, q, ctx_len, k_tail, v_tail, scale)
    finally:
        enc.loops[loop]["v"].alpha = saved


def _reconstruct_chain_via_anchor(enc, loop):
    cfg = enc.cfg
    if cfg.is_anchor(loop):
        return ORIG["reconstruct_f64"](enc, loop)
    a = cfg.anchor_of(loop)
    return tuple(enc.loops[loop][n].alpha.astype(np.float64)[..., None] * O.reference_f64(enc, n, a)
                 + O.residual_f64(enc.loops[loop][n]) for n in ("k", "v"))


def _chain_view_without_residual(qg, g, rotate, alpha_hat, ref):
    return (np.asarray(alpha_hat).astype(np.float32)[..., None] * np.asarray(ref, np.float32)).astype(np.float32)


def _decode_chain_drops_link_alpha(enc, loop, q, ctx_len, k_tail=None, v_tail=None, scale=1 / np.sqrt(128)):
    deeper = enc.cfg.chain(loop)[1:]
    saved = {c: enc.loops[c]["k"].alpha for c in deeper}
    for c in deeper:
        enc.loops[c]["k"].alpha = np.ones_like(saved[c])
    try:
        return ORIG["decode_attention_f64"](enc, loop, q, ctx_len, k_tail, v_tail, scale)
    finally:
        for c in deeper:
            enc.loops[c]["k"].alpha = saved[c]


def _multi_query_tail_excludes_self(enc, loop, q, ctx_len, k_tail, v_tail, scale=1 / np.sqrt(128)):
    n_q, n_tail = q.shape[1], k_tail.shape[2]
    out = np.zeros(q.shape)
    for i in range(n_q):
        n_vis = n_tail - n_q + i
        out[:, i] = O.decode_attention_f64(enc, loop, q[:, i], ctx_len, k_tail[:, :, :n_vis], v_tail[:, :, :n_vis], scale)
    return out


def _tree_dot_drops_last_lane(a, b):
    prod = (np.asarray(a, np.float32) * np.asarray(b, np.float32)).astype(np.float32)
    return prod[..., :120].sum(-1, dtype=np.float32)


ORIG = {n: getattr(O, n) for n in ("fwht_fp32", "ls_alpha_fp32", "reconstruct_f64", "residual_f64",
                                   "quantize_groups_fp32", "dequant_f64", "decode_attention_f64",
                                   "lane_tree_dot_fp32", "reconstruct_fp32", "decode_attention_multi_f64")}

PINS = [
    P.test_p1_alpha_minimises_squared_error,
    P.test_p1_tree_dot_matches_float64_within_rounding,
    lambda: [P.test_p2_scaled_copy_has_zero_residual(c, r) for c in (2.0, -0.5) for r in (0, 1)],
    lambda: [P.test_p3_alpha_zero_without_rotation_is_plain_group_quantisation(b, g)
             for b, g in ((2, 32), (4, 16))],
    P.test_p4_hadamard_matches_library_and_is_orthogonal,
    P.test_p4_fast_transform_equals_matrix,
    lambda: P.test_p5_quantiser_error_bound(2, 32),
    lambda: [P.test_p6_rotated_domain_decode_equals_brute_force(b, r)
             for b, r in (((2, 16), (1, 0)), ((2, 4), (0, 0)))],
    P.test_p6_two_token_softmax_by_hand,
    P.test_p7_ls_scaling_never_worse_than_unit_scale,
    lambda: [P.test_p8_full_precision_residual_reconstructs(r) for r in (0, 1)],
    lambda: [P.test_chained_scaled_copies_reconstruct_exactly(p, 1) for p in (O.ANCHOR_PREVIOUS, O.ANCHOR_NEXT)],
    lambda: P.test_chained_reconstruction_error_is_the_quantiser_error(O.ANCHOR_NEXT, 16),
    lambda: P.test_chained_decode_equals_brute_force(O.ANCHOR_NEXT, 4),
    P.test_multi_query_decode_equals_masked_brute_force,
    lambda: P.test_encoder_chain_view_is_the_decoders_reconstruction(O.ANCHOR_NEXT, 16, 1),
]


def _any_pin_fails():
    for pin in PINS:
        try:
            pin()
        except AssertionError:
            return True
    return False


@pytest.mark.parametrize("name,mutant", [
    ("fwht_fp32", _fwht_wrong_sign),
    ("ls_alpha_fp32", _alpha_swapped),
    ("reconstruct_f64", _reconstruct_no_alpha),
    ("residual_f64", _residual_unnormalised),
    ("quantize_groups_fp32", _quant_floor),
    ("dequant_f64", _dequant_strided_groups),
    ("decode_attention_f64", _decode_drop_value_alpha),
    ("lane_tree_dot_fp32", _tree_dot_drops_last_lane),
    ("reconstruct_f64", _reconstruct_chain_via_anchor),
    ("reconstruct_fp32", _chain_view_without_residual),
    ("decode_attention_f64", _decode_chain_drops_link_alpha),
    ("decode_attention_multi_f64", _multi_query_tail_excludes_self),
])
def test_planted_mistake_is_caught(monkeypatch, name, mutant):
    monkeypatch.setattr(O, name, mutant)
    assert _any_pin_fails(), f"no pin caught a planted mistake in {name}"


def test_unmutated_oracle_passes_all_pins():
    assert not _any_pin_fails()
