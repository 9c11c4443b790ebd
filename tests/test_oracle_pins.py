"""Pins of the CPU oracle against facts that do not come from the oracle.

Source of the method: "ResidualQuant: KV Cache Quantization for Looped
Transformers with 2-Bit Residuals" (Kim et al., 2026), cited as [RQ].

Each pin is chosen so that a plausible slip in the oracle (a dropped term, a
wrong sign, a transposed operand, an off-by-one group) fails at least one of
them; ``test_oracle_mutations.py`` plants such slips and checks that they do.
"""
import math
import os
from decimal import ROUND_HALF_UP, Decimal

import numpy as np
import pytest
import scipy.linalg

import oracle.rq_oracle as O

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def bf16_values(rng, shape, scale=1.0):
    """float32 arrays whose values are exactly representable in bf16."""
    x = (rng.standard_normal(shape) * scale).astype(np.float32)
    u = x.view(np.uint32)
    # round to nearest even on the 16 dropped bits
    u = ((u + 0x7FFF + ((u >> 16) & 1)) & 0xFFFF0000).astype(np.uint32)
    return u.view(np.float32)


# ---------------------------------------------------------------- P1: alpha

def brute_force_ls_scale(x, r):
    """argmin_a ||x - a r||^2 by a grid scan then golden-section refinement."""
    x = x.astype(np.float64)
    r = r.astype(np.float64)

    def f(a):
        d = x - a * r
        return float(d @ d)

    grid = np.linspace(-4.0, 4.0, 8001)
    vals = np.array([f(a) for a in grid])
    i = int(np.argmin(vals))
    lo, hi = grid[max(i - 1, 0)], grid[min(i + 1, len(grid) - 1)]
    phi = (math.sqrt(5) - 1) / 2
    for _ in range(200):
        a1 = hi - phi * (hi - lo)
        a2 = lo + phi * (hi - lo)
        if f(a1) < f(a2):
            hi = a2
        else:
            lo = a1
    return 0.5 * (lo + hi)


def test_p1_alpha_minimises_squared_error():
    rng = np.random.default_rng(11)
    for _ in range(12):
        ref = bf16_values(rng, (128,), scale=rng.uniform(0.5, 3))
        x = bf16_values(rng, (128,)) * np.float32(0.3) + np.float32(rng.uniform(-2, 2)) * ref
        a_star = brute_force_ls_scale(x, ref)
        a_hat = float(O.ls_alpha_fp32(x, ref))
        # fp16 storage: within half an fp16 ulp (plus fp32 noise) of the minimiser
        ulp16 = float(np.spacing(np.float16(abs(a_star))))
        assert abs(a_hat - a_star) <= 0.5 * ulp16 + 1e-6 * abs(a_star) + 1e-9


def test_p1_tree_dot_matches_float64_within_rounding():
    rng = np.random.default_rng(12)
    a = rng.standard_normal((64, 128)).astype(np.float32)
    b = rng.standard_normal((64, 128)).astype(np.float32)
    got = O.lane_tree_dot_fp32(a, b).astype(np.float64)
    exact = np.einsum("nd,nd->n", a.astype(np.float64), b.astype(np.float64))
    bound = 20 * 2.0 ** -24 * np.einsum("nd,nd->n", np.abs(a), np.abs(b))
    assert np.all(np.abs(got - exact) <= bound)


def test_p1_alpha_modes_and_zero_reference():
    rng = np.random.default_rng(13)
    x = bf16_values(rng, (4, 128))
    ref = bf16_values(rng, (4, 128))
    assert np.all(O.ls_alpha_fp32(x, ref, O.ALPHA_ONE) == 1)
    assert np.all(O.ls_alpha_fp32(x, ref, O.ALPHA_ZERO) == 0)
    assert np.all(O.ls_alpha_fp32(x, np.zeros_like(ref)) == 0)


# ---------------------------------------------------------- P2: zero residual

@pytest.mark.parametrize("c", [1.0, -1.0, 2.0, -2.0, 0.5, -0.5])
@pytest.mark.parametrize("rotate", [0, 1])
def test_p2_scaled_copy_has_zero_residual(c, rotate):
    rng = np.random.default_rng(21)
    B, H, T = 1, 2, 9
    ref = bf16_values(rng, (B, H, T, 128), scale=1.5)
    K = np.stack([np.float32(c) * ref, ref]).astype(np.float32)
    V = np.stack([np.float32(-c) * ref, ref]).astype(np.float32)
    cfg = O.CacheConfig(2, [2, 16], [32, 32], [rotate, 0], [O.ALPHA_LS, O.ALPHA_LS])
    enc = O.encode_fp32emu(K, V, cfg)
    pk = enc.loops[0]["k"]
    assert np.all(pk.alpha.astype(np.float64) == c)
    assert np.all(pk.codes == 0) and np.all(pk.scale == 0) and np.all(pk.zero == 0)
    kh, vh = O.reconstruct_f64(enc, 0)
    assert np.array_equal(kh, K[0].astype(np.float64))
    assert np.array_equal(vh, V[0].astype(np.float64))


# ------------------------------------------------ P3: direct quantisation

def nearest_level_codes(x, scale, zero, bits, g):
    """Textbook rounding: the level z + c*s (c in 0..2^b-1) nearest to x."""
    lead = x.shape[:-1]
    xs = x.reshape(lead + (128 // g, g)).astype(np.float64)
    levels = zero.astype(np.float64)[..., None, None] + \
        np.arange(1 << bits)[None, :] * scale.astype(np.float64)[..., None, None]
    # levels: [..., ng, 1, 2^b]; distances [..., ng, g, 2^b]
    d = np.abs(xs[..., None] - levels)
    return np.argmin(d, axis=-1).reshape(lead + (128,))


@pytest.mark.parametrize("bits,g", [(2, 32), (2, 16), (4, 32), (4, 16)])
def test_p3_alpha_zero_without_rotation_is_plain_group_quantisation(bits, g):
    rng = np.random.default_rng(31 + bits + g)
    B, H, T = 2, 2, 33
    K = bf16_values(rng, (2, B, H, T, 128), scale=2.0)
    V = bf16_values(rng, (2, B, H, T, 128), scale=0.7)
    cfg = O.CacheConfig(2, [bits, 16], [g, 32], [0, 0], [O.ALPHA_ZERO, O.ALPHA_LS])
    enc = O.encode_fp32emu(K, V, cfg)
    for name, X in (("k", K), ("v", V)):
        p = enc.loops[0][name]
        x = X[0]
        assert np.all(p.alpha == 0)
        xs = x.reshape(x.shape[:-1] + (128 // g, g)).astype(np.float64)
        mn, mx = xs.min(-1), xs.max(-1)
        # the stored offset is the fp16 value nearest the group minimum
        assert np.all(np.abs(p.zero.astype(np.float64) - mn) <= 0.5 * np.spacing(np.abs(mn).astype(np.float16)).astype(np.float64))
        # the stored scale is within one fp16 ulp of (max - min) / (2^b - 1)
        s = (mx - mn) / ((1 << bits) - 1)
        assert np.all(np.abs(p.scale.astype(np.float64) - s) <= np.spacing(s.astype(np.float16)).astype(np.float64))
        want = nearest_level_codes(x, p.scale, p.zero, bits, g)
        ok = ~p.near_tie
        assert np.array_equal(p.codes[ok], want[ok])
        # reconstruction is the textbook z + c * s
        kh, vh = O.reconstruct_f64(enc, 0)
        got = kh if name == "k" else vh
        c = p.codes.reshape(x.shape[:-1] + (128 // g, g)).astype(np.float64)
        want_rec = (p.zero.astype(np.float64)[..., None] + c * p.scale.astype(np.float64)[..., None])
        assert np.array_equal(got, want_rec.reshape(x.shape))


# --------------------------------------------------------------- P4: Hadamard

def test_p4_hadamard_matches_library_and_is_orthogonal():
    H = O.hadamard_pm1(128)
    assert np.array_equal(H, scipy.linalg.hadamard(128).astype(np.float64))
    Hi = H.astype(np.int64)
    assert np.array_equal(Hi @ Hi.T, 128 * np.eye(128, dtype=np.int64))
    Hn = O.hadamard_orthonormal(128)
    assert np.allclose(Hn @ Hn, np.eye(128), atol=1e-14)


def test_p4_fast_transform_equals_matrix():
    rng = np.random.default_rng(41)
    x = rng.standard_normal((50, 128)).astype(np.float32)
    got = O.fwht_fp32(x).astype(np.float64)
    want = x.astype(np.float64) @ scipy.linalg.hadamard(128).T / np.sqrt(128.0)
    err = np.abs(got - want).max(axis=1)
    assert np.all(err <= 16 * 2.0 ** -24 * np.abs(x).sum(axis=1) / np.sqrt(128))
    # basis vectors map to columns of H scaled by fl32(1/sqrt(128)) exactly
    eye = np.eye(128, dtype=np.float32)
    cols = O.fwht_fp32(eye)
    assert np.array_equal(cols, (scipy.linalg.hadamard(128).T * np.float32(1 / np.sqrt(128.0))).astype(np.float32))
    assert np.float32(1 / np.sqrt(128.0)).view(np.uint32) == 0x3DB504F3


# --------------------------------------------------------- P5: quantiser bounds

@pytest.mark.parametrize("bits,g", [(2, 32), (2, 16), (4, 32)])
def test_p5_quantiser_error_bound(bits, g):
    rng = np.random.default_rng(51)
    y = (rng.standard_normal((400, 128)) * rng.uniform(0.01, 5, (400, 1))).astype(np.float32)
    q = O.quantize_groups_fp32(y, bits, g)
    qmax = (1 << bits) - 1
    assert q.codes.max() <= qmax
    deq = O.dequant_f64(q.codes, q.scale, q.zero, g)
    ys = y.reshape(400, 128 // g, g).astype(np.float64)
    mn = ys.min(-1)
    s = (ys.max(-1) - mn) / qmax
    sh = q.scale.astype(np.float64)
    zh = q.zero.astype(np.float64)
    bound = 0.5 * sh + qmax * np.abs(sh - s) + np.abs(zh - mn) + 1e-7 * np.abs(ys).max(-1)
    err = np.abs(deq.reshape(ys.shape) - ys).max(-1)
    assert np.all(err <= bound)


# ------------------------------------------------------------- P6: decode

def _small_case(seed, B=2, Hkv=2, G=2, T=23, bits=(2, 16), group=(32, 32), rotate=(1, 0), n_tail=1,
                lens=None):
    rng = np.random.default_rng(seed)
    L = len(bits)
    ref = bf16_values(rng, (B, Hkv, T, 128), scale=1.3)
    K = [bf16_values(rng, (B, Hkv, T, 128), scale=0.2) + np.float32(0.9) * ref for _ in range(L - 1)]
    K = np.stack(K + [ref]).astype(np.float32)
    vref = bf16_values(rng, (B, Hkv, T, 128))
    V = [bf16_values(rng, (B, Hkv, T, 128), scale=0.3) + np.float32(1.1) * vref for _ in range(L - 1)]
    V = np.stack(V + [vref]).astype(np.float32)
    cfg = O.CacheConfig(L, list(bits), list(group), list(rotate), [0] * L)
    enc = O.encode_fp32emu(K, V, cfg)
    q = bf16_values(rng, (B, Hkv * G, 128))
    kt = bf16_values(rng, (B, Hkv, n_tail, 128))
    vt = bf16_values(rng, (B, Hkv, n_tail, 128))
    ctx = np.array(lens if lens is not None else [T] * B)
    return enc, q, ctx, kt, vt


@pytest.mark.parametrize("bits,rotate", [((2, 16), (1, 0)), ((4, 4), (1, 0)), ((2, 4), (0, 0))])
def test_p6_rotated_domain_decode_equals_brute_force(bits, rotate):
    enc, q, ctx, kt, vt = _small_case(61, bits=bits, rotate=rotate, lens=[23, 7])
    for loop in range(2):
        got = O.decode_attention_f64(enc, loop, q, ctx, kt, vt)
        Kh, Vh = O.reconstruct_f64(enc, loop)
        want = O.attention_f64(q, Kh, Vh, ctx, kt, vt)
        assert np.abs(got - want).max() <= 1e-12 * max(1.0, np.abs(want).max())


def test_p6_two_token_softmax_by_hand():
    enc, q, ctx, kt, vt = _small_case(62, B=1, Hkv=1, G=1, T=2, n_tail=0)
    Kh, Vh = O.reconstruct_f64(enc, 0)
    got = O.decode_attention_f64(enc, 0, q, ctx, kt[:, :, :0], vt[:, :, :0])[0, 0]
    tau = 1 / math.sqrt(128)
    s1 = tau * float(np.dot(q[0, 0].astype(np.float64), Kh[0, 0, 0]))
    s2 = tau * float(np.dot(q[0, 0].astype(np.float64), Kh[0, 0, 1]))
    w1 = 1.0 / (1.0 + math.exp(s2 - s1))
    want = w1 * Vh[0, 0, 0] + (1 - w1) * Vh[0, 0, 1]
    assert np.abs(got - want).max() <= 1e-12


def test_p6_empty_context_and_tail_only():
    enc, q, ctx, kt, vt = _small_case(63, lens=[0, 5])
    got = O.decode_attention_f64(enc, 0, q, ctx, kt, vt)
    # sequence 0 attends only to its single tail token: output == that token's value
    G = q.shape[1] // kt.shape[1]
    for qh in range(q.shape[1]):
        assert np.array_equal(got[0, qh], vt[0, qh // G, 0].astype(np.float64))
    none = O.decode_attention_f64(enc, 0, q, np.array([0, 0]), kt[:, :, :0], vt[:, :, :0])
    assert np.all(none == 0)


# ------------------------------------------------------------- P7: LS <= alpha=1

def test_p7_ls_scaling_never_worse_than_unit_scale():
    rng = np.random.default_rng(71)
    ref = bf16_values(rng, (500, 128), scale=1.0)
    x = (np.float32(0.7) * ref + bf16_values(rng, (500, 128), scale=0.3)).astype(np.float32)
    a = O.ls_alpha_fp32(x, ref).astype(np.float64)[:, None]
    e_ls = ((x - a * ref) ** 2).sum(1)
    e_one = ((x - ref) ** 2).sum(1)
    # fp16 storage of alpha can cost at most (0.5 ulp16)^2 * ||ref||^2 over the optimum
    slack = (0.5 * np.spacing(np.abs(a[:, 0]).astype(np.float16)).astype(np.float64)) ** 2 * (ref.astype(np.float64) ** 2).sum(1)
    assert np.all(e_ls <= e_one + slack + 1e-9)
    assert np.mean(e_ls) < 0.8 * np.mean(e_one)


# -------------------------------------------------------- P8: rotation is undone

@pytest.mark.parametrize("rotate", [0, 1])
def test_p8_full_precision_residual_reconstructs(rotate):
    rng = np.random.default_rng(81)
    ref = bf16_values(rng, (64, 128), scale=1.2)
    x = (np.float32(0.95) * ref + bf16_values(rng, (64, 128), scale=0.25)).astype(np.float32)
    a = O.ls_alpha_fp32(x, ref)
    r = (x - (a.astype(np.float32)[:, None] * ref).astype(np.float32)).astype(np.float32)
    y = O.fwht_fp32(r) if rotate else r
    # undo with the float64 machinery that reconstruction uses (no quantisation)
    back = y.astype(np.float64) @ O.hadamard_orthonormal(128) if rotate else y.astype(np.float64)
    xr = a.astype(np.float64)[:, None] * ref.astype(np.float64) + back
    assert np.abs(xr - x).max() <= 1e-6 * np.abs(x).max()


# --------------------------------------------------- P9: bitwidths on the pages

def _parse_blocks(s):
    s = s.strip()
    if "*" in s:
        n, blk = s.split("*", 1)
        blk = [int(v) for v in blk.strip("() ").split(",")]
        return [blk] * int(n)
    return [[int(v) for v in s.split(",")]]


def _round_printed(x, printed):
    places = len(printed.split(".")[1]) if "." in printed else 0
    q = Decimal(1).scaleb(-places)
    return Decimal(repr(x)).quantize(q, rounding=ROUND_HALF_UP)


def _rows(name):
    with open(os.path.join(GOLDEN, name)) as f:
        for line in f:
            line = line.strip()
            if line and not line.startswith("#"):
                yield [c.strip() for c in line.split("|")]


def test_p9_effective_bitwidth_matches_pages():
    n = 0
    for where, mode, blocks, g, hd, printed in _rows("beff_pages.txt"):
        b = O.effective_bitwidth(_parse_blocks(blocks), int(g), head_dim=int(hd),
                                 residual=(mode == "residual"))
        assert _round_printed(b, printed) == Decimal(printed), (where, b, printed)
        n += 1
    assert n == 13


def test_p9_storage_reduction_matches_abstract():
    for printed, blocks, g, hd in _rows("storage_reduction_pages.txt"):
        b = O.effective_bitwidth(_parse_blocks(blocks), int(g), head_dim=int(hd))
        assert _round_printed(100 * (1 - b / 16), printed) == Decimal(printed)


# ------------------------------------------- norm-ratio alpha ([RQ] Table 9)

def test_norm_ratio_alpha_matches_norms():
    rng = np.random.default_rng(91)
    ref = bf16_values(rng, (200, 128), scale=1.3)
    x = bf16_values(rng, (200, 128), scale=0.7)
    a = O.ls_alpha_fp32(x, ref, O.ALPHA_NORM).astype(np.float64)
    want = np.linalg.norm(x.astype(np.float64), axis=1) / np.linalg.norm(ref.astype(np.float64), axis=1)
    assert np.all(np.abs(a - want) <= 0.5 * np.spacing(want.astype(np.float16)).astype(np.float64) + 1e-6 * want)
    # a scaled copy: the ratio is |c| whatever the sign (it is not the LS scale)
    for c in (2.0, -0.5):
        assert np.all(O.ls_alpha_fp32(np.float32(c) * ref, ref, O.ALPHA_NORM).astype(np.float64) == abs(c))
    assert np.all(O.ls_alpha_fp32(x, np.zeros_like(ref), O.ALPHA_NORM) == 0)


# --------------------- anchor policies ([RQ] Table 1 First/Last-loop; Table 8)

def _loops_from(ref, scales, rng):
    return np.stack([np.float32(c) * ref for c in scales]).astype(np.float32)


def test_anchor_of_each_policy():
    cfg = O.CacheConfig(8, [2] * 8, [32] * 8, [1] * 8, [0] * 8, O.ANCHOR_INTERVAL, 4)
    assert [cfg.anchor_of(l) for l in range(8)] == [3, 3, 3, 3, 7, 7, 7, 7]
    assert cfg.anchors() == [3, 7]
    cfg6 = O.CacheConfig(6, [2] * 6, [32] * 6, [1] * 6, [0] * 6, O.ANCHOR_INTERVAL, 4)
    assert [cfg6.anchor_of(l) for l in range(6)] == [3, 3, 3, 3, 5, 5]
    first = O.CacheConfig(4, [16, 2, 2, 2], [32] * 4, [0, 1, 1, 1], [0] * 4, O.ANCHOR_FIRST)
    assert [first.anchor_of(l) for l in range(4)] == [0, 0, 0, 0]
    last = O.CacheConfig(4, [2, 2, 2, 16], [32] * 4, [1, 1, 1, 0], [0] * 4)
    assert [last.anchor_of(l) for l in range(4)] == [3, 3, 3, 3]


def test_interval_of_all_loops_equals_last_loop_policy():
    rng = np.random.default_rng(92)
    ref = bf16_values(rng, (1, 2, 11, 128))
    K = np.stack([bf16_values(rng, (1, 2, 11, 128)) for _ in range(3)] + [ref])
    V = np.stack([bf16_values(rng, (1, 2, 11, 128)) for _ in range(3)] + [ref])
    a = O.encode_fp32emu(K, V, O.CacheConfig(4, [2, 2, 4, 4], [32] * 4, [1, 1, 1, 0], [0] * 4))
    b = O.encode_fp32emu(K, V, O.CacheConfig(4, [2, 2, 4, 4], [32] * 4, [1, 1, 1, 0], [0] * 4, O.ANCHOR_INTERVAL, 4))
    for l in range(3):
        for n in "kv":
            assert np.array_equal(a.loops[l][n].codes, b.loops[l][n].codes)
            assert np.array_equal(a.loops[l][n].alpha, b.loops[l][n].alpha)


@pytest.mark.parametrize("policy,interval", [(O.ANCHOR_FIRST, 0), (O.ANCHOR_INTERVAL, 3)])
def test_scaled_copies_of_their_anchor_have_zero_residual(policy, interval):
    rng = np.random.default_rng(93)
    L = 6
    cfg = O.CacheConfig(L, [2] * L, [32] * L, [1] * L, [0] * L, policy, interval)
    bits = list(cfg.bits)
    for l in range(L):
        if cfg.is_anchor(l):
            bits[l] = 16
            cfg.rotate[l] = 0
    cfg.bits = bits
    base = {a: bf16_values(rng, (1, 1, 7, 128)) for a in cfg.anchors()}
    scales = [1.0, -2.0, 0.5, 2.0, -1.0, 0.5]
    K = np.stack([np.float32(scales[l]) * base[cfg.anchor_of(l)] if not cfg.is_anchor(l) else base[l]
                  for l in range(L)]).astype(np.float32)
    enc = O.encode_fp32emu(K, K.copy(), cfg)
    for l in range(L):
        kh, _ = O.reconstruct_f64(enc, l)
        assert np.array_equal(kh, K[l].astype(np.float64))
        if not cfg.is_anchor(l):
            assert np.all(enc.loops[l]["k"].codes == 0)
            assert np.all(enc.loops[l]["k"].alpha.astype(np.float64) == scales[l])


def test_anchor_interval_decode_equals_brute_force():
    rng = np.random.default_rng(94)
    L, B, H, T = 8, 2, 2, 19
    cfg = O.CacheConfig(L, [2, 2, 2, 4, 2, 4, 2, 16], [32, 16, 32, 32, 32, 32, 16, 32],
                        [1, 1, 0, 0, 1, 0, 1, 0], [0, 3, 0, 0, 1, 0, 0, 0], O.ANCHOR_INTERVAL, 4)
    K = np.stack([bf16_values(rng, (B, H, T, 128)) for _ in range(L)])
    V = np.stack([bf16_values(rng, (B, H, T, 128)) for _ in range(L)])
    enc = O.encode_fp32emu(K, V, cfg)
    q = bf16_values(rng, (B, 2 * H, 128))
    kt, vt = bf16_values(rng, (B, H, 1, 128)), bf16_values(rng, (B, H, 1, 128))
    ctx = np.array([19, 4])
    for loop in range(L):
        got = O.decode_attention_f64(enc, loop, q, ctx, kt, vt)
        Kh, Vh = O.reconstruct_f64(enc, loop)
        want = O.attention_f64(q, Kh, Vh, ctx, kt, vt)
        assert np.abs(got - want).max() <= 1e-12 * max(1.0, np.abs(want).max())


# ------------------------------------------- chained references (Previous-/Next-loop)
# [RQ] Table 9 ("Previous-loop", "Next-loop" rows) and Figure 3 caption (the
# Previous-/Next-loop reference family): each loop is stored against its
# neighbour, so a loop is reconstructed through the chain down to the anchor.

def test_ref_of_chain_policies():
    prev = O.CacheConfig(4, [4, 2, 2, 2], [32] * 4, [0, 1, 1, 1], [0] * 4, O.ANCHOR_PREVIOUS)
    assert [prev.ref_of(l) for l in range(4)] == [0, 0, 1, 2]
    assert [prev.anchor_of(l) for l in range(4)] == [0, 0, 0, 0]
    assert [prev.chain(l) for l in range(4)] == [[], [1], [2, 1], [3, 2, 1]]
    nxt = O.CacheConfig(4, [2, 2, 2, 4], [32] * 4, [1, 1, 1, 0], [0] * 4, O.ANCHOR_NEXT)
    assert [nxt.ref_of(l) for l in range(4)] == [1, 2, 3, 3]
    assert [nxt.anchor_of(l) for l in range(4)] == [3, 3, 3, 3]
    assert [nxt.chain(l) for l in range(4)] == [[0, 1, 2], [1, 2], [2], []]
    assert nxt.anchors() == [3] and prev.anchors() == [0]


@pytest.mark.parametrize("policy", [O.ANCHOR_PREVIOUS, O.ANCHOR_NEXT])
@pytest.mark.parametrize("rotate", [0, 1])
def test_chained_scaled_copies_reconstruct_exactly(policy, rotate):
    """Each loop an exact power-of-two multiple of its neighbour: every alpha is
    that factor, every residual and code is zero, and the reconstruction through
    the chain gives back the loops exactly (products of powers of two are exact)."""
    rng = np.random.default_rng(95)
    L = 4
    anchor = 0 if policy == O.ANCHOR_PREVIOUS else L - 1
    bits = [2] * L
    bits[anchor] = 16
    rot = [rotate] * L
    rot[anchor] = 0
    cfg = O.CacheConfig(L, bits, [32] * L, rot, [0] * L, policy)
    factor = {0: 2.0, 1: -0.5, 2: -2.0, 3: 0.5}
    X = [None] * L
    X[anchor] = bf16_values(rng, (1, 2, 9, 128))
    for l in sorted(range(L), key=lambda l: len(cfg.chain(l))):
        if l != anchor:
            X[l] = (np.float32(factor[l]) * X[cfg.ref_of(l)]).astype(np.float32)
    K = np.stack(X)
    enc = O.encode_fp32emu(K, -K, cfg)
    for l in range(L):
        kh, vh = O.reconstruct_f64(enc, l)
        assert np.array_equal(kh, K[l].astype(np.float64))
        assert np.array_equal(vh, -K[l].astype(np.float64))
        if l != anchor:
            assert np.all(enc.loops[l]["k"].codes == 0)
            assert np.all(enc.loops[l]["k"].alpha.astype(np.float64) == factor[l])


def _neighbour_chain_loops(rng, cfg, shape, noise=0.25):
    """Loops that each resemble their reference: x_l = a_l x_ref(l) + noise."""
    L = cfg.num_loops
    X = [None] * L
    for l in sorted(range(L), key=lambda l: len(cfg.chain(l))):
        if cfg.is_anchor(l):
            X[l] = bf16_values(rng, shape)
        else:
            x = (np.float32(rng.uniform(0.8, 1.2)) * X[cfg.ref_of(l)]
                 + np.float32(noise) * rng.standard_normal(shape).astype(np.float32))
            u = x.astype(np.float32).view(np.uint32)  # round to bf16, nearest even
            X[l] = ((u + 0x7FFF + ((u >> 16) & 1)) & 0xFFFF0000).astype(np.uint32).view(np.float32)
    return np.stack(X)


@pytest.mark.parametrize("policy,anchor_bits", [(O.ANCHOR_NEXT, 16), (O.ANCHOR_NEXT, 4), (O.ANCHOR_PREVIOUS, 4)])
def test_chained_reconstruction_error_is_the_quantiser_error(policy, anchor_bits):
    """In the rotated domain the chained reconstruction differs from the input
    loop only by the quantiser: H (x_hat_l - x_l) = deq - H (x_l - alpha x_hat_ref)
    with x_hat_ref the reconstruction of the reference, so every coordinate obeys
    the min-max quantiser's bound.  A residual taken against anything but the
    reconstructed reference breaks the bound at depth >= 2."""
    rng = np.random.default_rng(96)
    L = 4
    anchor = 0 if policy == O.ANCHOR_PREVIOUS else L - 1
    bits, group = [2] * L, [32] * L
    bits[anchor] = anchor_bits
    group[1] = 16
    rot = [1] * L
    rot[anchor] = 0
    cfg = O.CacheConfig(L, bits, group, rot, [0] * L, policy)
    K = _neighbour_chain_loops(rng, cfg, (2, 2, 40, 128))
    V = _neighbour_chain_loops(rng, cfg, (2, 2, 40, 128))
    enc = O.encode_fp32emu(K, V, cfg)
    Hn = scipy.linalg.hadamard(128) / np.sqrt(128.0)
    for l in range(L):
        if cfg.is_anchor(l):
            continue
        refs = O.reconstruct_f64(enc, cfg.ref_of(l))
        hats = O.reconstruct_f64(enc, l)
        for name, X, ref, hat in (("k", K, refs[0], hats[0]), ("v", V, refs[1], hats[1])):
            p = enc.loops[l][name]
            x = X[l].astype(np.float64)
            y = (x - p.alpha.astype(np.float64)[..., None] * ref)
            if p.rotate:
                y = y @ Hn
            g, qmax = p.group, (1 << p.bits) - 1
            ys = y.reshape(y.shape[:-1] + (128 // g, g))
            mn = ys.min(-1)
            s = (ys.max(-1) - mn) / qmax
            sh, zh = p.scale.astype(np.float64), p.zero.astype(np.float64)
            bound = 0.5 * sh + qmax * np.abs(sh - s) + np.abs(zh - mn) + 1e-5 * np.abs(x).max(-1)[..., None]
            err = hat - x
            if p.rotate:
                err = err @ Hn
            err = np.abs(err.reshape(ys.shape)).max(-1)
            assert np.all(err <= bound), (l, name)


@pytest.mark.parametrize("policy", [O.ANCHOR_PREVIOUS, O.ANCHOR_NEXT])
@pytest.mark.parametrize("anchor_bits", [16, 4])
def test_chained_decode_equals_brute_force(policy, anchor_bits):
    rng = np.random.default_rng(97)
    L, B, H, T = 5, 2, 2, 17
    anchor = 0 if policy == O.ANCHOR_PREVIOUS else L - 1
    bits, group = [2, 4, 2, 2, 4], [32, 32, 16, 32, 16]
    rot, modes = [1, 0, 1, 1, 1], [0, 3, 1, 0, 0]
    bits[anchor], group[anchor], rot[anchor] = anchor_bits, 32, 0
    cfg = O.CacheConfig(L, bits, group, rot, modes, policy)
    K = _neighbour_chain_loops(rng, cfg, (B, H, T, 128))
    V = _neighbour_chain_loops(rng, cfg, (B, H, T, 128))
    enc = O.encode_fp32emu(K, V, cfg)
    q = bf16_values(rng, (B, 2 * H, 128))
    kt, vt = bf16_values(rng, (B, H, 2, 128)), bf16_values(rng, (B, H, 2, 128))
    ctx = np.array([17, 5])
    for loop in range(L):
        got = O.decode_attention_f64(enc, loop, q, ctx, kt, vt)
        Kh, Vh = O.reconstruct_f64(enc, loop)
        want = O.attention_f64(q, Kh, Vh, ctx, kt, vt)
        assert np.abs(got - want).max() <= 1e-12 * max(1.0, np.abs(want).max())


def test_chain_of_one_link_equals_star_policies():
    """With two loops the Next-loop chain is the Last-loop policy and the
    Previous-loop chain the First-loop policy; with four loops the loop next to
    the anchor is stored identically under both families."""
    rng = np.random.default_rng(98)
    K = np.stack([bf16_values(rng, (1, 2, 13, 128)) for _ in range(4)])
    V = np.stack([bf16_values(rng, (1, 2, 13, 128)) for _ in range(4)])
    for star, chain, L, loop in ((O.ANCHOR_LAST, O.ANCHOR_NEXT, 2, 0), (O.ANCHOR_FIRST, O.ANCHOR_PREVIOUS, 2, 1),
                                 (O.ANCHOR_LAST, O.ANCHOR_NEXT, 4, 2), (O.ANCHOR_FIRST, O.ANCHOR_PREVIOUS, 4, 1)):
        anchor = L - 1 if star == O.ANCHOR_LAST else 0
        bits = [2] * L
        bits[anchor] = 16
        rot = [1] * L
        rot[anchor] = 0
        a = O.encode_fp32emu(K[:L], V[:L], O.CacheConfig(L, bits, [32] * L, rot, [0] * L, star))
        b = O.encode_fp32emu(K[:L], V[:L], O.CacheConfig(L, bits, [32] * L, rot, [0] * L, chain))
        for n in "kv":
            assert np.array_equal(a.loops[loop][n].codes, b.loops[loop][n].codes)
            assert np.array_equal(a.loops[loop][n].alpha, b.loops[loop][n].alpha)
            assert np.array_equal(a.loops[loop][n].scale, b.loops[loop][n].scale)


# ----------------------------------------------- multi-query (draft token) decode

def test_multi_query_decode_equals_masked_brute_force():
    """Each draft token's row equals softmax attention over the reconstructed
    cache and the whole tail under an explicit causal mask (tail token j is
    visible to draft token i iff j <= n_tail - n_q + i), built here as one score
    matrix instead of the oracle's truncated tails."""
    rng = np.random.default_rng(99)
    B, H, G, T, n_q, n_tail = 2, 2, 2, 21, 3, 5
    cfg = O.CacheConfig(4, [2, 2, 4, 16], [32, 16, 32, 32], [1, 1, 0, 0], [0, 3, 0, 0])
    K = np.stack([bf16_values(rng, (B, H, T, 128)) for _ in range(4)])
    V = np.stack([bf16_values(rng, (B, H, T, 128)) for _ in range(4)])
    enc = O.encode_fp32emu(K, V, cfg)
    q = bf16_values(rng, (B, n_q, G * H, 128))
    kt, vt = bf16_values(rng, (B, H, n_tail, 128)), bf16_values(rng, (B, H, n_tail, 128))
    ctx = np.array([21, 6])
    scale = 1 / np.sqrt(128)
    for loop in (0, 3):
        got = O.decode_attention_multi_f64(enc, loop, q, ctx, kt, vt)
        Kh, Vh = O.reconstruct_f64(enc, loop)
        for b in range(B):
            n = int(ctx[b])
            for qh in range(G * H):
                h = qh // G
                Kall = np.concatenate([Kh[b, h, :n], kt[b, h].astype(np.float64)])
                Vall = np.concatenate([Vh[b, h, :n], vt[b, h].astype(np.float64)])
                S = scale * (q[b, :, qh].astype(np.float64) @ Kall.T)          # [n_q, n + n_tail]
                visible = np.arange(n + n_tail)[None, :] <= (n + n_tail - n_q + np.arange(n_q))[:, None]
                S = np.where(visible, S, -np.inf)
                P_ = np.exp(S - S.max(1, keepdims=True))
                want = (P_ @ Vall) / P_.sum(1, keepdims=True)
                assert np.abs(got[b, :, qh] - want).max() <= 1e-12 * max(1.0, np.abs(want).max())


@pytest.mark.parametrize("policy,anchor_bits,rotate", [(O.ANCHOR_NEXT, 16, 1), (O.ANCHOR_PREVIOUS, 4, 1),
                                                       (O.ANCHOR_NEXT, 4, 0)])
def test_encoder_chain_view_is_the_decoders_reconstruction(policy, anchor_bits, rotate):
    """The binary32 view the encoder keeps of a chained reference equals the
    float64 reconstruction a decoder forms from the stored codes, up to binary32
    rounding: the two are written independently (fast transform in binary32
    against an explicit matrix in float64)."""
    rng = np.random.default_rng(100)
    L = 4
    anchor = 0 if policy == O.ANCHOR_PREVIOUS else L - 1
    bits = [2] * L
    bits[anchor] = anchor_bits
    rot = [rotate] * L
    rot[anchor] = 0
    cfg = O.CacheConfig(L, bits, [32] * L, rot, [0, 3, 0, 0], policy)
    K = _neighbour_chain_loops(rng, cfg, (2, 2, 30, 128))
    V = _neighbour_chain_loops(rng, cfg, (2, 2, 30, 128))
    enc = O.encode_fp32emu(K, V, cfg)
    for l in range(L):
        if cfg.is_anchor(l) or l not in enc.hat32:
            continue
        kh, vh = O.reconstruct_f64(enc, l)
        for view, ref in ((enc.hat32[l]["k"], kh), (enc.hat32[l]["v"], vh)):
            scale = np.abs(ref).max(-1, keepdims=True) + 1e-30
            assert np.abs(view.astype(np.float64) - ref).max() <= 2e-6 * scale.max()
