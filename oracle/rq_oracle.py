"""CPU oracle for the ResidualQuant hot path -- TEST INFRASTRUCTURE ONLY.

Only ``tests/``, ``__graft_entry__.smoke()`` and the CPU-baseline / reference
arm of ``bench.py`` may import this module.  The product path (the CUDA
library and its Python binding) never imports it, and this module imports
nothing from the product path: the two share no code, constant or table.

What it computes follows "ResidualQuant: KV Cache Quantization for Looped
Transformers with 2-Bit Residuals" (Kim et al., 2026), cited below as [RQ]:

* abstract: the final loop's KV states are the reference; the other loops are
  stored as low-precision residuals, with least-squares scaling, rotations
  applied to the residuals and loop-wise mixed precision;
* Figure 1, steps (1)-(5): direct INT2 quantisation, Last-loop residual,
  least-square scaling, rotation, mixed precision;
* Figure 2 caption: the residual ``K_2 - alpha_2 K_1``;
* Figure 3 caption: "alpha = 1" is the no-LS ablation;
* Table 5 caption: INT2 group size 16/32, INT4 group size 32;
* Table 8 caption: the effective bitwidth counts quantised values, scales,
  offsets and LS coefficients.

The pages print no equations, so the encoder's arithmetic is fixed by a written
specification that this module follows step for step (all in IEEE binary32
with round-to-nearest-even, each operation rounded separately):

  alpha  (per vector of 128, separately for K and V)
      lane j (0..15) owns elements 8j..8j+7; p_j = +0, then p_j += x_e * r_e
      for e in order; then p_j += p_{j xor o} for o = 8, 4, 2, 1;
      alpha = num / den (den == 0 -> 0), stored as fp16 (RNE).
      alpha mode "one" stores 1, mode "zero" stores 0.
  residual  r_e = x_e - (alpha_hat * ref_e)
  rotation  (if enabled) unnormalised fast Walsh-Hadamard transform, strides
      h = 1, 2, ..., 64, butterfly (a, b) -> (a + b, a - b) with a the lower
      index; then each element times fl32(1/sqrt(128)).  The rotation is the
      orthonormal Sylvester Hadamard matrix (the pages' OptR-H is not defined
      on them; this build uses the plain Hadamard it is built on).
  quantiser per group of g contiguous (rotated) coordinates, b bits:
      mn = min + 0, mx = max + 0 (the "+ 0" makes a zero unsigned),
      s = (mx - mn) / (2^b - 1); s_hat = fp16(s); z_hat = fp16(mn);
      code = clamp(rint((y - z_hat) / s_hat), 0, 2^b - 1), code = 0 if s_hat == 0.
  INT4 anchor: the reference loop is group-quantised directly (4 bits, g = 32,
      no alpha, no rotation); the other loops take their alpha and residual
      against its dequantised value  ref_hat = z_hat + (code * s_hat)  (fp32).
  Chained references ([RQ] Table 9 and Figure 3 caption: the "Previous-loop"
      and "Next-loop" reference families): loop l's reference is loop l-1
      (Previous) or l+1 (Next), and the chain ends at loop 0 or L-1, the anchor.
      A loop that is the reference of another is seen by the encoder as its
      binary32 reconstruction  x_hat = (alpha_hat * ref_hat) + u  with
      u = the rotation of deq (the rotation is its own inverse), deq = z_hat +
      (code * s_hat); alpha and the residual of the next loop are taken against
      that x_hat, since it is all a decoder has.

Reconstruction and decode attention are computed in float64 from the stored
codes and metadata.  The rotation there is an explicit 128x128 matrix built
from its definition, not a fast transform.

Every function here is pinned by ``tests/test_oracle_pins.py`` against facts
that do not come from this module (closed forms, brute force, a library
Hadamard, the bitwidths printed on the pages).  Parity unpinned: none of the
functions below; the pages' accuracy and NMSE tables need model weights and
are out of scope.
"""
from __future__ import annotations

from dataclasses import dataclass, field
from typing import Dict, List, Optional, Sequence

import numpy as np

D = 128
F32 = np.float32
F16 = np.float16
INV_SQRT_D_F32 = np.float32(1.0 / np.sqrt(128.0))
FP16_MAX = 65504.0

ALPHA_LS, ALPHA_ONE, ALPHA_ZERO, ALPHA_NORM = 0, 1, 2, 3
ANCHOR_LAST, ANCHOR_FIRST, ANCHOR_INTERVAL, ANCHOR_PREVIOUS, ANCHOR_NEXT = 0, 1, 2, 3, 4


# ---------------------------------------------------------------------------
# Rotation
# ---------------------------------------------------------------------------

def hadamard_pm1(n: int = D) -> np.ndarray:
    """Sylvester Hadamard matrix with entries (-1)^popcount(i & j), float64."""
    i = np.arange(n)[:, None]
    j = np.arange(n)[None, :]
    x = np.bitwise_and(i, j)
    parity = np.zeros_like(x)
    while np.any(x):
        parity ^= x & 1
        x = x >> 1
    return np.where(parity == 0, 1.0, -1.0)


def hadamard_orthonormal(n: int = D) -> np.ndarray:
    """H / sqrt(n): orthonormal and symmetric, so it is its own inverse."""
    return hadamard_pm1(n) / np.sqrt(float(n))


def fwht_fp32(x: np.ndarray) -> np.ndarray:
    """The encoder's rotation in binary32: butterflies at strides 1..64, then
    the fl32(1/sqrt(128)) scale.  ``x``: float32 [..., 128]."""
    y = np.asarray(x, dtype=F32).copy()
    lead = y.shape[:-1]
    h = 1
    while h < D:
        y = y.reshape(lead + (D // (2 * h), 2, h))
        a = y[..., 0, :]
        b = y[..., 1, :]
        y = np.stack([a + b, a - b], axis=-2).reshape(lead + (D,))
        h *= 2
    return (y * INV_SQRT_D_F32).astype(F32)


# ---------------------------------------------------------------------------
# Least-squares scale ([RQ] Figure 1 step (3); Figure 2 caption)
# ---------------------------------------------------------------------------

def lane_tree_dot_fp32(a: np.ndarray, b: np.ndarray) -> np.ndarray:
    """<a, b> over the last axis (128) in the specified binary32 order."""
    prod = (np.asarray(a, F32) * np.asarray(b, F32)).astype(F32)
    prod = prod.reshape(prod.shape[:-1] + (16, 8))
    p = np.zeros(prod.shape[:-1], dtype=F32)
    for e in range(8):
        p = (p + prod[..., e]).astype(F32)
    lane = np.arange(16)
    for o in (8, 4, 2, 1):
        p = (p + p[..., lane ^ o]).astype(F32)
    return p[..., 0]


def ls_alpha_fp32(x: np.ndarray, ref: np.ndarray, mode: int = ALPHA_LS) -> np.ndarray:
    """Stored (fp16) scale alpha_hat per vector; x, ref float32 [..., 128].

    LS mode: alpha = <x, ref> / <ref, ref>, the minimiser of ||x - a ref||^2
    ([RQ] Figure 1 step 3).  Norm-ratio mode ([RQ] Table 9, "Norm-ratio"):
    alpha = ||x|| / ||ref||, each norm the correctly rounded square root of
    the same fixed-order dot product.
    """
    lead = np.asarray(x).shape[:-1]
    if mode == ALPHA_ONE:
        return np.ones(lead, dtype=F16)
    if mode == ALPHA_ZERO:
        return np.zeros(lead, dtype=F16)
    if mode == ALPHA_NORM:
        nx = np.sqrt(lane_tree_dot_fp32(x, x)).astype(F32)
        nr = np.sqrt(lane_tree_dot_fp32(ref, ref)).astype(F32)
        with np.errstate(divide="ignore", invalid="ignore", over="ignore"):
            alpha = np.where(nr == 0, F32(0), nx / np.where(nr == 0, F32(1), nr)).astype(F32)
            return alpha.astype(F16)
    num = lane_tree_dot_fp32(x, ref)
    den = lane_tree_dot_fp32(ref, ref)
    with np.errstate(divide="ignore", invalid="ignore", over="ignore"):
        alpha = np.where(den == 0, F32(0), num / np.where(den == 0, F32(1), den)).astype(F32)
        return alpha.astype(F16)


# ---------------------------------------------------------------------------
# Asymmetric group quantiser ([RQ] Table 5 caption: INT2 g = 16/32, INT4 g = 32;
# Table 8 caption: scales and offsets per group)
# ---------------------------------------------------------------------------

@dataclass
class QuantGroups:
    codes: np.ndarray      # uint8 [..., 128]
    scale: np.ndarray      # float16 [..., 128 // g]
    zero: np.ndarray       # float16 [..., 128 // g]
    near_tie: np.ndarray   # bool [..., 128]: within 1 fp32 ulp of a rounding midpoint


def quantize_groups_fp32(y: np.ndarray, bits: int, g: int) -> QuantGroups:
    """Min-max asymmetric quantiser of float32 ``y`` [..., 128] in groups of g."""
    y = np.asarray(y, dtype=F32)
    lead = y.shape[:-1]
    ng = D // g
    yg = y.reshape(lead + (ng, g))
    qmax = F32((1 << bits) - 1)
    mn = (yg.min(axis=-1) + F32(0)).astype(F32)
    mx = (yg.max(axis=-1) + F32(0)).astype(F32)
    with np.errstate(over="ignore", invalid="ignore", divide="ignore"):
        s = ((mx - mn).astype(F32) / qmax).astype(F32)
        s_hat = s.astype(F16)
        z_hat = mn.astype(F16)
        sf = s_hat.astype(F32)[..., None]
        zf = z_hat.astype(F32)[..., None]
        ok = sf > 0
        u = ((yg - zf).astype(F32) / np.where(ok, sf, F32(1))).astype(F32)
        c = np.clip(np.rint(u), 0, qmax)
        c = np.where(ok, c, 0).astype(np.uint8)
        # exact quotient from the same binary32 operands: flag near-midpoints
        u64 = (yg.astype(np.float64) - zf.astype(np.float64)) / np.where(ok, sf, F32(1)).astype(np.float64)
        mid = np.floor(u64) + 0.5
        ulp = np.spacing(np.abs(mid).astype(F32)).astype(np.float64)
        near = ok & (np.abs(u64 - mid) <= ulp)
    return QuantGroups(codes=c.reshape(lead + (D,)), scale=s_hat, zero=z_hat,
                       near_tie=near.reshape(lead + (D,)))


def dequant_fp32(q: QuantGroups, g: int) -> np.ndarray:
    """z_hat + (code * s_hat) in binary32 (the encoder's view of an INT4 anchor)."""
    lead = q.codes.shape[:-1]
    c = q.codes.reshape(lead + (D // g, g)).astype(F32)
    v = (q.zero.astype(F32)[..., None] + (c * q.scale.astype(F32)[..., None]).astype(F32)).astype(F32)
    return v.reshape(lead + (D,))


def dequant_f64(codes: np.ndarray, scale: np.ndarray, zero: np.ndarray, g: int) -> np.ndarray:
    """z_hat + code * s_hat in float64."""
    lead = codes.shape[:-1]
    c = codes.reshape(lead + (D // g, g)).astype(np.float64)
    v = zero.astype(np.float64)[..., None] + c * scale.astype(np.float64)[..., None]
    return v.reshape(lead + (D,))


# ---------------------------------------------------------------------------
# Encode ([RQ] abstract; Figure 1 steps (2)-(5))
# ---------------------------------------------------------------------------

@dataclass
class CacheConfig:
    """Per-loop formats and which loop each loop takes as its reference.

    Anchor policies ([RQ] Table 1 "First-loop" / "Last-loop"; Table 8 anchor
    intervals "N x [2^n, 4]", each group ending in its own anchor; Table 9
    "Previous-loop" / "Next-loop"):
      ANCHOR_LAST: the final loop is every loop's reference;
      ANCHOR_FIRST: loop 0 is every loop's reference;
      ANCHOR_INTERVAL: blocks of `anchor_interval` consecutive loops, the last
        loop of each block (or the final loop, for a short last block) being
        the reference of the others in its block;
      ANCHOR_PREVIOUS: loop l's reference is loop l-1; loop 0 is the anchor;
      ANCHOR_NEXT: loop l's reference is loop l+1; the final loop is the anchor.
    Anchor loops use bits 16 (bf16) or 4 (INT4, g = 32); the others 2 or 4.
    """
    num_loops: int
    bits: Sequence[int]
    group: Sequence[int]
    rotate: Sequence[int]
    alpha_mode: Sequence[int]
    anchor_policy: int = ANCHOR_LAST
    anchor_interval: int = 0

    @staticmethod
    def from_dict(d: dict) -> "CacheConfig":
        return CacheConfig(d["num_loops"], list(d["bits"]), list(d["group"]),
                           list(d["rotate"]), list(d["alpha_mode"]),
                           d.get("anchor_policy", ANCHOR_LAST), d.get("anchor_interval", 0))

    def ref_of(self, loop: int) -> int:
        """The loop whose (reconstructed) values loop `loop` is stored against;
        `loop` itself for an anchor."""
        L = self.num_loops
        if self.anchor_policy == ANCHOR_LAST:
            return L - 1
        if self.anchor_policy == ANCHOR_FIRST:
            return 0
        if self.anchor_policy == ANCHOR_PREVIOUS:
            return max(loop - 1, 0)
        if self.anchor_policy == ANCHOR_NEXT:
            return min(loop + 1, L - 1)
        n = self.anchor_interval
        return min((loop // n) * n + n - 1, L - 1)

    def chain(self, loop: int) -> List[int]:
        """The residual loops from `loop` toward its anchor (the anchor itself
        excluded): [loop, ref_of(loop), ...]; empty for an anchor."""
        out = []
        while self.ref_of(loop) != loop:
            out.append(loop)
            loop = self.ref_of(loop)
        return out

    def anchor_of(self, loop: int) -> int:
        while self.ref_of(loop) != loop:
            loop = self.ref_of(loop)
        return loop

    def is_anchor(self, loop: int) -> bool:
        return self.anchor_of(loop) == loop

    def anchors(self) -> List[int]:
        return sorted({self.anchor_of(l) for l in range(self.num_loops)})


@dataclass
class EncodedPlane:
    """One loop's K or V as stored: codes/meta (+ alpha for residual loops)."""
    codes: np.ndarray
    scale: np.ndarray
    zero: np.ndarray
    alpha: Optional[np.ndarray]
    near_tie: np.ndarray
    bits: int
    group: int
    rotate: int


@dataclass
class Encoded:
    cfg: CacheConfig
    # per anchor loop a: 'k'/'v' float32 bf16 values, or the INT4 EncodedPlane
    anchor_bf16: Dict[int, Dict[str, np.ndarray]] = field(default_factory=dict)
    anchor_q: Dict[int, Dict[str, EncodedPlane]] = field(default_factory=dict)
    hat32: Dict[int, Dict[str, np.ndarray]] = field(default_factory=dict)  # encoder's fp32 view of references
    loops: List[Optional[Dict[str, EncodedPlane]]] = field(default_factory=list)  # None for anchors
    error: bool = False


def _check_range(x: np.ndarray) -> bool:
    return bool(np.all(np.isfinite(x)) and np.all(np.abs(x) <= FP16_MAX))


def reconstruct_fp32(qg: QuantGroups, g: int, rotate: int, alpha_hat: np.ndarray, ref: np.ndarray) -> np.ndarray:
    """The encoder's binary32 view of a stored residual loop, used as the next
    loop's reference under a chained policy:  (alpha_hat * ref) + u,  with u the
    rotation of z_hat + (code * s_hat) (the orthonormal Hadamard is symmetric,
    so the same transform undoes it)."""
    u = dequant_fp32(qg, g)
    if rotate:
        u = fwht_fp32(u)
    a32 = np.asarray(alpha_hat).astype(F32)[..., None]
    return ((a32 * np.asarray(ref, F32)).astype(F32) + u).astype(F32)


def encode_fp32emu(K: np.ndarray, V: np.ndarray, cfg: CacheConfig) -> Encoded:
    """Encode every loop of the cached tokens.

    K, V: float32 [L, ..., 128] holding bf16 values (any leading shape after
    the loop axis, e.g. [B, H, T]).  Anchors are stored first; every other loop
    is encoded against its reference after that reference (nearest the anchor
    first, so a chain is walked outward from its anchor).
    """
    L = cfg.num_loops
    assert K.shape[0] == L and V.shape == K.shape
    enc = Encoded(cfg=cfg)
    enc.error = not (_check_range(K) and _check_range(V))
    for a in cfg.anchors():
        rb = cfg.bits[a]
        enc.anchor_bf16[a], enc.anchor_q[a], enc.hat32[a] = {}, {}, {}
        for name, X in (("k", K), ("v", V)):
            ref = np.asarray(X[a], dtype=F32)
            if rb == 16:
                enc.anchor_bf16[a][name] = ref
                enc.hat32[a][name] = ref
            elif rb == 4:
                qg = quantize_groups_fp32(ref, 4, 32)
                enc.anchor_q[a][name] = EncodedPlane(qg.codes, qg.scale, qg.zero, None, qg.near_tie, 4, 32, 0)
                enc.hat32[a][name] = dequant_fp32(qg, 32)
            else:
                raise ValueError("anchor bits must be 16 or 4")
    enc.loops = [None] * L
    is_ref = {cfg.ref_of(l) for l in range(L) if not cfg.is_anchor(l)}
    for l in sorted((l for l in range(L) if not cfg.is_anchor(l)), key=lambda l: len(cfg.chain(l))):
        planes = {}
        if l in is_ref:
            enc.hat32[l] = {}
        for name, X in (("k", K), ("v", V)):
            x = np.asarray(X[l], dtype=F32)
            ref = enc.hat32[cfg.ref_of(l)][name]
            a_hat = ls_alpha_fp32(x, ref, cfg.alpha_mode[l])
            if not np.all(np.isfinite(a_hat.astype(np.float64))):
                enc.error = True
            a32 = a_hat.astype(F32)[..., None]
            r = (x - (a32 * ref).astype(F32)).astype(F32)
            y = fwht_fp32(r) if cfg.rotate[l] else r
            qg = quantize_groups_fp32(y, cfg.bits[l], cfg.group[l])
            if not (np.all(np.isfinite(qg.scale.astype(np.float64))) and
                    np.all(np.isfinite(qg.zero.astype(np.float64)))):
                enc.error = True
            planes[name] = EncodedPlane(qg.codes, qg.scale, qg.zero, a_hat, qg.near_tie,
                                        cfg.bits[l], cfg.group[l], cfg.rotate[l])
            if l in is_ref:
                enc.hat32[l][name] = reconstruct_fp32(qg, cfg.group[l], cfg.rotate[l], a_hat, ref)
        enc.loops[l] = planes
    return enc


# ---------------------------------------------------------------------------
# Reconstruction (float64)
# ---------------------------------------------------------------------------

def reference_f64(enc: Encoded, name: str, anchor: Optional[int] = None) -> np.ndarray:
    """The decoder's view of an anchor loop (default: the final loop): exact
    bf16 values, or the INT4 anchor dequantised in float64."""
    a = enc.cfg.num_loops - 1 if anchor is None else anchor
    if enc.cfg.bits[a] == 16:
        return enc.anchor_bf16[a][name].astype(np.float64)
    p = enc.anchor_q[a][name]
    return dequant_f64(p.codes, p.scale, p.zero, 32)


def residual_f64(p: EncodedPlane) -> np.ndarray:
    """Dequantised residual in the original (unrotated) domain, float64."""
    y = dequant_f64(p.codes, p.scale, p.zero, p.group)
    if p.rotate:
        y = y @ hadamard_orthonormal(D)  # H symmetric: row-vector form of H y
    return y


def reconstruct_f64(enc: Encoded, loop: int):
    """(K_hat, V_hat) float64 of one loop: alpha_hat * ref_hat + H^T deq(codes),
    where ref_hat is the anchor's values or, under a chained policy, the
    reconstruction of the loop's reference (computed the same way)."""
    cfg = enc.cfg
    if cfg.is_anchor(loop):
        return reference_f64(enc, "k", loop), reference_f64(enc, "v", loop)
    refs = reconstruct_f64(enc, cfg.ref_of(loop))
    out = []
    for name, ref in zip(("k", "v"), refs):
        p = enc.loops[loop][name]
        out.append(p.alpha.astype(np.float64)[..., None] * ref + residual_f64(p))
    return out[0], out[1]


# ---------------------------------------------------------------------------
# Decode attention (float64)
# ---------------------------------------------------------------------------

def _softmax_combine(scores: List[np.ndarray]):
    s = np.concatenate(scores)
    if s.size == 0:
        return None, None
    m = s.max()
    p = np.exp(s - m)
    return p, p.sum()


def decode_attention_f64(enc: Encoded, loop: int, q: np.ndarray, ctx_len: np.ndarray,
                         k_tail: Optional[np.ndarray] = None, v_tail: Optional[np.ndarray] = None,
                         scale: float = 1.0 / np.sqrt(128.0)) -> np.ndarray:
    """Decode attention of one loop, scored in the rotated domain.

    q: [B, Hq, 128]; ctx_len: [B]; k_tail/v_tail: [B, Hkv, n_tail, 128] (bf16
    values of the current token(s), attended unquantised).  For a residual loop
    each cached token's score is
        scale * (alpha_K (q . ref_k) + (H q) . deq(codes_K))
    and the output is
        (sum_t p_t alpha_V,t ref_v,t + H^T sum_t p_t deq(codes_V,t) + sum_tail p v) / sum p.
    Under a chained policy the loop's chain l = c_0 -> c_1 -> ... -> c_{n-1} ->
    anchor unrolls the recursion  x_hat_c = alpha_c x_hat_{ref(c)} + H^T deq_c:
        x_hat_l = beta_n ref + sum_i beta_i H^T deq(codes_{c_i}),
        beta_0 = 1, beta_{i+1} = beta_i * alpha_{c_i}   (per token, K and V apart),
    so the score takes beta_n (q . ref_k) + sum_i beta_i (H q) . deq_i and the
    value sums weigh each term by p_t times its beta.
    Returns float64 [B, Hq, 128].
    """
    cfg = enc.cfg
    q = np.asarray(q, dtype=np.float64)
    B, Hq, _ = q.shape
    a = cfg.anchor_of(loop)
    refk = reference_f64(enc, "k", a)
    refv = reference_f64(enc, "v", a)
    Hkv = refk.shape[1]
    G = Hq // Hkv
    Hn = hadamard_orthonormal(D)
    out = np.zeros((B, Hq, D))
    members = cfg.chain(loop)
    terms = []  # per chain member: (deq K, deq V, rotate, beta K, beta V), betas [B, Hkv, T]
    bk = np.ones(refk.shape[:-1])
    bv = np.ones(refv.shape[:-1])
    for c in members:
        pk, pv = enc.loops[c]["k"], enc.loops[c]["v"]
        terms.append((dequant_f64(pk.codes, pk.scale, pk.zero, pk.group),
                      dequant_f64(pv.codes, pv.scale, pv.zero, pv.group), pk.rotate, bk, bv))
        bk = bk * pk.alpha.astype(np.float64)
        bv = bv * pv.alpha.astype(np.float64)
    for b in range(B):
        n = int(ctx_len[b])
        for qh in range(Hq):
            h = qh // G
            qv = q[b, qh]
            s_c = bk[b, h, :n] * (refk[b, h, :n] @ qv)
            for yk, _, rot, tk, _ in terms:
                qr = Hn @ qv if rot else qv
                s_c = s_c + tk[b, h, :n] * (yk[b, h, :n] @ qr)
            scores = [scale * s_c]
            if k_tail is not None and k_tail.shape[2] > 0:
                scores.append(scale * (np.asarray(k_tail[b, h], np.float64) @ qv))
            p, lsum = _softmax_combine(scores)
            if p is None:
                continue
            pc, pt = p[:n], p[n:]
            o = (pc * bv[b, h, :n]) @ refv[b, h, :n]
            for _, yv, rot, _, tv in terms:
                acc_res = (pc * tv[b, h, :n]) @ yv[b, h, :n]
                o = o + (Hn @ acc_res if rot else acc_res)
            if pt.size:
                o = o + pt @ np.asarray(v_tail[b, h], np.float64)
            out[b, qh] = o / lsum
    return out


def decode_attention_multi_f64(enc: Encoded, loop: int, q: np.ndarray, ctx_len: np.ndarray,
                               k_tail: np.ndarray, v_tail: np.ndarray,
                               scale: float = 1.0 / np.sqrt(128.0)) -> np.ndarray:
    """Several query tokens per sequence (speculative verification of n_q draft
    tokens): q [B, n_q, Hq, 128]; the last n_q tail tokens are the draft tokens'
    keys and values.  Draft token i is an ordinary decode whose tail stops at
    itself: tail tokens 0 .. n_tail - n_q + i.  Returns float64 [B, n_q, Hq, 128]."""
    q = np.asarray(q)
    n_q, n_tail = q.shape[1], k_tail.shape[2]
    out = np.zeros(q.shape, dtype=np.float64)
    for i in range(n_q):
        n_vis = n_tail - n_q + i + 1
        out[:, i] = decode_attention_f64(enc, loop, q[:, i], ctx_len, k_tail[:, :, :n_vis], v_tail[:, :, :n_vis], scale)
    return out


def attention_f64(q: np.ndarray, Kc: np.ndarray, Vc: np.ndarray, ctx_len: np.ndarray,
                  k_tail: Optional[np.ndarray] = None, v_tail: Optional[np.ndarray] = None,
                  scale: float = 1.0 / np.sqrt(128.0)) -> np.ndarray:
    """Brute-force softmax(q K^T * scale) V over given (reconstructed or bf16)
    caches Kc, Vc [B, Hkv, T, 128] followed by the tail tokens."""
    q = np.asarray(q, dtype=np.float64)
    B, Hq, _ = q.shape
    Hkv = Kc.shape[1]
    G = Hq // Hkv
    out = np.zeros((B, Hq, D))
    for b in range(B):
        n = int(ctx_len[b])
        for qh in range(Hq):
            h = qh // G
            Kb = np.asarray(Kc[b, h, :n], np.float64)
            Vb = np.asarray(Vc[b, h, :n], np.float64)
            if k_tail is not None and k_tail.shape[2] > 0:
                Kb = np.concatenate([Kb, np.asarray(k_tail[b, h], np.float64)])
                Vb = np.concatenate([Vb, np.asarray(v_tail[b, h], np.float64)])
            if Kb.shape[0] == 0:
                continue
            s = scale * (Kb @ q[b, qh])
            w = np.exp(s - s.max())
            out[b, qh] = (w @ Vb) / w.sum()
    return out


# ---------------------------------------------------------------------------
# Effective bitwidth ([RQ] Table 5, Table 8 and Table 10 captions: values,
# scales, offsets and LS coefficients are counted)
# ---------------------------------------------------------------------------

def effective_bitwidth(blocks: Sequence[Sequence[int]], group: int, head_dim: int = 128,
                       residual: bool = True, meta_bits: int = 16, alpha_bits: int = 16,
                       anchor_group: int = 32) -> float:
    """Average stored bits per KV element over all loops.

    ``blocks``: one list of per-loop bit widths per anchor interval; the last
    entry of each list is that interval's anchor (reference) loop.  A loop
    quantised to b bits with group g costs b + meta_bits/g per element (g is
    ``group`` for 2-bit loops and ``anchor_group`` for 4-bit loops); a bf16
    loop costs 16.  In residual mode every non-anchor loop also stores one
    LS coefficient of ``alpha_bits`` per head_dim-element vector.
    """
    total, n = 0.0, 0
    for blk in blocks:
        for i, b in enumerate(blk):
            if b == 16:
                cost = 16.0
            else:
                g = group if b == 2 else anchor_group
                cost = b + meta_bits / g
            if residual and i != len(blk) - 1:
                cost += alpha_bits / head_dim
            total += cost
            n += 1
    return total / n
