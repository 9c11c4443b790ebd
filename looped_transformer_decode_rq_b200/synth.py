"""Seeded synthetic inputs for the ResidualQuant hot path.

This module only draws random numbers and shapes them into the workloads the
benchmark and the tests run. It holds none of the method's arithmetic (no
scaling coefficient, rotation or quantiser), so the CUDA path and the CPU
oracle can both take their inputs from it without sharing any computation.

Generator (the pages give no data, only the observation that keys and values of
the loops of a looped Transformer are close to those of the final loop --
"ResidualQuant: KV Cache Quantization for Looped Transformers with 2-Bit
Residuals", abstract and Figure 2/Figure 5 captions):

* reference (final-loop) keys/values ``K_ref = N(0,1) * s[h, c]`` with a
  per-(head, channel) scale ``s ~ LogNormal(0, 0.5)``; with probability
  ``outlier_p`` a channel is an outlier whose scale is multiplied by
  ``outlier_mult``; rounded to bf16;
* every other loop ``K_l = a_l[h] * K_ref + N(0, sigma_l^2)`` with
  ``a_l ~ U(0.8, 1.2)`` drawn per (loop, head); rounded to bf16;
* values are drawn the same way with their own scales and ``a_l``;
* queries ``q ~ N(0, 1)`` rounded to bf16, one per (loop, sequence, q-head);
  with probability ``q_outlier_p`` a query element is an outlier, multiplied
  by ``U(q_outlier_mult)`` (30-100x by default);
* the current token of every loop (the "tail", attended in bf16 before it is
  encoded) follows the same recipe as the cached tokens.
"""
from __future__ import annotations

from dataclasses import dataclass, field, replace
from typing import Optional, Sequence

import torch

HEAD_DIM = 128


@dataclass(frozen=True)
class Workload:
    """Shape, per-loop format and generator parameters of one synthetic case.

    ``bits[l]``/``group[l]``/``rotate[l]``/``alpha_mode[l]`` follow the cache
    configuration of the C ABI: the last loop is the reference loop, whose
    ``bits`` is 16 (bf16 reference) or 4 (INT4 anchor, group 32).
    """

    name: str
    num_loops: int = 4
    batch: int = 1
    kv_heads: int = 2
    q_heads: int = 2
    head_dim: int = HEAD_DIM
    context: int = 256
    lengths: Optional[Sequence[int]] = None  # ragged lengths (None: all == context)
    length_range: Optional[Sequence[int]] = None  # draw lengths U{lo..hi} from the seed
    bits: Sequence[int] = (2, 2, 2, 16)
    group: Sequence[int] = (32, 32, 32, 32)
    rotate: Sequence[int] = (1, 1, 1, 0)
    alpha_mode: Sequence[int] = (0, 0, 0, 0)
    sigma: Sequence[float] = (0.2, 0.2, 0.2)
    outlier_p: float = 0.0
    outlier_mult: float = 10.0
    n_tail: int = 1
    seed: int = 0
    layers: int = 1
    anchor_policy: int = 0      # 0: final loop is the reference; 1: loop 0; 2: blocks of anchor_interval;
                                # 3 / 4: chained, loop l against loop l-1 / l+1
    anchor_interval: int = 0
    q_outlier_p: float = 0.0    # per (loop, sequence, q-head, channel): the query element is an outlier
    q_outlier_mult: Sequence[float] = (30.0, 100.0)  # outlier query elements are multiplied by U(lo, hi)

    def with_(self, **kw) -> "Workload":
        return replace(self, **kw)

    @property
    def gqa(self) -> int:
        return self.q_heads // self.kv_heads


# ---------------------------------------------------------------------------
# Named workloads.  Sizes follow the looped-model shapes the benchmark uses
# (Ouro-1.4B-like attention: 16 KV heads, head_dim 128, 4 loops).
# ---------------------------------------------------------------------------

def tiny() -> Workload:
    """1 layer, 4 loops (loop 4 = bf16 reference), 2 KV heads, batch 1,
    context 256, loops 1-3 INT2 g=32 with the Hadamard rotation, noise 0.2."""
    return Workload(name="tiny_L4_H2_B1_T256_int2g32", batch=1, kv_heads=2, q_heads=2,
                    context=256, sigma=(0.2, 0.2, 0.2), seed=0)


def ouro_8k(batch: int = 16, context: int = 8192) -> Workload:
    """Ouro-1.4B-shaped single layer: 4 loops, 16 KV heads (MHA), batch 16,
    context 8192, loops 1-3 INT2 g=32 rotated, bf16 reference, noise
    0.3/0.2/0.1 per loop and 1% outlier channels at 10x."""
    return Workload(name=f"ouro_L4_H16_B{batch}_T{context}_int2g32_bf16ref", batch=batch,
                    kv_heads=16, q_heads=16, context=context, sigma=(0.3, 0.2, 0.1),
                    outlier_p=0.01, seed=1)


def ouro_8k_next_loop(batch: int = 16, context: int = 8192) -> Workload:
    """The Ouro-shaped 8k layer stored with the Next-loop chained reference
    (loop l against loop l+1, the final loop the bf16 anchor): decoding loop 1
    reads the codes of loops 1-3 and the anchor."""
    return ouro_8k(batch, context).with_(name=f"ouro_L4_H16_B{batch}_T{context}_int2g32_bf16ref_next_loop",
                                         anchor_policy=4)


def ouro_8k_next_loop_int4(batch: int = 16, context: int = 8192) -> Workload:
    """Next-loop chain with an INT4 anchor, loops 1-3 INT2 g=32 ([2,2,2,4], the
    mixed Next-loop setting of the pages' Table 9)."""
    return ouro_8k(batch, context).with_(name=f"ouro_L4_H16_B{batch}_T{context}_2224_int4ref_next_loop",
                                         bits=(2, 2, 2, 4), anchor_policy=4)


def mixed_int4_anchor(batch: int = 8, context: int = 8192) -> Workload:
    """Same shape, loops 1-2 INT2, loop 3 INT4, reference loop INT4 g=32."""
    return Workload(name=f"mixed_2244_H16_B{batch}_T{context}_int4ref", batch=batch,
                    kv_heads=16, q_heads=16, context=context, bits=(2, 2, 4, 4),
                    group=(32, 32, 32, 32), rotate=(1, 1, 1, 0), sigma=(0.3, 0.2, 0.1),
                    outlier_p=0.01, seed=2)


def capacity_24layer(batch: int = 1, context: int = 8192) -> Workload:
    """One layer of a 24-layer, 4-loop, 16-head model (INT2 loops 1-3, g=32)."""
    return Workload(name=f"capacity_24x_L4_H16_B{batch}_T{context}", batch=batch, kv_heads=16,
                    q_heads=16, context=context, sigma=(0.3, 0.2, 0.1), outlier_p=0.01,
                    seed=3, layers=24)


def gqa_long(batch: int = 8, context: int = 32768, q_heads: int = 32, int4_anchor: bool = False) -> Workload:
    """4 loops, 32 (or `q_heads`) query heads / 8 KV heads, batch 8, ragged
    lengths U{context/2 .. context}, INT2 loops 1-3 g=32, bf16 reference (or an
    INT4 g=32 anchor: the [2,2,2,4] setting)."""
    suffix = "_int4ref" if int4_anchor else ""
    return Workload(name=f"gqa_L4_Hq{q_heads}_Hkv8_B{batch}_T{context}_ragged{suffix}", batch=batch,
                    kv_heads=8, q_heads=q_heads, context=context, bits=(2, 2, 2, 4) if int4_anchor else (2, 2, 2, 16),
                    length_range=(context // 2, context), sigma=(0.3, 0.2, 0.1),
                    outlier_p=0.01, seed=4)


# ---------------------------------------------------------------------------

def _bf16(x: torch.Tensor) -> torch.Tensor:
    return x.to(torch.bfloat16)


def draw_lengths(wl: Workload, device="cpu") -> torch.Tensor:
    """Per-sequence context lengths (int32 [B])."""
    if wl.lengths is not None:
        assert len(wl.lengths) == wl.batch
        return torch.tensor(list(wl.lengths), dtype=torch.int32, device=device)
    if wl.length_range is not None:
        g = torch.Generator(device="cpu").manual_seed(wl.seed * 7919 + 17)
        lo, hi = wl.length_range
        return torch.randint(lo, hi + 1, (wl.batch,), generator=g, dtype=torch.int64).to(
            device=device, dtype=torch.int32)
    return torch.full((wl.batch,), wl.context, dtype=torch.int32, device=device)


def make_inputs(wl: Workload, device="cpu", layer: int = 0) -> dict:
    """Draw every input of one layer of ``wl`` on ``device``.

    Returns a dict of tensors:
      ``k``, ``v``: bf16 [L, B, Hkv, T, D]  -- the cached tokens of every loop
      ``k_tail``, ``v_tail``: bf16 [L, B, Hkv, n_tail, D] -- the current token(s)
      ``q``: bf16 [L, B, Hq, D]            -- one decode query per loop
      ``ctx_len``: int32 [B]                -- cached tokens per sequence
    """
    L, B, Hkv, Hq, D, T = wl.num_loops, wl.batch, wl.kv_heads, wl.q_heads, wl.head_dim, wl.context
    assert len(wl.sigma) == L - 1
    dev = torch.device(device)
    g = torch.Generator(device=dev).manual_seed(wl.seed * 1000003 + layer)

    def randn(*shape):
        return torch.randn(*shape, generator=g, device=dev, dtype=torch.float32)

    def rand(*shape):
        return torch.rand(*shape, generator=g, device=dev, dtype=torch.float32)

    def channel_scale():
        s = torch.exp(0.5 * randn(Hkv, D))
        if wl.outlier_p > 0:
            mask = rand(Hkv, D) < wl.outlier_p
            s = torch.where(mask, s * wl.outlier_mult, s)
        return s

    out = {}
    for name in ("k", "v"):
        scale = channel_scale()
        a = 0.8 + 0.4 * rand(L - 1, Hkv)
        planes = torch.empty((L, B, Hkv, T, D), dtype=torch.bfloat16, device=dev)
        tails = torch.empty((L, B, Hkv, wl.n_tail, D), dtype=torch.bfloat16, device=dev)
        for which, dst, n in (("cache", planes, T), ("tail", tails, wl.n_tail)):
            if n == 0:
                continue
            ref = _bf16(randn(B, Hkv, n, D) * scale[None, :, None, :])
            dst[L - 1].copy_(ref)
            reff = ref.float()
            for l in range(L - 1):
                noise = randn(B, Hkv, n, D)
                x = a[l][None, :, None, None] * reff + wl.sigma[l] * noise
                dst[l].copy_(_bf16(x))
                del noise, x
            del ref, reff
        out[name] = planes
        out[name + "_tail"] = tails
    q = randn(L, B, Hq, D)
    if wl.q_outlier_p > 0:
        # outlier query channels, from a generator of their own (the other
        # inputs of the workload are unchanged by it)
        go = torch.Generator(device=dev).manual_seed(wl.seed * 1000003 + layer + 7777)
        mask = torch.rand(L, B, Hq, D, generator=go, device=dev) < wl.q_outlier_p
        lo, hi = wl.q_outlier_mult
        mult = lo + (hi - lo) * torch.rand(L, B, Hq, D, generator=go, device=dev)
        q = torch.where(mask, q * mult, q)
    out["q"] = _bf16(q)
    out["ctx_len"] = draw_lengths(wl, device=dev)
    return out


def draft_queries(wl: Workload, n_q: int, device="cpu") -> torch.Tensor:
    """Queries of n_q draft tokens per sequence and loop, bf16 [L, B, n_q, Hq, D],
    drawn like the single decode queries (N(0, 1), rounded to bf16) from a
    generator of their own."""
    dev = torch.device(device)
    g = torch.Generator(device=dev).manual_seed(wl.seed * 1000003 + 7919 * n_q + 17)
    x = torch.randn(wl.num_loops, wl.batch, n_q, wl.q_heads, wl.head_dim, generator=g, device=dev)
    return _bf16(x)


def cache_config_dict(wl: Workload, capacity: Optional[int] = None) -> dict:
    """The cache configuration (fields of the C ABI's ``rq_config``)."""
    return dict(num_loops=wl.num_loops, batch=wl.batch, kv_heads=wl.kv_heads,
                q_heads=wl.q_heads, head_dim=wl.head_dim,
                capacity=capacity if capacity is not None else wl.context + wl.n_tail,
                bits=list(wl.bits), group=list(wl.group), rotate=list(wl.rotate),
                alpha_mode=list(wl.alpha_mode), anchor_policy=wl.anchor_policy,
                anchor_interval=wl.anchor_interval)
