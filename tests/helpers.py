"""Test-side helpers: unpack the cache planes the library writes (bit order as
documented in include/rq_api.h), run the oracle on the same seeded inputs, and
the error metrics the parity tests use.  Nothing here is shared with the CUDA
path."""
from __future__ import annotations

import numpy as np
import torch

import oracle.rq_oracle as O

# Tolerances (encode: bit-exact; reconstruct and attention: relative, vs float64)
RECON_TOL = 1e-3
ATTN_TOL = 2e-3


def to_np32(t: torch.Tensor) -> np.ndarray:
    return t.detach().to("cpu", torch.float32).numpy()


def unpack_codes(raw: np.ndarray, bits: int) -> np.ndarray:
    """raw uint8 [..., 128*bits/8] -> uint8 codes [..., 128].

    INT2: element d in bits 2*(d%16) of little-endian 32-bit word d/16;
    INT4: element d in bits 4*(d%8) of word d/8."""
    words = raw.view("<u4")
    per = 32 // bits
    d = np.arange(128)
    w = words[..., d // per]
    return ((w >> (bits * (d % per)).astype(np.uint32)) & ((1 << bits) - 1)).astype(np.uint8)


def unpack_meta(raw: np.ndarray):
    """raw uint8 [..., ng*4] -> (scale fp16 [..., ng], zero fp16 [..., ng])."""
    h = raw.view("<u2").reshape(raw.shape[:-1] + (-1, 2))
    return h[..., 0].view(np.float16), h[..., 1].view(np.float16)


def unpack_alpha(raw: np.ndarray):
    h = raw.view("<u2")
    return h[..., 0].view(np.float16), h[..., 1].view(np.float16)


def read_planes(cache, n_tokens: int = 0, positions=None):
    """Copy the cache's planes to numpy: the first n_tokens positions of every
    sequence, or (``positions``: one position per sequence) the one record of
    sequence b at positions[b], as a length-1 token axis."""
    from looped_transformer_decode_rq_b200 import rq  # noqa: F401
    cfg, lay = cache.cfg, cache.layout
    L = cfg.num_loops
    out = {"ref": {}, "loops": []}

    def grab(off, rec):
        pl = cache.plane(off, rec)
        if positions is None:
            return pl[:, :, :n_tokens].cpu().numpy()
        pos = torch.as_tensor(positions, dtype=torch.long, device=pl.device)
        idx = pos.view(-1, 1, 1, 1).expand(-1, pl.shape[1], 1, rec)
        return torch.gather(pl, 2, idx).cpu().numpy()

    for l in range(L):
        if lay.alpha_offset[l] >= 0:
            continue
        out["ref"][l] = {}
        for kv, name in enumerate("kv"):
            if cfg.bits[l] == 16:
                out["ref"][l][name] = grab(lay.codes_offset[l][kv], 256).view("<u2")
            else:
                codes = unpack_codes(grab(lay.codes_offset[l][kv], 64), 4)
                s, z = unpack_meta(grab(lay.meta_offset[l][kv], 16))
                out["ref"][l][name] = (codes, s, z)
    for l in range(L):
        if lay.alpha_offset[l] < 0:
            out["loops"].append(None)
            continue
        d = {}
        for kv, name in enumerate("kv"):
            codes = unpack_codes(grab(lay.codes_offset[l][kv], lay.codes_record_bytes[l]), cfg.bits[l])
            s, z = unpack_meta(grab(lay.meta_offset[l][kv], lay.meta_record_bytes[l]))
            d[name] = (codes, s, z)
        ak, av = unpack_alpha(grab(lay.alpha_offset[l], 4))
        d["alpha"] = (ak, av)
        out["loops"].append(d)
    return out


def oracle_encode(inputs: dict, cfg_dict: dict) -> O.Encoded:
    K = to_np32(inputs["k"])
    V = to_np32(inputs["v"])
    return O.encode_fp32emu(K, V, O.CacheConfig.from_dict(cfg_dict))


def compare_encoded(planes: dict, enc: O.Encoded) -> dict:
    """Bit-exact comparison; codes may differ only where the oracle flags a
    rounding near-tie.  Returns counts; raises AssertionError on mismatch."""
    stats = {"codes": 0, "near_tie": 0, "near_tie_diff": 0}
    cfg = enc.cfg
    assert sorted(planes["ref"]) == cfg.anchors()
    for a in cfg.anchors():
        for name in "kv":
            if cfg.bits[a] == 16:
                want = enc.anchor_bf16[a][name].view(np.uint32) >> 16
                assert np.array_equal(planes["ref"][a][name].astype(np.uint32), want), f"anchor {a} {name} differs"
            else:
                codes, s, z = planes["ref"][a][name]
                p = enc.anchor_q[a][name]
                assert np.array_equal(s.view(np.uint16), p.scale.view(np.uint16)), f"anchor {a} {name} scale differs"
                assert np.array_equal(z.view(np.uint16), p.zero.view(np.uint16)), f"anchor {a} {name} zero differs"
                diff = codes != p.codes
                assert not np.any(diff & ~p.near_tie), f"anchor {a} {name} codes differ"
    for l, d in enumerate(planes["loops"]):
        if d is None:
            assert cfg.is_anchor(l)
            continue
        ak, av = d["alpha"]
        assert np.array_equal(ak.view(np.uint16), enc.loops[l]["k"].alpha.view(np.uint16)), f"loop {l} alpha_K differs"
        assert np.array_equal(av.view(np.uint16), enc.loops[l]["v"].alpha.view(np.uint16)), f"loop {l} alpha_V differs"
        for name in "kv":
            codes, s, z = d[name]
            p = enc.loops[l][name]
            assert np.array_equal(s.view(np.uint16), p.scale.view(np.uint16)), f"loop {l} {name} scale differs"
            assert np.array_equal(z.view(np.uint16), p.zero.view(np.uint16)), f"loop {l} {name} zero differs"
            diff = codes != p.codes
            bad = diff & ~p.near_tie
            assert not np.any(bad), f"loop {l} {name} codes differ at {np.argwhere(bad)[:5]}"
            stats["codes"] += codes.size
            stats["near_tie"] += int(p.near_tie.sum())
            stats["near_tie_diff"] += int((diff & p.near_tie).sum())
    return stats


def rel_err_rows(got: np.ndarray, want: np.ndarray) -> np.ndarray:
    """Per-row ||got - want||_inf / ||want||_inf over the last axis."""
    num = np.abs(got.astype(np.float64) - want).max(axis=-1)
    den = np.maximum(np.abs(want).max(axis=-1), 1e-30)
    return num / den
