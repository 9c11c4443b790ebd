"""Parity at the benchmark's full sizes, in the launch configuration bench.py
times (persistent split over all pages of the whole batch).  The whole batch is
encoded and decoded on the GPU; sampled (sequence, kv-head) slabs are encoded
by the oracle and compared bit for bit, and their q-heads' attention outputs
compared with the float64 oracle over the full context."""
import numpy as np
import pytest
import torch

import oracle.rq_oracle as O
from looped_transformer_decode_rq_b200 import synth
from tests.helpers import ATTN_TOL, compare_encoded, rel_err_rows, unpack_alpha, unpack_codes, unpack_meta

pytestmark = pytest.mark.gpu

CASES = [
    (synth.ouro_8k(), [(0, 0), (7, 9), (15, 15)]),
    (synth.mixed_int4_anchor(batch=8), [(0, 3), (7, 15)]),
    (synth.mixed_int4_anchor(batch=32), [(31, 15)]),
    (synth.gqa_long(batch=8), [(0, 0), (5, 7)]),
    (synth.gqa_long(batch=8, q_heads=64), [(3, 4)]),
    (synth.gqa_long(batch=8, int4_anchor=True), [(0, 0), (6, 3)]),
    (synth.ouro_8k_next_loop(), [(0, 0), (15, 15)]),
    (synth.ouro_8k_next_loop_int4(), [(0, 0), (9, 12)]),
]


def _slab_planes(cache, b, h, n):
    """The cache planes of one (b, h) slab, unpacked like tests.helpers.read_planes."""
    cfg, lay = cache.cfg, cache.layout
    L = cfg.num_loops

    def grab(off, rec):
        return cache.plane(off, rec)[b:b + 1, h:h + 1, :n].cpu().numpy()

    out = {"ref": {}, "loops": []}
    for l in range(L):
        if lay.anchor_of[l] != l:
            continue
        out["ref"][l] = {}
        for kv, name in enumerate("kv"):
            if cfg.bits[l] == 16:
                out["ref"][l][name] = grab(lay.codes_offset[l][kv], 256).view("<u2")
            else:
                s, z = unpack_meta(grab(lay.meta_offset[l][kv], 16))
                out["ref"][l][name] = (unpack_codes(grab(lay.codes_offset[l][kv], 64), 4), s, z)
    for l in range(L):
        if lay.anchor_of[l] == l:
            out["loops"].append(None)
            continue
        d = {}
        for kv, name in enumerate("kv"):
            s, z = unpack_meta(grab(lay.meta_offset[l][kv], lay.meta_record_bytes[l]))
            d[name] = (unpack_codes(grab(lay.codes_offset[l][kv], lay.codes_record_bytes[l]), cfg.bits[l]), s, z)
        d["alpha"] = unpack_alpha(grab(lay.alpha_offset[l], 4))
        out["loops"].append(d)
    return out


@pytest.mark.parametrize("wl,samples", CASES, ids=lambda x: getattr(x, "name", "samples"))
def test_full_size_sampled_parity(librq, wl, samples):
    rq = librq
    dev = torch.device("cuda")
    inp = synth.make_inputs(wl, dev)
    cfgd = synth.cache_config_dict(wl)
    cache = rq.Cache(rq.config_from_dict(cfgd), device=dev)
    cache.encode(inp["k"], inp["v"])
    ctx = inp["ctx_len"]
    outs = [cache.decode_attention(l, inp["q"][l], ctx, inp["k_tail"][l], inp["v_tail"][l])
            for l in range(wl.num_loops)]
    torch.cuda.synchronize()
    assert cache.get_error() == 0
    G = wl.gqa
    ocfg = O.CacheConfig.from_dict(cfgd)
    for b, h in samples:
        n = int(ctx[b])
        sl = lambda t: t[:, b:b + 1, h:h + 1].float().cpu().numpy()  # noqa: E731
        K, V = sl(inp["k"])[:, :, :, :n], sl(inp["v"])[:, :, :, :n]
        enc = O.encode_fp32emu(K, V, ocfg)
        compare_encoded(_slab_planes(cache, b, h, n), enc)
        q = inp["q"][:, b:b + 1, h * G:(h + 1) * G].float().cpu().numpy()
        kt, vt = sl(inp["k_tail"]), sl(inp["v_tail"])
        for l in range(wl.num_loops):
            want = O.decode_attention_f64(enc, l, q[l], np.array([n]), kt[l], vt[l])
            got = outs[l][b:b + 1, h * G:(h + 1) * G].cpu().numpy()
            err = rel_err_rows(got, want).max()
            assert err <= ATTN_TOL, (wl.name, b, h, l, float(err))


def test_full_size_multi_query(librq):
    """Four draft tokens per sequence on the full Ouro-shaped cache, in the
    configuration bench.py times (the tensor-core kernel, 4 rows per kv-head)."""
    rq = librq
    n_q = 4
    wl = synth.ouro_8k().with_(n_tail=n_q)
    dev = torch.device("cuda")
    inp = synth.make_inputs(wl, dev)
    qm = synth.draft_queries(wl, n_q, dev)
    cfgd = synth.cache_config_dict(wl)
    cache = rq.Cache(rq.config_from_dict(cfgd), device=dev)
    cache.encode(inp["k"], inp["v"])
    ctx = inp["ctx_len"]
    outs = [cache.decode_attention_multi(l, qm[l], ctx, inp["k_tail"][l], inp["v_tail"][l]) for l in (0, 3)]
    torch.cuda.synchronize()
    assert cache.get_error() == 0
    ocfg = O.CacheConfig.from_dict(cfgd)
    for b, h in [(2, 5), (14, 0)]:
        n = int(ctx[b])
        sl = lambda t: t[:, b:b + 1, h:h + 1].float().cpu().numpy()  # noqa: E731
        enc = O.encode_fp32emu(sl(inp["k"])[:, :, :, :n], sl(inp["v"])[:, :, :, :n], ocfg)
        kt, vt = sl(inp["k_tail"]), sl(inp["v_tail"])
        for i, l in enumerate((0, 3)):
            q = qm[l][b:b + 1, :, h:h + 1].float().cpu().numpy()
            want = O.decode_attention_multi_f64(enc, l, q, np.array([n]), kt[l], vt[l])
            got = outs[i][b:b + 1, :, h:h + 1].cpu().numpy()
            err = rel_err_rows(got, want).max()
            assert err <= ATTN_TOL, (b, h, l, float(err))


def test_full_size_sixteen_rows_one_pass(librq):
    """Four draft tokens on the full 32k GQA cache (4 query heads per kv-head):
    16 rows per kv-head in one pass over the cache on the tensor cores, as the
    bench's verify line times them."""
    rq = librq
    n_q = 4
    wl = synth.gqa_long(batch=8).with_(n_tail=n_q)
    dev = torch.device("cuda")
    inp = synth.make_inputs(wl, dev)
    qm = synth.draft_queries(wl, n_q, dev)
    cfgd = synth.cache_config_dict(wl)
    cache = rq.Cache(rq.config_from_dict(cfgd), device=dev)
    cache.encode(inp["k"], inp["v"])
    ctx = inp["ctx_len"]
    G = wl.gqa
    for l in (0, 3):
        assert cache.decode_plan(l, n_q) == (rq.DECODE_KERNEL_TENSOR, n_q * G)
    outs = [cache.decode_attention_multi(l, qm[l], ctx, inp["k_tail"][l], inp["v_tail"][l]) for l in (0, 3)]
    torch.cuda.synchronize()
    assert cache.get_error() == 0
    ocfg = O.CacheConfig.from_dict(cfgd)
    for b, h in [(1, 2), (7, 7)]:
        n = int(ctx[b])
        sl = lambda t: t[:, b:b + 1, h:h + 1].float().cpu().numpy()  # noqa: E731
        enc = O.encode_fp32emu(sl(inp["k"])[:, :, :, :n], sl(inp["v"])[:, :, :, :n], ocfg)
        kt, vt = sl(inp["k_tail"]), sl(inp["v_tail"])
        for i, l in enumerate((0, 3)):
            q = qm[l][b:b + 1, :, h * G:(h + 1) * G].float().cpu().numpy()
            want = O.decode_attention_multi_f64(enc, l, q, np.array([n]), kt[l], vt[l])
            got = outs[i][b:b + 1, :, h * G:(h + 1) * G].cpu().numpy()
            err = rel_err_rows(got, want).max()
            assert err <= ATTN_TOL, (b, h, l, float(err))
