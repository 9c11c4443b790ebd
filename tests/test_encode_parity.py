"""GPU encode vs the oracle: packed codes, fp16 scales/offsets and alphas must
match bit for bit (codes may differ only where the oracle flags a rounding
near-tie); reconstruction within 1e-3 relative to the float64 oracle."""
import numpy as np
import pytest
import torch

import oracle.rq_oracle as O
from looped_transformer_decode_rq_b200 import synth
from tests.helpers import (RECON_TOL, compare_encoded, oracle_encode, read_planes, rel_err_rows,
                           to_np32)

pytestmark = pytest.mark.gpu

CASES = [
    synth.tiny(),
    synth.Workload(name="mixed_modes", batch=2, kv_heads=3, q_heads=3, context=33,
                   bits=(2, 4, 2, 16), group=(16, 32, 32, 32), rotate=(1, 1, 0, 0),
                   alpha_mode=(0, 1, 2, 0), sigma=(0.3, 0.2, 0.1), outlier_p=0.05, seed=5),
    synth.Workload(name="int4_anchor", batch=2, kv_heads=2, q_heads=2, context=65,
                   bits=(2, 2, 4, 4), group=(32, 16, 32, 32), rotate=(1, 1, 1, 0),
                   sigma=(0.3, 0.2, 0.1), outlier_p=0.02, seed=6),
    synth.Workload(name="two_loops", num_loops=2, batch=1, kv_heads=1, q_heads=1, context=1,
                   bits=(4, 16), group=(32, 32), rotate=(1, 0), alpha_mode=(0, 0), sigma=(0.2,), seed=7),
    synth.Workload(name="eight_loops", num_loops=8, batch=1, kv_heads=2, q_heads=2, context=17,
                   bits=(2, 2, 2, 2, 2, 2, 2, 4), group=(16,) * 7 + (32,), rotate=(1,) * 7 + (0,),
                   alpha_mode=(0,) * 8, sigma=(0.3, 0.25, 0.2, 0.15, 0.1, 0.1, 0.05), seed=8),
    # First-loop reference ([RQ] Table 1) with norm-ratio and LS scales ([RQ] Table 9)
    synth.Workload(name="first_loop_norm_ratio", batch=2, kv_heads=2, q_heads=2, context=45,
                   bits=(16, 2, 2, 4), group=(32, 32, 16, 32), rotate=(0, 1, 1, 1), alpha_mode=(0, 3, 0, 3),
                   sigma=(0.3, 0.2, 0.1), anchor_policy=1, seed=13),
    # anchor intervals 2 x [2^3, 4] ([RQ] Table 8), INT4 and bf16 anchors
    synth.Workload(name="anchor_interval_2x4", num_loops=8, batch=2, kv_heads=2, q_heads=2, context=33,
                   bits=(2, 2, 2, 4, 2, 2, 2, 16), group=(16, 32, 32, 32, 32, 16, 32, 32),
                   rotate=(1, 1, 1, 0, 1, 1, 0, 0), alpha_mode=(0, 0, 3, 0, 0, 1, 0, 0),
                   sigma=(0.3, 0.25, 0.2, 0.15, 0.1, 0.1, 0.05), anchor_policy=2, anchor_interval=4, seed=14),
    # chained references ([RQ] Table 9: Next-loop with [2,2,2,4]-style formats, Previous-loop with [4,2,2,2]):
    # each loop is stored against its neighbour's binary32 reconstruction
    synth.Workload(name="next_loop_chain", batch=2, kv_heads=3, q_heads=3, context=45,
                   bits=(2, 2, 2, 16), group=(32,) * 4, rotate=(1, 1, 1, 0), alpha_mode=(0, 3, 1, 0),
                   sigma=(0.3, 0.2, 0.1), outlier_p=0.02, anchor_policy=4, seed=15),
    synth.Workload(name="previous_loop_chain_int4", batch=2, kv_heads=2, q_heads=2, context=70,
                   bits=(4, 2, 2, 2), group=(32, 16, 16, 16), rotate=(0, 1, 1, 1),
                   sigma=(0.3, 0.2, 0.1), outlier_p=0.02, anchor_policy=3, seed=16),
    synth.Workload(name="next_loop_chain_int4_unrotated", batch=1, kv_heads=2, q_heads=2, context=33,
                   bits=(4, 4, 4, 4), group=(32,) * 4, rotate=(0, 0, 0, 0), sigma=(0.3, 0.2, 0.1),
                   anchor_policy=4, seed=17),
]


def _cache(wl, rq):
    return rq.Cache(rq.config_from_dict(synth.cache_config_dict(wl)), device="cuda")


@pytest.mark.parametrize("wl", CASES, ids=lambda w: w.name)
def test_encode_bit_exact(librq, wl):
    rq = librq
    inp = synth.make_inputs(wl, "cpu")
    cache = _cache(wl, rq)
    cache.encode(inp["k"].cuda(), inp["v"].cuda())
    assert cache.get_error() == 0
    planes = read_planes(cache, wl.context)
    enc = oracle_encode(inp, synth.cache_config_dict(wl))
    assert not enc.error
    stats = compare_encoded(planes, enc)
    assert stats["near_tie_diff"] <= stats["near_tie"]


@pytest.mark.parametrize("wl", CASES, ids=lambda w: w.name)
def test_reconstruct_within_tolerance(librq, wl):
    rq = librq
    inp = synth.make_inputs(wl, "cpu")
    cache = _cache(wl, rq)
    cache.encode(inp["k"].cuda(), inp["v"].cuda())
    enc = oracle_encode(inp, synth.cache_config_dict(wl))
    for loop in range(wl.num_loops):
        kg, vg = cache.reconstruct(loop, 0, wl.context)
        ko, vo = O.reconstruct_f64(enc, loop)
        for got, want in ((kg, ko), (vg, vo)):
            err = rel_err_rows(got.cpu().numpy(), want)
            assert err.max() <= RECON_TOL, (loop, float(err.max()))


def test_append_with_device_positions_matches_prefill(librq):
    rq = librq
    wl = synth.Workload(name="append", batch=3, kv_heads=2, q_heads=2, context=70, bits=(2, 2, 4, 4),
                        sigma=(0.3, 0.2, 0.1), seed=9)
    inp = synth.make_inputs(wl, "cpu")
    k, v = inp["k"].cuda(), inp["v"].cuda()
    cache = _cache(wl, rq)
    T = wl.context
    cache.encode(k[:, :, :, :T - 5].contiguous(), v[:, :, :, :T - 5].contiguous(), start_pos=0)
    cache.encode(k[:, :, :, T - 5:T - 3], v[:, :, :, T - 5:T - 3], start_pos=T - 5)  # strided views
    for i in range(T - 3, T):
        pos = torch.full((wl.batch,), i, dtype=torch.int32, device="cuda")
        cache.encode(k[:, :, :, i:i + 1], v[:, :, :, i:i + 1], positions=pos)
    assert cache.get_error() == 0
    compare_encoded(read_planes(cache, T), oracle_encode(inp, synth.cache_config_dict(wl)))


def test_ragged_append_positions(librq):
    """Each sequence appends at its own position."""
    rq = librq
    wl = synth.Workload(name="ragged_append", batch=3, kv_heads=1, q_heads=1, context=40, seed=10)
    inp = synth.make_inputs(wl, "cpu")
    k, v = inp["k"].cuda(), inp["v"].cuda()
    cache = _cache(wl, rq)
    cache.encode(k, v)
    before = read_planes(cache, wl.context)
    # overwrite position p_b of sequence b with token j=5's data
    pos = torch.tensor([3, 17, 39], dtype=torch.int32, device="cuda")
    cache.encode(k[:, :, :, 5:6], v[:, :, :, 5:6], positions=pos)
    after = read_planes(cache, wl.context)
    for b, p in enumerate([3, 17, 39]):
        for l in range(wl.num_loops - 1):
            codes_after = after["loops"][l]["k"][0][b, 0, p]
            codes_src = before["loops"][l]["k"][0][b, 0, 5]
            assert np.array_equal(codes_after, codes_src)
        untouched = [t for t in range(wl.context) if t != p]
        assert np.array_equal(after["loops"][0]["k"][0][b, 0, untouched], before["loops"][0]["k"][0][b, 0, untouched])


def test_capacity_errors(librq):
    rq = librq
    wl = synth.Workload(name="cap", batch=1, kv_heads=1, q_heads=1, context=8, n_tail=0, seed=11)
    inp = synth.make_inputs(wl, "cpu")
    cache = _cache(wl, rq)  # capacity 8
    k, v = inp["k"].cuda(), inp["v"].cuda()
    with pytest.raises(rq.RQError) as e:
        cache.encode(k, v, start_pos=1)
    assert e.value.status == rq.ERR_CAPACITY
    pos = torch.tensor([5], dtype=torch.int32, device="cuda")
    cache.encode(k, v, positions=pos)  # tokens 3..7 would land past capacity: dropped, flagged
    assert cache.get_error() & rq.FLAG_POSITION
    assert cache.get_error() == 0  # reading clears


def test_non_finite_input_sets_device_flag(librq):
    rq = librq
    wl = synth.Workload(name="nan", batch=1, kv_heads=1, q_heads=1, context=4, seed=12)
    inp = synth.make_inputs(wl, "cpu")
    k = inp["k"].clone()
    k[1, 0, 0, 2, 7] = float("nan")
    cache = _cache(wl, rq)
    cache.encode(k.cuda(), inp["v"].cuda())
    assert cache.get_error() & rq.FLAG_BAD_INPUT
    k[1, 0, 0, 2, 7] = 1e5  # beyond the fp16 range of the metadata
    cache.encode(k.cuda(), inp["v"].cuda())
    assert cache.get_error() & rq.FLAG_BAD_INPUT


@pytest.mark.parametrize("policy", [0, 4])
def test_degenerate_vectors_bit_exact(librq, policy):
    """Zero anchor vectors (alpha = 0), exact multiples of the reference (zero
    residual, zero scale, codes 0), constant vectors (min = max) and signed
    zeros, under the Last-loop and the Next-loop policies: the GPU matches the
    oracle bit for bit and decodes within tolerance."""
    rq = librq
    wl = synth.Workload(name=f"degenerate_{policy}", batch=2, kv_heads=2, q_heads=2, context=9,
                        sigma=(0.3, 0.2, 0.1), anchor_policy=policy, seed=18)
    inp = synth.make_inputs(wl, "cpu")
    k, v = inp["k"].clone(), inp["v"].clone()
    k[3, 0, 0, 0] = 0.0                       # zero anchor vector
    k[:3, 0, 0, 0] = 0.5                      # constant loops against it
    k[2, 0, 1, 1] = k[3, 0, 1, 1] * 2         # exact multiple of the anchor
    k[1, 0, 1, 1] = k[2, 0, 1, 1] * -0.5      # ... and of the neighbour (Next-loop)
    v[:, 1, 0, 2] = -0.0                      # signed zeros everywhere
    v[0, 1, 1, 3] = 1.25                      # one constant vector
    cfgd = synth.cache_config_dict(wl)
    cache = rq.Cache(rq.config_from_dict(cfgd), device="cuda")
    cache.encode(k.cuda(), v.cuda())
    assert cache.get_error() == 0
    planes = read_planes(cache, wl.context)
    enc = O.encode_fp32emu(to_np32(k), to_np32(v), O.CacheConfig.from_dict(cfgd))
    assert not enc.error
    compare_encoded(planes, enc)
    ctx = inp["ctx_len"]
    for loop in range(wl.num_loops):
        out = cache.decode_attention(loop, inp["q"][loop].cuda(), ctx.cuda(), inp["k_tail"][loop].cuda(),
                                     inp["v_tail"][loop].cuda())
        torch.cuda.synchronize()
        want = O.decode_attention_f64(enc, loop, to_np32(inp["q"][loop]), ctx.numpy(),
                                      to_np32(inp["k_tail"][loop]), to_np32(inp["v_tail"][loop]))
        assert rel_err_rows(out.cpu().numpy(), want).max() <= 2e-3
