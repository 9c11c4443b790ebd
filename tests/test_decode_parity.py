"""GPU decode attention vs the float64 oracle: max over (b, q-head) of
||o - o_ref||_inf / ||o_ref||_inf <= 2e-3, on shapes that span several pages,
several CTAs and ragged tails, for every reference/residual format."""
import numpy as np
import pytest
import torch

import oracle.rq_oracle as O
from looped_transformer_decode_rq_b200 import synth
from tests.helpers import ATTN_TOL, compare_encoded, oracle_encode, rel_err_rows, to_np32

pytestmark = pytest.mark.gpu


def run_case(rq, wl, loops=None, n_tail=None, lengths=None, scale=None, kernel=None):
    if n_tail is not None:
        wl = wl.with_(n_tail=n_tail)
    if lengths is not None:
        wl = wl.with_(lengths=tuple(lengths))
    inp = synth.make_inputs(wl, "cpu")
    cfgd = synth.cache_config_dict(wl)
    cache = rq.Cache(rq.config_from_dict(cfgd), device="cuda")
    if kernel is not None:
        cache.set_decode_kernel(kernel)
    cache.encode(inp["k"].cuda(), inp["v"].cuda())
    enc = oracle_encode(inp, cfgd)
    ctx = inp["ctx_len"]
    worst = 0.0
    for loop in (loops if loops is not None else range(wl.num_loops)):
        kt = inp["k_tail"][loop].cuda() if wl.n_tail else None
        vt = inp["v_tail"][loop].cuda() if wl.n_tail else None
        out = cache.decode_attention(loop, inp["q"][loop].cuda(), ctx.cuda(), kt, vt, softmax_scale=scale)
        torch.cuda.synchronize()
        want = O.decode_attention_f64(enc, loop, to_np32(inp["q"][loop]), ctx.numpy(),
                                      to_np32(inp["k_tail"][loop]) if wl.n_tail else None,
                                      to_np32(inp["v_tail"][loop]) if wl.n_tail else None,
                                      scale if scale is not None else 1 / np.sqrt(128))
        got = out.cpu().numpy()
        empty = (ctx.numpy() == 0) & (wl.n_tail == 0)
        if empty.any():
            assert np.all(got[empty] == 0)
        keep = ~empty
        if keep.any():
            err = rel_err_rows(got[keep], want[keep])
            worst = max(worst, float(err.max()))
            assert err.max() <= ATTN_TOL, (wl.name, loop, float(err.max()))
    assert cache.get_error() == 0
    return worst


def test_tiny_all_loops(librq):
    run_case(librq, synth.tiny())


@pytest.mark.parametrize("G", [1, 2, 4, 8])
def test_ragged_batch_gqa(librq, G):
    wl = synth.Workload(name=f"ragged_G{G}", batch=4, kv_heads=2, q_heads=2 * G, context=257,
                        sigma=(0.3, 0.2, 0.1), outlier_p=0.02, seed=20 + G)
    run_case(librq, wl, lengths=[1, 31, 257, 33])


@pytest.mark.parametrize("bits,group,ref_bits", [
    ((2, 2, 2), 16, 16), ((4, 4, 4), 32, 16), ((4, 4, 4), 16, 16),
    ((2, 2, 4), 32, 4), ((2, 2, 2), 16, 4),
])
def test_formats(librq, bits, group, ref_bits):
    wl = synth.Workload(name=f"fmt_{bits}_{group}_{ref_bits}", batch=3, kv_heads=2, q_heads=4, context=130,
                        bits=tuple(bits) + (ref_bits,), group=(group,) * 3 + (32,),
                        sigma=(0.3, 0.2, 0.1), outlier_p=0.02, seed=31)
    run_case(librq, wl, lengths=[64, 65, 130], n_tail=2)


def test_direct_and_unrotated_modes(librq):
    wl = synth.Workload(name="modes", batch=2, kv_heads=2, q_heads=2, context=100,
                        rotate=(0, 1, 0, 0), alpha_mode=(2, 1, 0, 0), sigma=(0.3, 0.2, 0.1), seed=32)
    run_case(librq, wl, lengths=[100, 37])


def test_empty_contexts_and_tail_only(librq):
    wl = synth.Workload(name="empty", batch=3, kv_heads=2, q_heads=4, context=70, seed=33)
    run_case(librq, wl, lengths=[0, 70, 0], n_tail=1)
    run_case(librq, wl, lengths=[0, 0, 0], n_tail=0)
    run_case(librq, wl, lengths=[0, 0, 0], n_tail=3)


def test_many_pages_many_ctas(librq):
    """Enough pages that every CTA of the persistent grid spans segment borders."""
    wl = synth.Workload(name="long", batch=2, kv_heads=4, q_heads=8, context=3001, sigma=(0.3, 0.2, 0.1),
                        outlier_p=0.01, seed=34)
    run_case(librq, wl, lengths=[3001, 1777], loops=[0, 3])


def test_softmax_scale_parameter(librq):
    wl = synth.Workload(name="scale", batch=1, kv_heads=2, q_heads=2, context=90, seed=35)
    run_case(librq, wl, scale=0.3, loops=[0, 3])


def test_ctx_len_beyond_capacity_is_clamped_and_flagged(librq):
    rq = librq
    wl = synth.Workload(name="clamp", batch=2, kv_heads=1, q_heads=1, context=64, n_tail=0, seed=36)
    inp = synth.make_inputs(wl, "cpu")
    cfgd = synth.cache_config_dict(wl)  # capacity 64
    cache = rq.Cache(rq.config_from_dict(cfgd), device="cuda")
    cache.encode(inp["k"].cuda(), inp["v"].cuda())
    ctx = torch.tensor([64, 1000], dtype=torch.int32, device="cuda")
    out = cache.decode_attention(0, inp["q"][0].cuda(), ctx)
    assert cache.get_error() & rq.FLAG_CTX_LEN
    enc = oracle_encode(inp, cfgd)
    want = O.decode_attention_f64(enc, 0, to_np32(inp["q"][0]), np.array([64, 64]))
    assert rel_err_rows(out.cpu().numpy(), want).max() <= ATTN_TOL


@pytest.mark.parametrize("G,lens", [(1, [200, 1, 64]), (4, [129, 0, 300])])
def test_bf16_cache_baseline(librq, G, lens):
    rq = librq
    wl = synth.Workload(name="bf16", batch=3, kv_heads=2, q_heads=2 * G, context=300, seed=37, n_tail=1)
    inp = synth.make_inputs(wl, "cpu")
    ctx = torch.tensor(lens, dtype=torch.int32)
    for loop in (0, 3):
        # strided view: the cache tensor has extra capacity and a head-major layout
        big = torch.zeros((wl.batch, wl.kv_heads, 320, 128), dtype=torch.bfloat16)
        big[:, :, :300] = inp["k"][loop]
        bigv = torch.zeros_like(big)
        bigv[:, :, :300] = inp["v"][loop]
        out = rq.bf16_decode_attention(big.cuda(), bigv.cuda(), inp["q"][loop].cuda(), ctx.cuda(),
                                       inp["k_tail"][loop].cuda(), inp["v_tail"][loop].cuda())
        want = O.attention_f64(to_np32(inp["q"][loop]), to_np32(inp["k"][loop]), to_np32(inp["v"][loop]),
                               ctx.numpy(), to_np32(inp["k_tail"][loop]), to_np32(inp["v_tail"][loop]))
        assert rel_err_rows(out.cpu().numpy(), want).max() <= ATTN_TOL


@pytest.mark.parametrize("policy,interval,L,bits,alpha", [
    (1, 0, 4, (16, 2, 2, 4), (0, 0, 3, 0)),                        # First-loop, norm ratio on loop 2
    (2, 4, 8, (2, 2, 2, 4, 2, 2, 4, 16), (0,) * 8),                # 2 x [2,2,2,4]-style blocks
    (2, 3, 7, (2, 2, 4, 2, 2, 4, 4), (0, 3, 0, 0, 1, 0, 0)),       # short last block [2, 4]
])
def test_anchor_policies(librq, policy, interval, L, bits, alpha):
    rot = tuple(0 if b in (16,) else 1 for b in bits)
    wl = synth.Workload(name=f"anchors_{policy}_{interval}", num_loops=L, batch=2, kv_heads=2, q_heads=4,
                        context=150, bits=bits, group=(32,) * L, rotate=rot, alpha_mode=alpha,
                        sigma=tuple(0.1 + 0.03 * i for i in range(L - 1)), anchor_policy=policy,
                        anchor_interval=interval, outlier_p=0.01, seed=40 + policy + interval)
    run_case(librq, wl, lengths=[150, 70])


@pytest.mark.parametrize("policy,bits,group,G", [
    (4, (2, 2, 2, 16), (32,) * 4, 1),          # Next-loop, bf16 anchor, INT2 g=32
    (4, (2, 2, 2, 4), (32,) * 4, 4),           # Next-loop, INT4 anchor ([RQ] Table 9's [2,2,2,4])
    (3, (4, 2, 2, 2), (32, 16, 16, 16), 2),    # Previous-loop, INT4 anchor ([4,2,2,2]), INT2 g=16
    (3, (16, 4, 4, 4), (32,) * 4, 8),          # Previous-loop, bf16 anchor, INT4 links
    (4, (2, 2, 2, 4), (32,) * 4, 1),           # INT4-anchor chains at G = 1 run three consumer groups
    (3, (4, 2, 2, 2), (32, 16, 16, 16), 1),
])
def test_chained_policies(librq, policy, bits, group, G):
    """Previous-/Next-loop references ([RQ] Table 9): a loop one, two or three
    links from its anchor is decoded from every link's codes."""
    anchor = 0 if policy == 3 else 3
    rot = tuple(0 if l == anchor else 1 for l in range(4))
    wl = synth.Workload(name=f"chain_{policy}_{G}", batch=3, kv_heads=2, q_heads=2 * G, context=300, bits=bits,
                        group=group, rotate=rot, sigma=(0.3, 0.2, 0.1), outlier_p=0.01, anchor_policy=policy,
                        seed=60 + policy + G)
    run_case(librq, wl, lengths=[300, 129, 1])


@pytest.mark.parametrize("policy,bits,group,G,loops", [
    (4, (2, 2, 2, 4), (32,) * 4, 4, [0, 1, 2, 3]),    # Next-loop [2,2,2,4]: 3, 2 and 1 links, and the anchor
    (4, (2, 2, 2, 4), (32,) * 4, 8, [1, 2, 3]),       # 8 rows: two links (value sums over the scores)
    (3, (4, 2, 2, 2), (32, 16, 16, 16), 4, [1, 2]),   # Previous-loop, INT2 g=16 links: 1 and 2 links
    (4, (4, 4, 4, 4), (32,) * 4, 4, [1, 2]),          # INT4 links: 2 and 1 links
])
def test_chained_loops_on_the_tensor_cores(librq, policy, bits, group, G, loops):
    """Chained (Previous-/Next-loop) INT4-anchor loops on the tensor-core
    kernel: every link's keys are scored against the one rotated query and
    combined by Horner's rule from the anchor outward, every link's values go
    into the one rotated accumulator with signed weights.  Forced onto the
    tensor cores against the float64 oracle; the automatic choice takes them
    from 4 rows (three links at 8 rows as two 4-row passes)."""
    rq = librq
    anchor = 0 if policy == 3 else 3
    rot = tuple(0 if l == anchor else 1 for l in range(4))
    wl = synth.Workload(name=f"chain_tc_{policy}_{G}", batch=3, kv_heads=2, q_heads=2 * G, context=300, bits=bits,
                        group=group, rotate=rot, sigma=(0.3, 0.2, 0.1), outlier_p=0.01, anchor_policy=policy,
                        seed=90 + policy + G)
    run_case(rq, wl, lengths=[300, 129, 1], loops=loops, kernel=rq.DECODE_KERNEL_TENSOR)
    cache = rq.Cache(rq.config_from_dict(synth.cache_config_dict(wl)), device="cuda")
    for l in loops:
        kernel, rows = cache.decode_plan(l, 1)
        assert kernel == rq.DECODE_KERNEL_TENSOR and rows == G, (l, kernel, rows)
    if G == 8 and anchor == 3:
        assert cache.decode_plan(0, 1) == (rq.DECODE_KERNEL_TENSOR, 4)  # three links: two 4-row passes


def test_chained_loops_run_on_the_cuda_core_kernel(librq):
    """With a bf16 anchor the tensor-core kernel decodes the anchor and the
    loop next to it (one link) but reports a longer chain as unsupported; the
    default then picks the CUDA-core kernel."""
    rq = librq
    wl = synth.Workload(name="chain_tc", batch=2, kv_heads=2, q_heads=8, context=260, sigma=(0.3, 0.2, 0.1),
                        anchor_policy=4, seed=66)
    run_case(rq, wl, loops=[2, 3], kernel=rq.DECODE_KERNEL_TENSOR)
    cache = rq.Cache(rq.config_from_dict(synth.cache_config_dict(wl)), device="cuda")
    inp = synth.make_inputs(wl, "cpu")
    cache.set_decode_kernel(rq.DECODE_KERNEL_TENSOR)
    with pytest.raises(rq.RQError) as e:
        cache.decode_attention(0, inp["q"][0].cuda(), inp["ctx_len"].cuda())
    assert e.value.status == rq.ERR_UNSUPPORTED
    run_case(rq, wl, loops=[0, 1])


OUTLIER_FORMATS = {"bf16ref_int2": ((2, 2, 2, 16), (32,) * 4), "int4anchor_2244": ((2, 2, 4, 4), (32,) * 4),
                   "int4anchor_int4g16": ((4, 4, 4, 4), (16, 16, 16, 32)),
                   "bf16ref_int4g16": ((4, 2, 4, 16), (16, 32, 16, 32))}


@pytest.mark.parametrize("G", [1, 2, 4])
@pytest.mark.parametrize("fmt", sorted(OUTLIER_FORMATS))
def test_outlier_query_channels(librq, fmt, G):
    """Queries with a few large channels (2% of elements at 30-100x) on the
    CUDA-core kernels: the INT4 anchor's unrotated query keeps 24 bits per
    lane, so the other channels keep their precision; the residual's rotated
    query has no outliers left to lose it to."""
    bits, group = OUTLIER_FORMATS[fmt]
    wl = synth.Workload(name=f"qout_{fmt}_{G}", batch=3, kv_heads=2, q_heads=2 * G, context=300, bits=bits,
                        group=group, sigma=(0.3, 0.2, 0.1), outlier_p=0.01, q_outlier_p=0.02, seed=170 + G)
    run_case(librq, wl, lengths=[300, 129, 1], n_tail=1, kernel=librq.DECODE_KERNEL_SIMT)


@pytest.mark.parametrize("n_tail", [64, 127])
def test_recent_window_bf16_tail(librq, n_tail):
    """A window of the most recent 64-127 tokens kept in bf16 next to the compact
    cache ([RQ] Table 10: "Recent 64" / "Recent 64-127" bf16 KV tokens)."""
    wl = synth.Workload(name=f"tail{n_tail}", batch=2, kv_heads=2, q_heads=4, context=200, bits=(2, 2, 4, 4),
                        sigma=(0.3, 0.2, 0.1), outlier_p=0.01, seed=50 + n_tail)
    run_case(librq, wl, lengths=[200, 0], n_tail=n_tail)


# ---------------------------------------------------------------------------
# both decode kernels on the same cases: the CUDA-core kernel (64-token pages)
# and the tensor-core kernel (128-token pages, G in {1, 2, 4, 8})
# ---------------------------------------------------------------------------
TC_FORMATS = {
    # name: (bits, group, rotate, alpha_mode, G values)
    "bf16ref_int2g32_int4g32": ((2, 4, 2, 16), (32, 32, 32, 32), (1, 1, 1, 0), (0, 0, 3, 0), (1, 2, 4)),
    "bf16ref_int2g32": ((2, 2, 2, 16), (32, 32, 32, 32), (1, 1, 1, 0), (0, 3, 1, 0), (8,)),
    "bf16ref_int2g16": ((2, 2, 2, 16), (16, 16, 16, 32), (1, 1, 0, 0), (0, 1, 0, 0), (1, 2, 4)),
    "int4anchor_int2g32_int4g16": ((2, 4, 2, 4), (32, 16, 16, 32), (1, 1, 1, 0), (0, 0, 3, 0), (1, 2, 4)),
    "int4anchor_2244_g32": ((2, 2, 4, 4), (32, 32, 32, 32), (1, 1, 1, 0), (0, 3, 0, 0), (1, 8)),
    "no_anchor_term": ((2, 4, 2, 16), (32, 32, 16, 32), (1, 0, 1, 0), (2, 2, 2, 0), (1, 2, 4, 8)),
}


@pytest.mark.parametrize("kernel", ["simt", "tensor"])
@pytest.mark.parametrize("fmt", sorted(TC_FORMATS))
def test_both_kernels_formats_and_pages(librq, fmt, kernel):
    """Every loop of the format (residual loops and the anchor loop) at each G the
    tensor-core kernel implements, over 0, 1, 127, 128, 129 and 300 cached tokens
    (several 128-token pages, partial pages and a partial last record block)."""
    rq = librq
    bits, group, rotate, alpha, Gs = TC_FORMATS[fmt]
    for G in Gs:
        wl = synth.Workload(name=f"{fmt}_G{G}", batch=6, kv_heads=2, q_heads=2 * G, context=300, bits=bits,
                            group=group, rotate=rotate, alpha_mode=alpha, sigma=(0.3, 0.2, 0.1), outlier_p=0.02,
                            seed=60 + G)
        k = rq.DECODE_KERNEL_SIMT if kernel == "simt" else rq.DECODE_KERNEL_TENSOR
        run_case(rq, wl, lengths=[300, 0, 128, 1, 129, 127], n_tail=2, kernel=k)


@pytest.mark.parametrize("G", [4, 8])
def test_tensor_kernel_many_pages(librq, G):
    """Enough 128-token pages that every CTA of the persistent grid spans
    segment borders, with ragged lengths."""
    wl = synth.Workload(name=f"tc_long_G{G}", batch=3, kv_heads=4, q_heads=4 * G, context=5000,
                        sigma=(0.3, 0.2, 0.1), outlier_p=0.01, seed=70 + G)
    run_case(librq, wl, lengths=[5000, 2222, 129], loops=[0, 3], kernel=librq.DECODE_KERNEL_TENSOR)


def test_tensor_kernel_rejects_unimplemented(librq):
    """INT4 anchor with 16-dim residual groups at G = 8 needs more tensor memory
    than the tensor-core kernel has: that kernel reports it, the default picks
    the CUDA-core kernel."""
    rq = librq
    wl = synth.Workload(name="tc_unsupported", batch=1, kv_heads=2, q_heads=16, context=64, bits=(2, 2, 4, 4),
                        group=(16, 32, 32, 32), seed=80)
    cache = rq.Cache(rq.config_from_dict(synth.cache_config_dict(wl)), device="cuda")
    inp = synth.make_inputs(wl, "cpu")
    cache.set_decode_kernel(rq.DECODE_KERNEL_TENSOR)
    with pytest.raises(rq.RQError) as e:
        cache.decode_attention(0, inp["q"][0].cuda(), inp["ctx_len"].cuda())
    assert e.value.status == rq.ERR_UNSUPPORTED
    cache.set_decode_kernel(rq.DECODE_KERNEL_AUTO)
    cache.encode(inp["k"].cuda(), inp["v"].cuda())
    out = cache.decode_attention(0, inp["q"][0].cuda(), inp["ctx_len"].cuda())
    torch.cuda.synchronize()
    enc = oracle_encode(inp, synth.cache_config_dict(wl))
    want = O.decode_attention_f64(enc, 0, to_np32(inp["q"][0]), inp["ctx_len"].numpy())
    assert rel_err_rows(out.cpu().numpy(), want).max() <= ATTN_TOL


@pytest.mark.parametrize("kernel", ["simt", "tensor", "tensor_g8", "simt_int4_anchor_g1", "tensor_int4_anchor_g1",
                                    "tensor_int4_anchor_g4", "tensor_chain_g4", "simt_chain_g1"])
def test_wait_limit_sets_flag_and_context_recovers(librq, kernel):
    """Failure path without a fault: the producers wait on a barrier nothing
    arrives at (test hook); every wait gives up after its limit, the call sets
    FLAG_PIPE_TIMEOUT and returns, and the next call on the same context is
    correct.  The int4_anchor_g1 cases are the byte-plane kernels (INT4 anchor,
    one query row per kv-head) on the CUDA cores and on the tensor cores; the
    two after them the tensor-core kernel with its register split (INT4 anchor,
    4 rows) and with a three-link chain; tensor_g8 the tensor-core kernel whose
    stages refill their key and value halves separately (bf16 anchor, 8 rows);
    simt_chain_g1 the byte-plane CUDA-core kernel with its register split (one
    row, three links)."""
    import time
    rq = librq
    wl = synth.Workload(name="stall", batch=2, kv_heads=2, q_heads=8, context=300, seed=90)
    if kernel.endswith("int4_anchor_g1"):
        wl = wl.with_(q_heads=2, bits=(2, 2, 4, 4))
    elif kernel.endswith("int4_anchor_g4"):
        wl = wl.with_(bits=(2, 2, 4, 4))
    elif kernel.endswith("chain_g4"):
        wl = wl.with_(bits=(2, 2, 2, 4), anchor_policy=4)  # loop 0 is three links from the anchor
    elif kernel.endswith("chain_g1"):
        wl = wl.with_(q_heads=2, bits=(2, 2, 2, 4), anchor_policy=4)
    elif kernel.endswith("_g8"):
        wl = wl.with_(q_heads=16)
    inp = synth.make_inputs(wl, "cpu")
    cfgd = synth.cache_config_dict(wl)
    cache = rq.Cache(rq.config_from_dict(cfgd), device="cuda")
    cache.set_decode_kernel(rq.DECODE_KERNEL_TENSOR if kernel.startswith("tensor") else rq.DECODE_KERNEL_SIMT)
    cache.encode(inp["k"].cuda(), inp["v"].cuda())
    assert cache.get_error() == 0
    q, ctx = inp["q"][0].cuda(), inp["ctx_len"].cuda()
    kt, vt = inp["k_tail"][0].cuda(), inp["v_tail"][0].cuda()
    with pytest.raises(rq.RQError):
        cache.set_debug_stall(-2)
    cache.set_debug_stall(0)
    t0 = time.time()
    cache.decode_attention(0, q, ctx, kt, vt)
    flags = cache.get_error()
    assert flags & rq.FLAG_PIPE_TIMEOUT
    assert time.time() - t0 < 60
    cache.set_debug_stall(-1)
    out = cache.decode_attention(0, q, ctx, kt, vt)
    torch.cuda.synchronize()
    assert cache.get_error() == 0
    enc = oracle_encode(inp, cfgd)
    want = O.decode_attention_f64(enc, 0, to_np32(inp["q"][0]), inp["ctx_len"].numpy(),
                                  to_np32(inp["k_tail"][0]), to_np32(inp["v_tail"][0]))
    assert rel_err_rows(out.cpu().numpy(), want).max() <= ATTN_TOL


def _same_planes(a, b):
    if isinstance(a, dict):
        assert a.keys() == b.keys()
        for key in a:
            _same_planes(a[key], b[key])
    elif isinstance(a, (list, tuple)):
        assert len(a) == len(b)
        for x, y in zip(a, b):
            _same_planes(x, y)
    elif a is None:
        assert b is None
    else:
        assert np.array_equal(np.ascontiguousarray(a).view(np.uint8), np.ascontiguousarray(b).view(np.uint8))


@pytest.mark.parametrize("kernel", ["simt", "tensor"])
@pytest.mark.parametrize("bits,policy", [((2, 2, 2, 16), 0), ((2, 2, 4, 4), 0), ((2, 2, 2, 16), 4)])
def test_decode_with_fused_append_matches_separate_calls(librq, kernel, bits, policy):
    """rq_decode_attention_append (the final loop's decode plus the per-step
    append of every loop's new token, one combine launch) gives the same output
    and the same cache bytes as a decode followed by an encode at device positions."""
    from tests.helpers import read_planes
    rq = librq
    wl = synth.Workload(name="fused_append", batch=3, kv_heads=2, q_heads=8, context=200, bits=bits,
                        sigma=(0.3, 0.2, 0.1), outlier_p=0.01, anchor_policy=policy, seed=95)
    inp = synth.make_inputs(wl, "cpu")
    cfgd = synth.cache_config_dict(wl)
    k, v = inp["k"].cuda(), inp["v"].cuda()
    caches = []
    lay = rq.cache_layout(rq.config_from_dict(cfgd))
    for _ in range(2):
        # zeroed buffers: positions neither call writes compare equal too
        c = rq.Cache(rq.config_from_dict(cfgd), buffer=torch.zeros(lay.total_bytes + 1024, dtype=torch.uint8,
                                                                    device="cuda"))
        c.set_decode_kernel(rq.DECODE_KERNEL_SIMT if kernel == "simt" else rq.DECODE_KERNEL_TENSOR)
        c.encode(k, v)
        caches.append(c)
    ctx = torch.tensor([200, 137, 5], dtype=torch.int32, device="cuda")
    last = wl.num_loops - 1
    q, kt, vt = inp["q"][last].cuda(), inp["k_tail"][last].cuda(), inp["v_tail"][last].cuda()
    k_new, v_new = inp["k_tail"].cuda(), inp["v_tail"].cuda()  # [L, B, Hkv, 1, 128]
    out_a = caches[0].decode_attention(last, q, ctx, kt, vt)
    caches[0].encode(k_new, v_new, positions=ctx)
    out_b = caches[1].decode_attention_append(last, q, ctx, kt, vt, k_new, v_new, ctx)
    torch.cuda.synchronize()
    assert caches[0].get_error() == 0 and caches[1].get_error() == 0
    assert torch.equal(out_a, out_b)
    _same_planes(read_planes(caches[0], wl.context + 1), read_planes(caches[1], wl.context + 1))
    # the fused call against the oracle: its attention output (the cache before
    # the append plus the tail) and the records it appended (the oracle's encode
    # of the new token, bit for bit)
    enc = oracle_encode(inp, cfgd)
    want = O.decode_attention_f64(enc, last, to_np32(inp["q"][last]), ctx.cpu().numpy(),
                                  to_np32(inp["k_tail"][last]), to_np32(inp["v_tail"][last]))
    assert rel_err_rows(out_b.cpu().numpy(), want).max() <= ATTN_TOL
    enc_new = O.encode_fp32emu(to_np32(inp["k_tail"]), to_np32(inp["v_tail"]), O.CacheConfig.from_dict(cfgd))
    compare_encoded(read_planes(caches[1], positions=ctx.cpu()), enc_new)


@pytest.mark.parametrize("kernel", ["simt", "tensor"])
def test_any_workspace_contents_repeated_calls_and_graph_replay(librq, kernel):
    """The workspace needs no initial contents; repeated calls and replays of a
    captured CUDA graph (split kernel, then the combine kernel as a programmatic
    dependent launch) give the same, correct output, with ragged and empty
    sequences."""
    rq = librq
    wl = synth.Workload(name="segment_combine", batch=5, kv_heads=3, q_heads=12, context=700,
                        sigma=(0.3, 0.2, 0.1), outlier_p=0.01, seed=97)
    wl = wl.with_(lengths=(700, 0, 1, 333, 64))
    inp = synth.make_inputs(wl, "cpu")
    cfgd = synth.cache_config_dict(wl)
    cache = rq.Cache(rq.config_from_dict(cfgd), device="cuda")
    cache.set_decode_kernel(rq.DECODE_KERNEL_SIMT if kernel == "simt" else rq.DECODE_KERNEL_TENSOR)
    cache.encode(inp["k"].cuda(), inp["v"].cuda())
    q, ctx = inp["q"][0].cuda(), inp["ctx_len"].cuda()
    kt, vt = inp["k_tail"][0].cuda(), inp["v_tail"][0].cuda()
    enc = oracle_encode(inp, cfgd)
    want = O.decode_attention_f64(enc, 0, to_np32(inp["q"][0]), inp["ctx_len"].numpy(),
                                  to_np32(inp["k_tail"][0]), to_np32(inp["v_tail"][0]))
    gen = torch.Generator(device="cuda").manual_seed(5)
    first = None
    for fill in ("ones", "random", "zeros"):
        if fill == "ones":
            cache.workspace.fill_(0xFF)
        elif fill == "random":
            cache.workspace.copy_(torch.randint(0, 256, cache.workspace.shape, generator=gen, device="cuda",
                                                dtype=torch.int32).to(torch.uint8))
        else:
            cache.workspace.zero_()
        for _ in range(3):
            out = cache.decode_attention(0, q, ctx, kt, vt)
            torch.cuda.synchronize()
            assert cache.get_error() == 0
            assert rel_err_rows(out.cpu().numpy(), want).max() <= ATTN_TOL, fill
            if first is None:
                first = out.clone()
            assert torch.equal(out, first), fill
    static_out = torch.zeros_like(first)
    side = torch.cuda.Stream()
    side.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(side):
        cache.decode_attention(0, q, ctx, kt, vt, out=static_out)  # warm-up outside the capture
    torch.cuda.current_stream().wait_stream(side)
    torch.cuda.synchronize()
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph):
        cache.decode_attention(0, q, ctx, kt, vt, out=static_out)
    for _ in range(3):
        static_out.zero_()
        graph.replay()
        torch.cuda.synchronize()
        assert torch.equal(static_out, first)
    del graph
    assert cache.get_error() == 0


@pytest.mark.parametrize("gq,n_q,bits,kernel", [
    (1, 2, (2, 2, 2, 16), None),          # two draft tokens on the Ouro-shaped rows: CUDA cores
    (1, 4, (2, 2, 2, 16), None),          # four rows per kv-head: tensor cores by default
    (1, 4, (2, 2, 2, 16), "simt"),
    (2, 4, (2, 2, 4, 4), None),           # GQA pairs x 4 drafts = 8 rows, INT4 anchor
    (1, 8, (2, 2, 2, 16), "simt"),
    (4, 4, (2, 2, 2, 16), None),          # 16 rows: one pass on the tensor cores
    (1, 16, (2, 2, 4, 4), None),
    (1, 4, (2, 2, 2, 16), "next_loop"),   # draft tokens on a Next-loop chained cache (CUDA cores)
    (2, 4, (2, 2, 2, 4), "next_loop"),    # 8 rows of a chain: two passes of 4 by default
])
def test_multi_query_decode(librq, gq, n_q, bits, kernel):
    """n_q draft tokens per sequence in one call: every draft token sees the
    cache, the earlier tail tokens and the draft tokens up to itself."""
    rq = librq
    wl = synth.Workload(name=f"multi_{gq}_{n_q}", batch=3, kv_heads=2, q_heads=2 * gq, context=300, bits=bits,
                        sigma=(0.3, 0.2, 0.1), outlier_p=0.01, n_tail=n_q + 1, seed=110 + n_q + gq,
                        anchor_policy=4 if kernel == "next_loop" else 0)
    wl = wl.with_(lengths=(300, 0, 129))
    inp = synth.make_inputs(wl, "cpu")
    qm = synth.draft_queries(wl, n_q, "cpu")
    cfgd = synth.cache_config_dict(wl)
    cache = rq.Cache(rq.config_from_dict(cfgd), device="cuda")
    if kernel == "simt":
        cache.set_decode_kernel(rq.DECODE_KERNEL_SIMT)
    cache.encode(inp["k"].cuda(), inp["v"].cuda())
    enc = oracle_encode(inp, cfgd)
    ctx = inp["ctx_len"]
    for loop in (0, wl.num_loops - 1):
        kt, vt = inp["k_tail"][loop], inp["v_tail"][loop]
        out = cache.decode_attention_multi(loop, qm[loop].cuda(), ctx.cuda(), kt.cuda(), vt.cuda())
        torch.cuda.synchronize()
        want = O.decode_attention_multi_f64(enc, loop, to_np32(qm[loop]), ctx.numpy(), to_np32(kt), to_np32(vt))
        err = rel_err_rows(out.cpu().numpy(), want)
        assert err.max() <= ATTN_TOL, (loop, float(err.max()))
    assert cache.get_error() == 0


@pytest.mark.parametrize("bits,rows_of_loop", [
    ((2, 2, 2, 16), {0: 16, 3: 16}),        # bf16 anchor, INT2 g=32: 16 rows in one pass
    ((2, 2, 4, 4), {0: 16, 2: 16, 3: 16}),  # INT4 anchor, INT2 and INT4 g=32 residuals
])
def test_sixteen_rows_per_pass(librq, bits, rows_of_loop):
    """4 query heads per kv-head x 4 draft tokens: where the tensor-core kernel
    has a 16-row variant the call reads each cached page once for all 16 rows
    (rq_decode_plan), and every loop matches the float64 oracle."""
    rq = librq
    gq, n_q = 4, 4
    wl = synth.Workload(name=f"rows16_{bits}", batch=2, kv_heads=2, q_heads=2 * gq, context=400, bits=bits,
                        sigma=(0.3, 0.2, 0.1), outlier_p=0.01, n_tail=n_q, seed=170 + bits[2])
    wl = wl.with_(lengths=(400, 131))
    inp = synth.make_inputs(wl, "cpu")
    qm = synth.draft_queries(wl, n_q, "cpu")
    cfgd = synth.cache_config_dict(wl)
    cache = rq.Cache(rq.config_from_dict(cfgd), device="cuda")
    cache.encode(inp["k"].cuda(), inp["v"].cuda())
    enc = oracle_encode(inp, cfgd)
    ctx = inp["ctx_len"]
    for loop, rows in rows_of_loop.items():
        assert cache.decode_plan(loop, n_q) == (rq.DECODE_KERNEL_TENSOR, rows), loop
        kt, vt = inp["k_tail"][loop], inp["v_tail"][loop]
        out = cache.decode_attention_multi(loop, qm[loop].cuda(), ctx.cuda(), kt.cuda(), vt.cuda())
        torch.cuda.synchronize()
        want = O.decode_attention_multi_f64(enc, loop, to_np32(qm[loop]), ctx.numpy(), to_np32(kt), to_np32(vt))
        err = rel_err_rows(out.cpu().numpy(), want)
        assert err.max() <= ATTN_TOL, (loop, float(err.max()))
    # forced onto the CUDA cores the same call runs in 4-row passes
    cache.set_decode_kernel(rq.DECODE_KERNEL_SIMT)
    assert cache.decode_plan(0, n_q) == (rq.DECODE_KERNEL_SIMT, 4)
    assert cache.get_error() == 0


def test_multi_query_of_one_token_is_the_single_decode(librq):
    rq = librq
    wl = synth.Workload(name="multi_one", batch=2, kv_heads=2, q_heads=4, context=200, sigma=(0.3, 0.2, 0.1),
                        seed=120)
    inp = synth.make_inputs(wl, "cpu")
    cache = rq.Cache(rq.config_from_dict(synth.cache_config_dict(wl)), device="cuda")
    cache.encode(inp["k"].cuda(), inp["v"].cuda())
    q, ctx, kt, vt = inp["q"][0].cuda(), inp["ctx_len"].cuda(), inp["k_tail"][0].cuda(), inp["v_tail"][0].cuda()
    one = cache.decode_attention(0, q, ctx, kt, vt)
    multi = cache.decode_attention_multi(0, q.unsqueeze(1).contiguous(), ctx, kt, vt)
    torch.cuda.synchronize()
    assert torch.equal(one, multi[:, 0])
    # rows per kv-head neither 1, 2, 4 nor a multiple of 8; fewer tail tokens than drafts
    q6 = torch.zeros((2, 3, 4, 128), dtype=torch.bfloat16, device="cuda")
    with pytest.raises(rq.RQError) as e:
        cache.decode_attention_multi(0, q6, ctx, kt, vt)
    assert e.value.status == rq.ERR_UNSUPPORTED
    q2 = torch.zeros((2, 2, 4, 128), dtype=torch.bfloat16, device="cuda")
    with pytest.raises(rq.RQError) as e:
        cache.decode_attention_multi(0, q2, ctx, kt, vt)
    assert e.value.status == rq.ERR_INVALID_ARG


@pytest.mark.parametrize("G,kernel", [(1, "simt"), (4, "tensor")])
def test_maximum_batch(librq, G, kernel):
    """RQ_MAX_BATCH sequences of ragged, partly empty lengths (the per-sequence
    page prefix lives in shared memory); sampled sequences against the oracle."""
    rq = librq
    B = rq.MAX_BATCH
    wl = synth.Workload(name=f"max_batch_G{G}", batch=B, kv_heads=1, q_heads=G, context=70,
                        length_range=(0, 70), sigma=(0.3, 0.2, 0.1), seed=130 + G)
    inp = synth.make_inputs(wl, "cpu")
    cfgd = synth.cache_config_dict(wl)
    cache = rq.Cache(rq.config_from_dict(cfgd), device="cuda")
    cache.set_decode_kernel(rq.DECODE_KERNEL_SIMT if kernel == "simt" else rq.DECODE_KERNEL_TENSOR)
    cache.encode(inp["k"].cuda(), inp["v"].cuda())
    ctx = inp["ctx_len"]
    idx = np.array([0, 1, 2, 511, 777, B - 2, B - 1])
    sub = O.CacheConfig.from_dict(cfgd)
    enc = O.encode_fp32emu(to_np32(inp["k"])[:, idx], to_np32(inp["v"])[:, idx], sub)
    for loop in (0, 3):
        out = cache.decode_attention(loop, inp["q"][loop].cuda(), ctx.cuda(), inp["k_tail"][loop].cuda(),
                                     inp["v_tail"][loop].cuda())
        torch.cuda.synchronize()
        want = O.decode_attention_f64(enc, loop, to_np32(inp["q"][loop])[idx], ctx.numpy()[idx],
                                      to_np32(inp["k_tail"][loop])[idx], to_np32(inp["v_tail"][loop])[idx])
        err = rel_err_rows(out.cpu().numpy()[idx], want)
        assert err.max() <= ATTN_TOL, (loop, float(err.max()))
    assert cache.get_error() == 0


def test_batch_beyond_maximum_is_refused(librq):
    rq = librq
    wl = synth.Workload(name="over_max_batch", batch=rq.MAX_BATCH + 1, kv_heads=1, q_heads=1, context=3, seed=140)
    inp = synth.make_inputs(wl, "cpu")
    cache = rq.Cache(rq.config_from_dict(synth.cache_config_dict(wl)), device="cuda")
    cache.encode(inp["k"].cuda(), inp["v"].cuda())
    with pytest.raises(rq.RQError) as e:
        cache.decode_attention(0, inp["q"][0].cuda(), inp["ctx_len"].cuda())
    assert e.value.status == rq.ERR_UNSUPPORTED
    assert cache.get_error() == 0
