"""rq_decode_attention_static_scratch: decode attention for callers that cannot
allocate device memory (for example code running inside a framework that owns
every allocation, or serving loops that must not call cudaMalloc once they are
running).  It keeps its split-K partials in the library's own fixed-size
device array instead of a caller workspace.

The test calls it through the C ABI twice in a row on each cache and checks
each output against rq_decode_attention (same kernels on the same grid, caller
workspace): the two must agree bit for bit, and both must match the float64
oracle within the attention tolerance of the other parity tests.  It lives in
a file of its own that pytest collects last and passes both alone and after
the other tests."""
import ctypes as C

import numpy as np
import pytest
import torch

import oracle.rq_oracle as O
from looped_transformer_decode_rq_b200 import synth
from tests.helpers import ATTN_TOL, oracle_encode, rel_err_rows, to_np32

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("q_heads", [8, 32])
def test_static_scratch_matches_workspace_entry_point_twice(librq, q_heads):
    """q_heads / kv_heads = 2 (the CUDA-core kernel) and 8 (the largest group:
    the tensor-core kernel's 8-row variant)."""
    rq = librq
    wl = synth.Workload(name="static_scratch", batch=3, kv_heads=4, q_heads=q_heads, context=700,
                        lengths=(700, 65, 333), sigma=(0.3, 0.2, 0.1), outlier_p=0.01, seed=77)
    inp = synth.make_inputs(wl, "cpu")
    cfgd = synth.cache_config_dict(wl)
    cache = rq.Cache(rq.config_from_dict(cfgd), device="cuda")
    assert cache.workspace.numel() <= rq.STATIC_SCRATCH_BYTES
    cache.encode(inp["k"].cuda(), inp["v"].cuda())
    enc = oracle_encode(inp, cfgd)
    ctx = inp["ctx_len"].cuda()
    lib = rq.lib()
    stream = torch.cuda.current_stream().cuda_stream
    # two calls in a row: a residual loop, then the reference loop with other queries
    for loop in (1, 3):
        q = inp["q"][loop].cuda()
        kt, vt = inp["k_tail"][loop].cuda(), inp["v_tail"][loop].cuda()
        want = cache.decode_attention(loop, q, ctx, kt, vt)
        got = torch.full_like(want, float("nan"))
        st = lib.rq_decode_attention_static_scratch(cache.handle, loop, q.data_ptr(), ctx.data_ptr(),
                                                    kt.data_ptr(), vt.data_ptr(), kt.shape[2],
                                                    C.c_float(128 ** -0.5), got.data_ptr(), stream)
        assert st == rq.OK, lib.rq_last_error_message()
        torch.cuda.synchronize()
        assert torch.isfinite(got).all()
        assert torch.equal(got, want)
        oracle = O.decode_attention_f64(enc, loop, to_np32(inp["q"][loop]), inp["ctx_len"].numpy(),
                                        to_np32(inp["k_tail"][loop]), to_np32(inp["v_tail"][loop]))
        assert rel_err_rows(got.cpu().numpy(), oracle).max() <= ATTN_TOL
    assert cache.get_error() == 0


def test_static_scratch_rejects_caches_beyond_its_size(librq):
    rq = librq
    # (128*8 + SMs) slots x 8 heads x 1040 B > 4 MiB
    cfg = rq.config_from_dict(dict(num_loops=2, batch=128, kv_heads=8, q_heads=64, capacity=64,
                                   bits=[2, 16], group=[32, 32], rotate=[1, 0], alpha_mode=[0, 0]))
    cache = rq.Cache(cfg, device="cuda")
    assert cache.workspace.numel() > rq.STATIC_SCRATCH_BYTES
    q = torch.zeros((128, 64, 128), dtype=torch.bfloat16, device="cuda")
    ctx = torch.zeros((128,), dtype=torch.int32, device="cuda")
    out = torch.empty((128, 64, 128), dtype=torch.float32, device="cuda")
    st = rq.lib().rq_decode_attention_static_scratch(cache.handle, 0, q.data_ptr(), ctx.data_ptr(), None, None, 0,
                                                     C.c_float(0.088), out.data_ptr(), None)
    assert st == rq.ERR_WORKSPACE
    assert b"static scratch" in rq.lib().rq_last_error_message()
