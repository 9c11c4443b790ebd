"""Bit-exact check of every packed code, scale, offset and alpha of the
Ouro-shaped 8k benchmark cache (16 sequences x 16 kv-heads x 8192 tokens x 4
loops, the configuration bench.py times): the GPU encodes the whole batch in
one call; the oracle encodes each (sequence, kv-head) slab in a pool of host
processes started with spawn, and the planes are compared slab by slab.  Codes
may differ only where the oracle flags a rounding near-tie."""
import multiprocessing as mp
import os
from concurrent.futures import ProcessPoolExecutor

import pytest
import torch

import oracle.rq_oracle as O
from looped_transformer_decode_rq_b200 import synth
from tests.helpers import compare_encoded
from tests.test_fullsize_parity import _slab_planes

pytestmark = pytest.mark.gpu


def _encode_and_compare(args):
    K, V, cfgd, planes = args
    enc = O.encode_fp32emu(K, V, O.CacheConfig.from_dict(cfgd))
    assert not enc.error
    return compare_encoded(planes, enc)


def test_ouro8k_every_slab_bit_exact(librq):
    rq = librq
    wl = synth.ouro_8k()
    dev = torch.device("cuda")
    inp = synth.make_inputs(wl, dev)
    cfgd = synth.cache_config_dict(wl)
    cache = rq.Cache(rq.config_from_dict(cfgd), device=dev)
    cache.encode(inp["k"], inp["v"])
    assert cache.get_error() == 0
    n = wl.context
    workers = max(1, min(32, len(os.sched_getaffinity(0))))
    totals = {"codes": 0, "near_tie": 0, "near_tie_diff": 0, "slabs": 0}
    with ProcessPoolExecutor(max_workers=workers, mp_context=mp.get_context("spawn")) as pool:
        for b in range(wl.batch):
            Kb = inp["k"][:, b:b + 1].float().cpu().numpy()  # [L, 1, Hkv, T, 128]
            Vb = inp["v"][:, b:b + 1].float().cpu().numpy()
            jobs = [pool.submit(_encode_and_compare,
                                (Kb[:, :, h:h + 1], Vb[:, :, h:h + 1], cfgd, _slab_planes(cache, b, h, n)))
                    for h in range(wl.kv_heads)]
            for j in jobs:
                st = j.result()
                for key in ("codes", "near_tie", "near_tie_diff"):
                    totals[key] += st[key]
                totals["slabs"] += 1
    assert totals["slabs"] == wl.batch * wl.kv_heads
    assert totals["codes"] == 3 * 2 * wl.batch * wl.kv_heads * n * 128
    assert totals["near_tie_diff"] <= totals["near_tie"]
