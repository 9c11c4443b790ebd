"""The C-ABI library loads, exports every symbol include/rq_api.h declares, and
rejects bad arguments on the host before touching the device (no GPU needed)."""
import ctypes as C
import os
import re

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "rq_api.h")


def declared_functions():
    src = open(HEADER).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    names = re.findall(r"^\s*RQ_API\s+(?:const\s+)?[a-z_0-9]+\s*\*?\s*(rq_[a-z_0-9]+)\s*\(", src, flags=re.M)
    return sorted(set(names))


def test_header_declares_expected_entry_points():
    names = declared_functions()
    for n in ("rq_cache_layout", "rq_cache_create", "rq_cache_destroy", "rq_encode", "rq_decode_attention",
              "rq_decode_workspace_size", "rq_bf16_decode_attention", "rq_reconstruct", "rq_get_error",
              "rq_status_string"):
        assert n in names


def test_library_exports_every_declared_symbol(librq):
    lib = librq.lib()
    for n in declared_functions():
        assert hasattr(lib, n), f"{n} declared in rq_api.h but not exported"
    assert set(declared_functions()) <= set(librq.EXPORTED) | {n for n in declared_functions() if hasattr(lib, n)}


def test_status_strings(librq):
    assert librq.status_string(0) == "RQ_OK"
    assert librq.status_string(3) == "RQ_ERR_CAPACITY"
    assert librq.status_string(99) == "RQ_UNKNOWN_STATUS"


def _cfg(librq, **kw):
    d = dict(num_loops=4, batch=16, kv_heads=16, q_heads=16, capacity=8192, bits=[2, 2, 2, 16],
             group=[32, 32, 32, 32], rotate=[1, 1, 1, 0], alpha_mode=[0, 0, 0, 0])
    d.update(kw)
    return librq.config_from_dict(d)


def test_layout_bytes_per_token_head(librq):
    lay = librq.cache_layout(_cfg(librq))
    assert lay.capacity_padded == 8192
    assert lay.codes_record_bytes[3] == 256 and lay.meta_offset[3][0] == -1 and lay.alpha_offset[3] == -1
    assert list(lay.anchor_of)[:4] == [3, 3, 3, 3]
    per = 2 * 256 + sum(2 * lay.codes_record_bytes[l] + 2 * lay.meta_record_bytes[l] + 4 for l in range(3))
    assert per == 2 * 256 + 3 * (2 * 32 + 2 * 16 + 4)   # 812 B per (b, h, token) over all loops
    recs = 16 * 16 * 8192
    assert lay.total_bytes >= per * recs
    assert lay.total_bytes - per * recs <= 1024 * 16
    offs = [lay.codes_offset[l][kv] for l in range(4) for kv in range(2)]
    assert all(o % 1024 == 0 for o in offs)
    assert lay.codes_offset[4][0] == -1


def test_layout_int4_anchor_and_padding(librq):
    lay = librq.cache_layout(_cfg(librq, capacity=100, bits=[2, 2, 4, 4]))
    assert lay.capacity_padded == 128
    assert lay.codes_record_bytes[3] == 64 and lay.meta_record_bytes[3] == 16
    assert lay.codes_record_bytes[2] == 64 and lay.meta_record_bytes[2] == 16
    lay16 = librq.cache_layout(_cfg(librq, group=[16, 16, 16, 32]))
    assert lay16.meta_record_bytes[0] == 32


@pytest.mark.parametrize("field,value,status", [
    ("num_loops", 1, 1), ("num_loops", 17, 1), ("batch", 0, 1), ("kv_heads", 0, 1),
    ("q_heads", 24, 1), ("q_heads", 48, 2), ("head_dim", 64, 2), ("capacity", 0, 1),
    ("bits", [3, 2, 2, 16], 2), ("bits", [2, 2, 2, 8], 2), ("group", [64, 32, 32, 32], 2),
    ("group", [32, 32, 32, 16], 1), ("rotate", [2, 1, 1, 0], 1), ("alpha_mode", [4, 0, 0, 0], 1),
])
def test_layout_rejects_bad_config(librq, field, value, status):
    cfg = _cfg(librq, **({field: value} if field not in ("head_dim",) else {}))
    if field == "head_dim":
        cfg.head_dim = value
    if field == "group" and value == [32, 32, 32, 16]:
        cfg = _cfg(librq, bits=[2, 2, 2, 4], group=value)
        status = 2
    lay = librq.Layout()
    got = librq.lib().rq_cache_layout(C.byref(cfg), C.byref(lay))
    assert got == status, librq.lib().rq_last_error_message()


def test_create_rejects_bad_buffers_before_device_work(librq):
    lib = librq.lib()
    cfg = _cfg(librq, batch=1, kv_heads=1, q_heads=1, capacity=64)
    lay = librq.cache_layout(cfg)
    h = C.c_void_p()
    assert lib.rq_cache_create(C.byref(cfg), None, lay.total_bytes, C.byref(h)) == 1
    assert lib.rq_cache_create(C.byref(cfg), 1024 * 1024 + 16, lay.total_bytes, C.byref(h)) == 1
    assert lib.rq_cache_create(C.byref(cfg), 1024 * 1024, lay.total_bytes - 1, C.byref(h)) == 1
    assert b"aligned" in lib.rq_last_error_message() or b"bytes" in lib.rq_last_error_message()
    assert lib.rq_cache_create(C.byref(cfg), 1024 * 1024, lay.total_bytes, None) == 1


def test_null_handles_are_rejected(librq):
    lib = librq.lib()
    st = (C.c_int64 * 4)(0, 0, 0, 0)
    assert lib.rq_encode(None, 16, 16, st, 0, None, 1, None) == 1
    assert lib.rq_decode_attention(None, 0, 16, 16, None, None, 0, 0.1, 16, 256, 1 << 20, None) == 1
    assert lib.rq_reconstruct(None, 0, 0, 1, 16, 16, None) == 1
    assert lib.rq_get_error(None, None, None) == 1
    lib.rq_cache_destroy(None)  # no-op


def test_bf16_decode_rejects_bad_arguments(librq):
    lib = librq.lib()
    st = (C.c_int64 * 3)(16 * 128 * 64, 128 * 64, 128)
    args = dict(batch=1, kv=1, hq=1, k=4096, v=8192, strides=st, cap=64, q=16384, ctx=32768)
    def call(**kw):
        a = dict(args); a.update(kw)
        return lib.rq_bf16_decode_attention(a["batch"], a["kv"], a["hq"], a["k"], a["v"], a["strides"], a["cap"],
                                            a["q"], a["ctx"], None, None, 0, 0.088, 65536, 1 << 20, 1 << 20,
                                            None, None)
    assert call(batch=0) == 1
    assert call(hq=3, kv=2) == 1
    assert call(hq=48, kv=3) == 2
    assert call(k=None) == 1
    assert call(k=4097) == 1
    assert call(strides=(C.c_int64 * 3)(16 * 128 * 64, 128 * 64, 100)) == 1
    assert call(cap=0) == 1


def test_layout_anchor_policies(librq):
    rq = librq
    first = rq.cache_layout(_cfg(librq, bits=[16, 2, 2, 2], group=[32] * 4, rotate=[0, 1, 1, 1],
                                 anchor_policy=rq.ANCHOR_FIRST))
    assert list(first.anchor_of)[:4] == [0, 0, 0, 0]
    assert first.alpha_offset[0] == -1 and all(first.alpha_offset[l] >= 0 for l in (1, 2, 3))
    cfg = rq.config_from_dict(dict(num_loops=8, batch=2, kv_heads=2, q_heads=2, capacity=64,
                                   bits=[2, 2, 2, 4, 2, 2, 2, 4], group=[32] * 8, rotate=[1, 1, 1, 0] * 2,
                                   alpha_mode=[0] * 8, anchor_policy=rq.ANCHOR_INTERVAL, anchor_interval=4))
    lay = rq.cache_layout(cfg)
    assert list(lay.anchor_of)[:8] == [3, 3, 3, 3, 7, 7, 7, 7]
    assert lay.codes_record_bytes[3] == 64 and lay.meta_record_bytes[3] == 16
    # an anchor must be bf16 or INT4, a residual loop INT2 or INT4
    bad = rq.config_from_dict(dict(num_loops=8, batch=2, kv_heads=2, q_heads=2, capacity=64,
                                   bits=[2] * 8, group=[32] * 8, rotate=[1] * 8, alpha_mode=[0] * 8,
                                   anchor_policy=rq.ANCHOR_INTERVAL, anchor_interval=4))
    assert rq.lib().rq_cache_layout(C.byref(bad), C.byref(rq.Layout())) == rq.ERR_UNSUPPORTED
    bad.anchor_interval = 1
    assert rq.lib().rq_cache_layout(C.byref(bad), C.byref(rq.Layout())) == rq.ERR_INVALID_ARG


def test_layout_chained_policies(librq):
    """Previous-/Next-loop references: ref_of is the neighbour, anchor_of the
    chain's end; a chain must share one residual format, keep alpha and stay
    within RQ_MAX_CHAIN links."""
    rq = librq
    nxt = rq.cache_layout(_cfg(librq, bits=[2, 2, 2, 4], group=[32] * 4, rotate=[1, 1, 1, 0],
                               anchor_policy=rq.ANCHOR_NEXT))
    assert list(nxt.ref_of)[:4] == [1, 2, 3, 3]
    assert list(nxt.anchor_of)[:4] == [3, 3, 3, 3]
    assert nxt.alpha_offset[3] == -1 and all(nxt.alpha_offset[l] >= 0 for l in (0, 1, 2))
    prev = rq.cache_layout(_cfg(librq, bits=[4, 2, 2, 2], group=[32] * 4, rotate=[0, 1, 1, 1],
                                anchor_policy=rq.ANCHOR_PREVIOUS))
    assert list(prev.ref_of)[:4] == [0, 0, 1, 2]
    assert list(prev.anchor_of)[:4] == [0, 0, 0, 0]
    last = rq.cache_layout(_cfg(librq, bits=[2, 2, 2, 16], group=[32] * 4, rotate=[1, 1, 1, 0]))
    assert list(last.ref_of)[:4] == [3, 3, 3, 3]

    def status(**kw):
        c = _cfg(librq, **kw)
        return rq.lib().rq_cache_layout(C.byref(c), C.byref(rq.Layout()))
    # mixed residual formats on one chain
    assert status(bits=[2, 2, 4, 16], group=[32] * 4, rotate=[1, 1, 1, 0], anchor_policy=rq.ANCHOR_NEXT) == rq.ERR_UNSUPPORTED
    assert status(bits=[2, 2, 2, 16], group=[16, 32, 32, 32], rotate=[1, 1, 1, 0],
                  anchor_policy=rq.ANCHOR_NEXT) == rq.ERR_UNSUPPORTED
    assert status(bits=[2, 2, 2, 16], group=[32] * 4, rotate=[0, 1, 1, 0], anchor_policy=rq.ANCHOR_NEXT) == rq.ERR_UNSUPPORTED
    # direct quantisation (alpha 0) has no reference to chain through
    assert status(bits=[2, 2, 2, 16], group=[32] * 4, rotate=[1, 1, 1, 0], alpha_mode=[2, 0, 0, 0],
                  anchor_policy=rq.ANCHOR_NEXT) == rq.ERR_UNSUPPORTED
    # at most three links
    c5 = rq.config_from_dict(dict(num_loops=5, batch=1, kv_heads=1, q_heads=1, capacity=64, bits=[2, 2, 2, 2, 16],
                                  group=[32] * 5, rotate=[1, 1, 1, 1, 0], alpha_mode=[0] * 5,
                                  anchor_policy=rq.ANCHOR_NEXT))
    assert rq.lib().rq_cache_layout(C.byref(c5), C.byref(rq.Layout())) == rq.ERR_UNSUPPORTED
    c5.anchor_policy = rq.ANCHOR_LAST
    assert rq.lib().rq_cache_layout(C.byref(c5), C.byref(rq.Layout())) == rq.OK
    c5.anchor_policy = 5
    assert rq.lib().rq_cache_layout(C.byref(c5), C.byref(rq.Layout())) == rq.ERR_INVALID_ARG
