"""Out-of-bounds write detection without a sanitizer: guard bands ("canaries").

Every buffer a call writes -- the cache buffer, the decode output, the
split-K workspace and the reconstruction outputs -- is cut from a larger
allocation filled with a byte pattern.  After encode, decode (both kernels),
the fused append and reconstruction on small shapes the test checks, byte for
byte, that nothing outside what the call may write has changed:

* the bands before and after every buffer;
* inside the cache buffer, the padding between planes and the records of
  every position the calls never wrote (positions past the encoded context up
  to the plane's padded capacity);
* the workspace past the size the library asked for.
"""
import numpy as np
import pytest
import torch

from looped_transformer_decode_rq_b200 import synth

pytestmark = pytest.mark.gpu

PATTERN = 0xA5
BAND = 4096  # bytes of guard on each side (a multiple of 1024 keeps the cache's alignment rule simple)


def guarded(nbytes, align=1024):
    """A uint8 view of `nbytes` inside a pattern-filled allocation with at
    least BAND guard bytes on each side; returns (view, whole, start)."""
    whole = torch.full((nbytes + 2 * BAND + align,), PATTERN, dtype=torch.uint8, device="cuda")
    start = BAND + (-(whole.data_ptr() + BAND)) % align
    return whole[start:start + nbytes], whole, start


def assert_bands(whole, start, nbytes, what):
    h = whole.cpu().numpy()
    assert np.all(h[:start] == PATTERN), f"{what}: bytes before the buffer changed"
    assert np.all(h[start + nbytes:] == PATTERN), f"{what}: bytes after the buffer changed"


def plane_spans(lay, cfg):
    """(offset, record_bytes) of every plane of the layout."""
    spans = []
    for l in range(cfg.num_loops):
        for kv in range(2):
            spans.append((lay.codes_offset[l][kv], lay.codes_record_bytes[l]))
            if lay.meta_offset[l][kv] >= 0:
                spans.append((lay.meta_offset[l][kv], lay.meta_record_bytes[l]))
        if lay.alpha_offset[l] >= 0:
            spans.append((lay.alpha_offset[l], 4))
    return spans


def assert_cache_untouched_outside(cache_bytes, lay, cfg, written):
    """Padding between planes and every record at a position not in
    written[b] (a set per sequence) must still hold the pattern."""
    h = cache_bytes.cpu().numpy()
    B, H, Tp = cfg.batch, cfg.kv_heads, lay.capacity_padded
    covered = np.zeros(h.size, dtype=bool)
    covered[lay.status_offset:lay.status_offset + 256] = True  # status word (cleared at create)
    for off, rec in plane_spans(lay, cfg):
        n = B * H * Tp * rec
        covered[off:off + n] = True
        plane = h[off:off + n].reshape(B, H, Tp, rec)
        for b in range(B):
            keep = np.ones(Tp, dtype=bool)
            keep[sorted(written[b])] = False
            assert np.all(plane[b, :, keep] == PATTERN), f"plane at {off}: sequence {b} has stray records"
    assert np.all(h[~covered] == PATTERN), "padding between planes changed"


@pytest.mark.parametrize("bits,G", [((2, 2, 2, 16), 1), ((2, 2, 4, 4), 1), ((2, 2, 4, 4), 4), ((2, 2, 2, 16), 8)])
def test_no_write_outside_buffers(librq, bits, G):
    rq = librq
    T, cap = 200, 300
    wl = synth.Workload(name=f"guard_{bits}_{G}", batch=3, kv_heads=2, q_heads=2 * G, context=T, bits=bits,
                        sigma=(0.3, 0.2, 0.1), outlier_p=0.01, seed=150 + G, lengths=(200, 77, 0))
    inp = synth.make_inputs(wl, "cpu")
    cfgd = synth.cache_config_dict(wl, capacity=cap)
    cfg = rq.config_from_dict(cfgd)
    lay = rq.cache_layout(cfg)
    cbuf, cwhole, cstart = guarded(lay.total_bytes)
    cache = rq.Cache(cfg, buffer=cbuf)
    assert cache.base.data_ptr() == cbuf.data_ptr()
    cache.encode(inp["k"].cuda(), inp["v"].cuda())  # positions 0 .. T-1 of every sequence
    written = [set(range(T)) for _ in range(wl.batch)]
    ws_bytes = cache.workspace.numel()
    wbuf, wwhole, wstart = guarded(ws_bytes + 512, align=256)
    cache.workspace = wbuf[:ws_bytes]
    B, Hq, L = wl.batch, wl.q_heads, wl.num_loops
    out_bytes = B * Hq * 128 * 4
    obuf, owhole, ostart = guarded(out_bytes, align=256)
    out = obuf.view(torch.float32).view(B, Hq, 128)
    ctx = inp["ctx_len"].cuda()
    kernels = [rq.DECODE_KERNEL_SIMT]
    if G >= 2:
        kernels.append(rq.DECODE_KERNEL_TENSOR)
    for kernel in kernels:
        cache.set_decode_kernel(kernel)
        for loop in range(L):
            cache.decode_attention(loop, inp["q"][loop].cuda(), ctx, inp["k_tail"][loop].cuda(),
                                   inp["v_tail"][loop].cuda(), out=out)
        # fused append of one new token per sequence at position ctx[b]
        cache.decode_attention_append(L - 1, inp["q"][L - 1].cuda(), ctx, inp["k_tail"][L - 1].cuda(),
                                      inp["v_tail"][L - 1].cuda(), inp["k_tail"].cuda(), inp["v_tail"].cuda(), ctx,
                                      out=out)
        for b in range(B):
            written[b].add(int(inp["ctx_len"][b]))
        torch.cuda.synchronize()
        assert cache.get_error() == 0
        assert_bands(owhole, ostart, out_bytes, "decode output")
        # the workspace past the library's size and the bands around it
        wh = wwhole.cpu().numpy()
        assert np.all(wh[wstart + ws_bytes:] == PATTERN), "workspace written past its size"
        assert np.all(wh[:wstart] == PATTERN), "bytes before the workspace changed"
    # reconstruction outputs of a token range
    n = 50
    rk, rkw, rks = guarded(B * wl.kv_heads * n * 128 * 4, align=256)
    rv, rvw, rvs = guarded(B * wl.kv_heads * n * 128 * 4, align=256)
    for loop in range(L):
        st = rq.lib().rq_reconstruct(cache.handle, loop, 100, n, rk.data_ptr(), rv.data_ptr(),
                                     torch.cuda.current_stream().cuda_stream)
        assert st == rq.OK
    torch.cuda.synchronize()
    assert_bands(rkw, rks, rk.numel(), "reconstruct k_out")
    assert_bands(rvw, rvs, rv.numel(), "reconstruct v_out")
    assert_bands(cwhole, cstart, lay.total_bytes, "cache buffer")
    assert_cache_untouched_outside(cbuf, lay, cfg, written)
