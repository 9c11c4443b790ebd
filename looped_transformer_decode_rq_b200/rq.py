"""Thin ctypes binding of ``librq_b200.so`` (the C ABI in ``include/rq_api.h``).

Argument marshalling only: torch tensors supply device memory and the current
CUDA stream; every step of encode and decode runs in the library's kernels.
Importing this module loads the library and raises ``ImportError`` if it has
not been built (``python -m looped_transformer_decode_rq_b200.build``) -- there
is no fallback implementation.
"""
from __future__ import annotations

import ctypes as C
import os
from dataclasses import dataclass
from typing import Optional, Sequence

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "librq_b200.so")
if not os.path.exists(LIB_PATH):
    raise ImportError(f"{LIB_PATH} is missing: build it with "
                      "`python -m looped_transformer_decode_rq_b200.build`")
_lib = C.CDLL(LIB_PATH)

MAX_LOOPS = 16
HEAD_DIM = 128
PAGE_TOKENS = 64
MAX_BATCH = 1024

OK, ERR_INVALID_ARG, ERR_UNSUPPORTED, ERR_CAPACITY, ERR_WORKSPACE, ERR_CUDA, ERR_DEVICE_FLAG = range(7)
FLAG_BAD_INPUT, FLAG_POSITION, FLAG_CTX_LEN, FLAG_PIPE_TIMEOUT, FLAG_META_OVERFLOW = 1, 2, 4, 8, 16
ALPHA_LS, ALPHA_ONE, ALPHA_ZERO, ALPHA_NORM_RATIO = 0, 1, 2, 3
ANCHOR_LAST, ANCHOR_FIRST, ANCHOR_INTERVAL, ANCHOR_PREVIOUS, ANCHOR_NEXT = 0, 1, 2, 3, 4
MAX_CHAIN = 3
MAX_DRAFT = 16
DECODE_KERNEL_AUTO, DECODE_KERNEL_SIMT, DECODE_KERNEL_TENSOR = 0, 1, 2

# every symbol the header declares (checked by the ABI tests)
EXPORTED = ("rq_cache_layout", "rq_cache_create", "rq_cache_destroy", "rq_cache_info", "rq_encode",
            "rq_decode_workspace_size", "rq_decode_attention", "rq_bf16_decode_workspace_size",
            "rq_bf16_decode_attention", "rq_reconstruct", "rq_get_error", "rq_status_string",
            "rq_last_error_message", "rq_decode_attention_static_scratch", "rq_cache_set_decode_kernel",
            "rq_cache_set_debug_stall", "rq_decode_attention_append", "rq_decode_multi_workspace_size",
            "rq_decode_attention_multi", "rq_decode_plan")
STATIC_SCRATCH_BYTES = 4 * 1024 * 1024


class Config(C.Structure):
    _fields_ = [("num_loops", C.c_int32), ("batch", C.c_int32), ("kv_heads", C.c_int32),
                ("q_heads", C.c_int32), ("head_dim", C.c_int32), ("capacity", C.c_int32),
                ("bits", C.c_int32 * MAX_LOOPS), ("group", C.c_int32 * MAX_LOOPS),
                ("rotate", C.c_int32 * MAX_LOOPS), ("alpha_mode", C.c_int32 * MAX_LOOPS),
                ("anchor_policy", C.c_int32), ("anchor_interval", C.c_int32)]


class Layout(C.Structure):
    _fields_ = [("capacity_padded", C.c_int64), ("total_bytes", C.c_int64), ("status_offset", C.c_int64),
                ("codes_offset", (C.c_int64 * 2) * MAX_LOOPS), ("meta_offset", (C.c_int64 * 2) * MAX_LOOPS),
                ("alpha_offset", C.c_int64 * MAX_LOOPS), ("codes_record_bytes", C.c_int64 * MAX_LOOPS),
                ("meta_record_bytes", C.c_int64 * MAX_LOOPS), ("anchor_of", C.c_int32 * MAX_LOOPS),
                ("ref_of", C.c_int32 * MAX_LOOPS)]


_vp, _i32, _i64, _f32 = C.c_void_p, C.c_int32, C.c_int64, C.c_float
_sig = {
    "rq_cache_layout": (C.c_int, [C.POINTER(Config), C.POINTER(Layout)]),
    "rq_cache_create": (C.c_int, [C.POINTER(Config), _vp, _i64, C.POINTER(_vp)]),
    "rq_cache_destroy": (None, [_vp]),
    "rq_cache_info": (C.c_int, [_vp, C.POINTER(Config), C.POINTER(Layout)]),
    "rq_encode": (C.c_int, [_vp, _vp, _vp, C.POINTER(_i64), _i32, _vp, _i32, _vp]),
    "rq_cache_set_decode_kernel": (C.c_int, [_vp, _i32]),
    "rq_cache_set_debug_stall": (C.c_int, [_vp, _i32]),
    "rq_decode_workspace_size": (C.c_int, [_vp, C.POINTER(_i64)]),
    "rq_decode_multi_workspace_size": (C.c_int, [_vp, _i32, C.POINTER(_i64)]),
    "rq_decode_plan": (C.c_int, [_vp, _i32, _i32, C.POINTER(_i32), C.POINTER(_i32)]),
    "rq_decode_attention_multi": (C.c_int, [_vp, _i32, _vp, _i32, _vp, _vp, _vp, _i32, _f32, _vp, _vp, _i64, _vp]),
    "rq_decode_attention": (C.c_int, [_vp, _i32, _vp, _vp, _vp, _vp, _i32, _f32, _vp, _vp, _i64, _vp]),
    "rq_decode_attention_static_scratch": (C.c_int, [_vp, _i32, _vp, _vp, _vp, _vp, _i32, _f32, _vp, _vp]),
    "rq_decode_attention_append": (C.c_int, [_vp, _i32, _vp, _vp, _vp, _vp, _i32, _f32, _vp, _vp, _i64, _vp, _vp,
                                             C.POINTER(_i64), _vp, _i32, _vp]),
    "rq_bf16_decode_workspace_size": (C.c_int, [_i32, _i32, _i32, C.POINTER(_i64)]),
    "rq_bf16_decode_attention": (C.c_int, [_i32, _i32, _i32, _vp, _vp, C.POINTER(_i64), _i32, _vp, _vp, _vp,
                                           _vp, _i32, _f32, _vp, _vp, _i64, _vp, _vp]),
    "rq_reconstruct": (C.c_int, [_vp, _i32, _i32, _i32, _vp, _vp, _vp]),
    "rq_get_error": (C.c_int, [_vp, _vp, C.POINTER(C.c_uint32)]),
    "rq_status_string": (C.c_char_p, [C.c_int]),
    "rq_last_error_message": (C.c_char_p, []),
}
for _name, (_res, _args) in _sig.items():
    _f = getattr(_lib, _name)
    _f.restype = _res
    _f.argtypes = _args


class RQError(RuntimeError):
    def __init__(self, status: int, where: str):
        self.status = status
        msg = _lib.rq_last_error_message().decode()
        super().__init__(f"{where}: {_lib.rq_status_string(status).decode()} ({msg})")


def _check(status: int, where: str) -> None:
    if status != OK:
        raise RQError(status, where)


def _ptr(t: Optional[torch.Tensor]) -> Optional[int]:
    return None if t is None else t.data_ptr()


def _stream(stream=None) -> Optional[int]:
    if stream is None:
        stream = torch.cuda.current_stream()
    return stream.cuda_stream


def make_config(num_loops: int, batch: int, kv_heads: int, q_heads: int, capacity: int,
                bits: Sequence[int], group: Sequence[int], rotate: Sequence[int],
                alpha_mode: Sequence[int], head_dim: int = HEAD_DIM, anchor_policy: int = ANCHOR_LAST,
                anchor_interval: int = 0) -> Config:
    c = Config()
    c.num_loops, c.batch, c.kv_heads, c.q_heads, c.head_dim, c.capacity = (
        num_loops, batch, kv_heads, q_heads, head_dim, capacity)
    c.anchor_policy, c.anchor_interval = anchor_policy, anchor_interval
    for i in range(min(num_loops, MAX_LOOPS, len(bits))):
        c.bits[i], c.group[i], c.rotate[i], c.alpha_mode[i] = bits[i], group[i], rotate[i], alpha_mode[i]
    return c


def config_from_dict(d: dict) -> Config:
    return make_config(d["num_loops"], d["batch"], d["kv_heads"], d["q_heads"], d["capacity"], d["bits"],
                       d["group"], d["rotate"], d["alpha_mode"], d.get("head_dim", HEAD_DIM),
                       d.get("anchor_policy", ANCHOR_LAST), d.get("anchor_interval", 0))


def cache_layout(cfg: Config) -> Layout:
    lay = Layout()
    _check(_lib.rq_cache_layout(C.byref(cfg), C.byref(lay)), "rq_cache_layout")
    return lay


class Cache:
    """A ResidualQuant KV cache: one device buffer (owned here, allocated with
    torch) carved into the planes ``rq_cache_layout`` describes."""

    def __init__(self, cfg: Config, device=None, buffer: Optional[torch.Tensor] = None):
        self.cfg = cfg
        self.layout = cache_layout(cfg)
        n = self.layout.total_bytes
        if buffer is None:
            buffer = torch.empty(n + 1024, dtype=torch.uint8, device=device or "cuda")
        off = (-buffer.data_ptr()) % 1024
        self.buffer = buffer
        self.base = buffer[off:off + n]
        h = _vp()
        _check(_lib.rq_cache_create(C.byref(cfg), self.base.data_ptr(), n, C.byref(h)), "rq_cache_create")
        self._h = h
        ws = _i64()
        _check(_lib.rq_decode_workspace_size(self._h, C.byref(ws)), "rq_decode_workspace_size")
        self.workspace = torch.zeros(ws.value, dtype=torch.uint8, device=self.base.device)
        self._multi_ws = {}

    @property
    def handle(self):
        return self._h

    def set_debug_stall(self, page: int) -> None:
        """Failure-path test hook: the decode producers wait out their limit before
        CTA-local page `page` (-1: off); the call then sets FLAG_PIPE_TIMEOUT."""
        _check(_lib.rq_cache_set_debug_stall(self._h, page), "rq_cache_set_debug_stall")

    def set_decode_kernel(self, kernel: int) -> None:
        """DECODE_KERNEL_AUTO (default), DECODE_KERNEL_SIMT or DECODE_KERNEL_TENSOR."""
        _check(_lib.rq_cache_set_decode_kernel(self._h, kernel), "rq_cache_set_decode_kernel")

    @property
    def G(self) -> int:
        return self.cfg.q_heads // self.cfg.kv_heads

    def close(self):
        if getattr(self, "_h", None):
            _lib.rq_cache_destroy(self._h)
            self._h = None

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass

    # ---- views of the planes (for tests and inspection)
    def plane(self, offset: int, record_bytes: int) -> torch.Tensor:
        cfg, lay = self.cfg, self.layout
        n = cfg.batch * cfg.kv_heads * lay.capacity_padded * record_bytes
        return self.base[offset:offset + n].view(cfg.batch, cfg.kv_heads, lay.capacity_padded, record_bytes)

    def encode(self, k: torch.Tensor, v: torch.Tensor, start_pos: int = 0,
               positions: Optional[torch.Tensor] = None, stream=None) -> None:
        """k, v: bf16 [L, B, Hkv, n, 128] (unit stride on the last dim)."""
        assert k.dtype == torch.bfloat16 and v.dtype == torch.bfloat16 and k.shape == v.shape
        assert k.stride() == v.stride() and k.stride(-1) == 1
        strides = (_i64 * 4)(*k.stride()[:4])
        _check(_lib.rq_encode(self._h, k.data_ptr(), v.data_ptr(), strides, start_pos, _ptr(positions),
                              k.shape[3], _stream(stream)), "rq_encode")

    def _check_decode_args(self, q, ctx_len, k_tail, v_tail, out):
        """Shapes, dtypes, devices and layouts of a single-query decode's tensors
        (the kernels read and write them as these shapes, so a wrong one must
        not reach the library)."""
        cfg = self.cfg
        dev = self.base.device
        B, Hq, Hkv = cfg.batch, cfg.q_heads, cfg.kv_heads
        if q.dtype != torch.bfloat16 or not q.is_contiguous() or tuple(q.shape) != (B, Hq, HEAD_DIM) or q.device != dev:
            raise ValueError(f"q must be a contiguous bf16 [{B}, {Hq}, {HEAD_DIM}] tensor on {dev}")
        if ctx_len.dtype != torch.int32 or tuple(ctx_len.shape) != (B,) or ctx_len.device != dev:
            raise ValueError(f"ctx_len must be an int32 [{B}] tensor on {dev}")
        n_tail = 0 if k_tail is None else k_tail.shape[2]
        if n_tail:
            for t in (k_tail, v_tail):
                if (t is None or t.dtype != torch.bfloat16 or not t.is_contiguous() or t.device != dev
                        or t.dim() != 4 or tuple(t.shape) != (B, Hkv, n_tail, HEAD_DIM)):
                    raise ValueError(f"k_tail and v_tail must be contiguous bf16 [{B}, {Hkv}, n_tail, {HEAD_DIM}] "
                                     f"tensors on {dev}")
        if out is None:
            out = torch.empty((B, Hq, HEAD_DIM), dtype=torch.float32, device=dev)
        elif (out.dtype != torch.float32 or not out.is_contiguous() or tuple(out.shape) != (B, Hq, HEAD_DIM)
              or out.device != dev):
            raise ValueError(f"out must be a contiguous fp32 [{B}, {Hq}, {HEAD_DIM}] tensor on {dev}")
        return q, ctx_len, k_tail, v_tail, out, n_tail

    def decode_attention(self, loop: int, q: torch.Tensor, ctx_len: torch.Tensor,
                         k_tail: Optional[torch.Tensor] = None, v_tail: Optional[torch.Tensor] = None,
                         softmax_scale: Optional[float] = None, out: Optional[torch.Tensor] = None,
                         stream=None) -> torch.Tensor:
        """q: bf16 [B, Hq, 128]; ctx_len: int32 [B]; tails bf16 [B, Hkv, n_tail, 128]."""
        q, ctx_len, k_tail, v_tail, out, n_tail = self._check_decode_args(q, ctx_len, k_tail, v_tail, out)
        scale = softmax_scale if softmax_scale is not None else HEAD_DIM ** -0.5
        _check(_lib.rq_decode_attention(self._h, loop, q.data_ptr(), ctx_len.data_ptr(), _ptr(k_tail),
                                        _ptr(v_tail), n_tail, scale, out.data_ptr(), self.workspace.data_ptr(),
                                        self.workspace.numel(), _stream(stream)), "rq_decode_attention")
        return out

    def decode_plan(self, loop: int, n_q: int = 1):
        """(kernel, rows per pass over the cache) that a decode of `loop` with
        n_q draft tokens takes on this handle (rq_decode_plan)."""
        k, rows = _i32(0), _i32(0)
        _check(_lib.rq_decode_plan(self._h, loop, n_q, C.byref(k), C.byref(rows)), "rq_decode_plan")
        return k.value, rows.value

    def decode_attention_multi(self, loop: int, q: torch.Tensor, ctx_len: torch.Tensor,
                               k_tail: torch.Tensor, v_tail: torch.Tensor, softmax_scale: Optional[float] = None,
                               out: Optional[torch.Tensor] = None, stream=None) -> torch.Tensor:
        """n_q query tokens per sequence: q bf16 [B, n_q, Hq, 128]; the last n_q of the
        tail tokens (bf16 [B, Hkv, n_tail, 128]) are the draft tokens.  Returns fp32
        [B, n_q, Hq, 128]."""
        cfg = self.cfg
        assert q.dtype == torch.bfloat16 and q.is_contiguous() and q.dim() == 4 and ctx_len.dtype == torch.int32
        n_q = q.shape[1]
        assert k_tail.is_contiguous() and v_tail.is_contiguous()
        if out is None:
            out = torch.empty((cfg.batch, n_q, cfg.q_heads, HEAD_DIM), dtype=torch.float32, device=q.device)
        ws = self._multi_ws.get(n_q)
        if ws is None:
            need = C.c_int64()
            _check(_lib.rq_decode_multi_workspace_size(self._h, n_q, C.byref(need)), "rq_decode_multi_workspace_size")
            ws = self._multi_ws[n_q] = torch.zeros(need.value, dtype=torch.uint8, device=self.base.device)
        scale = softmax_scale if softmax_scale is not None else HEAD_DIM ** -0.5
        _check(_lib.rq_decode_attention_multi(self._h, loop, q.data_ptr(), n_q, ctx_len.data_ptr(), _ptr(k_tail),
                                              _ptr(v_tail), k_tail.shape[2], scale, out.data_ptr(), ws.data_ptr(),
                                              ws.numel(), _stream(stream)), "rq_decode_attention_multi")
        return out

    def decode_attention_append(self, loop: int, q: torch.Tensor, ctx_len: torch.Tensor,
                                k_tail: Optional[torch.Tensor], v_tail: Optional[torch.Tensor],
                                k_new: torch.Tensor, v_new: torch.Tensor, positions: torch.Tensor,
                                softmax_scale: Optional[float] = None, out: Optional[torch.Tensor] = None,
                                stream=None) -> torch.Tensor:
        """decode_attention(loop, ...) and the encode of k_new/v_new (bf16 [L, B, Hkv, n, 128])
        at device positions (int32 [B]) in one call."""
        q, ctx_len, k_tail, v_tail, out, n_tail = self._check_decode_args(q, ctx_len, k_tail, v_tail, out)
        assert k_new.dtype == torch.bfloat16 and v_new.dtype == torch.bfloat16 and k_new.shape == v_new.shape
        assert k_new.stride() == v_new.stride() and k_new.stride(-1) == 1 and positions.dtype == torch.int32
        scale = softmax_scale if softmax_scale is not None else HEAD_DIM ** -0.5
        strides = (_i64 * 4)(*k_new.stride()[:4])
        _check(_lib.rq_decode_attention_append(self._h, loop, q.data_ptr(), ctx_len.data_ptr(), _ptr(k_tail),
                                               _ptr(v_tail), n_tail, scale, out.data_ptr(), self.workspace.data_ptr(),
                                               self.workspace.numel(), k_new.data_ptr(), v_new.data_ptr(), strides,
                                               positions.data_ptr(), k_new.shape[3], _stream(stream)),
               "rq_decode_attention_append")
        return out

    def decode_attention_static_scratch(self, loop: int, q: torch.Tensor, ctx_len: torch.Tensor,
                                        k_tail: Optional[torch.Tensor] = None, v_tail: Optional[torch.Tensor] = None,
                                        softmax_scale: Optional[float] = None, out: Optional[torch.Tensor] = None,
                                        stream=None) -> torch.Tensor:
        """decode_attention without a caller workspace: the library keeps the
        split-K partials in its own fixed 4 MiB device array (for callers that
        cannot allocate).  Calls that overlap on the GPU race on that array."""
        q, ctx_len, k_tail, v_tail, out, n_tail = self._check_decode_args(q, ctx_len, k_tail, v_tail, out)
        scale = softmax_scale if softmax_scale is not None else HEAD_DIM ** -0.5
        _check(_lib.rq_decode_attention_static_scratch(self._h, loop, q.data_ptr(), ctx_len.data_ptr(),
                                                       _ptr(k_tail), _ptr(v_tail), n_tail, scale, out.data_ptr(),
                                                       _stream(stream)), "rq_decode_attention_static_scratch")
        return out

    def reconstruct(self, loop: int, t0: int, n: int, stream=None):
        cfg = self.cfg
        k = torch.empty((cfg.batch, cfg.kv_heads, n, HEAD_DIM), dtype=torch.float32, device=self.base.device)
        v = torch.empty_like(k)
        _check(_lib.rq_reconstruct(self._h, loop, t0, n, k.data_ptr(), v.data_ptr(), _stream(stream)),
               "rq_reconstruct")
        return k, v

    def get_error(self, stream=None) -> int:
        flags = C.c_uint32(0)
        st = _lib.rq_get_error(self._h, _stream(stream), C.byref(flags))
        if st not in (OK, ERR_DEVICE_FLAG):
            _check(st, "rq_get_error")
        return flags.value


def bf16_workspace_bytes(batch: int, kv_heads: int, q_heads: int) -> int:
    ws = _i64()
    _check(_lib.rq_bf16_decode_workspace_size(batch, kv_heads, q_heads, C.byref(ws)),
           "rq_bf16_decode_workspace_size")
    return ws.value


def bf16_decode_attention(k_cache: torch.Tensor, v_cache: torch.Tensor, q: torch.Tensor, ctx_len: torch.Tensor,
                          k_tail: Optional[torch.Tensor] = None, v_tail: Optional[torch.Tensor] = None,
                          softmax_scale: Optional[float] = None, workspace: Optional[torch.Tensor] = None,
                          out: Optional[torch.Tensor] = None, status: Optional[torch.Tensor] = None,
                          stream=None) -> torch.Tensor:
    """Decode attention over a plain bf16 cache k_cache/v_cache [B, Hkv, cap, 128]."""
    B, Hkv, cap, D = k_cache.shape
    Hq = q.shape[1]
    assert D == HEAD_DIM and k_cache.stride() == v_cache.stride() and k_cache.stride(-1) == 1
    if workspace is None:
        workspace = torch.zeros(bf16_workspace_bytes(B, Hkv, Hq), dtype=torch.uint8, device=q.device)
    if out is None:
        out = torch.empty((B, Hq, HEAD_DIM), dtype=torch.float32, device=q.device)
    n_tail = 0 if k_tail is None else k_tail.shape[2]
    strides = (_i64 * 3)(*k_cache.stride()[:3])
    scale = softmax_scale if softmax_scale is not None else HEAD_DIM ** -0.5
    _check(_lib.rq_bf16_decode_attention(B, Hkv, Hq, k_cache.data_ptr(), v_cache.data_ptr(), strides, cap,
                                         q.data_ptr(), ctx_len.data_ptr(), _ptr(k_tail), _ptr(v_tail), n_tail,
                                         scale, out.data_ptr(), workspace.data_ptr(), workspace.numel(),
                                         _ptr(status), _stream(stream)), "rq_bf16_decode_attention")
    return out


def status_string(status: int) -> str:
    return _lib.rq_status_string(status).decode()


def lib():
    """The loaded ctypes library (for ABI tests)."""
    return _lib
