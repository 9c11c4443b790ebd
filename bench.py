#!/usr/bin/env python
"""Decode-step benchmark of the ResidualQuant hot path on B200.

One step = one decode step of a 4-loop looped model's attention layer over a
synthetic Ouro-1.4B-shaped cache (16 KV heads, head_dim 128, batch 16, 8192
cached tokens): decode attention of every loop (three INT2 residual loops and
the bf16 reference loop, each with the current token as a bf16 tail), and the
encode of the new token into every loop's cache, fused into the final loop's
decode call (rq_decode_attention_append).  ``value`` is decode tokens/s
(sequences x steps / s) over all ranks; the same step over a plain bf16 cache
(same library, same kernels without the residual) is reported beside it.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl rq|reference]
                    [--workload ouro8k|mixed|gqa|tiny] [--batch B]
    python bench.py --workload capacity       # 24-layer capacity sweep (own JSON line)
    python bench.py --workload mixed_sweep    # [2,2,4,4] INT4-anchor batch 1/8/32/64 vs bf16

Multi-GPU (torchrun) runs independent replicas, one per rank (the path has no
exchange step); timing is the max over ranks.  ``--impl reference`` times the
CPU oracle (the reference arm for this method) on bounded samples.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import os
import statistics
import subprocess
import sys
import tempfile
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import numpy as np  # noqa: E402
import torch  # noqa: E402

from looped_transformer_decode_rq_b200 import synth  # noqa: E402

METRIC = "RQ decode-attn tokens/s & HBM GB/s (% of B200 peak) at 8k ctx vs BF16 cache"
PROFILE_TRAFFIC = os.path.join(ROOT, "profiles", "rq_decode_split_ouro8k_traffic.txt")


def parse_args():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    # 100 steps of about 0.8 ms: a timed window long enough that run-to-run clock
    # drift averages out
    ap.add_argument("--steps", type=int, default=100)
    ap.add_argument("--warmup", type=int, default=10)
    ap.add_argument("--impl", choices=["rq", "reference"], default="rq")
    ap.add_argument("--workload", choices=["ouro8k", "mixed", "gqa", "gqa_int4", "next_loop", "next_loop_int4", "tiny",
                                           "capacity", "mixed_sweep", "verify_gqa"],
                    default="ouro8k")
    ap.add_argument("--decode-kernel", choices=["auto", "simt", "tensor"], default="auto",
                    help="decode kernel of the RQ cache (the automatic choice by default)")
    ap.add_argument("--batch", type=int, default=None)
    ap.add_argument("--q-heads", type=int, default=None, help="query heads of the workload (a multiple of its kv-heads)")
    ap.add_argument("--cpu-seconds", type=float, default=10.0)
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-bf16", action="store_true")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-extra", action="store_true", help="skip the mixed INT4-anchor and GQA side lines")
    ap.add_argument("--no-sweeps", action="store_true",
                    help="skip the mixed-format batch sweep and the 24-layer capacity sweep")
    return ap.parse_args()


def make_workload(args) -> synth.Workload:
    wl = _base_workload(args)
    if args.q_heads:
        wl = wl.with_(name=f"{wl.name}_Hq{args.q_heads}", q_heads=args.q_heads)
    return wl


def _base_workload(args) -> synth.Workload:
    if args.workload == "ouro8k":
        return synth.ouro_8k(batch=args.batch or 16)
    if args.workload == "mixed":
        return synth.mixed_int4_anchor(batch=args.batch or 8)
    if args.workload == "gqa":
        return synth.gqa_long(batch=args.batch or 8)
    if args.workload == "gqa_int4":
        return synth.gqa_long(batch=args.batch or 8, int4_anchor=True)
    if args.workload == "next_loop":
        return synth.ouro_8k_next_loop(batch=args.batch or 16)
    if args.workload == "next_loop_int4":
        return synth.ouro_8k_next_loop_int4(batch=args.batch or 16)
    return synth.tiny()


# ---------------------------------------------------------------------------
# distributed plumbing (replicas only)
# ---------------------------------------------------------------------------

def dist_setup(args):
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        import datetime
        import torch.distributed as dist
        torch.cuda.set_device(local)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=torch.device("cuda", local))
    elif torch.cuda.is_available():
        torch.cuda.set_device(0)
    return world, rank


def barrier(world):
    if world > 1:
        import torch.distributed as dist
        dist.barrier()


def max_over_ranks(x: float, world: int) -> float:
    """Max of a per-rank time over all ranks (the job is as slow as its slowest rank)."""
    if world == 1:
        return x
    import torch.distributed as dist
    dev = "cuda" if dist.get_backend() == "nccl" else "cpu"
    t = torch.tensor([x], dtype=torch.float64, device=dev)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def job_tokens_per_s(batch_per_rank: int, world: int, ms_per_step: float) -> float:
    """Whole-job decode throughput: every rank decodes its own batch each step."""
    return batch_per_rank * world / (ms_per_step * 1e-3)


# ---------------------------------------------------------------------------
# clocks
# ---------------------------------------------------------------------------
CLOCK_FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
                "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
                "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")


class ClockSampler:
    def __init__(self):
        self.proc = None
        self.path = None
        sel = []
        try:
            uuid = str(torch.cuda.get_device_properties(torch.cuda.current_device()).uuid)
            sel = ["-i", uuid if uuid.startswith("GPU-") else "GPU-" + uuid]
        except Exception:
            sel = []
        self.sel = sel

    def start(self):
        fd, self.path = tempfile.mkstemp(suffix=".csv")
        os.close(fd)
        try:
            self.proc = subprocess.Popen(["nvidia-smi", *self.sel, f"--query-gpu={CLOCK_FIELDS}",
                                          "--format=csv,noheader,nounits", "-lms", "200"],
                                         stdout=open(self.path, "w"), stderr=subprocess.DEVNULL)
        except Exception:
            self.proc = None
        time.sleep(0.3)

    def stop(self):
        if self.proc is None:
            return None
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except Exception:
            self.proc.kill()
        rows = []
        for line in open(self.path):
            parts = [p.strip() for p in line.split(",")]
            if len(parts) >= 9:
                rows.append(parts)
        os.unlink(self.path)
        if not rows:
            return None
        sm = [float(r[1]) for r in rows if r[1].replace(".", "").isdigit()]
        smax = [float(r[2]) for r in rows if r[2].replace(".", "").isdigit()]
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[i] for r in rows for i in range(4) if r[5 + i].lower() == "active"})
        return {"sm_mhz": statistics.median(sm) if sm else None,
                "sm_max_mhz": max(smax) if smax else None, "reasons": reasons, "samples": len(rows)}


# ---------------------------------------------------------------------------
# workload bytes (algorithmic: each record read once per call)
# ---------------------------------------------------------------------------

def record_bytes(lay, cfgd, loop):
    """Bytes one decode call of `loop` reads per (b, kv-head, token): its
    anchor's record and, for every residual link between the loop and the
    anchor (one, or up to three under a chained policy), codes, meta and alpha."""
    a = lay.anchor_of[loop]
    ref = 2 * lay.codes_record_bytes[a] + 2 * lay.meta_record_bytes[a]
    if loop == a:
        return ref
    if cfgd["alpha_mode"][loop] == 2:
        return 2 * lay.codes_record_bytes[loop] + 2 * lay.meta_record_bytes[loop]
    total, link = ref, loop
    while link != a:
        total += 2 * lay.codes_record_bytes[link] + 2 * lay.meta_record_bytes[link] + 4
        link = lay.ref_of[link]
    return total


def call_bytes(lay, cfgd, loop, tokens_total, B, Hq, Hkv, n_tail):
    return (tokens_total * Hkv * record_bytes(lay, cfgd, loop) + B * Hq * 128 * (2 + 4) +
            B * Hkv * n_tail * 512)


def source_hash(paths):
    h = hashlib.sha256()
    for p in paths:
        with open(p, "rb") as f:
            h.update(f.read())
    return h.hexdigest()[:16]


def read_profile_traffic(kernel_hash, workload):
    """Per-launch DRAM bytes of the split kernel from the committed ncu summary,
    if it was taken on the current kernel source and on this workload."""
    if not os.path.exists(PROFILE_TRAFFIC):
        return None
    vals = {}
    for line in open(PROFILE_TRAFFIC):
        if ":" in line and not line.startswith("#"):
            k, v = line.split(":", 1)
            vals[k.strip()] = v.strip()
    if vals.get("kernel_source_sha256_16") != kernel_hash or vals.get("workload") != workload:
        return None
    for key in ("dram_bytes_per_launch", "dram_bytes_per_launch_scaled"):
        try:
            return int(vals[key])
        except (KeyError, ValueError):
            continue
    return None


def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return float(d["hbm_gbs"]), "measured"
    return 6650.0, "fallback"


# ---------------------------------------------------------------------------
# CPU oracle timing (cpu_baseline and the reference arm)
# ---------------------------------------------------------------------------

class OracleSample:
    """One (sequence, kv-head) slab of the workload, encoded by the oracle.
    A sample step = decode attention of every loop for that slab's G q-heads
    plus the encode of its new token; the full step is B*Hkv such samples."""

    def __init__(self, wl, inp, b=0, h=0):
        import oracle.rq_oracle as O
        self.O = O
        self.wl = wl
        G = wl.gqa
        sl = lambda t: t[:, b:b + 1, h:h + 1].float().cpu().numpy()  # noqa: E731
        self.K, self.V = sl(inp["k"]), sl(inp["v"])
        self.kt, self.vt = sl(inp["k_tail"]), sl(inp["v_tail"])
        self.q = inp["q"][:, b:b + 1, h * G:(h + 1) * G].float().cpu().numpy()
        self.ctx = np.array([int(inp["ctx_len"][b])])
        self.cfg = O.CacheConfig.from_dict(synth.cache_config_dict(wl))
        self.enc = O.encode_fp32emu(self.K, self.V, self.cfg)
        self.b, self.h = b, h

    def step(self):
        O = self.O
        outs = [O.decode_attention_f64(self.enc, l, self.q[l], self.ctx, self.kt[l], self.vt[l])
                for l in range(self.wl.num_loops)]
        O.encode_fp32emu(self.kt, self.vt, self.cfg)
        return outs


def blas_threads():
    try:
        from threadpoolctl import threadpool_info
        n = [i.get("num_threads", 1) for i in threadpool_info() if i.get("user_api") == "blas"]
        return max(n) if n else 1
    except Exception:
        return 1


def time_oracle(sample, wl, seconds, min_reps=1):
    reps, t0 = 0, time.perf_counter()
    while True:
        sample.step()
        reps += 1
        el = time.perf_counter() - t0
        if reps >= min_reps and el >= seconds:
            break
    per_sample = el / reps
    full_step = per_sample * wl.batch * wl.kv_heads
    return wl.batch / full_step, per_sample, reps


# ---------------------------------------------------------------------------
# the GPU arm
# ---------------------------------------------------------------------------

def time_steps(step, steps, warmup, world, stream):
    """Mean device time of one step over `steps` timed steps (after `warmup`),
    max over ranks."""
    for _ in range(warmup):
        step()
    barrier(world)
    torch.cuda.synchronize()
    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    a.record(stream)
    for _ in range(steps):
        step()
    b.record(stream)
    torch.cuda.synchronize()
    barrier(world)
    return max_over_ranks(a.elapsed_time(b) / steps, world)


def workload_config(wl, world):
    """The `config` object of a bench line (the same keys for both arms)."""
    return {"workload": wl.name, "global_batch": wl.batch * world, "seq_len": wl.context, "loops": wl.num_loops,
            "kv_heads": wl.kv_heads, "q_heads": wl.q_heads, "head_dim": 128, "bits": list(wl.bits),
            "group": list(wl.group), "parallelism": f"replicas x{world}",
            "l2": "inputs larger than L2 (>= 1 GB read per call), no flush"}


def residual_call_ms(call, stream, reps=50, warmup=5):
    """Mean device time of one decode call issued `reps` times back to back
    (one event pair around the whole run, none between the calls)."""
    for _ in range(warmup):
        call()
    torch.cuda.synchronize()
    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    a.record(stream)
    for _ in range(reps):
        call()
    b.record(stream)
    torch.cuda.synchronize()
    return a.elapsed_time(b) / reps, reps


def measure_workload(wl, steps, warmup, world, rank, per_loop=False):
    """RQ decode step and bf16-cache step of one workload (side lines of the
    main result): tokens/s, residual-loop GB/s and the speed-up over bf16."""
    from looped_transformer_decode_rq_b200 import rq
    dev = torch.device("cuda", torch.cuda.current_device())
    wl = wl.with_(seed=wl.seed + 1000 * rank)
    inp = synth.make_inputs(wl, dev)
    L, B, Hkv, Hq, T = wl.num_loops, wl.batch, wl.kv_heads, wl.q_heads, wl.context
    cfgd = synth.cache_config_dict(wl, capacity=T + 1)
    cache = rq.Cache(rq.config_from_dict(cfgd), device=dev)
    cache.encode(inp["k"], inp["v"])
    ctx = inp["ctx_len"]
    tokens_total = int(ctx.sum().item())
    k_new = inp["k_tail"][:, :, :, :1].contiguous()
    v_new = inp["v_tail"][:, :, :, :1].contiguous()
    q = inp["q"]
    outs = torch.empty((L, B, Hq, 128), dtype=torch.float32, device=dev)
    stream = torch.cuda.current_stream()

    def rq_step():
        for l in range(L - 1):
            cache.decode_attention(l, q[l], ctx, k_new[l], v_new[l], out=outs[l])
        cache.decode_attention_append(L - 1, q[L - 1], ctx, k_new[L - 1], v_new[L - 1], k_new, v_new, ctx,
                                      out=outs[L - 1])

    ms = time_steps(rq_step, steps, warmup, world, stream)

    def loop_call(l):
        return lambda: cache.decode_attention(l, q[l], ctx, k_new[l], v_new[l], out=outs[l])

    call_ms, _ = residual_call_ms(loop_call(0), stream, reps=20)
    res_bytes = call_bytes(cache.layout, cfgd, 0, tokens_total, B, Hq, Hkv, 1)

    def call_gbs(kernel):
        cache.set_decode_kernel(kernel)
        try:
            t, _ = residual_call_ms(loop_call(0), stream, reps=10, warmup=3)
        finally:
            cache.set_decode_kernel(rq.DECODE_KERNEL_AUTO)
        return round(res_bytes / (t * 1e-3) / 1e9, 1)

    per_kernel = {"simt": call_gbs(rq.DECODE_KERNEL_SIMT)}
    if wl.gqa in (1, 2, 4, 8):
        try:
            per_kernel["tensor"] = call_gbs(rq.DECODE_KERNEL_TENSOR)
        except rq.RQError:
            per_kernel["tensor"] = None
    ws = torch.zeros(rq.bf16_workspace_bytes(B, Hkv, Hq), dtype=torch.uint8, device=dev)

    def bf16_step():
        for l in range(L):
            rq.bf16_decode_attention(inp["k"][l], inp["v"][l], q[l], ctx, k_new[l], v_new[l], workspace=ws, out=outs[l])

    bms = time_steps(bf16_step, steps, warmup, world, stream)
    loop_gbs = None
    if per_loop:  # every loop's decode call alone (a chained policy reads more links for farther loops)
        loop_gbs = {}
        for l in range(L):
            t, _ = residual_call_ms(loop_call(l), stream, reps=10, warmup=3)
            lb = call_bytes(cache.layout, cfgd, l, tokens_total, B, Hq, Hkv, 1)
            loop_gbs[str(l)] = {"bytes": lb, "gbs": round(lb / (t * 1e-3) / 1e9, 1)}
    flags = cache.get_error()
    out = {"workload": wl.name, "tokens_per_s": round(job_tokens_per_s(B, world, ms), 1),
           "ms_per_step": round(ms, 4), "residual_loop_gbs": round(res_bytes / (call_ms * 1e-3) / 1e9, 1),
           "residual_loop_bytes": res_bytes, "residual_loop_gbs_by_kernel": per_kernel,
           "bf16_tokens_per_s": round(job_tokens_per_s(B, world, bms), 1),
           "rq_speedup_vs_bf16": round(bms / ms, 3), "device_flags": flags}
    if loop_gbs is not None:
        out["loop_gbs"] = loop_gbs
    del cache, inp, outs, ws
    torch.cuda.empty_cache()
    return out


def measure_multi_query(wl, n_q, steps, warmup, world, rank):
    """Side line: one step of n_q draft tokens per sequence (speculative
    verification) through rq_decode_attention_multi on every loop, against the
    single-query step of the same cache; the cache is read once per call."""
    from looped_transformer_decode_rq_b200 import rq
    dev = torch.device("cuda", torch.cuda.current_device())
    wl = wl.with_(seed=wl.seed + 1000 * rank, n_tail=n_q)
    inp = synth.make_inputs(wl, dev)
    qm = synth.draft_queries(wl, n_q, dev)
    L, B, Hkv, Hq, T = wl.num_loops, wl.batch, wl.kv_heads, wl.q_heads, wl.context
    cfgd = synth.cache_config_dict(wl, capacity=T + n_q)
    cache = rq.Cache(rq.config_from_dict(cfgd), device=dev)
    cache.encode(inp["k"], inp["v"])
    ctx = inp["ctx_len"]
    tokens_total = int(ctx.sum().item())
    kt, vt = inp["k_tail"], inp["v_tail"]
    outs = torch.empty((L, B, n_q, Hq, 128), dtype=torch.float32, device=dev)
    out1 = torch.empty((L, B, Hq, 128), dtype=torch.float32, device=dev)
    stream = torch.cuda.current_stream()

    def multi_step():
        for l in range(L):
            cache.decode_attention_multi(l, qm[l], ctx, kt[l], vt[l], out=outs[l])

    kt1 = [kt[l][:, :, :1].contiguous() for l in range(L)]
    vt1 = [vt[l][:, :, :1].contiguous() for l in range(L)]

    def single_step():
        for l in range(L):
            cache.decode_attention(l, inp["q"][l], ctx, kt1[l], vt1[l], out=out1[l])

    ms = time_steps(multi_step, steps, warmup, world, stream)
    ms1 = time_steps(single_step, steps, warmup, world, stream)
    call_ms, _ = residual_call_ms(lambda: cache.decode_attention_multi(0, qm[0], ctx, kt[0], vt[0], out=outs[0]),
                                  stream, reps=10, warmup=3)
    # the same rows as blocks of half the draft tokens, one cache pass each
    # (the way rows beyond one pass run): the cost a single pass saves
    half = n_q // 2
    qh = [qm[0][:, :half].contiguous(), qm[0][:, half:].contiguous()]
    oh = [outs[0][:, :half].contiguous(), outs[0][:, half:].contiguous()]

    def two_calls():
        for i in range(2):
            cache.decode_attention_multi(0, qh[i], ctx, kt[0], vt[0], out=oh[i])

    call2_ms, _ = residual_call_ms(two_calls, stream, reps=10, warmup=3)
    res_bytes = (tokens_total * Hkv * record_bytes(cache.layout, cfgd, 0) + B * n_q * Hq * 128 * (2 + 4) +
                 B * Hkv * n_q * 512)
    flags = cache.get_error()
    kernel, rows_per_pass = cache.decode_plan(0, n_q)
    out = {"workload": f"{wl.name}_verify{n_q}", "n_q": n_q,
           "rows_per_kv_head": n_q * wl.gqa, "rows_per_pass": rows_per_pass,
           "passes": n_q * wl.gqa // rows_per_pass, "kernel": {1: "simt", 2: "tensor"}.get(kernel, kernel),
           "query_tokens_per_s": round(job_tokens_per_s(B * n_q, world, ms), 1), "ms_per_step": round(ms, 4),
           "single_query_tokens_per_s": round(job_tokens_per_s(B, world, ms1), 1),
           "single_query_ms_per_step": round(ms1, 4),
           "residual_loop_gbs": round(res_bytes / (call_ms * 1e-3) / 1e9, 1), "residual_loop_bytes": res_bytes,
           "residual_loop_ms": round(call_ms, 4), "residual_loop_ms_as_two_calls_of_half": round(call2_ms, 4),
           "device_flags": flags}
    del cache, inp, outs, out1, qm
    torch.cuda.empty_cache()
    return out


def measure_capacity(steps, warmup, world, rank, fractions=(1.0,)):
    """24-layer, 4-loop model at 8192 context: for a bf16 cache and for
    ResidualQuant caches (bf16 anchor, INT4 anchor), the largest batch whose 24
    layers of caches fit in HBM, and decode tokens/s of the full 24-layer
    attention step at `fractions` of that batch (1.0: the largest).  One
    synthetic sequence is encoded into every (layer, sequence) slot, each with
    its own cache memory: the timing does not depend on the values."""
    from looped_transformer_decode_rq_b200 import rq
    dev = torch.device("cuda", torch.cuda.current_device())
    layers, T = 24, 8192
    base = synth.capacity_24layer(batch=1, context=T)
    L, Hkv, Hq = base.num_loops, base.kv_heads, base.q_heads
    stream = torch.cuda.current_stream()
    one = synth.make_inputs(base.with_(batch=1, n_tail=1), dev)  # [L, 1, Hkv, T, 128]
    torch.cuda.empty_cache()
    free, _ = torch.cuda.mem_get_info()
    budget = int(free * 0.9) - (2 << 30)
    results = {}
    for fmt, bits in (("bf16", None), ("rq_bf16_anchor", (2, 2, 2, 16)), ("rq_int4_anchor", (2, 2, 2, 4))):
        torch.cuda.empty_cache()
        if fmt == "bf16":
            per_seq = layers * L * 2 * Hkv * (T + 1) * 128 * 2
        else:
            lay = rq.cache_layout(rq.config_from_dict(synth.cache_config_dict(base.with_(bits=bits), capacity=T + 1)))
            per_seq = layers * lay.total_bytes
        max_b = int(max(1, min(1024, budget // per_seq)))
        points = sorted({max(1, int(round(f * max_b))) for f in fractions})
        sweep = []
        for B in points:
            torch.cuda.empty_cache()
            wl = base.with_(batch=B) if bits is None else base.with_(batch=B, bits=bits)
            q = one["q"].expand(-1, B, -1, -1).contiguous()
            ctx = torch.full((B,), T, dtype=torch.int32, device=dev)
            k_new = one["k_tail"].expand(-1, B, -1, -1, -1).contiguous()
            v_new = one["v_tail"].expand(-1, B, -1, -1, -1).contiguous()
            outs = torch.empty((L, B, Hq, 128), dtype=torch.float32, device=dev)
            if fmt == "bf16":
                caches = []
                for _ in range(layers):
                    planes = []
                    for l in range(L):
                        kv = torch.empty((2, B, Hkv, T + 1, 128), dtype=torch.bfloat16, device=dev)
                        kv[0, :, :, :T].copy_(one["k"][l].expand(B, -1, -1, -1))
                        kv[1, :, :, :T].copy_(one["v"][l].expand(B, -1, -1, -1))
                        planes.append(kv)
                    caches.append(planes)
                ws = torch.zeros(rq.bf16_workspace_bytes(B, Hkv, Hq), dtype=torch.uint8, device=dev)

                def step():
                    for planes in caches:
                        for l in range(L):
                            kv = planes[l]
                            kv[0, :, :, T:T + 1].copy_(k_new[l])   # append the new token
                            kv[1, :, :, T:T + 1].copy_(v_new[l])
                            rq.bf16_decode_attention(kv[0], kv[1], q[l], ctx, k_new[l], v_new[l], workspace=ws,
                                                     out=outs[l])
            else:
                ws = None
                cfgd = synth.cache_config_dict(wl, capacity=T + 1)
                caches = [rq.Cache(rq.config_from_dict(cfgd), device=dev) for _ in range(layers)]
                kb = one["k"].expand(-1, B, -1, -1, -1)  # batch stride 0: the same values for every sequence
                vb = one["v"].expand(-1, B, -1, -1, -1)
                for c in caches:
                    c.encode(kb, vb)

                def step():
                    for c in caches:
                        for l in range(L - 1):
                            c.decode_attention(l, q[l], ctx, k_new[l], v_new[l], out=outs[l])
                        c.decode_attention_append(L - 1, q[L - 1], ctx, k_new[L - 1], v_new[L - 1], k_new, v_new,
                                                  ctx, out=outs[L - 1])
            ms = time_steps(step, steps, warmup, world, stream)
            flags = 0 if fmt == "bf16" else max(c.get_error() for c in caches)
            sweep.append({"batch": B, "tokens_per_s": round(job_tokens_per_s(B, world, ms), 1),
                          "ms_per_step": round(ms, 3), "device_flags": int(flags)})
            del caches, q, ctx, k_new, v_new, outs, ws
            torch.cuda.empty_cache()
        top = sweep[-1]
        results[fmt] = {"max_batch": max_b, "bytes_per_sequence": int(per_seq),
                        "tokens_per_s": top["tokens_per_s"], "ms_per_step": top["ms_per_step"],
                        "peak_tokens_per_s": max(r["tokens_per_s"] for r in sweep),
                        "device_flags": max(r["device_flags"] for r in sweep), "sweep": sweep}
    del one
    torch.cuda.empty_cache()
    return {"workload": "capacity_24layer_L4_H16_T8192", "metric": "decode tokens/s of the 24-layer attention step "
            "against batch, up to the largest batch whose caches fit", "results": results,
            "peak_vs_bf16": {k: round(v["peak_tokens_per_s"] / results["bf16"]["peak_tokens_per_s"], 3)
                             for k, v in results.items()},
            "max_batch_vs_bf16": {k: round(v["max_batch"] / results["bf16"]["max_batch"], 2)
                                  for k, v in results.items()},
            "hbm_budget_bytes": budget, "steps": steps, "warmup": warmup, "data": "synthetic", "n_gpus": world}


def run_capacity(args, world, rank):
    out = measure_capacity(max(2, min(args.steps, 5)), 3, world, rank, fractions=(0.25, 0.5, 0.75, 1.0))
    if rank == 0:
        print(json.dumps(out))


def measure_mixed_sweep(steps, warmup, world, rank, batches=(1, 8, 32, 64)):
    """Mixed-precision format [2,2,4,4] with an INT4 anchor at 8k context, batch
    1 / 8 / 32 / 64: the decode step (4 loop decodes + append-encode of the new
    token) against the bf16-cache step on the same values, and the
    append-encode alone.  A step that reads less than twice the L2 is timed
    alone after writing a 256 MB buffer (L2 flushed between timed steps)."""
    from looped_transformer_decode_rq_b200 import rq
    dev = torch.device("cuda", torch.cuda.current_device())
    stream = torch.cuda.current_stream()
    flush_buf = torch.empty(256 << 20, dtype=torch.uint8, device=dev)

    def timed(step, flush):
        for _ in range(warmup):
            step()
        barrier(world)
        torch.cuda.synchronize()
        if not flush:
            return time_steps(step, steps, 0, world, stream)
        total = 0.0
        for _ in range(steps):
            flush_buf.fill_(1)
            a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            a.record(stream)
            step()
            b.record(stream)
            b.synchronize()
            total += a.elapsed_time(b)
        barrier(world)
        return max_over_ranks(total / steps, world)

    results = []
    for B in batches:
        wl = synth.mixed_int4_anchor(batch=B).with_(seed=2 + 1000 * rank)
        inp = synth.make_inputs(wl, dev)
        L, Hkv, Hq, T = wl.num_loops, wl.kv_heads, wl.q_heads, wl.context
        cfgd = synth.cache_config_dict(wl, capacity=T + 1)
        cache = rq.Cache(rq.config_from_dict(cfgd), device=dev)
        cache.encode(inp["k"], inp["v"])
        ctx = inp["ctx_len"]
        k_new = inp["k_tail"][:, :, :, :1].contiguous()
        v_new = inp["v_tail"][:, :, :, :1].contiguous()
        q = inp["q"]
        outs = torch.empty((L, B, Hq, 128), dtype=torch.float32, device=dev)
        lay = cache.layout
        step_bytes = sum(B * Hkv * T * record_bytes(lay, cfgd, l) for l in range(L))
        flush = step_bytes < 2 * (126 << 20)

        def rq_step():
            for l in range(L - 1):
                cache.decode_attention(l, q[l], ctx, k_new[l], v_new[l], out=outs[l])
            cache.decode_attention_append(L - 1, q[L - 1], ctx, k_new[L - 1], v_new[L - 1], k_new, v_new, ctx,
                                          out=outs[L - 1])

        def append():
            cache.encode(k_new, v_new, positions=ctx)

        ws = torch.zeros(rq.bf16_workspace_bytes(B, Hkv, Hq), dtype=torch.uint8, device=dev)

        def bf16_step():
            for l in range(L):
                rq.bf16_decode_attention(inp["k"][l], inp["v"][l], q[l], ctx, k_new[l], v_new[l], workspace=ws,
                                         out=outs[l])

        ms = timed(rq_step, flush)
        enc_ms = timed(append, flush)
        bms = timed(bf16_step, flush)
        flags = cache.get_error()
        results.append({"batch": B, "tokens_per_s": round(job_tokens_per_s(B, world, ms), 1),
                        "ms_per_step": round(ms, 4), "hbm_gbs": round(step_bytes / (ms * 1e-3) / 1e9, 1),
                        "step_bytes": step_bytes, "append_encode_us": round(enc_ms * 1e3, 1),
                        "bf16_tokens_per_s": round(job_tokens_per_s(B, world, bms), 1),
                        "bf16_ms_per_step": round(bms, 4), "rq_speedup_vs_bf16": round(bms / ms, 3),
                        "l2_flushed": flush, "device_flags": int(flags)})
        del cache, inp, outs, ws
        torch.cuda.empty_cache()
    del flush_buf
    torch.cuda.empty_cache()
    return {"workload": "mixed_2244_H16_T8192_int4ref_batch_sweep",
            "metric": "decode step tokens/s (4 loops + append-encode) vs BF16 cache",
            "results": results, "steps": steps, "warmup": warmup, "data": "synthetic", "n_gpus": world}


def run_mixed_sweep(args, world, rank):
    out = measure_mixed_sweep(max(3, min(args.steps, 20)), max(3, args.warmup), world, rank)
    if rank == 0:
        print(json.dumps(out))


def run_rq(args, world, rank):
    from looped_transformer_decode_rq_b200 import rq

    wl = make_workload(args).with_(seed=make_workload(args).seed + 1000 * rank)
    dev = torch.device("cuda", torch.cuda.current_device())
    inp = synth.make_inputs(wl, dev)
    L, B, Hkv, Hq, T = wl.num_loops, wl.batch, wl.kv_heads, wl.q_heads, wl.context
    # room for the end-to-end leg, whose decode run grows the cache by a token per step
    e2e_warm = 3
    cfgd = synth.cache_config_dict(wl, capacity=T + 1 + (0 if args.no_e2e else e2e_warm + args.steps))
    cache = rq.Cache(rq.config_from_dict(cfgd), device=dev)
    cache.set_decode_kernel({"auto": rq.DECODE_KERNEL_AUTO, "simt": rq.DECODE_KERNEL_SIMT,
                             "tensor": rq.DECODE_KERNEL_TENSOR}[args.decode_kernel])
    cache.encode(inp["k"], inp["v"])
    ctx = inp["ctx_len"]
    tokens_total = int(ctx.sum().item())
    pos = ctx.clone()  # the new token goes to position ctx_len[b]
    k_new = inp["k_tail"][:, :, :, :1].contiguous()
    v_new = inp["v_tail"][:, :, :, :1].contiguous()
    q = inp["q"]
    outs = torch.empty((L, B, Hq, 128), dtype=torch.float32, device=dev)
    lay = cache.layout
    stream = torch.cuda.current_stream()
    n_tail = 1

    def step():
        # loops 0 .. L-2, then the final loop's decode with the new token's
        # append-encode (every loop) fused into its combine launch
        for l in range(L - 1):
            cache.decode_attention(l, q[l], ctx, k_new[l], v_new[l], out=outs[l])
        cache.decode_attention_append(L - 1, q[L - 1], ctx, k_new[L - 1], v_new[L - 1], k_new, v_new, pos,
                                      out=outs[L - 1])

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()
    flags = cache.get_error()

    # parity spot check of the timed launch configuration (rank 0: sequence 0, kv-head 0)
    parity = None
    sample = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        sample = OracleSample(wl, inp, 0, 0)
        want = sample.step()
        G = wl.gqa
        errs = []
        for l in range(L):
            got = outs[l, 0, :G].cpu().numpy()
            w = want[l][0]
            errs.append(float((np.abs(got - w).max(-1) / np.abs(w).max(-1)).max()))
        parity = {"max_rel_err": max(errs), "tol": 2e-3, "sampled": f"b=0, q-heads 0..{G - 1}, all {L} loops"}

    clocks = ClockSampler()
    clocks.start()
    barrier(world)
    torch.cuda.synchronize()
    t_start, t_end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    t_start.record(stream)
    for _ in range(args.steps):
        step()
    t_end.record(stream)
    torch.cuda.synchronize()
    barrier(world)
    clk = clocks.stop()
    ms = t_start.elapsed_time(t_end) / args.steps
    ms = max_over_ranks(ms, world)
    # Per-launch time of the dominant call (a residual loop's split + combine),
    # in a pass of its own so that no event sits inside the timed steps: the
    # call is issued back to back, as in the step, where each split kernel
    # overlaps the previous combine (programmatic dependent launches).
    call_ms, call_reps = residual_call_ms(lambda: cache.decode_attention(0, q[0], ctx, k_new[0], v_new[0],
                                                                         out=outs[0]), stream)
    flags |= cache.get_error()

    res_bytes = call_bytes(lay, cfgd, 0, tokens_total, B, Hq, Hkv, n_tail)
    step_bytes = sum(call_bytes(lay, cfgd, l, tokens_total, B, Hq, Hkv, n_tail) for l in range(L))
    step_bytes += L * B * Hkv * 512 + B * Hkv * (sum(record_bytes(lay, cfgd, l) for l in range(L)))
    peak, peak_kind = load_peaks()
    kernel_hash = source_hash([os.path.join(ROOT, "looped_transformer_decode_rq_b200", "csrc", f)
                               for f in ("rq_decode_split.cuh", "rq_common.cuh", "rq_internal.h")])
    achieved = res_bytes / (call_ms * 1e-3) / 1e9
    traffic = read_profile_traffic(kernel_hash, wl.name)
    value = job_tokens_per_s(B, world, ms)

    # ---- e2e through the public API with host buffers
    e2e = None
    if not args.no_e2e:
        # A decode run through the public API: every step copies its inputs
        # (the queries, the new token of every loop and the context lengths)
        # from pinned host memory and its outputs back, and the cache grows by
        # one token per step (step i attends ctx_len + i cached tokens plus the
        # new token, which it appends at position ctx_len + i).  As in a serving
        # loop, the copies run on their own streams and overlap the neighbouring
        # steps' decode (inputs and outputs double-buffered, ordered by events);
        # the timed region spans the first input copy to the last output copy.
        hq = torch.empty(q.shape, dtype=q.dtype, pin_memory=True).copy_(q.cpu())
        hk = torch.empty(k_new.shape, dtype=k_new.dtype, pin_memory=True).copy_(k_new.cpu())
        hv = torch.empty(v_new.shape, dtype=v_new.dtype, pin_memory=True).copy_(v_new.cpu())
        ctx0 = ctx.cpu()
        n_total = e2e_warm + args.steps
        hctx = torch.empty((n_total, B), dtype=torch.int32, pin_memory=True)
        for i in range(n_total):
            hctx[i].copy_(ctx0 + i)
        hout = [torch.empty(outs.shape, dtype=outs.dtype, pin_memory=True) for _ in range(2)]
        dbuf = [(torch.empty_like(q), torch.empty_like(k_new), torch.empty_like(v_new), torch.empty_like(outs),
                 torch.empty_like(ctx)) for _ in range(2)]
        h2d_s, d2h_s = torch.cuda.Stream(), torch.cuda.Stream()
        ev = {name: [torch.cuda.Event() for _ in range(2)] for name in ("h2d", "comp", "d2h")}

        def e2e_run(first, nsteps, start_ev=None):
            if start_ev is not None:
                h2d_s.wait_event(start_ev)
            for i in range(nsteps):
                j = i % 2
                dq, dk, dv, do, dctx = dbuf[j]
                if i >= 2:
                    h2d_s.wait_event(ev["comp"][j])  # step i-2 no longer reads these inputs
                with torch.cuda.stream(h2d_s):
                    dq.copy_(hq, non_blocking=True)
                    dk.copy_(hk, non_blocking=True)
                    dv.copy_(hv, non_blocking=True)
                    dctx.copy_(hctx[first + i], non_blocking=True)
                ev["h2d"][j].record(h2d_s)
                stream.wait_event(ev["h2d"][j])
                if i >= 2:
                    stream.wait_event(ev["d2h"][j])  # step i-2's output has left the device
                for l in range(L - 1):
                    cache.decode_attention(l, dq[l], dctx, dk[l], dv[l], out=do[l])
                cache.decode_attention_append(L - 1, dq[L - 1], dctx, dk[L - 1], dv[L - 1], dk, dv, dctx,
                                              out=do[L - 1])
                ev["comp"][j].record(stream)
                d2h_s.wait_event(ev["comp"][j])
                with torch.cuda.stream(d2h_s):
                    hout[j].copy_(do, non_blocking=True)
                ev["d2h"][j].record(d2h_s)
            stream.wait_stream(d2h_s)
            stream.wait_stream(h2d_s)

        e2e_run(0, e2e_warm)
        torch.cuda.synchronize()
        barrier(world)
        torch.cuda.synchronize()
        a, b2 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record(stream)
        e2e_run(e2e_warm, args.steps, start_ev=a)
        b2.record(stream)
        torch.cuda.synchronize()
        barrier(world)
        ems = max_over_ranks(a.elapsed_time(b2) / args.steps, world)
        e2e = {"value": round(job_tokens_per_s(B, world, ems), 1), "unit": "tokens/s",
               "h2d_bytes_per_step": int(hq.numel() * 2 + hk.numel() * 2 + hv.numel() * 2 + B * 4),
               "d2h_bytes_per_step": int(hout[0].numel() * 4),
               "context": f"decode run: ctx_len grows from {int(ctx0.min()) + e2e_warm} by one token per step",
               "copies": "own streams, overlapping the neighbouring steps (double-buffered)"}

    # ---- the same step over a bf16 cache (same library)
    bf16 = None
    if not args.no_bf16:
        kc = [inp["k"][l] for l in range(L)]
        vc = [inp["v"][l] for l in range(L)]
        ws = torch.zeros(rq.bf16_workspace_bytes(B, Hkv, Hq), dtype=torch.uint8, device=dev)

        def bf16_step():
            for l in range(L):
                rq.bf16_decode_attention(kc[l], vc[l], q[l], ctx, k_new[l], v_new[l], workspace=ws, out=outs[l])

        for _ in range(args.warmup):
            bf16_step()
        barrier(world)
        torch.cuda.synchronize()
        a, b2 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record(stream)
        for _ in range(args.steps):
            bf16_step()
        b2.record(stream)
        torch.cuda.synchronize()
        bms = max_over_ranks(a.elapsed_time(b2) / args.steps, world)
        bf_bytes = L * (tokens_total * Hkv * 512 + B * Hq * 128 * 6 + B * Hkv * n_tail * 512)
        bf16 = {"tokens_per_s": round(job_tokens_per_s(B, world, bms), 1), "ms_per_step": round(bms, 4),
                "hbm_gbs": round(bf_bytes / (bms * 1e-3) / 1e9, 1),
                "bytes_per_step": bf_bytes, "rq_speedup": round(bms / ms, 3)}
        del kc, vc, ws

    # ---- CPU oracle on a bounded sample (rank 0, N = 1 only)
    cpu = None
    if sample is not None:
        v, per, reps = time_oracle(sample, wl, args.cpu_seconds)
        cpu = {"value": round(v, 3), "unit": "tokens/s", "cores": blas_threads(), "kind": "oracle",
               "sample": (f"float64 NumPy oracle: decode of all {L} loops for sequence 0, kv-head 0 "
                          f"({wl.gqa} q-head(s), {int(ctx[0])} cached tokens + 1 tail) plus the encode "
                          f"of its new token, {reps} reps of {per:.3f} s; scaled by B*Hkv={B * Hkv}")}

    extra = None
    side = args.workload == "ouro8k" and not (args.no_extra and args.no_sweeps)
    if side:  # free the main workload's memory for the side lines
        del cache, inp, outs
        torch.cuda.empty_cache()
    if not args.no_extra and args.workload == "ouro8k":
        extra = [measure_workload(synth.mixed_int4_anchor(batch=32), 30, 3, world, rank, per_loop=True),
                 measure_workload(synth.gqa_long(batch=8), 30, 3, world, rank),
                 measure_workload(synth.gqa_long(batch=8, q_heads=64), 30, 3, world, rank),
                 measure_workload(synth.gqa_long(batch=8, int4_anchor=True), 30, 3, world, rank),
                 measure_workload(synth.ouro_8k_next_loop(), 30, 3, world, rank, per_loop=True),
                 measure_workload(synth.ouro_8k_next_loop_int4(), 30, 3, world, rank, per_loop=True),
                 # the same chain with 4 query heads per kv-head (chained loops on the tensor cores)
                 measure_workload(synth.ouro_8k_next_loop_int4(batch=8).with_(
                     name="ouro_L4_Hq64_H16_B8_T8192_2224_int4ref_next_loop", q_heads=64), 20, 3, world, rank,
                     per_loop=True),
                 measure_multi_query(synth.ouro_8k(), 4, 30, 3, world, rank),
                 measure_multi_query(synth.gqa_long(batch=8), 4, 20, 3, world, rank)]
    sweeps = None
    if not args.no_sweeps and args.workload == "ouro8k":
        # the mixed-precision [2,2,4,4] batch sweep and the 24-layer capacity
        # sweep, each its own workload (side results, not the headline)
        sweeps = {"mixed_2244_batch_sweep": measure_mixed_sweep(10, 3, world, rank),
                  "capacity_24layer_sweep": measure_capacity(3, 2, world, rank,
                                                             fractions=(0.25, 0.5, 0.75, 1.0))}

    out = {
        "metric": METRIC, "value": round(value, 1), "unit": "tokens/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(ms, 4),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16+int2 (fp32 math)",
        "data": "synthetic (seeded generator; Ouro-1.4B-shaped caches, random values)",
        "config": workload_config(wl, world),
        "hbm_gbs_step": round(step_bytes / (ms * 1e-3) / 1e9, 1),
        "bytes_per_step": step_bytes,
        "roofline": {"bound": "hbm", "achieved": round(achieved, 1), "peak": peak, "unit": "GB/s",
                     "frac": round(achieved / peak, 4), "traffic": traffic,
                     "kernel": "rq_decode_attention on a residual loop (split + combine kernels)",
                     "algorithmic_bytes_per_launch": res_bytes, "launch_ms": round(call_ms, 4),
                     "launch_timing": f"mean of {call_reps} back-to-back calls, one event pair, outside the timed steps",
                     "peak_kind": f"{peak_kind} (MEASURED_PEAKS.json hbm_gbs)" if peak_kind == "measured" else "fallback",
                     "frac_of_8tbs": round(achieved / 8000.0, 4)},
        "cpu_baseline": cpu, "e2e": e2e, "bf16_cache": bf16, "parity": parity, "other_workloads": extra,
        "sweeps": sweeps,
        # per step: a split and a combine kernel per loop (the final loop's combine also appends)
        "gpu_launches": args.steps * (2 * L), "clocks": clk, "device_flags": flags,
    }
    if rank == 0:
        print(json.dumps(out))


def run_reference(args, world, rank):
    """The reference arm: the CPU oracle, as it stands, on the GPU arm's
    workload.  Each step times one (sequence, kv-head) slab (decode of every
    loop plus the encode of its new token); the full step is B*Hkv such slabs,
    so the reported step time is that sample time times B*Hkv (stated in
    `extrapolation`)."""
    if rank != 0:
        return
    wl = make_workload(args)
    inp = synth.make_inputs(wl.with_(context=wl.context), "cuda" if torch.cuda.is_available() else "cpu")
    sample = OracleSample(wl, inp, 0, 0)
    for _ in range(args.warmup):
        sample.step()
    t = []
    for _ in range(args.steps):
        t0 = time.perf_counter()
        sample.step()
        t.append(time.perf_counter() - t0)
    per = statistics.mean(t)
    slabs = wl.batch * wl.kv_heads
    full = per * slabs
    value = wl.batch / full
    cpu = {"value": round(value, 3), "unit": "tokens/s", "cores": blas_threads(), "kind": "oracle",
           "sample": (f"one (sequence, kv-head) slab per step: decode of all {wl.num_loops} loops over "
                      f"{wl.context} tokens + encode of the new token; scaled by B*Hkv={slabs}")}
    out = {"metric": METRIC, "value": round(value, 3), "unit": "tokens/s", "n_gpus": world, "steps": args.steps,
           "warmup": args.warmup, "ms_per_step": round(full * 1e3, 3), "higher_is_better": True,
           "scaling": "weak", "vs_baseline": None, "dtype": "f64 (oracle)", "data": "synthetic",
           "config": workload_config(wl, 1),
           "extrapolation": {"slabs_timed_per_step": 1, "slabs_per_step": slabs,
                             "factor": slabs, "measured_ms_per_timed_step": round(per * 1e3, 3),
                             "timed_wall_s": round(sum(t), 3)},
           "impl": "reference", "cpu_baseline": cpu,
           "e2e": {"value": round(value, 3), "unit": "tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(out))


def main():
    args = parse_args()
    world, rank = dist_setup(args)
    try:
        if args.impl == "reference":
            run_reference(args, world, rank)
        elif args.workload == "capacity":
            run_capacity(args, world, rank)
        elif args.workload == "mixed_sweep":
            run_mixed_sweep(args, world, rank)
        elif args.workload == "verify_gqa":
            out = measure_multi_query(synth.gqa_long(batch=args.batch or 8), 4, max(3, args.steps),
                                      max(3, args.warmup), world, rank)
            if rank == 0:
                print(json.dumps(out))
        else:
            run_rq(args, world, rank)
    finally:
        if world > 1:
            import torch.distributed as dist
            dist.destroy_process_group()


if __name__ == "__main__":
    main()
