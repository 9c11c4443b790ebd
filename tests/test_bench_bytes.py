"""Host-side checks of bench.py's algorithmic byte counts (no GPU): the bytes a
decode call reads per (b, kv-head, token) follow the cache layout, including
every link of a chained policy, and the committed traffic figure is bound to
its workload and kernel sources."""
import bench
from looped_transformer_decode_rq_b200 import rq, synth


def _layout(wl):
    cfgd = synth.cache_config_dict(wl)
    return rq.cache_layout(rq.config_from_dict(cfgd)), cfgd


def test_record_bytes_last_loop_policy(librq):
    lay, cfgd = _layout(synth.ouro_8k())
    # bf16 anchor 2 x 256; INT2 g=32 residual: codes 2 x 32, meta 2 x 16, alpha 4
    assert [bench.record_bytes(lay, cfgd, l) for l in range(4)] == [612, 612, 612, 512]
    lay, cfgd = _layout(synth.mixed_int4_anchor())
    # INT4 anchor: codes 2 x 64 + meta 2 x 16 = 160; INT4 residual: 2 x 64 + 2 x 16 + 4 = 164
    assert [bench.record_bytes(lay, cfgd, l) for l in range(4)] == [260, 260, 324, 160]


def test_record_bytes_chained_policy_counts_every_link(librq):
    lay, cfgd = _layout(synth.ouro_8k_next_loop())
    assert [bench.record_bytes(lay, cfgd, l) for l in range(4)] == [812, 712, 612, 512]
    lay, cfgd = _layout(synth.ouro_8k_next_loop_int4())
    assert [bench.record_bytes(lay, cfgd, l) for l in range(4)] == [460, 360, 260, 160]


def test_traffic_figure_is_bound_to_workload_and_sources():
    import os
    h = bench.source_hash([os.path.join(bench.ROOT, "looped_transformer_decode_rq_b200", "csrc", f)
                           for f in ("rq_decode_split.cuh", "rq_common.cuh", "rq_internal.h")])
    assert bench.read_profile_traffic(h, "some_other_workload") is None
    assert bench.read_profile_traffic("0" * 16, synth.ouro_8k().name) is None
