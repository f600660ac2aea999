"""Host-side pins of bench.py's roofline arithmetic (no GPU).

The algorithmic bytes of the Qwen2-1.5B shape in bf16, written out from the
shapes: per layer the q/k/v weight [2048, 1536] and bias, o [1536, 1536],
gate/up/down 3 x [8960, 1536], two norms; the untied lm_head [151936, 1536]
and the final norm; one embedding row per token; 28,672 bytes of K/V per
cached position over all layers.
"""
import importlib.util
import os

import synth

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _bench():
    spec = importlib.util.spec_from_file_location("bench_mod", os.path.join(ROOT, "bench.py"))
    m = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(m)
    return m


def test_layer_and_step_weight_bytes():
    b = _bench()
    s = synth.QWEN2_1P5B
    per_layer = 2 * (2048 * 1536 + 2048 + 1536 * 1536 + 3 * 8960 * 1536 + 2 * 1536)
    assert per_layer == 93_595_648
    assert b.layer_weight_bytes(s) == per_layer
    weights = 28 * per_layer + 2 * (151936 * 1536 + 1536) + 2 * 1536  # + lm_head, final norm, one embedding row
    assert weights == 3_087_431_680
    kv_per_pos = 2 * 28 * 2 * 128 * 2
    assert kv_per_pos == 28_672
    # a step at context c reads every cached position plus the new one
    assert b.decode_step_bytes(s, 1, 512) == weights + 513 * kv_per_pos
    assert b.decode_step_bytes(s, 64, 4096) == 28 * per_layer + 2 * (151936 * 1536 + 1536) + 64 * 2 * 1536 \
        + 64 * 4097 * kv_per_pos


def test_recorded_traffic_is_tied_to_the_kernel_sources():
    """A recorded DRAM figure is reported only while the profiled kernel's
    sources hash to the value stored with it."""
    import json
    b = _bench()
    recs = json.load(open(os.path.join(ROOT, "profiles", "traffic.json")))
    assert recs
    for key, rec in recs.items():
        kernel, workload = key.split("@")
        assert kernel in b.KERNEL_SOURCES, key
        t = b.recorded_traffic(kernel, workload)
        if rec["src_hash"] == b.kernel_src_hash(kernel):
            assert t == rec["dram_bytes_per_launch"]
        else:
            assert t is None
        assert b.recorded_traffic(kernel, "another-workload") is None
