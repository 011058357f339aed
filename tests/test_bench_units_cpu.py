"""The algorithmic units bench.py divides by, pinned to figures computed by
hand from the workload shapes: decode bytes per launch (K and V of every valid
slot, q, k_new/v_new read, ring write, output) and causal prefill FLOPs
(4 H d P (P + 1) / 2 per sequence and layer)."""
import os
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

import bench  # noqa: E402
from ring_sliding_window_b200 import synth  # noqa: E402

ROW = 10 * 128 * 2  # one token's K (or V, q, ...) over all heads, bf16: 2,560 bytes


def test_decode_bytes_near_max_steady_state():
    w = synth.workload("near_max_context")
    # 4 sequences x (2 x 32,768 cached rows + q + k_new + v_new + ring write x 2 + out)
    want = 4 * (2 * (32640 + 128) * ROW + 6 * ROW)
    assert want == 671_150_080
    assert bench.kv_bytes_per_layer(w, [128] * 4) == want
    assert bench.kv_bytes_per_layer(w, [10_000] * 4) == want  # any t >= W


def test_decode_bytes_during_warm_up_count_only_held_entries():
    w = synth.workload("near_max_context")
    # t generated tokens before this step: P + t + 1 keys after the ring write
    for t in (0, 1, 63, 127):
        assert bench.kv_bytes_per_layer(w, [t] * 4) == 4 * (2 * (32640 + t + 1) * ROW + 6 * ROW)


def test_decode_bytes_single_page():
    w = synth.workload("single_page_decode")
    assert bench.kv_bytes_per_layer(w, [500]) == 2 * (1088 + 128) * ROW + 6 * ROW == 6_241_280


def test_prefill_flops_multi_page_and_near_max():
    mp = synth.workload("multi_page_decode")
    nm = synth.workload("near_max_context")
    assert bench.prefill_flops_per_layer(mp) == 8 * 4 * 10 * 128 * 8256 * 8257 // 2
    assert bench.prefill_flops_per_layer(nm) == 4 * 4 * 10 * 128 * 32640 * 32641 // 2
    # the 12-layer totals the workload table quotes: 16.75 and 130.9 TFLOP
    assert round(12 * bench.prefill_flops_per_layer(mp) / 1e12, 2) == 16.75
    assert round(12 * bench.prefill_flops_per_layer(nm) / 1e12, 1) == 130.9
