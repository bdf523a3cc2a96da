"""The synthetic workloads use the DiT shapes the pages print.

"Joy-face_change_optimized" model card, section "strip the text-stream
weights", parameter table: 201 M Linear parameters per block and stream,
8.05 B over 40 blocks, each stream 49.5% of the model.
"""
import os

import wlq_inputs as wi

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "dit_weights.txt")


def load_golden():
    vals = {}
    for line in open(GOLDEN):
        line = line.split("#", 1)[0].strip()
        if line:
            k, v = line.split()
            vals[k] = float(v)
    return vals


def block_linear_params():
    return 4 * wi.HIDDEN * wi.HIDDEN + 2 * wi.HIDDEN * wi.MLP


def test_params_per_block_match_page():
    g = load_golden()
    assert round(block_linear_params() / 1e6) == g["params_per_block_per_stream_M"]
    assert round(block_linear_params() * g["blocks"] / 1e9, 2) == g["params_per_stream_x40_B"]


def test_mixed_block_layers_cover_the_block():
    total = sum(N * K for _, N, K, _, _ in wi.MIXED_LAYERS)
    assert total == block_linear_params()
