"""The sizes the pages print (tests/golden/page_values.json, each with its
citation), checked against the workloads, the oracle and the library's
workspace arithmetic (CPU only)."""
import json
import os

import linear_attention_recurrence_gdr2_b200 as gdr2
import oracle
from linear_attention_recurrence_gdr2_b200 import inputs as gen

HERE = os.path.dirname(os.path.abspath(__file__))
GOLD = {v["name"]: v["value"] for v in
        json.load(open(os.path.join(HERE, "golden", "page_values.json")))["values"]}


def test_state_size_per_layer_matches_the_page():
    """One batch element's recurrent state in the layer-shaped workload holds
    the printed number of floats, both as the workload defines it and as the
    oracle returns it."""
    inp = gen.make_inputs(1, 3, 16, 128, 128, "bf16", seed=0)     # the layer head shape, 3 tokens
    H, dk, dv = inp.q.shape[2], inp.q.shape[3], inp.v.shape[3]
    assert H * dk * dv == GOLD["state_floats_per_layer_per_batch_element"]
    _, final = oracle.forward(inp.q, inp.k, inp.v, inp.log_alpha, inp.b, inp.w, None)
    assert final[0].size == GOLD["state_floats_per_layer_per_batch_element"]


def test_chunk_length_matches_the_page():
    """The backward keeps one checkpoint slot per printed chunk length of
    tokens: its workspace grows by one slot at every multiple of C."""
    C = GOLD["chunk_length"]
    size = lambda T: gdr2.bwd_workspace_size(1, T, 1, 64, 64, 1, gdr2.GDR2_FP32)
    per_token = 2 * 64 * 4                    # u and du, fp32
    per_slot = 2 * 64 * 64 * 4                # state and cotangent checkpoints, fp32
    for T in (C - 1, C, 2 * C - 1, 2 * C, 5 * C + 3):
        expect = ((T // C + 1) * per_slot + T * per_token + 255) // 256 * 256
        assert size(T) == expect
