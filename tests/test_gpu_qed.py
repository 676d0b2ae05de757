"""GPU parity of the QED forward (gdr2_qed_fwd) against the fp64 QED oracle.

QED is the second erase direction of "The Query Knows What to Forget"
(thelatestinai.com listing, abstract and Table 1); the page does not print the
update, so both sides compute the same stated reading and the comparison pins
the kernel to the oracle, not to the paper. Every element of o and of the
final state is checked at the usual bounds (fp32 1e-4, bf16 5e-3), over the
paper's arms (gate and projection on or off, query or fixed direction),
packed batches and both head sizes.
"""
import numpy as np
import pytest

import oracle
from helpers import assert_close, to_np, upload
from linear_attention_recurrence_gdr2_b200 import inputs as gen

pytestmark = pytest.mark.gpu


def gdr2():
    import linear_attention_recurrence_gdr2_b200 as m
    return m


def run(inp, device, strength, direction=None, flags=3):
    import torch
    t = upload(inp, device)
    lam = torch.tensor(strength, dtype=torch.float32, device=device)
    dirs = torch.tensor(direction, dtype=torch.float32, device=device) if direction is not None else None
    o, sf = gdr2().qed_fwd(t["q"], t["k"], t["v"], t["log_alpha"], t["b"], t["w"], lam, dirs, flags,
                           t["init_state"], t["cu_seqlens"])
    torch.cuda.synchronize()
    o_r, sf_r = oracle.qed_forward(inp.q, inp.k, inp.v, inp.log_alpha, inp.b, inp.w, np.asarray(strength),
                                   direction, flags, inp.init_state, inp.cu_seqlens)
    return to_np(o), to_np(sf), o_r, sf_r


@pytest.mark.parametrize("flags", [3, 1, 2, 0])
@pytest.mark.parametrize("dtype,d", [("bf16", 128), ("fp32", 64), ("fp32", 128), ("bf16", 64)])
def test_qed_arms(cuda_device, flags, dtype, d):
    inp = gen.make_inputs(2, 150, 3, d, d, dtype, seed=51, init_std=0.05)
    strength = [0.1, 0.5, 1.0]
    o, sf, o_r, sf_r = run(inp, cuda_device, strength, flags=flags)
    assert_close(f"qed flags={flags} {dtype} d={d} o", o, o_r, dtype)
    assert_close(f"qed flags={flags} {dtype} d={d} state", sf, sf_r, dtype)


@pytest.mark.parametrize("dtype", ["bf16", "fp32"])
def test_qed_fixed_direction_arm(cuda_device, dtype):
    inp = gen.make_inputs(1, 200, 2, 128, 128, dtype, seed=52, init_std=0.05)
    rng = np.random.default_rng(53)
    direction = rng.standard_normal((2, 128))
    direction /= np.linalg.norm(direction, axis=1, keepdims=True)
    o, sf, o_r, sf_r = run(inp, cuda_device, [0.3, 0.8], direction=direction)
    assert_close(f"qed fixed direction {dtype} o", o, o_r, dtype)
    assert_close(f"qed fixed direction {dtype} state", sf, sf_r, dtype)


def test_qed_packed_batch(cuda_device):
    lengths = [1, 64, 0, 130, 63, 7]
    inp = gen.make_inputs(1, 0, 2, 128, 128, "bf16", seed=54, init_std=0.05, lengths=lengths)
    o, sf, o_r, sf_r = run(inp, cuda_device, [0.4, 0.9])
    assert_close("qed packed o", o, o_r, "bf16")
    assert_close("qed packed state", sf, sf_r, "bf16")


def test_qed_zero_strength_matches_the_chunk_forward(cuda_device):
    """Strength 0 is the plain rule: the token path agrees with the chunk
    forward within both paths' bounds against the oracle."""
    import torch
    inp = gen.make_inputs(2, 300, 2, 128, 128, "fp32", seed=55, init_std=0.05)
    o, sf, o_r, sf_r = run(inp, cuda_device, [0.0, 0.0])
    o_p, sf_p = oracle.forward(inp.q, inp.k, inp.v, inp.log_alpha, inp.b, inp.w, inp.init_state)
    assert np.array_equal(o_r, o_p) and np.array_equal(sf_r, sf_p)
    t = upload(inp, cuda_device)
    o_c, sf_c = gdr2().chunk_fwd(t["q"], t["k"], t["v"], t["log_alpha"], t["b"], t["w"], t["init_state"])
    torch.cuda.synchronize()
    assert_close("qed strength 0 vs chunk forward", o, to_np(o_c), "fp32")
    assert_close("qed strength 0 state vs chunk forward", sf, to_np(sf_c), "fp32")


def test_qed_query_parallel_to_key_is_the_plain_rule(cuda_device):
    """Degenerate case of the reading: a query parallel to the key has no part
    orthogonal to it, so the second erase vanishes and the step is the plain
    rule (both sides decide u = 0 by the same relative threshold)."""
    inp = gen.make_inputs(1, 90, 2, 64, 64, "fp32", seed=56, init_std=0.05)
    inp.q[...] = 2.0 * inp.k
    o, sf, _, _ = run(inp, cuda_device, [0.7, 1.0])
    o_p, sf_p = oracle.forward(inp.q, inp.k, inp.v, inp.log_alpha, inp.b, inp.w, inp.init_state)
    assert_close("qed q || k o", o, o_p, "fp32")
    assert_close("qed q || k state", sf, sf_p, "fp32")
