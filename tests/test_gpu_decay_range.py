"""GPU parity over the whole decay domain (alpha anywhere in (0, 1]).

The rule admits any per-channel decay ("Gated Delta Rule-2: two gates instead
of one", ainews.random.gg article on Gated DeltaNet-2), including channels
that forget almost everything at every token. The chunk kernels absorb the
decay into factors e^{+-(g_r - g_31)}; where a chunk's decay takes those past
their range (|g_r - g_31| > 64), the tensor-core kernel recomputes the whole
(sequence, head) unit with the exact token recurrence and the CUDA-core
kernel runs that chunk token by token. These cases check every element
against the fp64 oracle at the usual bounds (fp32 1e-4, bf16 5e-3):
  strong  every key channel: log alpha ~ U(-20, -5)   (chunk sums near -800)
  mixed   a third of the key channels strong, the rest the usual weak decay
  none    alpha = 1
  edge    half-chunk sums near -60 (the chunk form at the edge of its factor
          range)
  window  about -74 over every 64 consecutive tokens (the chunk form at the
          edge of its chunk-to-chunk state factor)
"""
import numpy as np
import pytest

import oracle
from helpers import assert_close, rel_l2, to_np, upload
from linear_attention_recurrence_gdr2_b200 import inputs as gen

pytestmark = pytest.mark.gpu

REGIMES = ["strong", "mixed", "none", "edge", "window"]


def gdr2():
    import linear_attention_recurrence_gdr2_b200 as m
    return m


def run_and_check(inp, device, label, prologue=0):
    import torch
    t = upload(inp, device)
    o, sf = gdr2().chunk_fwd(t["q"], t["k"], t["v"], t["log_alpha"], t["b"], t["w"],
                             t["init_state"], t["cu_seqlens"], prologue=prologue)
    torch.cuda.synchronize()
    gdr2().check_device_error()
    if prologue:
        q, k, la, b, w = oracle.prologue(inp.q, inp.k, inp.log_alpha, inp.b, inp.w, prologue)
    else:
        q, k, la, b, w = inp.q, inp.k, inp.log_alpha, inp.b, inp.w
    o_r, sf_r = oracle.forward(q, k, inp.v, la, b, w, inp.init_state, inp.cu_seqlens)
    assert_close(f"{label} o", to_np(o), o_r, inp.dtype)
    assert_close(f"{label} state", to_np(sf), sf_r, inp.dtype)


@pytest.mark.parametrize("regime", REGIMES)
@pytest.mark.parametrize("dtype,d", [("bf16", 128), ("bf16", 64), ("fp32", 64), ("fp32", 128)])
def test_decay_regimes(cuda_device, regime, dtype, d):
    """Two sequences of 200 tokens (ragged last chunk), three heads, nonzero
    initial states."""
    inp = gen.make_inputs(2, 200, 3, d, d, dtype, seed=31, init_std=0.05)
    gen.with_decay_regime(inp, regime, seed=32)
    run_and_check(inp, cuda_device, f"{regime} {dtype} d={d}")


@pytest.mark.parametrize("dtype,d", [("bf16", 128), ("fp32", 64)])
def test_one_strong_head_among_weak_ones(cuda_device, dtype, d):
    """Only head 1 of three has strong decay: units that leave the factor
    range and units that do not run side by side in one launch."""
    inp = gen.make_inputs(2, 300, 3, d, d, dtype, seed=33, init_std=0.05)
    strong = gen.with_decay_regime(gen.make_inputs(2, 300, 3, d, d, dtype, seed=33), "strong", seed=34)
    inp.log_alpha[:, :, 1] = strong.log_alpha[:, :, 1]
    run_and_check(inp, cuda_device, f"one strong head {dtype} d={d}")


def test_strong_decay_in_one_chunk_only(cuda_device):
    """A single chunk (tokens 128..191) of strong decay inside weak decay:
    the first chunks run fast, then the unit is recomputed exactly."""
    inp = gen.make_inputs(1, 400, 2, 128, 128, "bf16", seed=35, init_std=0.05)
    strong = gen.with_decay_regime(gen.make_inputs(1, 400, 2, 128, 128, "bf16", seed=35), "strong", seed=36)
    inp.log_alpha[:, 128:192] = strong.log_alpha[:, 128:192]
    run_and_check(inp, cuda_device, "one strong chunk")


@pytest.mark.parametrize("regime", ["strong", "mixed"])
def test_decay_regimes_packed_batch(cuda_device, regime):
    lengths = [1, 64, 0, 130, 63, 65, 7, 192]
    inp = gen.make_inputs(1, 0, 2, 128, 128, "bf16", seed=37, init_std=0.05, lengths=lengths)
    gen.with_decay_regime(inp, regime, seed=38)
    run_and_check(inp, cuda_device, f"packed {regime}")


@pytest.mark.parametrize("regime", ["strong", "mixed", "edge", "window"])
def test_decay_regimes_segment_split(cuda_device, regime):
    """Few long bf16 sequences (segment-parallel scan, 4 segments): segment
    jobs and identity jobs that leave the factor range are recomputed exactly
    before the segments are combined."""
    assert gdr2().workspace_size(1, 2048, 2, 128, 128, 1, gdr2().GDR2_BF16) > 0  # split in use
    inp = gen.make_inputs(1, 2048, 2, 128, 128, "bf16", seed=39, init_std=0.05)
    gen.with_decay_regime(inp, regime, seed=40)
    run_and_check(inp, cuda_device, f"segments {regime}")


@pytest.mark.parametrize("dtype,d", [("bf16", 128), ("fp32", 64)])
def test_strong_decay_with_fused_prologue(cuda_device, dtype, d):
    """Pre-activation inputs whose decay branch is about +10 before the
    -softplus (log alpha about -10 per token): the exact path applies the
    same activations on load."""
    inp = gen.preact_inputs(2, 150, 2, d, dtype, seed=41, init_std=0.05, decay_shift=10.0)
    run_and_check(inp, cuda_device, f"preact strong {dtype} d={d}", prologue=gdr2().GDR2_PROLOGUE_ALL)


def test_strong_decay_noalloc_matches(cuda_device):
    """The allocation-free entry point takes the same exact path."""
    import torch
    inp = gen.make_inputs(2, 200, 2, 128, 128, "bf16", seed=42, init_std=0.05)
    gen.with_decay_regime(inp, "mixed", seed=43)
    t = upload(inp, cuda_device)
    o1, s1 = gdr2().chunk_fwd(t["q"], t["k"], t["v"], t["log_alpha"], t["b"], t["w"], t["init_state"])
    o2 = torch.empty_like(o1)
    s2 = torch.empty_like(s1)
    gdr2().chunk_fwd_noalloc(t["q"], t["k"], t["v"], t["log_alpha"], t["b"], t["w"], t["init_state"],
                             o=o2, final_state=s2)
    torch.cuda.synchronize()
    assert np.array_equal(to_np(o1), to_np(o2)) and np.array_equal(to_np(s1), to_np(s2))


def test_strong_decay_deterministic(cuda_device):
    import torch
    inp = gen.make_inputs(2, 260, 2, 128, 128, "bf16", seed=44, init_std=0.05)
    gen.with_decay_regime(inp, "strong", seed=45)
    t = upload(inp, cuda_device)
    runs = []
    for _ in range(2):
        o, s = gdr2().chunk_fwd(t["q"], t["k"], t["v"], t["log_alpha"], t["b"], t["w"], t["init_state"])
        torch.cuda.synchronize()
        runs.append((to_np(o), to_np(s)))
    assert np.array_equal(runs[0][0], runs[1][0]) and np.array_equal(runs[0][1], runs[1][1])
    assert rel_l2(runs[0][0], runs[1][0]) == 0.0
