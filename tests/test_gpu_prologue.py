"""GPU parity of the fused prologue (gdr2_chunk_fwd_preact,
gdr2_recurrent_step_preact): pre-activation q, k, b, w, log_alpha through the
kernels' on-load activations, against the fp64 prologue followed by the fp64
oracle. Same bounds as the plain path (rel-L2 <= 1e-4 fp32, <= 5e-3 bf16)."""
import numpy as np
import pytest

import oracle
from helpers import assert_close, to_np, upload
from linear_attention_recurrence_gdr2_b200 import inputs as gen

pytestmark = pytest.mark.gpu

ALL = 7


def gdr2():
    import linear_attention_recurrence_gdr2_b200 as m
    return m


def run(inp, device, flags):
    import torch
    t = upload(inp, device)
    o, sf = gdr2().chunk_fwd(t["q"], t["k"], t["v"], t["log_alpha"], t["b"], t["w"],
                             t["init_state"], t["cu_seqlens"], prologue=flags)
    torch.cuda.synchronize()
    gdr2().check_device_error()
    return to_np(o), to_np(sf)


def reference(inp, flags):
    q, k, la, b, w = oracle.prologue(inp.q, inp.k, inp.log_alpha, inp.b, inp.w, flags)
    return oracle.forward(q, k, inp.v, la, b, w, inp.init_state, inp.cu_seqlens)


@pytest.mark.parametrize("dtype,d", [("bf16", 128), ("fp32", 64), ("fp32", 128), ("bf16", 64)])
def test_chunk_prologue_all_flags(cuda_device, dtype, d):
    inp = gen.preact_inputs(2, 200, 2, d, dtype, seed=21, init_std=0.05)
    o, sf = run(inp, cuda_device, ALL)
    o_r, sf_r = reference(inp, ALL)
    assert_close(f"prologue {dtype} d{d} o", o, o_r, dtype)
    assert_close(f"prologue {dtype} d{d} state", sf, sf_r, dtype)


@pytest.mark.parametrize("flags", [1, 2, 4])
def test_chunk_prologue_single_flags(cuda_device, flags):
    """One activation at a time; the other inputs already in their final form."""
    raw = gen.preact_inputs(1, 130, 2, 128, "bf16", seed=22 + flags)
    ready = gen.make_inputs(1, 130, 2, 128, 128, "bf16", seed=40 + flags)
    pick = lambda name, bit: getattr(raw if flags & bit else ready, name)
    inp = gen.Inputs(pick("q", 1), pick("k", 1), ready.v, pick("log_alpha", 4), pick("b", 2),
                     pick("w", 2), None, None, "bf16")
    o, sf = run(inp, cuda_device, flags)
    o_r, sf_r = reference(inp, flags)
    assert_close(f"prologue flag {flags} o", o, o_r, "bf16")
    assert_close(f"prologue flag {flags} state", sf, sf_r, "bf16")


def test_chunk_prologue_segment_split(cuda_device):
    """The prologue inside both passes of the segment-parallel scan."""
    assert gdr2().workspace_size(1, 2048, 2, 128, 128, 1, gdr2().GDR2_BF16) > 0
    inp = gen.preact_inputs(1, 2048, 2, 128, "bf16", seed=23, init_std=0.05, decay_shift=-5.0)
    o, sf = run(inp, cuda_device, ALL)
    o_r, sf_r = reference(inp, ALL)
    assert_close("prologue split o", o, o_r, "bf16")
    assert_close("prologue split state", sf, sf_r, "bf16")


@pytest.mark.parametrize("dtype,d", [("bf16", 128), ("fp32", 64)])
def test_decode_prologue(cuda_device, dtype, d):
    import torch
    N, H, steps = 3, 2, 3
    raw = gen.preact_inputs(1, N * steps, H, d, dtype, seed=24, init_std=0.05)
    s0 = np.ascontiguousarray(np.repeat(raw.init_state, N, axis=0))  # [N, H, d, d]
    cut = lambda x, t: np.ascontiguousarray(x[0, t * N:(t + 1) * N])  # [N, H, d]
    state = torch.from_numpy(s0).to(cuda_device)
    s_ref = s0.astype(np.float64)
    tdt = torch.bfloat16 if dtype == "bf16" else torch.float32
    for t in range(steps):
        dev = {n: torch.from_numpy(cut(getattr(raw, n), t)).to(cuda_device).to(
            tdt if n != "log_alpha" else torch.float32) for n in ("q", "k", "v", "log_alpha", "b", "w")}
        o = gdr2().recurrent_step(dev["q"], dev["k"], dev["v"], dev["log_alpha"], dev["b"], dev["w"],
                                  state, prologue=ALL)
        torch.cuda.synchronize()
        q, k, la, b, w = oracle.prologue(cut(raw.q, t), cut(raw.k, t), cut(raw.log_alpha, t),
                                         cut(raw.b, t), cut(raw.w, t), ALL)
        o_r, s_ref = oracle.step(q, k, cut(raw.v, t), la, b, w, s_ref)
        assert_close(f"decode prologue {dtype} step {t} o", to_np(o), o_r, dtype)
    assert_close(f"decode prologue {dtype} state", to_np(state), s_ref, dtype)

