"""gdr2_chunk_fwd_noalloc: the chunk forward for callers that cannot allocate
device memory (they get only their input and output buffers). It keeps its
scratch in a fixed array inside the library; this checks, through the C ABI,
that two calls in a row give the same results as gdr2_chunk_fwd with a
caller-provided workspace, and that oversized packed batches are rejected.
The file is named to be collected last."""
import ctypes

import numpy as np
import pytest

from helpers import TOL, rel_l2, to_np, upload
from linear_attention_recurrence_gdr2_b200 import inputs as gen

pytestmark = pytest.mark.gpu


def _run_both(inp, device):
    import torch
    import linear_attention_recurrence_gdr2_b200 as gdr2
    t = upload(inp, device)
    B, T, H, dk = inp.q.shape
    N = inp.num_seqs
    o_ref, s_ref = gdr2.chunk_fwd(t["q"], t["k"], t["v"], t["log_alpha"], t["b"], t["w"],
                                  t["init_state"], t["cu_seqlens"])
    o = torch.empty_like(o_ref)
    s = torch.empty_like(s_ref)
    p = lambda x: ctypes.c_void_p(x.data_ptr()) if x is not None else None
    st = gdr2.lib().gdr2_chunk_fwd_noalloc(
        p(t["q"]), p(t["k"]), p(t["v"]), p(t["log_alpha"]), p(t["b"]), p(t["w"]),
        p(t["init_state"]), p(t["cu_seqlens"]), B, T, H, dk, dk, N, gdr2.GDR2_BF16,
        p(o), p(s), ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))
    assert st == 0, gdr2.status_string(st)
    torch.cuda.synchronize()
    gdr2.check_device_error()
    return to_np(o), to_np(s), to_np(o_ref), to_np(s_ref)


def test_noalloc_matches_workspace_entry_point_twice(cuda_device):
    # two different packed batches back to back: the second call must not
    # depend on what the first one left in the library's scratch array
    for seed, n in ((21, 40), (22, 7)):
        lengths = np.random.default_rng(seed).integers(1, 300, size=n)
        inp = gen.make_inputs(1, 0, 4, 128, 128, "bf16", seed=seed, init_std=0.02, lengths=lengths)
        o, s, o_ref, s_ref = _run_both(inp, cuda_device)
        assert rel_l2(o, o_ref) <= TOL["bf16"] and rel_l2(s, s_ref) <= TOL["bf16"]
        assert np.array_equal(o, o_ref) and np.array_equal(s, s_ref)


def test_noalloc_fixed_length_batch(cuda_device):
    inp = gen.make_inputs(2, 130, 3, 128, 128, "bf16", seed=23, init_std=0.02)
    o, s, o_ref, s_ref = _run_both(inp, cuda_device)
    assert rel_l2(o, o_ref) <= TOL["bf16"] and rel_l2(s, s_ref) <= TOL["bf16"]


def test_noalloc_rejects_too_many_sequences(cuda_device):
    import linear_attention_recurrence_gdr2_b200 as gdr2
    fake = ctypes.c_void_p(0x10000)
    st = gdr2.lib().gdr2_chunk_fwd_noalloc(fake, fake, fake, fake, fake, fake, None, fake,
                                           1, 20000, 2, 128, 128, 16385, gdr2.GDR2_BF16,
                                           fake, fake, None)
    assert st == 2  # GDR2_ERR_UNSUPPORTED, before any launch
