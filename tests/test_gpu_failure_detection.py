"""Failure detection on the GPU without a fault: a bounded device wait that
runs out is reported through gdr2_check_device_error, and the context stays
usable for the next operator call."""
import ctypes

import numpy as np
import pytest

import oracle
from helpers import assert_close, to_np, upload
from linear_attention_recurrence_gdr2_b200 import inputs as gen

pytestmark = pytest.mark.gpu


def test_bounded_wait_times_out_and_context_survives(cuda_device):
    import torch
    import linear_attention_recurrence_gdr2_b200 as gdr2
    L = gdr2.lib()
    L.gdr2_selftest_bounded_wait.restype = ctypes.c_int
    L.gdr2_selftest_bounded_wait.argtypes = [ctypes.c_uint32, ctypes.c_void_p]
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    gdr2.check_device_error()                      # start from a clean error word
    assert L.gdr2_selftest_bounded_wait(0, stream) == 1
    assert L.gdr2_selftest_bounded_wait(20000, stream) == 0   # 20 ms limit
    st = L.gdr2_check_device_error(stream)
    assert st == 5, gdr2.status_string(st)         # GDR2_ERR_DEVICE_TIMEOUT
    assert L.gdr2_check_device_error(stream) == 0  # the word was cleared
    # the context is still usable: a normal call succeeds and is correct
    inp = gen.make_inputs(1, 100, 2, 128, 128, "bf16", seed=31, init_std=0.02)
    t = upload(inp, cuda_device)
    o, sf = gdr2.chunk_fwd(t["q"], t["k"], t["v"], t["log_alpha"], t["b"], t["w"], t["init_state"])
    torch.cuda.synchronize()
    gdr2.check_device_error()
    o_r, s_r = oracle.forward(inp.q, inp.k, inp.v, inp.log_alpha, inp.b, inp.w, inp.init_state)
    assert_close("after self-test o", to_np(o), o_r, "bf16")
    assert_close("after self-test state", to_np(sf), s_r, "bf16")
