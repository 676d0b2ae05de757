"""GPU parity of the gate-aware backward (gdr2_chunk_bwd) against the fp64
oracle's reverse loop: every gradient (dq, dk, dv, dlog_alpha, db, dw,
d_init_state) within relative L2 1e-4 for fp32 inputs and 5e-3 for bf16
inputs; the per-element max error is printed beside it. Small cases compare
every element; the layer-shaped workload compares whole (sequence, head) units
recomputed one by one by the oracle."""
import numpy as np
import pytest

import oracle
from helpers import assert_close, to_np, unit_slices, upload
from linear_attention_recurrence_gdr2_b200 import inputs as gen

pytestmark = pytest.mark.gpu
NAMES = ("dq", "dk", "dv", "dlog_alpha", "db", "dw", "d_init_state")


def run_bwd(inp, d_o, d_final, device, alias=False):
    import torch
    import linear_attention_recurrence_gdr2_b200 as m
    t = upload(inp, device)
    dt = t["q"].dtype
    do_t = torch.from_numpy(d_o).to(device=device, dtype=dt)
    df_t = torch.from_numpy(d_final).to(device) if d_final is not None else None
    if alias:
        # d_init_state written over d_final_state through the C ABI directly
        B, T, H, dk = t["q"].shape
        N = inp.num_seqs
        outs = [torch.empty_like(t["q"]) for _ in range(2)] + [torch.empty_like(t["v"])]
        dla = torch.empty_like(t["log_alpha"])
        db, dw = torch.empty_like(t["b"]), torch.empty_like(t["w"])
        code = m.GDR2_BF16 if dt == torch.bfloat16 else m.GDR2_FP32
        need = m.bwd_workspace_size(B, T, H, dk, dk, N, code)
        ws = torch.empty(need, dtype=torch.uint8, device=device)
        p = lambda x: None if x is None else x.data_ptr()
        st = m.lib().gdr2_chunk_bwd(
            p(t["q"]), p(t["k"]), p(t["v"]), p(t["log_alpha"]), p(t["b"]), p(t["w"]),
            p(t["init_state"]), p(t["cu_seqlens"]), p(do_t), p(df_t), B, T, H, dk, dk, N, code,
            p(outs[0]), p(outs[1]), p(outs[2]), p(dla), p(db), p(dw), p(df_t), p(ws), need,
            torch.cuda.current_stream().cuda_stream)
        assert st == 0
        res = (outs[0], outs[1], outs[2], dla, db, dw, df_t)
    else:
        res = m.chunk_bwd(t["q"], t["k"], t["v"], t["log_alpha"], t["b"], t["w"], do_t,
                          t["init_state"], df_t, t["cu_seqlens"])
    torch.cuda.synchronize()
    return [to_np(x) for x in res]


def oracle_bwd(inp, d_o, d_final):
    """The oracle per sequence (it takes fixed-length batches)."""
    if inp.cu_seqlens is None:
        return oracle.backward(inp.q, inp.k, inp.v, inp.log_alpha, inp.b, inp.w,
                               inp.init_state, d_o, d_final)
    H, dk = inp.q.shape[2], inp.q.shape[3]
    outs = [np.zeros(x.shape) for x in (inp.q, inp.k, inp.v, inp.log_alpha, inp.b, inp.w)]
    d_init = np.zeros((inp.num_seqs, H, dk, inp.v.shape[-1]))
    for n in range(inp.num_seqs):
        a, e = int(inp.cu_seqlens[n]), int(inp.cu_seqlens[n + 1])
        sl = lambda x: x[:, a:e]
        s0 = inp.init_state[n:n + 1] if inp.init_state is not None else None
        df = d_final[n:n + 1] if d_final is not None else None
        g = oracle.backward(sl(inp.q), sl(inp.k), sl(inp.v), sl(inp.log_alpha), sl(inp.b),
                            sl(inp.w), s0, sl(d_o), df)
        for o, x in zip(outs, g[:6]):
            o[:, a:e] = x
        d_init[n] = g[6][0]
    return outs + [d_init]


def check(inp, label, device, with_final=True, alias=False):
    d_o, d_final = gen.cotangents(inp, seed=inp.meta.get("seed", 0) + 101)
    if not with_final:
        d_final = None
    got = run_bwd(inp, d_o, d_final, device, alias=alias)
    ref = oracle_bwd(inp, d_o, d_final)
    for name, g, r in zip(NAMES, got, ref):
        assert_close(f"{label} {name}", g, r, inp.dtype)


@pytest.mark.parametrize("dtype", ["fp32", "bf16"])
@pytest.mark.parametrize("d", [64, 128])
@pytest.mark.parametrize("T", [1, 63, 64, 65, 200])
def test_bwd_small_shapes(cuda_device, T, d, dtype):
    inp = gen.make_inputs(2, T, 2, d, d, dtype, seed=T * 5 + d, init_std=0.05)
    check(inp, f"bwd T={T} d={d} {dtype}", cuda_device)


def test_bwd_tiny_fp32_workload(cuda_device):
    """The tiny fp32 workload (B=1, H=1, T=256, d=64, zero initial state), no
    final-state cotangent: every element."""
    check(gen.tiny_fp32(), "bwd tiny fp32", cuda_device, with_final=False)


@pytest.mark.parametrize("dtype,d", [("fp32", 64), ("bf16", 128)])
def test_bwd_varlen(cuda_device, dtype, d):
    """Packed batch with an empty sequence, partial chunks and a 1-token one."""
    lengths = [1, 64, 0, 130, 63, 65, 7, 192]
    inp = gen.make_inputs(1, 0, 2, d, d, dtype, seed=d + 3, init_std=0.05, lengths=lengths)
    check(inp, f"bwd varlen d={d} {dtype}", cuda_device)


def test_bwd_strong_decay_and_no_state(cuda_device):
    """Faster forgetting (log_alpha scale 1.0), no initial state, no final cotangent."""
    inp = gen.make_inputs(2, 150, 2, 64, 64, "fp32", seed=9, la_scale=1.0)
    check(inp, "bwd strong decay", cuda_device, with_final=False)


def test_bwd_d_init_aliases_d_final(cuda_device):
    inp = gen.make_inputs(2, 100, 3, 128, 128, "bf16", seed=4, init_std=0.05)
    check(inp, "bwd alias", cuda_device, alias=True)


def test_bwd_layer_prefill_units(cuda_device):
    """The layer-shaped workload (B=4, T=2048, H=16, d=128, bf16) in one call;
    two (sequence, head) units recomputed by the oracle."""
    inp = gen.layer_prefill()
    d_o, d_final = gen.cotangents(inp, seed=7)
    got = run_bwd(inp, d_o, d_final, cuda_device)
    for n, h in ((0, 0), (3, 15)):
        sl, rows, s0 = unit_slices(inp, n, h)
        ref = oracle.backward(sl(inp.q), sl(inp.k), sl(inp.v), sl(inp.log_alpha), sl(inp.b),
                              sl(inp.w), s0, sl(d_o), d_final[n:n + 1, h:h + 1])
        for name, g, r in zip(NAMES[:6], got[:6], ref[:6]):
            assert_close(f"layer unit({n},{h}) {name}", g[rows], r[0, :, 0], "bf16")
        assert_close(f"layer unit({n},{h}) d_init_state", got[6][n, h], ref[6][0, 0], "bf16")


def test_bwd_deterministic(cuda_device):
    """No atomics and a fixed reduction order: two calls agree bit for bit."""
    inp = gen.make_inputs(2, 300, 4, 128, 128, "bf16", seed=21, init_std=0.05)
    d_o, d_final = gen.cotangents(inp, seed=22)
    a = run_bwd(inp, d_o, d_final, cuda_device)
    b = run_bwd(inp, d_o, d_final, cuda_device)
    for name, x, y in zip(NAMES, a, b):
        assert np.array_equal(x, y), f"{name} differs between two identical calls"
