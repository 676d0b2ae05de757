"""GPU parity: the CUDA path through the C ABI against the fp64 oracle.

Small cases compare every element; the full-size workloads compare whole
(sequence, head) units that the oracle recomputes one by one, in the same
launch configuration the benchmark times. Bound: relative L2 error <= 1e-4
for fp32 inputs and <= 5e-3 for bf16 inputs (fp32 state), on o and on the
final state; the per-element max error is printed beside it.
"""
import numpy as np
import pytest

import oracle
from helpers import TOL, assert_close, rel_l2, to_np, unit_slices, upload
from linear_attention_recurrence_gdr2_b200 import inputs as gen

pytestmark = pytest.mark.gpu


def gdr2():
    import linear_attention_recurrence_gdr2_b200 as m
    return m


def run_chunk(inp, device, final=True):
    t = upload(inp, device)
    o, sf = gdr2().chunk_fwd(t["q"], t["k"], t["v"], t["log_alpha"], t["b"], t["w"],
                             t["init_state"], t["cu_seqlens"], output_final_state=final)
    import torch
    torch.cuda.synchronize()
    gdr2().check_device_error()
    return to_np(o), (to_np(sf) if sf is not None else None)


def check_full(inp, device, label):
    o, sf = run_chunk(inp, device)
    o_r, sf_r = oracle.forward(inp.q, inp.k, inp.v, inp.log_alpha, inp.b, inp.w,
                               inp.init_state, inp.cu_seqlens)
    assert_close(f"{label} o", o, o_r, inp.dtype)
    assert_close(f"{label} state", sf, sf_r, inp.dtype)


def check_full_by_head(inp, device, label):
    """Every element of o and of the final states, the oracle run one head at
    a time (bounded host memory); the relative L2 errors are those of the
    whole tensors, accumulated over the heads."""
    import torch
    t = upload(inp, device)
    o_d, sf_d = gdr2().chunk_fwd(t["q"], t["k"], t["v"], t["log_alpha"], t["b"], t["w"],
                                 t["init_state"], t["cu_seqlens"])
    torch.cuda.synchronize()
    gdr2().check_device_error()
    del t
    H = inp.q.shape[2]
    err = {"o": [0.0, 0.0], "state": [0.0, 0.0]}
    worst = {"o": 0.0, "state": 0.0}
    for h in range(H):
        sl = lambda x: np.ascontiguousarray(x[:, :, h:h + 1])
        s0 = np.ascontiguousarray(inp.init_state[:, h:h + 1]) if inp.init_state is not None else None
        o_r, sf_r = oracle.forward(sl(inp.q), sl(inp.k), sl(inp.v), sl(inp.log_alpha), sl(inp.b),
                                   sl(inp.w), s0, inp.cu_seqlens)
        o_h = o_d[:, :, h:h + 1].float().cpu().numpy()
        sf_h = sf_d[:, h:h + 1].cpu().numpy()
        for key, x, r in (("o", o_h, o_r), ("state", sf_h, sf_r)):
            d = np.asarray(x, np.float64) - r
            err[key][0] += float(np.sum(d * d))
            err[key][1] += float(np.sum(r * r))
            worst[key] = max(worst[key], float(np.max(np.abs(d))) if d.size else 0.0)
            assert np.all(np.isfinite(x)), f"{label} {key}: non-finite values"
    for key in ("o", "state"):
        e = float(np.sqrt(err[key][0] / err[key][1]))
        print(f"{label} {key}: rel_l2={e:.3e} max_abs={worst[key]:.3e} (tol {TOL[inp.dtype]:.0e})")
        assert e <= TOL[inp.dtype], f"{label} {key}: rel_l2 {e:.3e} > {TOL[inp.dtype]:.0e}"


def check_units(inp, device, units, label):
    o, sf = run_chunk(inp, device)
    for n, h in units:
        sl, rows, s0 = unit_slices(inp, n, h)
        o_r, sf_r = oracle.forward(sl(inp.q), sl(inp.k), sl(inp.v), sl(inp.log_alpha),
                                   sl(inp.b), sl(inp.w), s0)
        assert_close(f"{label} unit({n},{h}) o", o[rows], o_r[0, :, 0], inp.dtype)
        assert_close(f"{label} unit({n},{h}) state", sf[n, h], sf_r[0, 0], inp.dtype)
    return o, sf


# ---------------------------------------------------------------- chunk fwd
def test_tiny_fp32_workload(cuda_device):
    """B=1, H=1, T=256, d=64, fp32, zero initial state, seed 0: every element."""
    check_full(gen.tiny_fp32(), cuda_device, "tiny fp32")


@pytest.mark.parametrize("dtype", ["fp32", "bf16"])
@pytest.mark.parametrize("d", [64, 128])
@pytest.mark.parametrize("T", [1, 63, 64, 65, 200])
def test_chunk_small_shapes(cuda_device, T, d, dtype):
    inp = gen.make_inputs(2, T, 3, d, d, dtype, seed=T * 7 + d, init_std=0.05)
    check_full(inp, cuda_device, f"T={T} d={d} {dtype}")


@pytest.mark.parametrize("dtype", ["fp32", "bf16"])
@pytest.mark.parametrize("d", [64, 128])
def test_chunk_varlen_small(cuda_device, d, dtype):
    lengths = [1, 64, 0, 130, 63, 65, 7, 192]
    inp = gen.make_inputs(1, 0, 2, d, d, dtype, seed=d, init_std=0.05, lengths=lengths)
    check_full(inp, cuda_device, f"varlen d={d} {dtype}")


def test_chunk_varlen_many_sequences(cuda_device):
    """300 packed sequences (lengths 0..200, ties included): exercises the
    longest-first ordering with a non-power-of-two count."""
    lengths = np.random.default_rng(12).integers(0, 201, size=300)
    inp = gen.make_inputs(1, 0, 2, 128, 128, "bf16", seed=12, init_std=0.05, lengths=lengths)
    check_full(inp, cuda_device, "varlen 300 seqs")


def test_chunk_varlen_above_sort_limit(cuda_device):
    """More sequences than the on-device sort handles: identity order."""
    lengths = np.random.default_rng(13).integers(0, 4, size=16400)
    inp = gen.make_inputs(1, 0, 1, 64, 64, "fp32", seed=13, init_std=0.05, lengths=lengths)
    check_full(inp, cuda_device, "varlen 16400 seqs")


def test_chunk_zero_initial_state_and_no_final_state(cuda_device):
    inp = gen.make_inputs(1, 100, 2, 128, 128, "bf16", seed=3)
    o, sf = run_chunk(inp, cuda_device, final=False)
    assert sf is None
    o_r, _ = oracle.forward(inp.q, inp.k, inp.v, inp.log_alpha, inp.b, inp.w)
    assert_close("no-final o", o, o_r, "bf16")


def test_chunk_final_state_may_alias_initial_state(cuda_device):
    import torch
    inp = gen.make_inputs(2, 130, 2, 64, 64, "fp32", seed=4, init_std=0.1)
    t = upload(inp, cuda_device)
    s = t["init_state"].clone()
    o, sf = gdr2().chunk_fwd(t["q"], t["k"], t["v"], t["log_alpha"], t["b"], t["w"], s,
                             final_state=s)
    torch.cuda.synchronize()
    o_r, sf_r = oracle.forward(inp.q, inp.k, inp.v, inp.log_alpha, inp.b, inp.w, inp.init_state)
    assert_close("alias o", to_np(o), o_r, "fp32")
    assert_close("alias state", to_np(s), sf_r, "fp32")


def test_chunk_empty_sequence_keeps_state(cuda_device):
    inp = gen.make_inputs(1, 0, 2, 64, 64, "bf16", seed=5, init_std=0.1, lengths=[0, 0])
    o, sf = run_chunk(inp, cuda_device)
    assert o.shape[1] == 0
    assert np.array_equal(sf, inp.init_state.astype(np.float64))


def test_chunk_deterministic(cuda_device):
    inp = gen.make_inputs(2, 300, 4, 128, 128, "bf16", seed=6, init_std=0.01)
    o1, s1 = run_chunk(inp, cuda_device)
    o2, s2 = run_chunk(inp, cuda_device)
    assert np.array_equal(o1, o2) and np.array_equal(s1, s2)


def test_chunk_strong_decay_in_range(cuda_device):
    """Per-token log-decay down to about -1 (chunk sums near -64) stays finite
    and accurate: the pairwise factors keep e^{g_r - g_s} <= 1."""
    inp = gen.make_inputs(1, 256, 2, 128, 128, "bf16", seed=8, la_scale=1.2, init_std=0.01)
    check_full(inp, cuda_device, "strong decay")


@pytest.mark.parametrize("B,T,H,la_scale,init", [
    (1, 2048, 2, 0.01, 0.05),    # 4 segments of 512 tokens, nonzero initial state
    (2, 1000, 3, 0.02, None),    # 2 segments, ragged last chunk
    (1, 8192, 1, 0.005, 0.02),   # 16 segments: the longest combine chain
    (1, 1700, 1, 0.02, 0.05),    # 3 segments of 576 tokens: correction tiles of 128 rows
                                 # straddle the segment boundaries; ragged end
])
def test_chunk_segment_split(cuda_device, B, T, H, la_scale, init):
    """Few long bf16 sequences run as concurrent segments (from the segment's
    entry state 0, or the true one for the first; and from the identity with
    z = 0), then the affine combine of the segment states and the o
    correction. Weak decay keeps each segment's entry state influential.
    Every element against the oracle."""
    assert gdr2().workspace_size(B, T, H, 128, 128, B, gdr2().GDR2_BF16) > 0  # split in use
    inp = gen.make_inputs(B, T, H, 128, 128, "bf16", seed=11, la_scale=la_scale, init_std=init)
    check_full(inp, cuda_device, f"segments B{B} T{T} H{H}")


def test_chunk_segment_split_matches_serial_scan(cuda_device):
    """The split and the serial scan (the allocation-free entry point never
    splits) agree with each other as well as with the oracle."""
    import torch
    inp = gen.make_inputs(1, 2048, 2, 128, 128, "bf16", seed=12, la_scale=0.01, init_std=0.05)
    o_split, s_split = run_chunk(inp, cuda_device)
    t = upload(inp, cuda_device)
    o2 = torch.empty_like(t["v"])
    s2 = torch.empty_like(t["init_state"])
    gdr2().chunk_fwd_noalloc(t["q"], t["k"], t["v"], t["log_alpha"], t["b"], t["w"],
                             t["init_state"], t["cu_seqlens"], o=o2, final_state=s2)
    torch.cuda.synchronize()
    o_r, s_r = oracle.forward(inp.q, inp.k, inp.v, inp.log_alpha, inp.b, inp.w, inp.init_state)
    assert_close("serial o", to_np(o2), o_r, "bf16")
    assert_close("serial state", to_np(s2), s_r, "bf16")
    assert_close("split o", o_split, o_r, "bf16")
    assert_close("split state", s_split, s_r, "bf16")
    assert rel_l2(o_split, to_np(o2)) < TOL["bf16"] and rel_l2(s_split, to_np(s2)) < TOL["bf16"]


@pytest.mark.slow
def test_layer_prefill_full_size(cuda_device):
    """B=4, H=16, T=2048, d=128, bf16: all 64 (sequence, head) units, every element."""
    check_full_by_head(gen.layer_prefill(), cuda_device, "prefill")


@pytest.mark.slow
def test_long_context_full_size(cuda_device):
    """B=1, H=16, T=32768, d=128, bf16, slow forgetting, nonzero initial state
    (segment-parallel scan, 2 segments): all 16 heads, every element."""
    check_full_by_head(gen.long_context(), cuda_device, "long")


@pytest.mark.slow
def test_varlen_packed_full_size(cuda_device):
    """64 packed sequences, lengths in [128, 8192], H=16, bf16, per-sequence
    states: every sequence and head, every element."""
    check_full_by_head(gen.varlen_packed(), cuda_device, "varlen")


@pytest.mark.slow
def test_long_single_head_sixteen_segments(cuda_device):
    """B=1, H=1, T=32768, d=128, bf16, slow forgetting: the segment split at
    its most segments (16 of 2048 tokens), the longest combine chain."""
    import linear_attention_recurrence_gdr2_b200 as m
    ws = m.workspace_size(1, 32768, 1, 128, 128, 1, m.GDR2_BF16)
    assert ws >= 32768 * 256 + 2 * 16 * 65536  # psi and two arrays of 16 segment states
    check_full(gen.long_context(T=32768, H=1), cuda_device, "long H=1 P=16")


# ------------------------------------------------------- method edge cases
def edge_case_inputs(case, dtype, d, seed):
    """The method's degenerate settings on otherwise usual inputs (two
    sequences of 200 tokens, three heads, nonzero initial states):
      no_erase     b = 0: decayed linear attention (nothing is erased)
      exact_recall b = w = 1, alpha = 1, unit keys: the delta rule at full
                   strength, where (I + A) is least well conditioned
      no_write     w = 0: pure erase (the state only decays and is erased)
    """
    inp = gen.make_inputs(2, 200, 3, d, d, dtype, seed=seed, init_std=0.05)
    if case == "no_erase":
        inp.b[...] = 0.0
    elif case == "exact_recall":
        inp.b[...] = 1.0
        inp.w[...] = 1.0
        inp.log_alpha[...] = 0.0
    elif case == "no_write":
        inp.w[...] = 0.0
    else:
        raise ValueError(case)
    return inp


@pytest.mark.parametrize("case", ["no_erase", "exact_recall", "no_write"])
@pytest.mark.parametrize("dtype,d", [("bf16", 128), ("bf16", 64), ("fp32", 64), ("fp32", 128)])
def test_method_edge_cases(cuda_device, case, dtype, d):
    check_full(edge_case_inputs(case, dtype, d, seed=51), cuda_device, f"{case} {dtype} d={d}")


def test_exact_recall_reads_back_the_value(cuda_device):
    """With b = w = 1, alpha = 1 and the query equal to the key, the readout
    is the token's own value (S_t^T k_t = v_t for a unit key): checked on the
    GPU output itself, for fp32 inputs whose keys are unit vectors."""
    inp = edge_case_inputs("exact_recall", "fp32", 64, seed=52)
    inp.q[...] = inp.k
    o, _ = run_chunk(inp, cuda_device)
    assert rel_l2(o, inp.v.astype(np.float64)) < 1e-4


# ------------------------------------------------------------------- decode
def run_decode(dec, device, steps):
    import torch
    dt = torch.bfloat16 if dec.dtype == "bf16" else torch.float32
    t = lambda x, d: torch.from_numpy(np.ascontiguousarray(x)).to(device=device, dtype=d)
    state = t(dec.state, torch.float32)
    outs = []
    for s in range(steps):
        o = gdr2().recurrent_step(t(dec.q[s], dt), t(dec.k[s], dt), t(dec.v[s], dt),
                                  t(dec.log_alpha[s], torch.float32), t(dec.b[s], dt),
                                  t(dec.w[s], dt), state)
        outs.append(to_np(o))
    torch.cuda.synchronize()
    return np.stack(outs), to_np(state)


def oracle_decode(dec, steps):
    S = dec.state
    outs = []
    for s in range(steps):
        o, S = oracle.step(dec.q[s], dec.k[s], dec.v[s], dec.log_alpha[s], dec.b[s], dec.w[s], S)
        outs.append(o)
    return np.stack(outs), S


@pytest.mark.parametrize("dtype", ["fp32", "bf16"])
@pytest.mark.parametrize("d", [64, 128])
def test_decode_small(cuda_device, d, dtype):
    dec = gen.make_decode_inputs(3, 5, d, d, 6, dtype, seed=d + 1)
    o, S = run_decode(dec, cuda_device, 6)
    o_r, S_r = oracle_decode(dec, 6)
    for s in range(6):
        assert_close(f"decode step {s} o", o[s], o_r[s], dtype)
    assert_close("decode state", S, S_r, dtype)


@pytest.mark.slow
def test_decode_full_size(cuda_device):
    """N=256 x H=16, d=128, fp32 state, 64 consecutive bf16 steps; all heads."""
    dec = gen.decode_batch()
    o, S = run_decode(dec, cuda_device, 64)
    o_r, S_r = oracle_decode(dec, 64)
    worst = max(rel_l2(o[s], o_r[s]) for s in range(64))
    print(f"decode full: worst per-step o rel_l2 {worst:.3e}")
    assert worst <= TOL["bf16"]
    assert_close("decode full state", S, S_r, "bf16")


def test_decode_matches_chunk_forward(cuda_device):
    """T decode steps from S0 and one chunk_fwd over the same T tokens agree."""
    import torch
    inp = gen.make_inputs(2, 70, 3, 128, 128, "fp32", seed=9, init_std=0.05)
    o_c, s_c = run_chunk(inp, cuda_device)
    t = upload(inp, cuda_device)
    state = t["init_state"].clone()
    o_d = []
    for s in range(70):
        sl = lambda x: x[:, s].contiguous()
        o_d.append(to_np(gdr2().recurrent_step(sl(t["q"]), sl(t["k"]), sl(t["v"]),
                                               sl(t["log_alpha"]), sl(t["b"]), sl(t["w"]),
                                               state)))
    torch.cuda.synchronize()
    assert rel_l2(np.stack(o_d, axis=1), o_c) < 1e-4
    assert rel_l2(to_np(state), s_c) < 1e-4


# ------------------------------------------------ malformed packed offsets
@pytest.mark.parametrize("dtype,d", [("bf16", 128), ("fp32", 64)])
def test_malformed_offsets_stay_in_bounds(cuda_device, dtype, d):
    """Packed-batch offsets that are negative, past the end or decreasing are
    clamped to [0, tokens] by the kernels (end >= start): every write stays
    inside o and the final states (guard rows around both are untouched) and
    no device error is raised. The values of overlapping ranges are not
    checked (two units then write the same rows)."""
    import torch
    T = 130
    inp = gen.make_inputs(1, T, 2, d, d, dtype, seed=61, init_std=0.05)
    t = upload(inp, cuda_device)
    cu = torch.tensor([0, 5, 3, 500, -7, T], dtype=torch.int32, device=cuda_device)
    N = cu.shape[0] - 1
    g = 8
    tdt = t["q"].dtype
    o_big = torch.full((1, T + 2 * g, 2, d), 7.0, dtype=tdt, device=cuda_device)
    s_big = torch.full((N + 2, 2, d, d), 7.0, dtype=torch.float32, device=cuda_device)
    o = o_big[:, g:g + T]
    s = s_big[1:N + 1]
    s0 = torch.zeros((N, 2, d, d), dtype=torch.float32, device=cuda_device)
    gdr2().chunk_fwd(t["q"], t["k"], t["v"], t["log_alpha"], t["b"], t["w"], s0, cu, o=o, final_state=s)
    torch.cuda.synchronize()
    gdr2().check_device_error()
    assert bool((o_big[:, :g] == 7.0).all()) and bool((o_big[:, g + T:] == 7.0).all())
    assert bool((s_big[0] == 7.0).all()) and bool((s_big[N + 1] == 7.0).all())
    assert bool(torch.isfinite(o.float()).all()) and bool(torch.isfinite(s).all())
