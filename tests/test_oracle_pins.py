"""Pin the fp64 oracle to what the pages fix, and show the pins have teeth.

The first group runs every check in ``pins.py`` against the compiled oracle.
The second group plants one plausible mistake at a time in a small
pure-Python copy of the token loop (CPU only) and asserts that at least one
pin rejects it, while the unmutated copy passes them all.
"""
import numpy as np
import pytest

import oracle
import pins
from linear_attention_recurrence_gdr2_b200 import inputs as gen


def oracle_fwd(q, k, v, la, b, w, s0=None, cu=None):
    return oracle.forward(q, k, v, la, b, w, s0, cu)


def oracle_step(q, k, v, la, b, w, s):
    return oracle.step(q, k, v, la, b, w, s)


@pytest.mark.parametrize("pin", pins.FORWARD_PINS, ids=lambda p: p.__name__)
def test_oracle_pin(pin):
    pin(oracle_fwd, np.random.default_rng(1234))


def test_oracle_fast_weight_argmin():
    pins.pin_fast_weight_argmin(oracle_step, np.random.default_rng(7))


def test_oracle_step_matches_single_token_forward():
    rng = np.random.default_rng(3)
    q, k, v, la, b, w, s0 = pins.rand_problem(rng, T=1)
    o_f, s_f = oracle.forward(q, k, v, la, b, w, s0)
    sq = lambda x: x[:, 0]
    o_s, s_s = oracle.step(sq(q), sq(k), sq(v), sq(la), sq(b), sq(w), s0)
    assert np.array_equal(o_f[:, 0], o_s) and np.array_equal(s_f, s_s)


def test_oracle_zero_length_and_rejects_bad_args():
    rng = np.random.default_rng(5)
    q, k, v, la, b, w, s0 = pins.rand_problem(rng, T=0)
    o, sf = oracle.forward(q, k, v, la, b, w, s0)
    assert o.shape == (2, 0, 2, 5) and np.array_equal(sf, s0)
    q, k, v, la, b, w, _ = pins.rand_problem(rng, B=1, T=4)
    with pytest.raises(ValueError):
        oracle.forward(q, k, v, la, b, w, None, np.array([0, 3, 2, 4]))
    with pytest.raises(ValueError):
        oracle.forward(q, k, v, la, b, w, None, np.array([0, 2, 3]))


def test_oracle_threads_do_not_change_results():
    rng = np.random.default_rng(11)
    q, k, v, la, b, w, s0 = pins.rand_problem(rng, B=3, T=20, H=3)
    o1, s1 = oracle.forward(q, k, v, la, b, w, s0, num_threads=1)
    o4, s4 = oracle.forward(q, k, v, la, b, w, s0, num_threads=4)
    assert np.array_equal(o1, o4) and np.array_equal(s1, s4)


# --------------------------------------------------------------------------
# Mutation tests: a small pure-Python token loop with one planted mistake.
# --------------------------------------------------------------------------
def loop_forward(q, k, v, la, b, w, s0=None, cu=None, mutation=None):
    B, T, H, dk = q.shape
    dv = v.shape[-1]
    if cu is None:
        spans = [(n, n * T, n * T + T) for n in range(B)]
        flat = lambda x: x.reshape(B * T, H, x.shape[-1])
    else:
        spans = [(n, int(cu[n]), int(cu[n + 1])) for n in range(len(cu) - 1)]
        flat = lambda x: x.reshape(T, H, x.shape[-1])
    qf, kf, vf, laf, bf, wf = (flat(x) for x in (q, k, v, la, b, w))
    o = np.zeros((qf.shape[0], H, dv))
    sf = np.zeros((len(spans), H, dk, dv))
    for n, t0, t1 in spans:
        for h in range(H):
            S = s0[n, h].copy() if s0 is not None else np.zeros((dk, dv))
            for t in range(t0, t1):
                kt, qt, bt = kf[t, h], qf[t, h], bf[t, h]
                a = np.exp(laf[t, h])
                e = bt * kt
                z = wf[t, h] * vf[t, h]
                if mutation == "drop_erase_gate":
                    e = kt
                if mutation == "drop_write_gate":
                    z = vf[t, h]
                if mutation == "readout_before_update":
                    o[t, h] = S.T @ qt
                if mutation != "decay_after_edit":
                    S = a[:, None] * S
                if mutation == "erase_gate_on_left":
                    S = S + np.outer(bt * kt, z - kt @ S)
                elif mutation == "wrong_sign":
                    S = S + np.outer(kt, z + e @ S)
                else:
                    S = S + np.outer(kt, z - e @ S)
                if mutation == "decay_after_edit":
                    S = a[:, None] * S
                if mutation == "decay_inverse":
                    S = S / (a * a)[:, None]
                if mutation != "readout_before_update":
                    o[t, h] = S.T @ qt
            sf[n, h] = S
    return o.reshape(q.shape[:-1] + (dv,)), sf


def loop_step(q, k, v, la, b, w, s, mutation=None):
    ex = lambda x: x[:, None]
    o, sf = loop_forward(ex(q), ex(k), ex(v), ex(la), ex(b), ex(w), s, mutation=mutation)
    return o[:, 0], sf


MUTATIONS = ["drop_erase_gate", "drop_write_gate", "readout_before_update",
             "decay_after_edit", "erase_gate_on_left", "wrong_sign", "decay_inverse"]


def _run_all_pins(fwd, step):
    failures = []
    for pin in pins.FORWARD_PINS:
        try:
            pin(fwd, np.random.default_rng(99))
        except AssertionError as e:
            failures.append(f"{pin.__name__}: {e}")
    try:
        pins.pin_fast_weight_argmin(step, np.random.default_rng(98))
    except AssertionError as e:
        failures.append(f"argmin: {e}")
    return failures


def test_unmutated_loop_passes_every_pin():
    assert _run_all_pins(loop_forward, loop_step) == []


@pytest.mark.parametrize("mutation", MUTATIONS)
def test_planted_mistake_is_caught(mutation):
    fwd = lambda *a, **kw: loop_forward(*a, mutation=mutation, **kw)
    step = lambda *a, **kw: loop_step(*a, mutation=mutation, **kw)
    assert _run_all_pins(fwd, step), f"no pin caught mutation {mutation!r}"


def test_segment_split_identity():
    """The segment-parallel scan's decomposition, on the oracle alone (fp64):
    running each segment from a zero state, and from the identity with z = 0
    (giving its transition Phi and readout map psi_t = Phi_t^T q_t), then
    chaining S_start(p+1) = Phi_p S_start(p) + S0_p and adding S_start^T psi_t,
    reproduces one serial run (the affine structure of the rule)."""
    inp = gen.make_inputs(2, 300, 2, 16, 16, "fp32", seed=31, la_scale=0.01, init_std=0.1)
    o_ref, s_ref = oracle.forward(inp.q, inp.k, inp.v, inp.log_alpha, inp.b, inp.w, inp.init_state)
    L, T = 128, 300
    eye = np.broadcast_to(np.eye(16, dtype=np.float32), inp.init_state.shape).copy()
    o = np.zeros_like(o_ref)
    s_start = inp.init_state.astype(np.float64)
    for p0 in range(0, T, L):
        sl = slice(p0, min(p0 + L, T))
        cut = lambda x: np.ascontiguousarray(x[:, sl])
        zero = np.zeros_like(inp.init_state)
        o_a, s_a = oracle.forward(cut(inp.q), cut(inp.k), cut(inp.v), cut(inp.log_alpha), cut(inp.b),
                                  cut(inp.w), inp.init_state if p0 == 0 else zero)
        o_b, phi = oracle.forward(cut(inp.q), cut(inp.k), np.zeros_like(cut(inp.v)), cut(inp.log_alpha),
                                  cut(inp.b), cut(inp.w), eye)
        if p0 == 0:
            o[:, sl] = o_a
            s_start = s_a
        else:
            o[:, sl] = o_a + np.einsum("ntha,nhab->ntbh", o_b, s_start).transpose(0, 1, 3, 2)
            s_start = np.einsum("nhik,nhkj->nhij", phi, s_start) + s_a
    assert np.max(np.abs(o - o_ref)) < 1e-12 * max(1.0, np.max(np.abs(o_ref)))
    assert np.max(np.abs(s_start - s_ref)) < 1e-12 * max(1.0, np.max(np.abs(s_ref)))


def test_prologue_against_library_routines():
    """The fused prologue's activations equal library routines: the logistic
    function (scipy.special.expit), softplus (numpy.logaddexp(0, x)) and the
    Euclidean norm (numpy.linalg.norm); no flag leaves the inputs unchanged;
    each flag touches only its own tensors."""
    from scipy.special import expit
    rng = np.random.default_rng(5)
    shp = (2, 7, 3, 16)
    q, k, la, b, w = (rng.standard_normal(shp) * 3 for _ in range(5))
    la[0, 0, 0, :4] = [-50.0, 50.0, 0.0, 700.0]   # extremes of softplus
    same = oracle.prologue(q, k, la, b, w, 0)
    for x, y in zip(same, (q, k, la, b, w)):
        assert np.array_equal(x, y)
    qn, kn, la2, bs, ws = oracle.prologue(q, k, la, b, w, 7)
    eps = 1e-6
    np.testing.assert_allclose(qn, q / np.sqrt(np.linalg.norm(q, axis=-1, keepdims=True) ** 2 + eps), rtol=1e-14)
    np.testing.assert_allclose(kn, k / np.sqrt(np.linalg.norm(k, axis=-1, keepdims=True) ** 2 + eps), rtol=1e-14)
    np.testing.assert_allclose(np.linalg.norm(qn, axis=-1), 1.0, rtol=1e-6)  # unit rows
    np.testing.assert_allclose(bs, expit(b), rtol=1e-14)
    np.testing.assert_allclose(ws, expit(w), rtol=1e-14)
    np.testing.assert_allclose(la2, -np.logaddexp(0.0, la), rtol=1e-14)
    assert np.all(la2 <= 0) and np.isfinite(la2).all()
    # one flag at a time
    q1, k1, la1, b1, w1 = oracle.prologue(q, k, la, b, w, oracle.PROLOGUE_GATE_SIGMOID)
    assert np.array_equal(q1, q) and np.array_equal(k1, k) and np.array_equal(la1, la)
    q1, k1, la1, b1, w1 = oracle.prologue(q, k, la, b, w, oracle.PROLOGUE_DECAY_SOFTPLUS)
    assert np.array_equal(b1, b) and np.array_equal(w1, w) and np.array_equal(q1, q)
