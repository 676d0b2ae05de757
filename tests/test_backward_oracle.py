"""Pins of the fp64 backward oracle (vector-Jacobian product of the token
recurrence; SURVEY's next row, the gate-aware backward): central finite
differences of the forward oracle on tiny inputs, linearity in the output and
final-state cotangents, and planted mistakes (in a test-local copy of the
reverse loop) that the finite-difference pin must reject. CPU only."""
import numpy as np
import pytest

import oracle

NAMES = ("q", "k", "v", "log_alpha", "b", "w", "init_state")


def tiny(seed, B=2, T=5, H=1, dk=3, dv=4):
    rng = np.random.default_rng(seed)
    q, k, b = (rng.standard_normal((B, T, H, dk)) for _ in range(3))
    la = -0.3 * np.abs(rng.standard_normal((B, T, H, dk)))
    v, w = (rng.standard_normal((B, T, H, dv)) for _ in range(2))
    s0 = rng.standard_normal((B, H, dk, dv))
    d_o = rng.standard_normal((B, T, H, dv))
    d_f = rng.standard_normal((B, H, dk, dv))
    return [q, k, v, la, b, w, s0], d_o, d_f


def loss(args, d_o, d_f):
    o, sf = oracle.forward(*args)
    return float(np.sum(o * d_o) + np.sum(sf * d_f))


def finite_differences(args, d_o, d_f, h=1e-6):
    out = []
    for idx in range(len(args)):
        x = args[idx]
        g = np.zeros_like(x)
        for i in np.ndindex(x.shape):
            ap, am = list(args), list(args)
            xp, xm = x.copy(), x.copy()
            xp[i] += h
            xm[i] -= h
            ap[idx], am[idx] = xp, xm
            g[i] = (loss(ap, d_o, d_f) - loss(am, d_o, d_f)) / (2 * h)
        out.append(g)
    return out


def assert_matches_fd(grads, fd):
    for name, g, f in zip(NAMES, grads, fd):
        err = np.abs(g - f).max() / max(1.0, np.abs(f).max())
        assert err < 1e-7, f"d{name}: relative error {err:.2e} against finite differences"


@pytest.mark.parametrize("seed", [0, 1])
def test_backward_matches_finite_differences(seed):
    args, d_o, d_f = tiny(seed)
    assert_matches_fd(oracle.backward(*args, d_o, d_f), finite_differences(args, d_o, d_f))


def test_backward_without_final_cotangent_and_state():
    args, d_o, _ = tiny(2)
    args[6] = None
    zero = np.zeros((2, 1, 3, 4))
    grads = oracle.backward(*args, d_o, None)
    fd = finite_differences(args[:6] + [zero], d_o, zero)
    assert_matches_fd(grads, fd)


def test_backward_is_linear_in_the_cotangents():
    args, d_o, d_f = tiny(3)
    g1 = oracle.backward(*args, d_o, d_f)
    g2 = oracle.backward(*args, 2.0 * d_o, -d_f)
    g12 = oracle.backward(*args, 3.0 * d_o, 0.0 * d_f)
    for a, b, c in zip(g1, g2, g12):
        np.testing.assert_allclose(a + b, c, rtol=1e-12, atol=1e-12)


def test_empty_sequence_passes_the_final_cotangent_through():
    args, _, d_f = tiny(4, T=0)
    grads = oracle.backward(*args, np.zeros((2, 0, 1, 4)), d_f)
    np.testing.assert_array_equal(grads[6], d_f)


def mutated_backward(args, d_o, d_f, mutation):
    """A copy of the reverse loop with one planted mistake."""
    q, k, v, la, b, w, s0 = args
    B, T, H, dk = q.shape
    alpha, e, z = np.exp(la), b * k, w * v
    S = s0.copy()
    prev = []
    for t in range(T):
        prev.append(S)
        Sp = alpha[:, t, :, :, None] * S
        r = np.einsum("bhij,bhi->bhj", Sp, e[:, t])
        S = Sp + k[:, t, :, :, None] * (z[:, t] - r)[:, :, None, :]
    G = d_f.copy()
    out = [np.zeros_like(x) for x in args[:6]]
    for t in range(T - 1, -1, -1):
        Sp = alpha[:, t, :, :, None] * prev[t]
        r = np.einsum("bhij,bhi->bhj", Sp, e[:, t])
        u = z[:, t] - r
        S_t = Sp + k[:, t, :, :, None] * u[:, :, None, :]
        G = G + q[:, t, :, :, None] * d_o[:, t, :, None, :]
        out[0][:, t] = np.einsum("bhij,bhj->bhi", S_t if mutation != "dq_prev_state" else prev[t], d_o[:, t])
        du = np.einsum("bhij,bhi->bhj", G, k[:, t])
        dk_t = np.einsum("bhij,bhj->bhi", G, u)
        dr = -du
        dSp = G + (e[:, t, :, :, None] * dr[:, :, None, :] if mutation != "drop_erase_read" else 0.0)
        de = np.einsum("bhij,bhj->bhi", Sp, dr)
        dalpha = np.sum(dSp * prev[t], axis=-1)
        G = alpha[:, t, :, :, None] * dSp if mutation != "no_decay_in_state_grad" else dSp
        out[4][:, t] = de * (k[:, t] if mutation != "erase_gate_wrong_factor" else b[:, t])
        out[1][:, t] = dk_t + (de * b[:, t] if mutation != "drop_key_in_erase" else 0.0)
        out[5][:, t] = du * v[:, t]
        out[2][:, t] = du * (w[:, t] if mutation != "write_gate_missing" else 1.0)
        out[3][:, t] = dalpha * (alpha[:, t] if mutation != "log_decay_chain_rule" else 1.0)
    return out + [G]


@pytest.mark.parametrize("mutation", [
    None, "dq_prev_state", "drop_erase_read", "no_decay_in_state_grad", "erase_gate_wrong_factor",
    "drop_key_in_erase", "write_gate_missing", "log_decay_chain_rule"])
def test_planted_mistakes_are_caught(mutation):
    args, d_o, d_f = tiny(5)
    fd = finite_differences(args, d_o, d_f)
    grads = mutated_backward(args, d_o, d_f, mutation)
    if mutation is None:
        assert_matches_fd(grads, fd)          # the unmutated copy passes
    else:
        with pytest.raises(AssertionError):
            assert_matches_fd(grads, fd)
