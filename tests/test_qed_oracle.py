"""Pins of the QED oracle (CPU).

QED ("The Query Knows What to Forget: A Second Erase Direction for Linear
Attention", thelatestinai.com listing: abstract and Table 1) adds to the
Gated Delta Rule-2 step a second erase direction taken from the query,
projected orthogonal to the key, gated by b_t, with a per-head strength. The
page does not print the update (its equation (6)), so the oracle is a reading
and its parity against the paper is unpinned. These tests pin the reading
itself: the reductions to the plain rule, the exact annihilation of both erase
directions at full strength, a brute-force product of explicit transition
matrices (with the direction from a QR factorisation instead of the
projection formula), and splitting into sequences.
"""
import numpy as np
import pytest

import oracle

pytestmark = pytest.mark.filterwarnings("ignore")


def rand_inputs(rng, B, T, H, dk, dv, la_scale=0.1):
    q = rng.standard_normal((B, T, H, dk))
    k = rng.standard_normal((B, T, H, dk))
    la = -la_scale * np.abs(rng.standard_normal((B, T, H, dk)))
    b = 1.0 / (1.0 + np.exp(-rng.standard_normal((B, T, H, dk))))
    v = rng.standard_normal((B, T, H, dv))
    w = 1.0 / (1.0 + np.exp(-rng.standard_normal((B, T, H, dv))))
    return q, k, v, la, b, w


@pytest.mark.parametrize("flags", [oracle.QED_FULL, oracle.QED_GATE, oracle.QED_PROJECT, 0])
def test_zero_strength_is_the_plain_rule(flags):
    rng = np.random.default_rng(1)
    q, k, v, la, b, w = rand_inputs(rng, 2, 9, 3, 8, 6)
    s0 = rng.standard_normal((2, 3, 8, 6))
    o1, s1 = oracle.forward(q, k, v, la, b, w, s0)
    o2, s2 = oracle.qed_forward(q, k, v, la, b, w, np.zeros(3), flags=flags, init_state=s0)
    assert np.array_equal(o1, o2) and np.array_equal(s1, s2)


def test_closed_erase_gate_leaves_decay_and_write_only():
    """b = 0: neither erase acts (the correction is gated by b), whatever the
    strength: S_t = D_t S_{t-1} + k_t (w_t . v_t)^T, the plain rule's b = 0 form."""
    rng = np.random.default_rng(2)
    q, k, v, la, b, w = rand_inputs(rng, 1, 7, 2, 8, 8)
    b = np.zeros_like(b)
    s0 = rng.standard_normal((1, 2, 8, 8))
    o1, s1 = oracle.forward(q, k, v, la, b, w, s0)
    o2, s2 = oracle.qed_forward(q, k, v, la, b, w, np.array([0.7, 2.0]), init_state=s0)
    np.testing.assert_allclose(o2, o1, rtol=0, atol=1e-12)
    np.testing.assert_allclose(s2, s1, rtol=0, atol=1e-12)


@pytest.mark.parametrize("dk", [4, 16])
def test_full_strength_erases_the_query_plane(dk):
    """Unit key, b = 1, alpha = 1, no write, strength 1: the step applies
    I - k k^T - u u^T with u the unit part of q orthogonal to k, the projector
    onto the complement of span{k, q}. So the new state has no content along
    k, and the query (which lies in that plane) reads exactly zero."""
    rng = np.random.default_rng(3)
    dv = 5
    q = rng.standard_normal((1, 1, 1, dk))
    k = rng.standard_normal((1, 1, 1, dk))
    k /= np.linalg.norm(k)
    la = np.zeros((1, 1, 1, dk))
    b = np.ones((1, 1, 1, dk))
    v = rng.standard_normal((1, 1, 1, dv))
    w = np.zeros((1, 1, 1, dv))
    s0 = rng.standard_normal((1, 1, dk, dv))
    o, s1 = oracle.qed_forward(q, k, v, la, b, w, np.ones(1), init_state=s0)
    scale = np.abs(s0).max() * np.linalg.norm(q)
    assert np.abs(o).max() < 1e-12 * scale
    assert np.abs(k[0, 0, 0] @ s1[0, 0]).max() < 1e-12 * np.abs(s0).max()
    # a second application changes nothing (projector)
    o2, s2 = oracle.qed_forward(q, k, v, la, b, w, np.ones(1), init_state=s1)
    np.testing.assert_allclose(s2, s1, rtol=0, atol=1e-12 * np.abs(s0).max())
    # without the projection the two erases do not form a projector: the
    # query still reads something (the pin above would catch a dropped P^perp)
    o3, _ = oracle.qed_forward(q, k, v, la, b, w, np.ones(1), flags=oracle.QED_GATE, init_state=s0)
    assert np.abs(o3).max() > 1e-3 * scale


def test_ungated_correction_acts_with_a_closed_key_gate():
    """flags = project only: the query-derived erase ignores b_t. With b = 0
    (no key erase) and strength 1 it still removes the state's content along
    u, the unit part of q orthogonal to k."""
    rng = np.random.default_rng(4)
    dk, dv = 8, 4
    q, k, v, la, b, w = rand_inputs(rng, 1, 1, 1, dk, dv)
    la = np.zeros_like(la)
    b = np.zeros_like(b)
    w = np.zeros_like(w)
    s0 = rng.standard_normal((1, 1, dk, dv))
    _, s1 = oracle.qed_forward(q, k, v, la, b, w, np.ones(1), flags=oracle.QED_PROJECT, init_state=s0)
    Q, _ = np.linalg.qr(np.stack([k[0, 0, 0], q[0, 0, 0]], axis=1))
    u = Q[:, 1]
    assert np.abs(u @ s1[0, 0]).max() < 1e-12 * np.abs(s0).max()
    # and with the gate on, b = 0 closes it
    _, s2 = oracle.qed_forward(q, k, v, la, b, w, np.ones(1), flags=oracle.QED_FULL, init_state=s0)
    np.testing.assert_allclose(s2, s0, rtol=0, atol=1e-12)


@pytest.mark.parametrize("flags", [oracle.QED_FULL, oracle.QED_GATE, oracle.QED_PROJECT, 0])
def test_brute_force_transition_products(flags):
    """T = 3: the state equals the product of explicit transition matrices
    M_t = (I - k e^T - lam u f^T) D_t applied to S0 plus the propagated writes,
    with u from a QR factorisation of [k, q] (projected) or q / |q|."""
    rng = np.random.default_rng(5)
    dk, dv, T = 6, 3, 3
    q, k, v, la, b, w = rand_inputs(rng, 1, T, 1, dk, dv, la_scale=0.3)
    lam = 0.45
    s0 = rng.standard_normal((1, 1, dk, dv))
    o, sf = oracle.qed_forward(q, k, v, la, b, w, np.array([lam]), flags=flags, init_state=s0)
    S = s0[0, 0].copy()
    for t in range(T):
        qt, kt, lt, bt = q[0, t, 0], k[0, t, 0], la[0, t, 0], b[0, t, 0]
        if flags & oracle.QED_PROJECT:
            Q, _ = np.linalg.qr(np.stack([kt, qt], axis=1))
            u = Q[:, 1]
        else:
            u = qt / np.linalg.norm(qt)
        f = bt * u if flags & oracle.QED_GATE else u
        M = (np.eye(dk) - np.outer(kt, bt * kt) - lam * np.outer(u, f)) @ np.diag(np.exp(lt))
        S = M @ S + np.outer(kt, w[0, t, 0] * v[0, t, 0])
        np.testing.assert_allclose(o[0, t, 0], S.T @ qt, rtol=1e-12, atol=1e-12)
    np.testing.assert_allclose(sf[0, 0], S, rtol=1e-12, atol=1e-12)


def test_fixed_direction_arm_and_parallel_direction():
    """The control arm takes a fixed per-head direction instead of q. A
    direction parallel to k_t projects to zero: no correction at all."""
    rng = np.random.default_rng(6)
    dk, dv, T = 8, 8, 4
    q, k, v, la, b, w = rand_inputs(rng, 1, T, 2, dk, dv)
    k[:, :, 0] = k[:, :1, 0]  # head 0: the same key at every token
    direction = rng.standard_normal((2, dk))
    direction[0] = 3.0 * k[0, 0, 0]
    s0 = rng.standard_normal((1, 2, dk, dv))
    o1, s1 = oracle.forward(q, k, v, la, b, w, s0)
    o2, s2 = oracle.qed_forward(q, k, v, la, b, w, np.array([0.8, 0.8]), direction=direction, init_state=s0)
    np.testing.assert_allclose(o2[:, :, 0], o1[:, :, 0], rtol=1e-12, atol=1e-12)
    assert np.abs(o2[:, :, 1] - o1[:, :, 1]).max() > 1e-3


def test_packed_sequences_equal_separate_runs():
    rng = np.random.default_rng(7)
    lengths = [3, 0, 5, 1]
    T = sum(lengths)
    q, k, v, la, b, w = rand_inputs(rng, 1, T, 2, 8, 4)
    lam = np.array([0.2, 1.1])
    cu = np.concatenate([[0], np.cumsum(lengths)])
    s0 = rng.standard_normal((4, 2, 8, 4))
    o, sf = oracle.qed_forward(q, k, v, la, b, w, lam, init_state=s0, cu_seqlens=cu)
    for n in range(4):
        sl = slice(cu[n], cu[n + 1])
        on, sn = oracle.qed_forward(q[:, sl], k[:, sl], v[:, sl], la[:, sl], b[:, sl], w[:, sl], lam,
                                    init_state=s0[n:n + 1])
        np.testing.assert_array_equal(o[:, sl], on)
        np.testing.assert_array_equal(sf[n], sn[0])
