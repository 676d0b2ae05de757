"""The backward decomposition the CUDA kernels implement, checked in fp64
against the oracle's reverse loop (CPU; no GPU, no import of the CUDA path).

The vector-Jacobian product of the token recurrence ("Chunkwise training and
gate-aware backward", ainews.random.gg article on Gated DeltaNet-2) is split
into three sweeps:
  A. forward, per value column: u_t = z_t - (alpha_t . S_{t-1})^T e_t and the
     state at every chunk start (and after the last token);
  B. reverse, per value column: the state cotangent G (from d_final), with
     H_t = G + q_t do_t^T, du_t = H_t^T k_t, G <- alpha_t . (H_t - e_t du_t^T),
     storing du_t and G at every chunk end; dv = du . w, dw = du . v, and the
     last G is d_init_state;
  C. per chunk and key row, given u, du and the two chunk checkpoints:
     dq_t = S_t do_t, de_t = -(alpha_t . S_{t-1}) du_t, dkW_t = H_t u_t,
     dk = dkW + b . de, db = k . de, and
     dlog_alpha_t = sum_{s >= t in the chunk} (q.dq - k.dkW + e.de)_s
                    + rowsum(G_end . S_end),
     the last line because both recurrences telescope: the decay gradient of
     token t equals that of token t+1 plus the three per-token terms, and at a
     chunk end it is the row-wise product of the incoming cotangent with the
     state there.
Each sweep only needs reductions along one axis: A and B along key rows (per
value column), C along value columns (per key row).

The second half restates the same backward in the chunk (WY) form, with the
forward's decay reference at chunk row 31: every per-chunk step is a product
of 64-row tiles, and a chunk-to-chunk recurrence carries the state cotangent.
It is checked against the oracle the same way.
"""
import numpy as np
import pytest

import oracle

C = 64


def sweeps(q, k, v, la, b, w, s0, do, dfin):
    """One (sequence, head): q, k, la, b [T, dk]; v, w, do [T, dv]."""
    T_len, dk = q.shape
    dv_ = v.shape[1]
    alpha, e, z = np.exp(la), b * k, w * v
    nck = -(-T_len // C)
    # sweep A
    ck = np.zeros((nck + 1, dk, dv_))
    U = np.zeros((T_len, dv_))
    S = s0.copy()
    for t in range(T_len):
        if t % C == 0:
            ck[t // C] = S
        Sp = alpha[t][:, None] * S
        U[t] = z[t] - Sp.T @ e[t]
        S = Sp + np.outer(k[t], U[t])
    ck[nck] = S
    # sweep B
    gk = np.zeros((nck, dk, dv_))
    dU = np.zeros((T_len, dv_))
    G = dfin.copy()
    for t in range(T_len - 1, -1, -1):
        if t == T_len - 1 or t % C == C - 1:
            gk[t // C] = G
        Hm = G + np.outer(q[t], do[t])
        dU[t] = Hm.T @ k[t]
        G = alpha[t][:, None] * (Hm - np.outer(e[t], dU[t]))
    d_init = G
    dvv, dww = dU * w, dU * v
    # sweep C
    dq, dkk, db, dla = (np.zeros((T_len, dk)) for _ in range(4))
    for c in range(nck):
        t0, t1 = c * C, min(T_len, (c + 1) * C)
        dkW = np.zeros((t1 - t0, dk))
        Hm = gk[c].copy()
        for t in range(t1 - 1, t0 - 1, -1):          # pass R
            Hm = Hm + np.outer(q[t], do[t])
            dkW[t - t0] = Hm @ U[t]
            Hm = alpha[t][:, None] * (Hm - np.outer(e[t], dU[t]))
        S = ck[c].copy()
        dg = np.zeros((t1 - t0, dk))
        for t in range(t0, t1):                       # pass F
            Sp = alpha[t][:, None] * S
            de = -(Sp @ dU[t])
            S = Sp + np.outer(k[t], U[t])
            dq[t] = S @ do[t]
            dkk[t] = dkW[t - t0] + b[t] * de
            db[t] = k[t] * de
            dg[t - t0] = q[t] * dq[t] - k[t] * dkW[t - t0] + e[t] * de
        acc = np.sum(gk[c] * S, axis=1)               # rowsum(G_end . S_end)
        for t in range(t1 - 1, t0 - 1, -1):
            acc = acc + dg[t - t0]
            dla[t] = acc
    return dq, dkk, dvv, dla, db, dww, d_init


def rel(a, b):
    return np.abs(a - b).max() / max(1e-30, np.abs(b).max())


@pytest.mark.parametrize("T,la_scale,with_state", [(200, 0.1, True), (64, 0.5, False), (1, 0.1, True),
                                                   (130, 1.0, True)])
def test_three_sweeps_match_oracle_backward(T, la_scale, with_state):
    rng = np.random.default_rng(T)
    dk, dv = 16, 12
    q = rng.standard_normal((1, T, 1, dk))
    k = rng.standard_normal((1, T, 1, dk))
    q /= np.linalg.norm(q, axis=-1, keepdims=True)
    k /= np.linalg.norm(k, axis=-1, keepdims=True)
    v = rng.standard_normal((1, T, 1, dv))
    la = -la_scale * np.log1p(np.exp(rng.standard_normal((1, T, 1, dk))))
    b = 1 / (1 + np.exp(-rng.standard_normal((1, T, 1, dk))))
    w = 1 / (1 + np.exp(-rng.standard_normal((1, T, 1, dv))))
    s0 = 0.1 * rng.standard_normal((1, 1, dk, dv)) if with_state else None
    do = rng.standard_normal((1, T, 1, dv))
    dfin = rng.standard_normal((1, 1, dk, dv)) if with_state else np.zeros((1, 1, dk, dv))
    ref = oracle.backward(q, k, v, la, b, w, s0, do, dfin)
    s0_ = s0[0, 0] if with_state else np.zeros((dk, dv))
    got = sweeps(q[0, :, 0], k[0, :, 0], v[0, :, 0], la[0, :, 0], b[0, :, 0], w[0, :, 0],
                 s0_, do[0, :, 0], dfin[0, 0])
    names = ("dq", "dk", "dv", "dlog_alpha", "db", "dw", "d_init_state")
    for name, g, r in zip(names, got, ref):
        r = r[0, 0] if r.ndim == 4 and name == "d_init_state" else r[0, :, 0]
        assert rel(g, r) < 1e-11, f"{name}: {rel(g, r):.2e}"


# ---------------------------------------------------------------------------
# The chunk (WY) form of the same backward: every per-chunk step is a dense
# product of 64-row tiles, the form a tensor-core backward takes. With the
# forward's chunk quantities (decay exponents d = g - g_31 about the chunk's
# row 31, Qm = q e^d, Km = k e^-d, Em = e e^d, Sm = e^{g_31} S0, A, P, T and U)
# and Ghat, the cotangent of the state at the chunk end:
#   dU   = T^T (P^T dO + (Km . e^{d_end}) Ghat)            (du of every token)
#   dQ   = e^d . (dO Sm^T + tril(dO U^T) Km)
#   dE   = -e^d . (dU Sm^T + stril(dU U^T) Km)
#   dKW  = e^-d . (triu(U dO^T) Qm - striu(U dU^T) Em) + e^{d_end - d} . (U Ghat^T)
#   Ghat_prev = e^{g_31} . (Qm^T dO - Em^T dU) + e^{g_end} . Ghat
# and the per-token combinations of the three-sweep form above (dk, db, the
# decay terms, restarted at the chunk end with rowsum(Ghat . S_end)).
from chunk_bwd_form import chunk_backward  # noqa: E402  (the exact form: no operand rounding)


@pytest.mark.parametrize("T,la_scale,with_state", [(200, 0.1, True), (64, 0.5, False), (1, 0.1, True),
                                                   (130, 1.0, True), (31, 0.3, True)])
def test_chunk_form_backward_matches_oracle(T, la_scale, with_state):
    rng = np.random.default_rng(100 + T)
    dk, dv = 16, 12
    q = rng.standard_normal((1, T, 1, dk))
    k = rng.standard_normal((1, T, 1, dk))
    q /= np.linalg.norm(q, axis=-1, keepdims=True)
    k /= np.linalg.norm(k, axis=-1, keepdims=True)
    v = rng.standard_normal((1, T, 1, dv))
    la = -la_scale * np.log1p(np.exp(rng.standard_normal((1, T, 1, dk))))
    b = 1 / (1 + np.exp(-rng.standard_normal((1, T, 1, dk))))
    w = 1 / (1 + np.exp(-rng.standard_normal((1, T, 1, dv))))
    s0 = 0.1 * rng.standard_normal((1, 1, dk, dv)) if with_state else None
    do = rng.standard_normal((1, T, 1, dv))
    dfin = rng.standard_normal((1, 1, dk, dv)) if with_state else np.zeros((1, 1, dk, dv))
    ref = oracle.backward(q, k, v, la, b, w, s0, do, dfin)
    s0_ = s0[0, 0] if with_state else np.zeros((dk, dv))
    got = chunk_backward(q[0, :, 0], k[0, :, 0], v[0, :, 0], la[0, :, 0], b[0, :, 0], w[0, :, 0],
                         s0_, do[0, :, 0], dfin[0, 0])
    names = ("dq", "dk", "dv", "dlog_alpha", "db", "dw", "d_init_state")
    for name, g, r in zip(names, got, ref):
        r = r[0, 0] if name == "d_init_state" else r[0, :, 0]
        assert rel(g, r) < 1e-10, f"{name}: {rel(g, r):.2e}"


# ---------------------------------------------------------------------------
# Segment split of the two sweeps (for few long sequences). Both sweeps are
# affine in their state, so a sequence cut into P segments can run every
# segment at once and chain the segments afterwards:
#   A: S_end(p) = Phi_p S_start(p) + S0_p, with Phi_p the product of the
#      segment's transition matrices M_t = (I - k_t e_t^T) Diag(alpha_t);
#      the segment run from the identity (z = 0) gives Phi_p and, per token,
#      psi_t = Phi_{<t}^T (alpha_t . e_t), so that u_t = u0_t - S_start^T psi_t.
#   B: G_start(p) = Phi_p^T G_end(p) + G0_p; the reverse run from the identity
#      with dO = 0 gives Phi_p^T as its last cotangent and, as its du,
#      chi_t = M_end ... M_{t+1} k_t, so that du_t = du0_t + G_end^T chi_t.
# The chunk checkpoints follow the same way: a chunk-start state is the zero
# run's plus the identity run's checkpoint times S_start, a chunk-end
# cotangent the zero run's plus the identity run's times G_end.


def sweep_a(alpha, e, k, z, s_init):
    """Sweep A over a token range: per-token u and the state before each token."""
    S = s_init.copy()
    us, before = [], []
    for t in range(alpha.shape[0]):
        before.append(S)
        Sp = alpha[t][:, None] * S
        u = z[t] - Sp.T @ e[t]
        S = Sp + np.outer(k[t], u)
        us.append(u)
    return np.array(us), np.array(before), S


def sweep_b(alpha, e, k, q, do, g_init):
    """Sweep B over a token range: per-token du and the cotangent after each token."""
    G = g_init.copy()
    dus, after = [None] * alpha.shape[0], [None] * alpha.shape[0]
    for t in range(alpha.shape[0] - 1, -1, -1):
        after[t] = G
        Hm = G + np.outer(q[t], do[t])
        dus[t] = Hm.T @ k[t]
        G = alpha[t][:, None] * (Hm - np.outer(e[t], dus[t]))
    return np.array(dus), np.array(after), G


@pytest.mark.parametrize("T,P,la_scale", [(256, 4, 0.1), (200, 3, 0.5), (97, 2, 1.0)])
def test_segment_split_of_the_sweeps(T, P, la_scale):
    rng = np.random.default_rng(T + P)
    dk, dv = 12, 10
    q = rng.standard_normal((T, dk))
    k = rng.standard_normal((T, dk))
    k /= np.linalg.norm(k, axis=-1, keepdims=True)
    alpha = np.exp(-la_scale * np.log1p(np.exp(rng.standard_normal((T, dk)))))
    b = 1 / (1 + np.exp(-rng.standard_normal((T, dk))))
    e = b * k
    z = rng.standard_normal((T, dv))
    do = rng.standard_normal((T, dv))
    s0 = 0.1 * rng.standard_normal((dk, dv))
    dfin = rng.standard_normal((dk, dv))
    u_ref, st_ref, _ = sweep_a(alpha, e, k, z, s0)
    du_ref, gt_ref, ginit_ref = sweep_b(alpha, e, k, q, do, dfin)

    cuts = np.linspace(0, T, P + 1).astype(int)
    I, zeros_z, zeros_do = np.eye(dk), np.zeros((T, dk)), np.zeros((T, dk))   # identity runs are dk wide
    # every segment at once: from zero (A, B) and from the identity (z = 0, dO = 0)
    segA, segB = [], []
    for p in range(P):
        a, c = cuts[p], cuts[p + 1]
        sl = slice(a, c)
        u0, b0, e0 = sweep_a(alpha[sl], e[sl], k[sl], z[sl], np.zeros((dk, dv)))
        uI, bI, Phi = sweep_a(alpha[sl], e[sl], k[sl], zeros_z[sl], I)
        segA.append((u0, b0, e0, -uI, bI, Phi))     # -uI[t] = psi_t (u from the identity, z = 0)
        d0, a0, g0 = sweep_b(alpha[sl], e[sl], k[sl], q[sl], do[sl], np.zeros((dk, dv)))
        chi, aI, PhiT = sweep_b(alpha[sl], e[sl], k[sl], q[sl], zeros_do[sl], I)
        segB.append((d0, a0, g0, chi, aI, PhiT))
    # chain the segments: A forward, B in reverse
    s_start, g_end = [s0], [None] * P
    for p in range(P - 1):
        _, _, e0, _, _, Phi = segA[p]
        s_start.append(Phi @ s_start[p] + e0)
    g_end[P - 1] = dfin
    for p in range(P - 1, 0, -1):
        _, _, g0, _, _, PhiT = segB[p]
        g_end[p - 1] = PhiT @ g_end[p] + g0
    np.testing.assert_allclose(segB[0][5] @ g_end[0] + segB[0][2], ginit_ref, rtol=1e-11, atol=1e-11)
    # per-token corrections and checkpoints
    for p in range(P):
        a, c = cuts[p], cuts[p + 1]
        u0, b0, _, psi, bI, _ = segA[p]
        d0, a0, _, chi, aI, _ = segB[p]
        u = u0 - psi @ s_start[p]                    # u_t = u0_t - S_start^T psi_t
        du = d0 + chi @ g_end[p]                     # du_t = du0_t + G_end^T chi_t
        np.testing.assert_allclose(u, u_ref[a:c], rtol=1e-10, atol=1e-11)
        np.testing.assert_allclose(du, du_ref[a:c], rtol=1e-10, atol=1e-11)
        before = b0 + np.einsum("tij,jv->tiv", bI, s_start[p])
        after = a0 + np.einsum("tij,jv->tiv", aI, g_end[p])     # G_t = G0_t + G^I_t G_end
        np.testing.assert_allclose(before, st_ref[a:c], rtol=1e-10, atol=1e-11)
        np.testing.assert_allclose(after, gt_ref[a:c], rtol=1e-10, atol=1e-11)
