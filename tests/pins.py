"""Independent checks that pin the fp64 oracle to what the pages fix.

Each check takes an implementation ``fwd(q, k, v, la, b, w, s0=None,
cu=None) -> (o, final_state)`` (token tensors [B, T, H, d], states
[N, H, d_k, d_v]) and raises AssertionError when the implementation disagrees
with a statement that does not come from the implementation itself:

* reductions to KDA and to Gated DeltaNet ("Gated Delta Rule-2" section of the
  zhichai.net summary; "two gates instead of one" section of the ainews
  article): separately written recurrences of those two models;
* exact recall of the delta rule (alpha = 1, b = w = 1, unit keys);
* b = 0 turns the operator into decayed linear attention, whose output and
  state have a closed form in the cumulative log-decay;
* on short sequences, explicit products of the per-token transition matrices
  (I - k e^T) Diag(alpha);
* the fast-weight view: S_t minimises
  ||S - Sbar_t||_F^2 - 2 <S^T k_t, z_t - Sbar_t^T e_t> with Sbar_t = D_t S_{t-1};
* state passing, packed variable-length batches, and joint linearity in the
  write target and the initial state.

Shapes use d_k != d_v so that a transposed operand cannot pass.
"""
from __future__ import annotations

import numpy as np

RTOL = 1e-11


def rel_err(x, ref):
    x = np.asarray(x, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    den = np.linalg.norm(ref.ravel())
    num = np.linalg.norm((x - ref).ravel())
    return num / den if den > 0 else num


def _unit(x):
    return x / np.linalg.norm(x, axis=-1, keepdims=True)


def rand_problem(rng, B=2, T=9, H=2, dk=6, dv=5, init=True):
    q = _unit(rng.standard_normal((B, T, H, dk)))
    k = _unit(rng.standard_normal((B, T, H, dk)))
    v = rng.standard_normal((B, T, H, dv))
    la = -np.logaddexp(0.0, rng.standard_normal((B, T, H, dk))) * 0.3
    b = 1.0 / (1.0 + np.exp(-rng.standard_normal((B, T, H, dk))))
    w = 1.0 / (1.0 + np.exp(-rng.standard_normal((B, T, H, dv))))
    s0 = rng.standard_normal((B, H, dk, dv)) * 0.3 if init else None
    return q, k, v, la, b, w, s0


# --------------------------------------------------------------------------
# Separately written recurrences of the two models GDR-2 generalises.
# --------------------------------------------------------------------------
def kda_reference(q, k, v, la, beta, s0):
    """Kimi Delta Attention, channel-wise decay, scalar edit gate beta_t:
    S_t = (I - beta_t k_t k_t^T) Diag(alpha_t) S_{t-1} + beta_t k_t v_t^T."""
    B, T, H, dk = q.shape
    dv = v.shape[-1]
    o = np.zeros((B, T, H, dv))
    sf = np.zeros((B, H, dk, dv))
    for n in range(B):
        for h in range(H):
            S = s0[n, h].copy() if s0 is not None else np.zeros((dk, dv))
            for t in range(T):
                kt = k[n, t, h][:, None]
                P = np.eye(dk) - beta[n, t, h] * (kt @ kt.T)
                S = P @ np.diag(np.exp(la[n, t, h])) @ S + beta[n, t, h] * kt @ v[n, t, h][None, :]
                o[n, t, h] = S.T @ q[n, t, h]
            sf[n, h] = S
    return o, sf


def gdn_reference(q, k, v, log_a, beta, s0):
    """Gated DeltaNet, scalar decay alpha_t and scalar edit gate beta_t:
    S_t = alpha_t (I - beta_t k_t k_t^T) S_{t-1} + beta_t k_t v_t^T."""
    B, T, H, dk = q.shape
    dv = v.shape[-1]
    o = np.zeros((B, T, H, dv))
    sf = np.zeros((B, H, dk, dv))
    for n in range(B):
        for h in range(H):
            S = s0[n, h].copy() if s0 is not None else np.zeros((dk, dv))
            for t in range(T):
                kt = k[n, t, h]
                S = np.exp(log_a[n, t, h]) * (S - beta[n, t, h] * np.outer(kt, kt @ S)) \
                    + beta[n, t, h] * np.outer(kt, v[n, t, h])
                o[n, t, h] = q[n, t, h] @ S
            sf[n, h] = S
    return o, sf


def pin_kda(fwd, rng):
    q, k, v, la, _, _, s0 = rand_problem(rng)
    beta = 1.0 / (1.0 + np.exp(-rng.standard_normal(q.shape[:3])))
    b = np.repeat(beta[..., None], q.shape[-1], axis=-1)
    w = np.repeat(beta[..., None], v.shape[-1], axis=-1)
    o, sf = fwd(q, k, v, la, b, w, s0)
    o_r, sf_r = kda_reference(q, k, v, la, beta, s0)
    assert rel_err(o, o_r) < RTOL and rel_err(sf, sf_r) < RTOL, "KDA reduction"


def pin_gdn(fwd, rng):
    q, k, v, _, _, _, s0 = rand_problem(rng)
    log_a = -np.logaddexp(0.0, rng.standard_normal(q.shape[:3])) * 0.3
    la = np.repeat(log_a[..., None], q.shape[-1], axis=-1)
    beta = 1.0 / (1.0 + np.exp(-rng.standard_normal(q.shape[:3])))
    b = np.repeat(beta[..., None], q.shape[-1], axis=-1)
    w = np.repeat(beta[..., None], v.shape[-1], axis=-1)
    o, sf = fwd(q, k, v, la, b, w, s0)
    o_r, sf_r = gdn_reference(q, k, v, log_a, beta, s0)
    assert rel_err(o, o_r) < RTOL and rel_err(sf, sf_r) < RTOL, "Gated DeltaNet reduction"


def pin_exact_recall(fwd, rng):
    """alpha = 1, b = w = 1, ||k_t|| = 1: the delta rule stores v_t under k_t
    exactly, so reading with q_t = k_t returns v_t at every step."""
    q, k, v, la, b, w, s0 = rand_problem(rng, T=12)
    q = k.copy()
    la = np.zeros_like(la)
    b = np.ones_like(b)
    w = np.ones_like(w)
    o, _ = fwd(q, k, v, la, b, w, s0)
    assert np.max(np.abs(o - v)) < 1e-12 * max(1.0, np.max(np.abs(v))), "exact recall"


def pin_no_erase_closed_form(fwd, rng):
    """b = 0: S_T = Diag(e^{G_T}) S_0 + sum_s Diag(e^{G_T - G_s}) k_s z_s^T and
    o_t = S_0^T (q_t . e^{G_t}) + sum_{s<=t} <q_t . e^{G_t - G_s}, k_s> z_s,
    with G_t = sum_{i<=t} log alpha_i."""
    q, k, v, la, b, w, s0 = rand_problem(rng)
    b = np.zeros_like(b)
    o, sf = fwd(q, k, v, la, b, w, s0)
    B, T, H, dk = q.shape
    z = w * v
    G = np.cumsum(la, axis=1)
    o_r = np.zeros_like(o)
    sf_r = np.zeros_like(sf)
    for n in range(B):
        for h in range(H):
            for t in range(T):
                acc = s0[n, h].T @ (q[n, t, h] * np.exp(G[n, t, h]))
                for s in range(t + 1):
                    acc = acc + np.dot(q[n, t, h] * np.exp(G[n, t, h] - G[n, s, h]),
                                       k[n, s, h]) * z[n, s, h]
                o_r[n, t, h] = acc
            S = np.exp(G[n, T - 1, h])[:, None] * s0[n, h]
            for s in range(T):
                S = S + np.outer(np.exp(G[n, T - 1, h] - G[n, s, h]) * k[n, s, h], z[n, s, h])
            sf_r[n, h] = S
    assert rel_err(o, o_r) < RTOL and rel_err(sf, sf_r) < RTOL, "b=0 closed form"


def pin_transition_products(fwd, rng, T=16):
    """S_T = M_T...M_1 S_0 + sum_s M_T...M_{s+1} k_s z_s^T with
    M_t = (I - k_t e_t^T) Diag(alpha_t); o_t from the same partial products."""
    q, k, v, la, b, w, s0 = rand_problem(rng, T=T)
    o, sf = fwd(q, k, v, la, b, w, s0)
    B, _, H, dk = q.shape
    z = w * v
    for n in range(B):
        for h in range(H):
            M = [(np.eye(dk) - np.outer(k[n, t, h], b[n, t, h] * k[n, t, h]))
                 @ np.diag(np.exp(la[n, t, h])) for t in range(T)]
            for t in range(T):
                prod = np.eye(dk)
                for i in range(t, -1, -1):
                    prod = prod @ M[i]
                St = prod @ s0[n, h]
                for s in range(t + 1):
                    tail = np.eye(dk)
                    for i in range(t, s, -1):
                        tail = tail @ M[i]
                    St = St + tail @ np.outer(k[n, s, h], z[n, s, h])
                assert rel_err(o[n, t, h], St.T @ q[n, t, h]) < 1e-10, "transition products (o)"
                if t == T - 1:
                    assert rel_err(sf[n, h], St) < 1e-10, "transition products (state)"


def pin_fast_weight_argmin(step, rng):
    """The step's new state minimises the fast-weight objective
    f(S) = ||S - Sbar||^2 - 2 <S^T k, z - Sbar^T e>, Sbar = Diag(alpha) S_prev.
    f is quadratic with Hessian 2I, so S* is the minimiser iff
    f(S* + X) - f(S*) = ||X||^2 for every X."""
    q, k, v, la, b, w, s0 = rand_problem(rng, T=1)
    sq = lambda x: x[:, 0]
    _, S1 = step(sq(q), sq(k), sq(v), sq(la), sq(b), sq(w), s0)
    N, H = S1.shape[:2]
    for n in range(N):
        for h in range(H):
            Sbar = np.exp(la[n, 0, h])[:, None] * s0[n, h]
            e = b[n, 0, h] * k[n, 0, h]
            z = w[n, 0, h] * v[n, 0, h]
            kt = k[n, 0, h]

            def f(S):
                return np.sum((S - Sbar) ** 2) - 2.0 * np.dot(S.T @ kt, z - Sbar.T @ e)
            for _ in range(3):
                X = rng.standard_normal(S1[n, h].shape)
                gap = f(S1[n, h] + X) - f(S1[n, h]) - np.sum(X * X)
                assert abs(gap) < 1e-9 * max(1.0, np.sum(X * X)), "fast-weight argmin"


def pin_state_passing(fwd, rng):
    q, k, v, la, b, w, s0 = rand_problem(rng, T=11)
    o, sf = fwd(q, k, v, la, b, w, s0)
    t1 = 4
    o1, s1 = fwd(q[:, :t1], k[:, :t1], v[:, :t1], la[:, :t1], b[:, :t1], w[:, :t1], s0)
    o2, s2 = fwd(q[:, t1:], k[:, t1:], v[:, t1:], la[:, t1:], b[:, t1:], w[:, t1:], s1)
    assert rel_err(np.concatenate([o1, o2], axis=1), o) < RTOL, "state passing (o)"
    assert rel_err(s2, sf) < RTOL, "state passing (state)"


def pin_varlen(fwd, rng):
    lengths = [3, 0, 7, 1, 5]
    H, dk, dv = 2, 6, 5
    T = sum(lengths)
    q, k, v, la, b, w, _ = rand_problem(rng, B=1, T=T, H=H, dk=dk, dv=dv, init=False)
    s0 = rng.standard_normal((len(lengths), H, dk, dv)) * 0.3
    cu = np.concatenate([[0], np.cumsum(lengths)]).astype(np.int64)
    o, sf = fwd(q, k, v, la, b, w, s0, cu)
    for n, L in enumerate(lengths):
        a, e = cu[n], cu[n + 1]
        if L == 0:
            assert np.array_equal(sf[n], s0[n]), "varlen empty sequence keeps its state"
            continue
        o_n, s_n = fwd(q[:, a:e], k[:, a:e], v[:, a:e], la[:, a:e], b[:, a:e], w[:, a:e],
                       s0[n:n + 1])
        assert rel_err(o[:, a:e], o_n) < RTOL and rel_err(sf[n], s_n[0]) < RTOL, "varlen"


def pin_linearity(fwd, rng):
    """For fixed q, k, alpha, b the map (z, S_0) -> (o, S_T) is linear."""
    q, k, v1, la, b, w, s1 = rand_problem(rng)
    v2 = rng.standard_normal(v1.shape)
    s2 = rng.standard_normal(s1.shape)
    c = 0.7
    oa, sa = fwd(q, k, v1, la, b, w, s1)
    ob, sb = fwd(q, k, v2, la, b, w, s2)
    oc, sc = fwd(q, k, v1 + c * v2, la, b, w, s1 + c * s2)
    assert rel_err(oc, oa + c * ob) < 1e-10 and rel_err(sc, sa + c * sb) < 1e-10, "linearity"


FORWARD_PINS = [pin_kda, pin_gdn, pin_exact_recall, pin_no_erase_closed_form,
                pin_transition_products, pin_state_passing, pin_varlen, pin_linearity]
