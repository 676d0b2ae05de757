"""The chunk form the kernels implement, checked in fp64 against the oracle
(CPU; no GPU, no import of the CUDA path).

This restates the algorithm of the chunk kernels step by step in numpy:
cumulative log-decay per chunk, decay factors taken about row 31
(d_r = g_r - g_31), the asymmetric erase factors Qm, Km, Em, A and P, T =
(I + A)^{-1} by the kernels' doubling on 16-row blocks, W = T Em, U = T Z - W Sm,
O = Qm Sm + P U and S <- Diag(e^{g_C - g_31}) (Sm + Km^T U). The chunk form is
derived in the "Chunkwise training and gate-aware backward" section of the
ainews.random.gg article on Gated DeltaNet-2; equality with the token-by-token
oracle (to fp64 rounding) pins the derivation the GPU code relies on.
"""
import numpy as np
import pytest

import oracle
from linear_attention_recurrence_gdr2_b200 import inputs as gen

C = 64
MID = 31


def inverse_by_doubling(A):
    """(I + A)^{-1} for strictly lower-triangular 64x64 A, as the kernels do it:
    16x16 diagonal blocks by forward substitution, then T_10 = -T_11 A_10 T_00
    inside each 32-block and across the two 32-blocks."""
    n = A.shape[0]
    T = np.zeros_like(A)
    for b0 in range(0, n, 16):
        blk = A[b0:b0 + 16, b0:b0 + 16]
        for j in range(16):           # column j of the block inverse
            x = np.zeros(16)
            x[j] = 1.0
            for i in range(16):       # right-looking forward substitution
                x[i + 1:] -= blk[i + 1:, i] * x[i]
            T[b0:b0 + 16, b0 + j] = x
    for size in (16, 32):
        for b0 in range(0, n, 2 * size):
            t00 = T[b0:b0 + size, b0:b0 + size]
            t11 = T[b0 + size:b0 + 2 * size, b0 + size:b0 + 2 * size]
            a10 = A[b0 + size:b0 + 2 * size, b0:b0 + size]
            T[b0 + size:b0 + 2 * size, b0:b0 + size] = -t11 @ (a10 @ t00)
    return T


def chunk_form(q, k, v, la, b, w, s0):
    """One (sequence, head): q, k, la, b [T, dk]; v, w [T, dv]; s0 [dk, dv]."""
    T_len, dk = q.shape
    S = s0.copy()
    o = np.zeros((T_len, v.shape[1]))
    for t0 in range(0, T_len, C):
        L = min(C, T_len - t0)
        pad = lambda x: np.vstack([x[t0:t0 + L], np.zeros((C - L, x.shape[1]))])
        qc, kc, vc, lac, bc, wc = (pad(x) for x in (q, k, v, la, b, w))
        g = np.cumsum(lac, axis=0)                 # rows past the end add nothing
        d = g - g[MID]
        qm, km, em = qc * np.exp(d), kc * np.exp(-d), bc * kc * np.exp(d)
        z = wc * vc
        sm = np.exp(g[MID])[:, None] * S
        A = np.tril(em @ km.T, -1)
        P = np.tril(qm @ km.T)
        Tinv = inverse_by_doubling(A)
        W = Tinv @ em
        U = Tinv @ z - W @ sm
        oc = qm @ sm + P @ U
        o[t0:t0 + L] = oc[:L]
        S = np.exp(g[C - 1] - g[MID])[:, None] * (sm + km.T @ U)
    return o, S


def test_doubling_inverse_is_exact():
    rng = np.random.default_rng(0)
    A = np.tril(rng.standard_normal((64, 64)) * 0.2, -1)
    np.testing.assert_allclose(inverse_by_doubling(A) @ (np.eye(64) + A), np.eye(64), atol=1e-12)


@pytest.mark.parametrize("T,la_scale,init", [(300, 0.1, 0.1), (64, 0.5, None), (131, 1.2, 0.05)])
def test_chunk_form_matches_oracle(T, la_scale, init):
    inp = gen.make_inputs(2, T, 2, 32, 24, "fp32", seed=7, la_scale=la_scale, init_std=init)
    o_r, s_r = oracle.forward(inp.q, inp.k, inp.v, inp.log_alpha, inp.b, inp.w, inp.init_state)
    for n in range(2):
        for h in range(2):
            s0 = (inp.init_state[n, h].astype(np.float64) if inp.init_state is not None
                  else np.zeros((32, 24)))
            f = lambda x: x[n, :, h].astype(np.float64)
            o, S = chunk_form(f(inp.q), f(inp.k), f(inp.v), f(inp.log_alpha), f(inp.b), f(inp.w), s0)
            scale = max(1.0, np.abs(o_r[n, :, h]).max())
            assert np.abs(o - o_r[n, :, h]).max() < 1e-12 * scale
            assert np.abs(S - s_r[n, h]).max() < 1e-12 * max(1.0, np.abs(s_r[n, h]).max())
