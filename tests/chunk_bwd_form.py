"""The chunk (WY) form of the gate-aware backward in numpy, with an optional
rounding of every matrix-product operand and result (test helper; CPU only).

Without rounding it is the exact fp64 restatement that tests/test_backward_form.py
matches to the oracle's reverse loop. With rounding it emulates a tensor-core
kernel that feeds bf16 or tf32 operands and accumulates in fp32:

    python tests/chunk_bwd_form.py [T]

prints the relative L2 error of every gradient against the fp64 oracle for
fp32, tf32 (10 mantissa bits, truncated) and bf16 (round to nearest even)
operands, and for the two mixed choices (chains in one format, per-chunk row
products in the other), on one head of the layer shape (d = 128, bf16 inputs).
Formulas (decay exponents d = g - g_31 about chunk row 31, Qm = q e^d,
Km = k e^-d, Em = b k e^d, Sm = e^{g_31} S0, Ghat the cotangent of the state at
the chunk end):
    dU   = T^T (P^T dO + (Km e^{d_end}) Ghat)
    dQ   = e^d (dO Sm^T + tril(dO U^T) Km)
    dE   = -e^d (dU Sm^T + stril(dU U^T) Km)
    dKW  = e^-d (triu(U dO^T) Qm - striu(U dU^T) Em) + e^{d_end - d} (U Ghat^T)
    Ghat_prev = e^{g_31} (Qm^T dO - Em^T dU) + e^{g_end} Ghat
"""
import os
import sys

import numpy as np

C = 64
MID = 31


def bf16(x):
    x32 = np.ascontiguousarray(x, dtype=np.float32)
    bits = x32.view(np.uint32).astype(np.uint64)
    bits = ((bits + 0x7FFF + ((bits >> 16) & 1)) >> 16) << 16
    return bits.astype(np.uint32).view(np.float32).astype(np.float64)


def tf32(x):
    x32 = np.ascontiguousarray(x, dtype=np.float32)
    return (x32.view(np.uint32) & np.uint32(0xFFFFE000)).view(np.float32).astype(np.float64)


def fp32(x):
    return np.asarray(x, dtype=np.float32).astype(np.float64)


def _product(rnd):
    return (lambda a, c: a @ c) if rnd is None else (lambda a, c: fp32(rnd(a) @ rnd(c)))


def chunk_backward(q, k, v, la, b, w, s0, do, dfin, rnd=None, rnd_rows="same"):
    """One (sequence, head): q, k, la, b [T, dk]; v, w, do [T, dv]; s0, dfin [dk, dv].
    `rnd` rounds the operands of the chain products (A, P, U, dU, the state and
    cotangent updates); `rnd_rows` those of the per-chunk row products (dQ, dE,
    dKW), by default the same. Returns dq, dk, dv, dlog_alpha, db, dw, d_init_state."""
    mm = _product(rnd)
    mr = mm if rnd_rows == "same" else _product(rnd_rows)
    T_len, dk = q.shape
    dv_ = v.shape[1]
    nck = -(-T_len // C)
    pad = lambda x, t0, L: np.vstack([x[t0:t0 + L], np.zeros((C - L, x.shape[1]))])
    S = s0.copy()
    saved = []
    for c in range(nck):                                    # forward over chunks
        t0 = c * C
        L = min(C, T_len - t0)
        qc, kc, vc, lac, bc, wc, doc = (pad(x, t0, L) for x in (q, k, v, la, b, w, do))
        g = np.cumsum(lac, axis=0)
        d = g - g[MID]
        qm, km, em = qc * np.exp(d), kc * np.exp(-d), bc * kc * np.exp(d)
        sm = np.exp(g[MID])[:, None] * S
        A = np.tril(mm(em, km.T), -1)
        P = np.tril(mm(qm, km.T))
        Tinv = np.linalg.solve(np.eye(C) + A, np.eye(C))
        U = mm(Tinv, wc * vc - mm(em, sm))
        X = sm + mm(km.T, U)                                # S_end = e^{d_end} X
        saved.append((t0, L, qc, kc, vc, bc, wc, doc, g, d, qm, km, em, sm, P, Tinv, U, X))
        S = np.exp(d[C - 1])[:, None] * X
    dq, dkk, db, dla = (np.zeros((T_len, dk)) for _ in range(4))
    dvv, dww = np.zeros((T_len, dv_)), np.zeros((T_len, dv_))
    Gh = dfin.copy()
    for c in range(nck - 1, -1, -1):                        # reverse over chunks
        t0, L, qc, kc, vc, bc, wc, doc, g, d, qm, km, em, sm, P, Tinv, U, X = saved[c]
        ed = np.exp(d)
        dend = d[C - 1]
        dU = mm(Tinv.T, mm(P.T, doc) + mm(km * np.exp(dend), Gh))
        dQ = ed * (mr(doc, sm.T) + mr(np.tril(mr(doc, U.T)), km))
        dE = -ed * (mr(dU, sm.T) + mr(np.tril(mr(dU, U.T), -1), km))
        dKW = (np.exp(-d) * (mr(np.triu(mr(U, doc.T)), qm) - mr(np.triu(mr(U, dU.T), 1), em))
               + np.exp(dend - d) * mr(U, Gh.T))
        dg = qc * dQ - kc * dKW + bc * kc * dE
        acc = np.exp(dend) * np.sum(Gh * X, axis=1)         # rowsum(Ghat . S_end)
        for t in range(L - 1, -1, -1):
            acc = acc + dg[t]
            dla[t0 + t] = acc
        dq[t0:t0 + L] = dQ[:L]
        dkk[t0:t0 + L] = (dKW + bc * dE)[:L]
        db[t0:t0 + L] = (kc * dE)[:L]
        dvv[t0:t0 + L] = (dU * wc)[:L]
        dww[t0:t0 + L] = (dU * vc)[:L]
        Gh = np.exp(g[MID])[:, None] * (mm(qm.T, doc) - mm(em.T, dU)) + np.exp(g[C - 1])[:, None] * Gh
    return dq, dkk, dvv, dla, db, dww, Gh


def operand_precision_errors(T=512, seed=3, rnd=tf32, rnd_rows="same"):
    """Relative L2 error of every gradient of the rounded chunk form against
    the fp64 oracle, on one head of the layer shape with bf16 inputs."""
    import oracle
    from linear_attention_recurrence_gdr2_b200 import inputs as gen
    inp = gen.make_inputs(1, T, 1, 128, 128, "bf16", seed=seed, init_std=0.01)
    d_o, d_f = gen.cotangents(inp, seed=seed + 1)
    ref = oracle.backward(inp.q, inp.k, inp.v, inp.log_alpha, inp.b, inp.w, inp.init_state, d_o, d_f)
    f = lambda x: x[0, :, 0].astype(np.float64)
    got = chunk_backward(f(inp.q), f(inp.k), f(inp.v), f(inp.log_alpha), f(inp.b), f(inp.w),
                         inp.init_state[0, 0].astype(np.float64), f(d_o),
                         d_f[0, 0].astype(np.float64), rnd, rnd_rows)
    names = ("dq", "dk", "dv", "dlog_alpha", "db", "dw", "d_init_state")
    out = {}
    for name, g, r in zip(names, got, ref):
        r = r[0, 0] if name == "d_init_state" else r[0, :, 0]
        out[name] = float(np.linalg.norm((g - r).ravel()) / np.linalg.norm(r.ravel()))
    return out


if __name__ == "__main__":
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    sys.path.insert(0, root)
    T = int(sys.argv[1]) if len(sys.argv) > 1 else 512
    for name, rnd, rows in (("fp32", fp32, "same"), ("tf32", tf32, "same"), ("bf16", bf16, "same"),
                            ("chains tf32, rows bf16", tf32, bf16),
                            ("chains bf16, rows tf32", bf16, tf32)):
        e = operand_precision_errors(T, rnd=rnd, rnd_rows=rows)
        print(name, " ".join(f"{k}={v:.1e}" for k, v in e.items()))
