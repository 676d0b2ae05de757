"""Gated Delta Rule-2 oracle (fp64, CPU) -- TEST INFRASTRUCTURE ONLY.

Only ``tests/``, ``__graft_entry__.smoke()`` and ``bench.py``'s CPU-baseline
leg may import this package. The CUDA library never calls it and shares no
code with it.

The forward arithmetic lives in ``gdr2_oracle.c`` (plain sequential fp64 C,
one token at a time); this module compiles it with gcc on first use and wraps
it for numpy arrays. The backward (``backward``, the vector-Jacobian product
of the same token rule) and the prologue are plain numpy in this module. Every input is upcast to float64 before the call, so bf16 inputs
enter the oracle with exactly the values the GPU sees.

Pinned by: tests/test_oracle_pins.py (KDA and Gated DeltaNet reductions,
exact recall, b=0 closed form, brute-force transition products, the
fast-weight argmin identity, state passing, varlen splitting, linearity; the
prologue against scipy's logistic function, numpy's logaddexp and norm);
tests/test_qed_oracle.py (the QED reading: its reductions to the plain rule,
the annihilation of both erase directions, brute-force products; PARITY
UNPINNED against the paper, which does not print the update);
tests/test_backward_oracle.py (the backward against central finite
differences of the forward, linearity in the cotangents, planted mistakes).
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import threading

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "gdr2_oracle.c")
_LIB = os.path.join(_HERE, "libgdr2_oracle.so")
_lock = threading.Lock()
_lib = None

_D = ctypes.POINTER(ctypes.c_double)
_I64 = ctypes.POINTER(ctypes.c_int64)


def build(force: bool = False) -> str:
    """Compile the oracle into ``oracle/libgdr2_oracle.so`` (gcc, -O2, OpenMP)."""
    if (not force and os.path.exists(_LIB)
            and os.path.getmtime(_LIB) >= os.path.getmtime(_SRC)):
        return _LIB
    tmp = _LIB + f".tmp{os.getpid()}"
    cmd = ["gcc", "-O2", "-fopenmp", "-shared", "-fPIC", "-std=c99",
           "-o", tmp, _SRC, "-lm"]
    subprocess.run(cmd, check=True)
    os.replace(tmp, _LIB)
    return _LIB


def _load():
    global _lib
    with _lock:
        if _lib is None:
            lib = ctypes.CDLL(build())
            lib.gdr2_oracle_forward.restype = ctypes.c_int
            lib.gdr2_oracle_forward.argtypes = [
                _D, _D, _D, _D, _D, _D, _D, _I64,
                ctypes.c_int64, ctypes.c_int64, ctypes.c_int64, ctypes.c_int64,
                ctypes.c_int64, ctypes.c_int64, _D, _D, ctypes.c_int]
            lib.gdr2_oracle_step.restype = ctypes.c_int
            lib.gdr2_oracle_step.argtypes = [
                _D, _D, _D, _D, _D, _D, _D,
                ctypes.c_int64, ctypes.c_int64, ctypes.c_int64, ctypes.c_int64,
                _D, ctypes.c_int]
            lib.gdr2_oracle_qed_forward.restype = ctypes.c_int
            lib.gdr2_oracle_qed_forward.argtypes = [
                _D, _D, _D, _D, _D, _D, _D, _D, ctypes.c_int, _D, _I64,
                ctypes.c_int64, ctypes.c_int64, ctypes.c_int64, ctypes.c_int64,
                ctypes.c_int64, ctypes.c_int64, _D, _D, ctypes.c_int]
            lib.gdr2_oracle_max_threads.restype = ctypes.c_int
            lib.gdr2_oracle_max_threads.argtypes = []
            _lib = lib
    return _lib


def _f64(x):
    return np.ascontiguousarray(np.asarray(x, dtype=np.float64))


def _p(a):
    return a.ctypes.data_as(_D) if a is not None else None


def max_threads() -> int:
    """Threads the oracle's OpenMP loop uses by default on this host."""
    return int(_load().gdr2_oracle_max_threads())


def forward(q, k, v, log_alpha, b, w, init_state=None, cu_seqlens=None,
            num_threads: int = 0):
    """Token-by-token fp64 forward of Gated Delta Rule-2.

    q, k, log_alpha, b: [B, T, H, d_k]; v, w: [B, T, H, d_v] (any float dtype,
    upcast to fp64). init_state: [N, H, d_k, d_v] or None (zeros).
    cu_seqlens: int array of N+1 offsets (then B must be 1) or None (N = B).
    Returns (o [B, T, H, d_v], final_state [N, H, d_k, d_v]) as float64.
    """
    q, k, v, la, b, w = (_f64(x) for x in (q, k, v, log_alpha, b, w))
    B, T, H, dk = q.shape
    dv = v.shape[-1]
    for name, x, d in (("k", k, dk), ("log_alpha", la, dk), ("b", b, dk),
                       ("v", v, dv), ("w", w, dv)):
        if x.shape != (B, T, H, d):
            raise ValueError(f"{name} has shape {x.shape}, expected {(B, T, H, d)}")
    if cu_seqlens is not None:
        cu = np.ascontiguousarray(np.asarray(cu_seqlens, dtype=np.int64))
        N = cu.shape[0] - 1
    else:
        cu = None
        N = B
    s0 = _f64(init_state) if init_state is not None else None
    if s0 is not None and s0.shape != (N, H, dk, dv):
        raise ValueError(f"init_state has shape {s0.shape}, expected {(N, H, dk, dv)}")
    o = np.zeros((B, T, H, dv), dtype=np.float64)
    sf = np.zeros((N, H, dk, dv), dtype=np.float64)
    rc = _load().gdr2_oracle_forward(
        _p(q), _p(k), _p(v), _p(la), _p(b), _p(w), _p(s0),
        cu.ctypes.data_as(_I64) if cu is not None else None,
        B, T, H, dk, dv, N, _p(o), _p(sf), int(num_threads))
    if rc != 0:
        raise ValueError(f"oracle forward rejected its arguments (code {rc})")
    return o, sf


QED_GATE = 1      # gate the query-derived erase by b_t
QED_PROJECT = 2   # project its direction orthogonal to k_t
QED_FULL = QED_GATE | QED_PROJECT


def qed_forward(q, k, v, log_alpha, b, w, strength, direction=None, flags: int = QED_FULL,
                init_state=None, cu_seqlens=None, num_threads: int = 0):
    """Token-by-token fp64 forward of Gated Delta Rule-2 with the QED second
    erase direction ("The Query Knows What to Forget", thelatestinai.com
    listing: abstract, Table 1). PARITY UNPINNED against the paper, which does
    not print the update: this is the reading in gdr2_oracle.c's QED section
    (a unit direction from the query, or from `direction` [H, d_k], projected
    orthogonal to k_t with flags & QED_PROJECT, erased with strength
    `strength` [H] and, with flags & QED_GATE, the erase gate b_t).

    Shapes and return values as forward()."""
    q, k, v, la, b, w = (_f64(x) for x in (q, k, v, log_alpha, b, w))
    B, T, H, dk = q.shape
    dv = v.shape[-1]
    for name, x, d in (("k", k, dk), ("log_alpha", la, dk), ("b", b, dk),
                       ("v", v, dv), ("w", w, dv)):
        if x.shape != (B, T, H, d):
            raise ValueError(f"{name} has shape {x.shape}, expected {(B, T, H, d)}")
    lam = _f64(strength).reshape(-1)
    if lam.shape != (H,):
        raise ValueError(f"strength has shape {lam.shape}, expected ({H},)")
    dirs = _f64(direction) if direction is not None else None
    if dirs is not None and dirs.shape != (H, dk):
        raise ValueError(f"direction has shape {dirs.shape}, expected {(H, dk)}")
    if cu_seqlens is not None:
        cu = np.ascontiguousarray(np.asarray(cu_seqlens, dtype=np.int64))
        N = cu.shape[0] - 1
    else:
        cu = None
        N = B
    s0 = _f64(init_state) if init_state is not None else None
    if s0 is not None and s0.shape != (N, H, dk, dv):
        raise ValueError(f"init_state has shape {s0.shape}, expected {(N, H, dk, dv)}")
    o = np.zeros((B, T, H, dv), dtype=np.float64)
    sf = np.zeros((N, H, dk, dv), dtype=np.float64)
    rc = _load().gdr2_oracle_qed_forward(
        _p(q), _p(k), _p(v), _p(la), _p(b), _p(w), _p(lam), _p(dirs), int(flags), _p(s0),
        cu.ctypes.data_as(_I64) if cu is not None else None,
        B, T, H, dk, dv, N, _p(o), _p(sf), int(num_threads))
    if rc != 0:
        raise ValueError(f"oracle QED forward rejected its arguments (code {rc})")
    return o, sf


def step(q, k, v, log_alpha, b, w, state, num_threads: int = 0):
    """One fp64 decode step. Token tensors [N, H, d]; state [N, H, d_k, d_v].

    Returns (o [N, H, d_v], new_state) without modifying the caller's array.
    """
    q, k, v, la, b, w = (_f64(x) for x in (q, k, v, log_alpha, b, w))
    N, H, dk = q.shape
    dv = v.shape[-1]
    S = np.array(state, dtype=np.float64, order="C", copy=True)
    if S.shape != (N, H, dk, dv):
        raise ValueError(f"state has shape {S.shape}, expected {(N, H, dk, dv)}")
    o = np.zeros((N, H, dv), dtype=np.float64)
    rc = _load().gdr2_oracle_step(_p(q), _p(k), _p(v), _p(la), _p(b), _p(w),
                                  _p(S), N, H, dk, dv, _p(o), int(num_threads))
    if rc != 0:
        raise ValueError(f"oracle step rejected its arguments (code {rc})")
    return o, S


# Fused-prologue flags (the same bit values as GDR2_PROLOGUE_* in gdr2.h).
PROLOGUE_QK_L2NORM = 1
PROLOGUE_GATE_SIGMOID = 2
PROLOGUE_DECAY_SOFTPLUS = 4


def prologue(q, k, log_alpha, b, w, flags: int):
    """The element-wise ends of the Gated DeltaNet-2 block's input branches, in
    fp64 ("Block design and hybrid model", ainews.random.gg article: q and k
    are L2-normalised, the erase and write gates are sigmoid projections; the
    decay branch's activation is not printed, -softplus is the reading taken).

    Per token and head, according to ``flags``:
      PROLOGUE_QK_L2NORM:      q, k <- x / sqrt(sum_c x_c^2 + 1e-6)
      PROLOGUE_GATE_SIGMOID:   b, w <- 1 / (1 + exp(-x))
      PROLOGUE_DECAY_SOFTPLUS: log_alpha <- -log(1 + exp(x))
    Returns (q, k, log_alpha, b, w) as float64 arrays.
    """
    q, k, la, b, w = (np.array(x, dtype=np.float64) for x in (q, k, log_alpha, b, w))
    if flags & PROLOGUE_QK_L2NORM:
        q = q / np.sqrt(np.sum(q * q, axis=-1, keepdims=True) + 1e-6)
        k = k / np.sqrt(np.sum(k * k, axis=-1, keepdims=True) + 1e-6)
    if flags & PROLOGUE_GATE_SIGMOID:
        b = 1.0 / (1.0 + np.exp(-b))
        w = 1.0 / (1.0 + np.exp(-w))
    if flags & PROLOGUE_DECAY_SOFTPLUS:
        # log(1 + e^x) = max(x, 0) + log(1 + e^{-|x|})  (no overflow)
        la = -(np.maximum(la, 0.0) + np.log1p(np.exp(-np.abs(la))))
    return q, k, la, b, w


def backward(q, k, v, log_alpha, b, w, init_state, d_o, d_final=None):
    """Vector-Jacobian product of the token recurrence (fp64, plain numpy,
    one token at a time in reverse, vectorised over (sequence, head) only).

    The "Chunkwise training and gate-aware backward" section of the
    ainews.random.gg article notes that with two different diagonal gates the
    gate factors must appear inside the gradient's dot products; here they do
    so by construction, by reverse-mode differentiation of the rule itself:
        S'_t = Diag(alpha_t) S_{t-1},  e_t = b_t . k_t,  z_t = w_t . v_t,
        r_t = S'_t^T e_t,  S_t = S'_t + k_t (z_t - r_t)^T,  o_t = S_t^T q_t.
    With G = dL/dS_t (accumulated from the end, starting at d_final), each
    step applies the chain rule to these five lines in reverse order (one line
    of the body per term).
    Fixed-length batches: tensors [B, T, H, d]; init_state [B, H, d_k, d_v] or
    None; d_o like o; d_final [B, H, d_k, d_v] or None (zero).
    Returns dq, dk, dv, dlog_alpha, db, dw, dinit_state (float64).
    """
    q, k, v, la, b, w, do = (np.asarray(x, dtype=np.float64) for x in (q, k, v, log_alpha, b, w, d_o))
    B, T, H, dk_ = q.shape
    dv_ = v.shape[-1]
    S = (np.zeros((B, H, dk_, dv_)) if init_state is None
         else np.array(init_state, dtype=np.float64, copy=True))
    alpha = np.exp(la)
    e = b * k
    z = w * v
    # forward, keeping every state S_{t-1} (input of step t)
    prev = np.empty((T, B, H, dk_, dv_))
    for t in range(T):
        prev[t] = S
        Sp = alpha[:, t, :, :, None] * S                       # S'_t = Diag(alpha_t) S_{t-1}
        r = np.einsum("bhij,bhi->bhj", Sp, e[:, t])            # r_t = S'^T e_t
        S = Sp + k[:, t, :, :, None] * (z[:, t] - r)[:, :, None, :]
    G = np.zeros((B, H, dk_, dv_)) if d_final is None else np.array(d_final, dtype=np.float64, copy=True)
    dq, dk, dv, dla, db, dw = (np.zeros_like(x) for x in (q, k, v, la, b, w))
    for t in range(T - 1, -1, -1):
        S_prev = prev[t]
        Sp = alpha[:, t, :, :, None] * S_prev
        r = np.einsum("bhij,bhi->bhj", Sp, e[:, t])
        u = z[:, t] - r
        S_t = Sp + k[:, t, :, :, None] * u[:, :, None, :]
        # o_t = S_t^T q_t
        G = G + q[:, t, :, :, None] * do[:, t, :, None, :]
        dq[:, t] = np.einsum("bhij,bhj->bhi", S_t, do[:, t])
        # S_t = S'_t + k_t u^T,  u = z_t - r_t
        du = np.einsum("bhij,bhi->bhj", G, k[:, t])
        dk_t = np.einsum("bhij,bhj->bhi", G, u)
        dz = du
        dr = -du
        # r_t = S'^T e_t:  dS' += e dr^T,  de = S' dr
        dSp = G + e[:, t, :, :, None] * dr[:, :, None, :]
        de = np.einsum("bhij,bhj->bhi", Sp, dr)
        # S'_t = Diag(alpha_t) S_{t-1}
        dalpha = np.sum(dSp * S_prev, axis=-1)
        G = alpha[:, t, :, :, None] * dSp
        # e = b . k,  z = w . v,  alpha = exp(log_alpha)
        db[:, t] = de * k[:, t]
        dk[:, t] = dk_t + de * b[:, t]
        dw[:, t] = dz * v[:, t]
        dv[:, t] = dz * w[:, t]
        dla[:, t] = dalpha * alpha[:, t]
    return dq, dk, dv, dla, db, dw, G
