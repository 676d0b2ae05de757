"""Seeded synthetic inputs for the Gated Delta Rule-2 operator.

This module draws random numbers and shapes them into the input
distributions of the workloads; it holds none of the operator's arithmetic.
Both the CUDA path (through the tests and the benchmark) and the fp64 oracle
take their inputs from here, so the two see identical bits.

Distributions (the layer-shaped workloads of the operator):
  q, k    ~ N(0,1), then L2-normalised per token and head over d_k
  v       ~ N(0,1)
  log_alpha = -softplus(N(0,1)) * la_scale        (per key channel, fp32)
  b, w    = sigmoid(N(0,1))                        (erase / write gates)
  states  = init_std * N(0,1)  when a nonzero initial state is requested
For bf16 workloads every token tensor except log_alpha is rounded once to
bf16 (round-to-nearest-even) on the host; the arrays returned are float32
arrays whose values are exactly representable in bf16. log_alpha and the
states stay fp32.

Seeding: the lengths of a packed batch come from
numpy.random.default_rng(seed). Each token tensor and state is drawn in
blocks of 2^22 values; block i of tensor number m (q, k, v, log_alpha, b, w,
initial state = 0..6) comes from a PCG64 generator seeded with
SeedSequence(seed, spawn_key=(m, i)). The values therefore depend only on the
seed and the shapes, not on how many threads draw the blocks.
"""
from __future__ import annotations

import os
from concurrent.futures import ThreadPoolExecutor
from dataclasses import dataclass, field
from typing import Optional

import numpy as np

FP32 = "fp32"
BF16 = "bf16"


def round_to_bf16(x: np.ndarray) -> np.ndarray:
    """Round float32 values to the nearest bf16 (ties to even); returns float32."""
    x = np.ascontiguousarray(x, dtype=np.float32)
    bits = x.view(np.uint32)
    lsb = (bits >> np.uint32(16)) & np.uint32(1)
    out = (bits + (np.uint32(0x7FFF) + lsb)) & np.uint32(0xFFFF0000)
    return out.view(np.float32)


_BLOCK = 1 << 22
_THREADS = max(1, min(32, os.cpu_count() or 1))


def _rows_parallel(fn, x: np.ndarray) -> np.ndarray:
    """fn applied to row blocks of x (rows = all axes but the last) in threads
    (numpy releases the GIL in its loops); fn must act on rows independently."""
    flat = x.reshape(-1, x.shape[-1]) if x.ndim > 1 else x.reshape(-1, 1)
    n = flat.shape[0]
    step = max(1, -(-n // (4 * _THREADS)))
    parts = [(a, min(n, a + step)) for a in range(0, n, step)] or [(0, 0)]
    out = [None] * len(parts)

    def run(i):
        a, e = parts[i]
        out[i] = fn(flat[a:e])

    with ThreadPoolExecutor(_THREADS) as ex:
        list(ex.map(run, range(len(parts))))
    return np.concatenate(out, axis=0).reshape(x.shape)


def _normal(seed: int, tensor: int, shape) -> np.ndarray:
    """Standard normal float32 draws of `shape`, block-parallel (module doc)."""
    n = int(np.prod(shape)) if len(shape) else 1
    out = np.empty(n, dtype=np.float32)
    nblk = max(1, -(-n // _BLOCK))

    def run(i):
        ss = np.random.SeedSequence(seed, spawn_key=(tensor, i))
        a, e = i * _BLOCK, min(n, (i + 1) * _BLOCK)
        np.random.Generator(np.random.PCG64(ss)).standard_normal(e - a, dtype=np.float32, out=out[a:e])

    if nblk == 1:
        run(0)
    else:
        with ThreadPoolExecutor(_THREADS) as ex:
            list(ex.map(run, range(nblk)))
    return out.reshape(shape)


def _softplus64(x: np.ndarray) -> np.ndarray:
    x = x.astype(np.float64)
    return np.logaddexp(0.0, x)


def _sigmoid32(x: np.ndarray) -> np.ndarray:
    return _rows_parallel(lambda r: (1.0 / (1.0 + np.exp(-r.astype(np.float64)))).astype(np.float32), x)


def _l2_normalise(x: np.ndarray) -> np.ndarray:
    def rows(r):
        r64 = r.astype(np.float64)
        n = np.sqrt((r64 * r64).sum(axis=-1, keepdims=True))
        return (r64 / np.maximum(n, 1e-30)).astype(np.float32)
    return _rows_parallel(rows, x)


def _neg_softplus_scaled(x: np.ndarray, scale: float) -> np.ndarray:
    return _rows_parallel(lambda r: (-_softplus64(r) * scale).astype(np.float32), x)


@dataclass
class Inputs:
    """One batch of operator inputs (numpy, host)."""
    q: np.ndarray
    k: np.ndarray
    v: np.ndarray
    log_alpha: np.ndarray
    b: np.ndarray
    w: np.ndarray
    init_state: Optional[np.ndarray]
    cu_seqlens: Optional[np.ndarray]
    dtype: str
    meta: dict = field(default_factory=dict)

    @property
    def num_seqs(self) -> int:
        if self.cu_seqlens is not None:
            return int(self.cu_seqlens.shape[0] - 1)
        return int(self.q.shape[0])

    @property
    def num_tokens(self) -> int:
        return int(self.q.shape[0] * self.q.shape[1])


def _token_tensors(seed, shape_k, shape_v, dtype, la_scale):
    q = _l2_normalise(_normal(seed, 0, shape_k))
    k = _l2_normalise(_normal(seed, 1, shape_k))
    v = _normal(seed, 2, shape_v)
    la = _neg_softplus_scaled(_normal(seed, 3, shape_k), la_scale)
    b = _sigmoid32(_normal(seed, 4, shape_k))
    w = _sigmoid32(_normal(seed, 5, shape_v))
    if dtype == BF16:
        q, k, v, b, w = (_rows_parallel(round_to_bf16, x) for x in (q, k, v, b, w))
    elif dtype != FP32:
        raise ValueError(f"unknown dtype {dtype!r}")
    return q, k, v, la, b, w


def make_inputs(B: int, T: int, H: int, dk: int, dv: int, dtype: str = BF16,
                seed: int = 0, la_scale: float = 0.1,
                init_std: Optional[float] = None,
                lengths: Optional[np.ndarray] = None,
                length_range: Optional[tuple] = None,
                num_seqs: Optional[int] = None) -> Inputs:
    """Draw one batch.

    Fixed-length batch: token tensors [B, T, H, d].
    Packed variable-length batch: pass ``lengths`` (explicit) or
    ``length_range=(lo, hi)`` with ``num_seqs`` (drawn first, integers in
    [lo, hi] inclusive); token tensors are [1, sum(lengths), H, d] and
    ``cu_seqlens`` holds the N+1 offsets. ``init_std`` draws a nonzero initial
    state init_std * N(0,1) of shape [N, H, dk, dv]; None means no state.
    """
    rng = np.random.default_rng(seed)
    cu = None
    if length_range is not None:
        lo, hi = length_range
        lengths = rng.integers(lo, hi, size=int(num_seqs), endpoint=True)
    if lengths is not None:
        lengths = np.asarray(lengths, dtype=np.int64)
        cu = np.zeros(lengths.shape[0] + 1, dtype=np.int64)
        cu[1:] = np.cumsum(lengths)
        B, T = 1, int(cu[-1])
    q, k, v, la, b, w = _token_tensors(seed, (B, T, H, dk), (B, T, H, dv),
                                       dtype, la_scale)
    N = B if cu is None else int(cu.shape[0] - 1)
    s0 = None
    if init_std is not None:
        s0 = (_normal(seed, 6, (N, H, dk, dv)) * np.float32(init_std)).astype(np.float32)
    return Inputs(q, k, v, la, b, w, s0, cu, dtype,
                  meta=dict(B=B, T=T, H=H, dk=dk, dv=dv, seed=seed,
                            la_scale=la_scale, init_std=init_std))


def with_decay_regime(inp: Inputs, regime: str, seed: int = 0) -> Inputs:
    """Replace log_alpha by another decay regime (in place; returns `inp`),
    drawn from its own generator seeded with `seed`:
      "strong"  every key channel forgets fast: log alpha ~ U(-20, -5)
      "mixed"   about a third of the key channels (the same ones for every
                token and head) as in "strong", the others unchanged
      "none"    alpha = 1 (log alpha = 0): no decay at all
      "edge"    decay at the edge of a 64-token chunk form with factors taken
                about the middle row: log alpha ~ U(-1.95, -1.85) on the first
                32 tokens of every 64 (half-chunk sums near -60) and
                U(-0.1, -0.05) on the other 32 (token positions counted from
                the start of the token axis, so fixed-length batches only)
      "window"  log alpha ~ U(-1.2, -1.1) everywhere: every 64 consecutive
                tokens decay by about -74
    """
    rng = np.random.default_rng(seed)
    la = inp.log_alpha
    if regime == "strong":
        la[...] = -rng.uniform(5.0, 20.0, size=la.shape).astype(np.float32)
    elif regime == "mixed":
        strong = rng.random(la.shape[-1]) < 1.0 / 3.0
        draw = -rng.uniform(5.0, 20.0, size=la.shape).astype(np.float32)
        la[..., strong] = draw[..., strong]
    elif regime == "none":
        la[...] = 0.0
    elif regime == "edge":
        first = (np.arange(la.shape[1]) % 64) < 32
        strong = -rng.uniform(1.85, 1.95, size=la.shape).astype(np.float32)
        weak = -rng.uniform(0.05, 0.1, size=la.shape).astype(np.float32)
        la[...] = np.where(first[None, :, None, None], strong, weak)
    elif regime == "window":
        la[...] = -rng.uniform(1.1, 1.2, size=la.shape).astype(np.float32)
    else:
        raise ValueError(f"unknown decay regime {regime!r}")
    inp.meta["decay"] = regime
    return inp


@dataclass
class DecodeInputs:
    """A run of single-token decode steps: token tensors [steps, N, H, d]."""
    q: np.ndarray
    k: np.ndarray
    v: np.ndarray
    log_alpha: np.ndarray
    b: np.ndarray
    w: np.ndarray
    state: np.ndarray
    dtype: str


def make_decode_inputs(N: int, H: int, dk: int, dv: int, steps: int,
                       dtype: str = BF16, seed: int = 0, la_scale: float = 0.1,
                       init_std: float = 0.01) -> DecodeInputs:
    """An initial state init_std * N(0,1) [N, H, dk, dv] and, for all steps
    at once, q, k, v, log_alpha, b, w of shape [steps, N, H, d]."""
    state = (_normal(seed, 6, (N, H, dk, dv)) * np.float32(init_std)).astype(np.float32)
    stack = _token_tensors(seed, (steps, N, H, dk), (steps, N, H, dv), dtype, la_scale)
    return DecodeInputs(*stack, state=state, dtype=dtype)


# The five workloads, by what they are.
def tiny_fp32(seed: int = 0) -> Inputs:
    """B=1, H=1, T=256, d_k=d_v=64, fp32, zero initial state."""
    return make_inputs(1, 256, 1, 64, 64, FP32, seed)


def layer_prefill(seed: int = 0) -> Inputs:
    """B=4, H=16, T=2048, d_k=d_v=128, bf16, zero initial state."""
    return make_inputs(4, 2048, 16, 128, 128, BF16, seed)


def long_context(seed: int = 0, T: int = 32768, H: int = 16) -> Inputs:
    """B=1, H=16, T=32768, d=128, bf16, slow forgetting (log-decay x0.02),
    initial state 0.01 * N(0,1)."""
    return make_inputs(1, T, H, 128, 128, BF16, seed, la_scale=0.02,
                       init_std=0.01)


def varlen_packed(seed: int = 0, num_seqs: int = 64, lo: int = 128,
                  hi: int = 8192) -> Inputs:
    """64 sequences, lengths uniform in [128, 8192], packed via cu_seqlens,
    H=16, d=128, bf16, per-sequence initial states 0.01 * N(0,1)."""
    return make_inputs(1, 0, 16, 128, 128, BF16, seed, init_std=0.01,
                       length_range=(lo, hi), num_seqs=num_seqs)


def decode_batch(seed: int = 0, steps: int = 64, N: int = 256) -> DecodeInputs:
    """N=256 sequences x H=16 heads, d=128, fp32 state 0.01 * N(0,1),
    64 consecutive bf16 decode steps."""
    return make_decode_inputs(N, 16, 128, 128, steps, BF16, seed)


def preact_inputs(B: int, T: int, H: int, d: int, dtype: str = BF16, seed: int = 0,
                  init_std: Optional[float] = None, decay_shift: float = -2.5) -> Inputs:
    """Pre-activation inputs for the fused prologue (gdr2_chunk_fwd_preact):
    q, k ~ 2 N(0,1) (not normalised), v ~ N(0,1), b, w ~ 2 N(0,1) (before the
    sigmoid), log_alpha ~ N(decay_shift, 1) (before -softplus: about -0.1 per
    token for the default shift). Same rounding and seeding scheme as make_inputs."""
    sk, sv = (B, T, H, d), (B, T, H, d)
    q = 2.0 * _normal(seed, 0, sk)
    k = 2.0 * _normal(seed, 1, sk)
    v = _normal(seed, 2, sv)
    la = (_normal(seed, 3, sk) + np.float32(decay_shift)).astype(np.float32)
    b = 2.0 * _normal(seed, 4, sk)
    w = 2.0 * _normal(seed, 5, sv)
    if dtype == BF16:
        q, k, v, b, w = (round_to_bf16(x) for x in (q, k, v, b, w))
    elif dtype != FP32:
        raise ValueError(f"unknown dtype {dtype!r}")
    s0 = None
    if init_std is not None:
        s0 = (_normal(seed, 6, (B, H, d, d)) * np.float32(init_std)).astype(np.float32)
    return Inputs(q, k, v, la, b, w, s0, None, dtype, {"preact": True})


def cotangents(inp: Inputs, seed: int = 1, final_std: float = 0.1):
    """Seeded cotangents for the backward: d_o ~ N(0,1) shaped like o (rounded
    to bf16 for bf16 workloads) and d_final ~ final_std * N(0,1), fp32
    [N, H, dk, dv] (tensor numbers 0 and 1 of the seeding scheme)."""
    B, T, H, dv = inp.v.shape
    dk = inp.q.shape[-1]
    d_o = _normal(seed, 0, (B, T, H, dv))
    if inp.dtype == BF16:
        d_o = round_to_bf16(d_o)
    d_final = (_normal(seed, 1, (inp.num_seqs, H, dk, dv)) * np.float32(final_std)).astype(np.float32)
    return d_o, d_final
