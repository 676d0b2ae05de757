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
states stay fp32. Draw order from numpy.random.default_rng(seed):
[lengths,] q, k, v, log_alpha, b, w, [initial state].
"""
from __future__ import annotations

from dataclasses import dataclass, field
from typing import Optional

import numpy as np

FP32 = "fp32"
BF16 = "bf16"


def round_to_bf16(x: np.ndarray) -> np.ndarray:
    """Round float32 values to the nearest bf16 (ties to even); returns float32."""
    x = np.ascontiguousarray(x, dtype=np.float32)
    bits = x.view(np.uint32).astype(np.uint64)
    lsb = (bits >> 16) & 1
    bits = ((bits + 0x7FFF + lsb) >> 16) << 16
    return bits.astype(np.uint32).view(np.float32)


def _softplus64(x: np.ndarray) -> np.ndarray:
    x = x.astype(np.float64)
    return np.logaddexp(0.0, x)


def _sigmoid32(x: np.ndarray) -> np.ndarray:
    return (1.0 / (1.0 + np.exp(-x.astype(np.float64)))).astype(np.float32)


def _l2_normalise(x: np.ndarray) -> np.ndarray:
    x64 = x.astype(np.float64)
    n = np.sqrt((x64 * x64).sum(axis=-1, keepdims=True))
    return (x64 / np.maximum(n, 1e-30)).astype(np.float32)


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


def _token_tensors(rng, shape_k, shape_v, dtype, la_scale):
    q = _l2_normalise(rng.standard_normal(shape_k, dtype=np.float32))
    k = _l2_normalise(rng.standard_normal(shape_k, dtype=np.float32))
    v = rng.standard_normal(shape_v, dtype=np.float32)
    la = (-_softplus64(rng.standard_normal(shape_k, dtype=np.float32))
          * la_scale).astype(np.float32)
    b = _sigmoid32(rng.standard_normal(shape_k, dtype=np.float32))
    w = _sigmoid32(rng.standard_normal(shape_v, dtype=np.float32))
    if dtype == BF16:
        q, k, v, b, w = (round_to_bf16(x) for x in (q, k, v, b, w))
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
    q, k, v, la, b, w = _token_tensors(rng, (B, T, H, dk), (B, T, H, dv),
                                       dtype, la_scale)
    N = B if cu is None else int(cu.shape[0] - 1)
    s0 = None
    if init_std is not None:
        s0 = (rng.standard_normal((N, H, dk, dv), dtype=np.float32)
              * np.float32(init_std)).astype(np.float32)
    return Inputs(q, k, v, la, b, w, s0, cu, dtype,
                  meta=dict(B=B, T=T, H=H, dk=dk, dv=dv, seed=seed,
                            la_scale=la_scale, init_std=init_std))


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
    """Draw an initial state init_std * N(0,1) [N, H, dk, dv], then for each
    step, in step order, q, k, v, log_alpha, b, w of shape [N, H, d]."""
    rng = np.random.default_rng(seed)
    state = (rng.standard_normal((N, H, dk, dv), dtype=np.float32)
             * np.float32(init_std)).astype(np.float32)
    per = [_token_tensors(rng, (N, H, dk), (N, H, dv), dtype, la_scale)
           for _ in range(steps)]
    stack = [np.stack([p[i] for p in per]) for i in range(6)]
    return DecodeInputs(*stack, state=state, dtype=dtype)


# The five workloads, by what they are.
def tiny_fp32(seed: int = 0) -> Inputs:
    """B=1, H=1, T=256, d_k=d_v=64, fp32, zero initial state."""
    return make_inputs(1, 256, 1, 64, 64, FP32, seed)


def layer_prefill(seed: int = 0) -> Inputs:
    """B=4, H=16, T=2048, d_k=d_v=128, bf16, zero initial state."""
    return make_inputs(4, 2048, 16, 128, 128, BF16, seed)


def long_context(seed: int = 0, T: int = 32768) -> Inputs:
    """B=1, H=16, T=32768, d=128, bf16, slow forgetting (log-decay x0.02),
    initial state 0.01 * N(0,1)."""
    return make_inputs(1, T, 16, 128, 128, BF16, seed, la_scale=0.02,
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
    token for the default shift). Same rounding and draw order as make_inputs."""
    rng = np.random.default_rng(seed)
    sk, sv = (B, T, H, d), (B, T, H, d)
    q = 2.0 * rng.standard_normal(sk, dtype=np.float32)
    k = 2.0 * rng.standard_normal(sk, dtype=np.float32)
    v = rng.standard_normal(sv, dtype=np.float32)
    la = (rng.standard_normal(sk, dtype=np.float32) + np.float32(decay_shift)).astype(np.float32)
    b = 2.0 * rng.standard_normal(sk, dtype=np.float32)
    w = 2.0 * rng.standard_normal(sv, dtype=np.float32)
    if dtype == BF16:
        q, k, v, b, w = (round_to_bf16(x) for x in (q, k, v, b, w))
    elif dtype != FP32:
        raise ValueError(f"unknown dtype {dtype!r}")
    s0 = None
    if init_std is not None:
        s0 = (rng.standard_normal((B, H, d, d), dtype=np.float32) * np.float32(init_std)).astype(np.float32)
    return Inputs(q, k, v, la, b, w, s0, None, dtype, {"preact": True})


def cotangents(inp: Inputs, seed: int = 1, final_std: float = 0.1):
    """Seeded cotangents for the backward: d_o ~ N(0,1) shaped like o (rounded
    to bf16 for bf16 workloads) and d_final ~ final_std * N(0,1), fp32
    [N, H, dk, dv]. Draw order: d_o, d_final."""
    rng = np.random.default_rng(seed)
    B, T, H, dv = inp.v.shape
    dk = inp.q.shape[-1]
    d_o = rng.standard_normal((B, T, H, dv), dtype=np.float32)
    if inp.dtype == BF16:
        d_o = round_to_bf16(d_o)
    d_final = (rng.standard_normal((inp.num_seqs, H, dk, dv), dtype=np.float32)
               * np.float32(final_std)).astype(np.float32)
    return d_o, d_final
