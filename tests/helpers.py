"""Shared helpers for the GPU parity tests: upload seeded inputs, run the CUDA
path through the binding, and compare with the fp64 oracle."""
from __future__ import annotations

import numpy as np

# Tolerances on the relative L2 error against the fp64 oracle, per input
# precision (fp32 inputs: 1e-4; bf16 inputs with fp32 state: 5e-3).
TOL = {"fp32": 1e-4, "bf16": 5e-3}


def rel_l2(x, ref) -> float:
    x = np.asarray(x, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    den = np.linalg.norm(ref.ravel())
    num = np.linalg.norm((x - ref).ravel())
    return float(num / den) if den > 0 else float(num)


def max_abs(x, ref) -> float:
    if np.asarray(ref).size == 0:
        return 0.0
    return float(np.max(np.abs(np.asarray(x, np.float64) - np.asarray(ref, np.float64))))


def assert_close(name, x, ref, dtype):
    e = rel_l2(x, ref)
    m = max_abs(x, ref)
    print(f"{name}: rel_l2={e:.3e} max_abs={m:.3e} (tol {TOL[dtype]:.0e})")
    assert np.all(np.isfinite(np.asarray(x, np.float64))), f"{name}: non-finite values"
    assert e <= TOL[dtype], f"{name}: rel_l2 {e:.3e} > {TOL[dtype]:.0e} (max_abs {m:.3e})"


def torch_dtype(dtype: str):
    import torch
    return torch.bfloat16 if dtype == "bf16" else torch.float32


def upload(inp, device):
    """Inputs (numpy, host) -> dict of device tensors in the operator's dtypes."""
    import torch
    dt = torch_dtype(inp.dtype)
    t = lambda x, d: torch.from_numpy(np.ascontiguousarray(x)).to(device=device, dtype=d)
    out = dict(q=t(inp.q, dt), k=t(inp.k, dt), v=t(inp.v, dt),
               log_alpha=t(inp.log_alpha, torch.float32), b=t(inp.b, dt), w=t(inp.w, dt))
    out["init_state"] = (t(inp.init_state, torch.float32)
                         if inp.init_state is not None else None)
    out["cu_seqlens"] = (t(inp.cu_seqlens, torch.int32)
                         if inp.cu_seqlens is not None else None)
    return out


def to_np(x):
    import torch
    return x.detach().to(torch.float64).cpu().numpy()


def unit_slices(inp, n, h):
    """Token range and arrays of one (sequence, head) unit, for the oracle."""
    if inp.cu_seqlens is not None:
        a, e = int(inp.cu_seqlens[n]), int(inp.cu_seqlens[n + 1])
        sl = lambda x: x[0:1, a:e, h:h + 1]
        rows = (0, slice(a, e), h)
    else:
        sl = lambda x: x[n:n + 1, :, h:h + 1]
        rows = (n, slice(None), h)
    s0 = inp.init_state[n:n + 1, h:h + 1] if inp.init_state is not None else None
    return sl, rows, s0
