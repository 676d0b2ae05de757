"""Gated Delta Rule-2 on B200: Python binding of the C-ABI library libgdr2.so.

This module only marshals arguments: it checks tensor shapes, dtypes and
devices, allocates outputs with PyTorch (device memory and streams are the
only things PyTorch is used for) and calls the ``extern "C"`` entry points
declared in ``include/gdr2.h`` on the current CUDA stream. Every step of the
operator runs in the library's CUDA kernels; there is no fallback. If the
library has not been built, the first call raises ``RuntimeError``.

Entry points (same names as the C ABI):
  chunk_fwd(q, k, v, log_alpha, b, w, init_state=None, cu_seqlens=None)
      -> (o, final_state)
  recurrent_step(q, k, v, log_alpha, b, w, state) -> o   (state in place)
  chunk_bwd(q, k, v, log_alpha, b, w, d_o, init_state=None, d_final_state=None,
            cu_seqlens=None) -> (dq, dk, dv, d_log_alpha, db, dw, d_init_state)
"""
from __future__ import annotations

import ctypes
import os
import threading
from typing import Optional, Tuple

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libgdr2.so")

GDR2_OK = 0
GDR2_FP32 = 0
GDR2_BF16 = 1
# fused prologue flags (gdr2.h)
GDR2_PROLOGUE_QK_L2NORM = 1
GDR2_PROLOGUE_GATE_SIGMOID = 2
GDR2_PROLOGUE_DECAY_SOFTPLUS = 4
GDR2_PROLOGUE_ALL = 7

_lock = threading.Lock()
_lib = None

_vp = ctypes.c_void_p
_i64 = ctypes.c_int64


class GDR2Error(RuntimeError):
    """A non-OK status returned by the C library."""

    def __init__(self, fn: str, status: int):
        self.status = status
        super().__init__(f"{fn} failed: {status_string(status)} (status {status})")


def lib() -> ctypes.CDLL:
    """Load libgdr2.so (raises RuntimeError if it has not been built)."""
    global _lib
    with _lock:
        if _lib is None:
            if not os.path.exists(LIB_PATH):
                raise RuntimeError(
                    f"{LIB_PATH} is missing: build the CUDA library first "
                    "(python -m linear_attention_recurrence_gdr2_b200.build)")
            L = ctypes.CDLL(LIB_PATH)
            L.gdr2_status_string.restype = ctypes.c_char_p
            L.gdr2_status_string.argtypes = [ctypes.c_int]
            L.gdr2_version.restype = ctypes.c_int
            L.gdr2_version.argtypes = []
            L.gdr2_chunk_fwd_workspace_size.restype = ctypes.c_int
            L.gdr2_chunk_fwd_workspace_size.argtypes = [
                _i64, _i64, _i64, _i64, _i64, _i64, ctypes.c_int, ctypes.POINTER(ctypes.c_size_t)]
            L.gdr2_chunk_fwd.restype = ctypes.c_int
            L.gdr2_chunk_fwd.argtypes = [
                _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp,
                _i64, _i64, _i64, _i64, _i64, _i64, ctypes.c_int,
                _vp, _vp, _vp, ctypes.c_size_t, _vp]
            L.gdr2_chunk_fwd_noalloc.restype = ctypes.c_int
            L.gdr2_chunk_fwd_noalloc.argtypes = [
                _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp,
                _i64, _i64, _i64, _i64, _i64, _i64, ctypes.c_int,
                _vp, _vp, _vp]
            L.gdr2_qed_fwd.restype = ctypes.c_int
            L.gdr2_qed_fwd.argtypes = [
                _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, ctypes.c_uint32, _vp, _vp,
                _i64, _i64, _i64, _i64, _i64, _i64, ctypes.c_int, _vp, _vp, _vp]
            L.gdr2_check_device_error.restype = ctypes.c_int
            L.gdr2_check_device_error.argtypes = [_vp]
            L.gdr2_recurrent_step.restype = ctypes.c_int
            L.gdr2_recurrent_step.argtypes = [
                _vp, _vp, _vp, _vp, _vp, _vp, _vp,
                _i64, _i64, _i64, _i64, ctypes.c_int, _vp, _vp]
            L.gdr2_chunk_fwd_preact.restype = ctypes.c_int
            L.gdr2_chunk_fwd_preact.argtypes = [
                _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp,
                _i64, _i64, _i64, _i64, _i64, _i64, ctypes.c_int,
                _vp, _vp, _vp, ctypes.c_size_t, ctypes.c_uint32, _vp]
            L.gdr2_recurrent_step_preact.restype = ctypes.c_int
            L.gdr2_recurrent_step_preact.argtypes = [
                _vp, _vp, _vp, _vp, _vp, _vp, _vp,
                _i64, _i64, _i64, _i64, ctypes.c_int, _vp, ctypes.c_uint32, _vp]
            L.gdr2_chunk_bwd_workspace_size.restype = ctypes.c_int
            L.gdr2_chunk_bwd_workspace_size.argtypes = [
                _i64, _i64, _i64, _i64, _i64, _i64, ctypes.c_int, ctypes.POINTER(ctypes.c_size_t)]
            L.gdr2_chunk_bwd.restype = ctypes.c_int
            L.gdr2_chunk_bwd.argtypes = [
                _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp,
                _i64, _i64, _i64, _i64, _i64, _i64, ctypes.c_int,
                _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, ctypes.c_size_t, _vp]
            _lib = L
    return _lib


def status_string(status: int) -> str:
    return lib().gdr2_status_string(int(status)).decode()


def version() -> int:
    return int(lib().gdr2_version())


def check_device_error(stream=None) -> None:
    """Synchronise `stream` and raise GDR2Error if a kernel of the library gave
    up a bounded device-side wait since the last check (gdr2_check_device_error)."""
    st = lib().gdr2_check_device_error(_stream_handle(stream))
    if st != GDR2_OK:
        raise GDR2Error("gdr2_check_device_error", st)


def _dtype_code(t) -> int:
    import torch
    if t.dtype == torch.bfloat16:
        return GDR2_BF16
    if t.dtype == torch.float32:
        return GDR2_FP32
    raise TypeError(f"unsupported dtype {t.dtype}; use torch.bfloat16 or torch.float32")


def _ptr(t) -> Optional[int]:
    return None if t is None else t.data_ptr()


def _check(t, name, shape, dtype, device):
    if t.device != device:
        raise ValueError(f"{name} is on {t.device}, expected {device}")
    if tuple(t.shape) != tuple(shape):
        raise ValueError(f"{name} has shape {tuple(t.shape)}, expected {tuple(shape)}")
    if t.dtype != dtype:
        raise TypeError(f"{name} has dtype {t.dtype}, expected {dtype}")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")


def _stream_handle(stream) -> int:
    import torch
    if stream is None:
        stream = torch.cuda.current_stream()
    return stream.cuda_stream


def workspace_size(B: int, T: int, H: int, d_k: int, d_v: int, num_seqs: int,
                   dtype_code: int) -> int:
    out = ctypes.c_size_t(0)
    st = lib().gdr2_chunk_fwd_workspace_size(B, T, H, d_k, d_v, num_seqs, dtype_code,
                                             ctypes.byref(out))
    if st != GDR2_OK:
        raise GDR2Error("gdr2_chunk_fwd_workspace_size", st)
    return int(out.value)


def bwd_workspace_size(B: int, T: int, H: int, d_k: int, d_v: int, num_seqs: int,
                       dtype_code: int) -> int:
    out = ctypes.c_size_t(0)
    st = lib().gdr2_chunk_bwd_workspace_size(B, T, H, d_k, d_v, num_seqs, dtype_code,
                                             ctypes.byref(out))
    if st != GDR2_OK:
        raise GDR2Error("gdr2_chunk_bwd_workspace_size", st)
    return int(out.value)


def chunk_bwd(q, k, v, log_alpha, b, w, d_o, init_state=None, d_final_state=None,
              cu_seqlens=None, *, output_d_init_state: bool = True, workspace=None,
              stream=None):
    """Gate-aware backward of Gated Delta Rule-2 (see gdr2_chunk_bwd in gdr2.h).

    Same inputs as chunk_fwd plus d_o (cotangent of o, like o) and
    d_final_state ([N, H, d_k, d_v] fp32 or None = zero). Returns
    (dq, dk, dv, d_log_alpha, db, dw, d_init_state): the first six like their
    inputs (d_log_alpha fp32), d_init_state [N, H, d_k, d_v] fp32 or None.
    """
    import torch
    dev = q.device
    if dev.type != "cuda":
        raise ValueError("chunk_bwd needs CUDA tensors")
    B, T, H, dk = q.shape
    dv = v.shape[-1]
    dt = q.dtype
    code = _dtype_code(q)
    for name, t, d in (("k", k, dk), ("b", b, dk), ("v", v, dv), ("w", w, dv), ("d_o", d_o, dv)):
        _check(t, name, (B, T, H, d), dt, dev)
    _check(q, "q", (B, T, H, dk), dt, dev)
    _check(log_alpha, "log_alpha", (B, T, H, dk), torch.float32, dev)
    if cu_seqlens is not None:
        if cu_seqlens.dtype != torch.int32 or cu_seqlens.device != dev or cu_seqlens.dim() != 1:
            raise ValueError("cu_seqlens must be a 1-D int32 tensor on the same device")
        N = cu_seqlens.shape[0] - 1
    else:
        N = B
    for name, t in (("init_state", init_state), ("d_final_state", d_final_state)):
        if t is not None:
            _check(t, name, (N, H, dk, dv), torch.float32, dev)
    dq, dk_, db = (torch.empty((B, T, H, dk), dtype=dt, device=dev) for _ in range(3))
    dv_, dw = (torch.empty((B, T, H, dv), dtype=dt, device=dev) for _ in range(2))
    dla = torch.empty((B, T, H, dk), dtype=torch.float32, device=dev)
    d_init = (torch.empty((N, H, dk, dv), dtype=torch.float32, device=dev)
              if output_d_init_state else None)
    need = bwd_workspace_size(B, T, H, dk, dv, N, code)
    if workspace is None or workspace.numel() * workspace.element_size() < need:
        workspace = torch.empty(max(need, 256), dtype=torch.uint8, device=dev)
    st = lib().gdr2_chunk_bwd(
        _ptr(q), _ptr(k), _ptr(v), _ptr(log_alpha), _ptr(b), _ptr(w), _ptr(init_state),
        _ptr(cu_seqlens), _ptr(d_o), _ptr(d_final_state), B, T, H, dk, dv, N, code,
        _ptr(dq), _ptr(dk_), _ptr(dv_), _ptr(dla), _ptr(db), _ptr(dw), _ptr(d_init),
        _ptr(workspace), workspace.numel() * workspace.element_size(), _stream_handle(stream))
    if st != GDR2_OK:
        raise GDR2Error("gdr2_chunk_bwd", st)
    return dq, dk_, dv_, dla, db, dw, d_init


def chunk_fwd(q, k, v, log_alpha, b, w, init_state=None, cu_seqlens=None, *,
              o=None, final_state=None, output_final_state: bool = True,
              workspace=None, prologue: int = 0,
              stream=None) -> Tuple["torch.Tensor", Optional["torch.Tensor"]]:
    """Chunkwise forward of Gated Delta Rule-2 (see gdr2_chunk_fwd in gdr2.h).

    q, k, b: [B, T, H, d_k]; v, w: [B, T, H, d_v] (bf16 or fp32, all alike);
    log_alpha: [B, T, H, d_k] fp32; init_state: [N, H, d_k, d_v] fp32 or None;
    cu_seqlens: int32 [N+1] on the device (then B == 1) or None.
    prologue: GDR2_PROLOGUE_* flags (gdr2_chunk_fwd_preact): activations the
    kernels apply to pre-activation q, k, b, w, log_alpha on load.
    Returns (o [B, T, H, d_v], final_state [N, H, d_k, d_v] fp32 or None).
    """
    import torch
    dev = q.device
    if dev.type != "cuda":
        raise ValueError("chunk_fwd needs CUDA tensors")
    B, T, H, dk = q.shape
    dv = v.shape[-1]
    dt = q.dtype
    code = _dtype_code(q)
    for name, t, d in (("k", k, dk), ("b", b, dk), ("v", v, dv), ("w", w, dv)):
        _check(t, name, (B, T, H, d), dt, dev)
    _check(q, "q", (B, T, H, dk), dt, dev)
    _check(log_alpha, "log_alpha", (B, T, H, dk), torch.float32, dev)
    if cu_seqlens is not None:
        if cu_seqlens.dtype != torch.int32 or cu_seqlens.device != dev or cu_seqlens.dim() != 1:
            raise ValueError("cu_seqlens must be a 1-D int32 tensor on the same device")
        N = cu_seqlens.shape[0] - 1
    else:
        N = B
    if init_state is not None:
        _check(init_state, "init_state", (N, H, dk, dv), torch.float32, dev)
    if o is None:
        o = torch.empty((B, T, H, dv), dtype=dt, device=dev)
    else:
        _check(o, "o", (B, T, H, dv), dt, dev)
    if final_state is None and output_final_state:
        final_state = torch.empty((N, H, dk, dv), dtype=torch.float32, device=dev)
    elif final_state is not None:
        _check(final_state, "final_state", (N, H, dk, dv), torch.float32, dev)
    need = workspace_size(B, T, H, dk, dv, N, code)
    if need > 0 and (workspace is None or workspace.numel() * workspace.element_size() < need):
        workspace = torch.empty(need, dtype=torch.uint8, device=dev)
    ws_bytes = 0 if workspace is None else workspace.numel() * workspace.element_size()
    if prologue:
        st = lib().gdr2_chunk_fwd_preact(
            _ptr(q), _ptr(k), _ptr(v), _ptr(log_alpha), _ptr(b), _ptr(w), _ptr(init_state),
            _ptr(cu_seqlens), B, T, H, dk, dv, N, code, _ptr(o), _ptr(final_state),
            _ptr(workspace), ws_bytes, int(prologue), _stream_handle(stream))
        if st != GDR2_OK:
            raise GDR2Error("gdr2_chunk_fwd_preact", st)
        return o, final_state
    st = lib().gdr2_chunk_fwd(
        _ptr(q), _ptr(k), _ptr(v), _ptr(log_alpha), _ptr(b), _ptr(w), _ptr(init_state),
        _ptr(cu_seqlens), B, T, H, dk, dv, N, code, _ptr(o), _ptr(final_state),
        _ptr(workspace), ws_bytes, _stream_handle(stream))
    if st != GDR2_OK:
        raise GDR2Error("gdr2_chunk_fwd", st)
    return o, final_state


def chunk_fwd_noalloc(q, k, v, log_alpha, b, w, init_state=None, cu_seqlens=None, *,
                      o, final_state=None, stream=None):
    """gdr2_chunk_fwd_noalloc: the chunk forward with caller-provided outputs
    and no workspace (for callers that cannot allocate; see gdr2.h). `o` (and
    `final_state`, if wanted) must be preallocated; nothing is allocated here."""
    import torch
    dev = q.device
    if dev.type != "cuda":
        raise ValueError("chunk_fwd_noalloc needs CUDA tensors")
    B, T, H, dk = q.shape
    dv = v.shape[-1]
    dt = q.dtype
    code = _dtype_code(q)
    for name, t, d in (("k", k, dk), ("b", b, dk), ("v", v, dv), ("w", w, dv)):
        _check(t, name, (B, T, H, d), dt, dev)
    _check(q, "q", (B, T, H, dk), dt, dev)
    _check(log_alpha, "log_alpha", (B, T, H, dk), torch.float32, dev)
    if cu_seqlens is not None:
        if cu_seqlens.dtype != torch.int32 or cu_seqlens.device != dev or cu_seqlens.dim() != 1:
            raise ValueError("cu_seqlens must be a 1-D int32 tensor on the same device")
        N = cu_seqlens.shape[0] - 1
    else:
        N = B
    _check(o, "o", (B, T, H, dv), dt, dev)
    if init_state is not None:
        _check(init_state, "init_state", (N, H, dk, dv), torch.float32, dev)
    if final_state is not None:
        _check(final_state, "final_state", (N, H, dk, dv), torch.float32, dev)
    st = lib().gdr2_chunk_fwd_noalloc(
        _ptr(q), _ptr(k), _ptr(v), _ptr(log_alpha), _ptr(b), _ptr(w), _ptr(init_state),
        _ptr(cu_seqlens), B, T, H, dk, dv, N, code, _ptr(o), _ptr(final_state),
        _stream_handle(stream))
    if st != GDR2_OK:
        raise GDR2Error("gdr2_chunk_fwd_noalloc", st)
    return o, final_state


GDR2_QED_GATE = 1
GDR2_QED_PROJECT = 2


def qed_fwd(q, k, v, log_alpha, b, w, strength, direction=None,
            flags: int = GDR2_QED_GATE | GDR2_QED_PROJECT, init_state=None, cu_seqlens=None, *,
            o=None, final_state=None, output_final_state: bool = True,
            stream=None) -> Tuple["torch.Tensor", Optional["torch.Tensor"]]:
    """Forward with the QED second erase direction (gdr2_qed_fwd in gdr2.h; a
    reading of a page that does not print the update). Inputs and outputs as
    chunk_fwd, plus strength: fp32 [H] on the device, direction: fp32 [H, d_k]
    or None (the query), flags: GDR2_QED_* bits."""
    import torch
    dev = q.device
    if dev.type != "cuda":
        raise ValueError("qed_fwd needs CUDA tensors")
    B, T, H, dk = q.shape
    dv = v.shape[-1]
    dt = q.dtype
    code = _dtype_code(q)
    for name, t, d in (("k", k, dk), ("b", b, dk), ("v", v, dv), ("w", w, dv)):
        _check(t, name, (B, T, H, d), dt, dev)
    _check(q, "q", (B, T, H, dk), dt, dev)
    _check(log_alpha, "log_alpha", (B, T, H, dk), torch.float32, dev)
    _check(strength, "strength", (H,), torch.float32, dev)
    if direction is not None:
        _check(direction, "direction", (H, dk), torch.float32, dev)
    if cu_seqlens is not None:
        if cu_seqlens.dtype != torch.int32 or cu_seqlens.device != dev or cu_seqlens.dim() != 1:
            raise ValueError("cu_seqlens must be a 1-D int32 tensor on the same device")
        N = cu_seqlens.shape[0] - 1
    else:
        N = B
    if init_state is not None:
        _check(init_state, "init_state", (N, H, dk, dv), torch.float32, dev)
    if o is None:
        o = torch.empty((B, T, H, dv), dtype=dt, device=dev)
    else:
        _check(o, "o", (B, T, H, dv), dt, dev)
    if final_state is None and output_final_state:
        final_state = torch.empty((N, H, dk, dv), dtype=torch.float32, device=dev)
    elif final_state is not None:
        _check(final_state, "final_state", (N, H, dk, dv), torch.float32, dev)
    st = lib().gdr2_qed_fwd(
        _ptr(q), _ptr(k), _ptr(v), _ptr(log_alpha), _ptr(b), _ptr(w), _ptr(strength), _ptr(direction),
        int(flags), _ptr(init_state), _ptr(cu_seqlens), B, T, H, dk, dv, N, code, _ptr(o),
        _ptr(final_state), _stream_handle(stream))
    if st != GDR2_OK:
        raise GDR2Error("gdr2_qed_fwd", st)
    return o, final_state


def recurrent_step(q, k, v, log_alpha, b, w, state, *, o=None, prologue: int = 0, stream=None):
    """One decode step (see gdr2_recurrent_step in gdr2.h); state updated in place.

    q, k, b: [N, H, d_k]; v, w: [N, H, d_v] (bf16 or fp32, all alike);
    log_alpha: [N, H, d_k] fp32; state: [N, H, d_k, d_v] fp32. Returns o [N, H, d_v].
    prologue: GDR2_PROLOGUE_* flags (gdr2_recurrent_step_preact).
    """
    import torch
    dev = q.device
    if dev.type != "cuda":
        raise ValueError("recurrent_step needs CUDA tensors")
    N, H, dk = q.shape
    dv = v.shape[-1]
    dt = q.dtype
    code = _dtype_code(q)
    for name, t, d in (("k", k, dk), ("b", b, dk), ("v", v, dv), ("w", w, dv)):
        _check(t, name, (N, H, d), dt, dev)
    _check(log_alpha, "log_alpha", (N, H, dk), torch.float32, dev)
    _check(state, "state", (N, H, dk, dv), torch.float32, dev)
    if o is None:
        o = torch.empty((N, H, dv), dtype=dt, device=dev)
    else:
        _check(o, "o", (N, H, dv), dt, dev)
    if prologue:
        st = lib().gdr2_recurrent_step_preact(
            _ptr(q), _ptr(k), _ptr(v), _ptr(log_alpha), _ptr(b), _ptr(w), _ptr(state),
            N, H, dk, dv, code, _ptr(o), int(prologue), _stream_handle(stream))
        if st != GDR2_OK:
            raise GDR2Error("gdr2_recurrent_step_preact", st)
        return o
    st = lib().gdr2_recurrent_step(
        _ptr(q), _ptr(k), _ptr(v), _ptr(log_alpha), _ptr(b), _ptr(w), _ptr(state),
        N, H, dk, dv, code, _ptr(o), _stream_handle(stream))
    if st != GDR2_OK:
        raise GDR2Error("gdr2_recurrent_step", st)
    return o
