"""The product path has no CPU fallback: every entry point of the binding
refuses host tensors loudly instead of computing anything on the CPU, and a
missing library raises instead of degrading (no GPU needed)."""
import importlib

import pytest
import torch

import linear_attention_recurrence_gdr2_b200 as gdr2


def host_inputs(B=1, T=8, H=1, d=64):
    z = lambda *s: torch.zeros(*s, dtype=torch.float32)
    return dict(q=z(B, T, H, d), k=z(B, T, H, d), v=z(B, T, H, d), log_alpha=z(B, T, H, d),
                b=z(B, T, H, d), w=z(B, T, H, d))


def test_chunk_fwd_refuses_host_tensors():
    x = host_inputs()
    with pytest.raises(ValueError, match="CUDA"):
        gdr2.chunk_fwd(x["q"], x["k"], x["v"], x["log_alpha"], x["b"], x["w"])


def test_chunk_bwd_refuses_host_tensors():
    x = host_inputs()
    with pytest.raises(ValueError, match="CUDA"):
        gdr2.chunk_bwd(x["q"], x["k"], x["v"], x["log_alpha"], x["b"], x["w"], x["v"])


def test_chunk_fwd_noalloc_refuses_host_tensors():
    x = host_inputs()
    with pytest.raises(ValueError, match="CUDA"):
        gdr2.chunk_fwd_noalloc(x["q"], x["k"], x["v"], x["log_alpha"], x["b"], x["w"],
                               o=torch.zeros_like(x["v"]))


def test_recurrent_step_refuses_host_tensors():
    z = lambda *s: torch.zeros(*s, dtype=torch.float32)
    q = z(2, 1, 64)
    with pytest.raises(ValueError, match="CUDA"):
        gdr2.recurrent_step(q, q, q, q, q, q, z(2, 1, 64, 64))


def test_missing_library_raises(monkeypatch, tmp_path):
    """With the shared library absent, loading it raises a RuntimeError that
    says how to build it."""
    m = importlib.reload(gdr2)
    try:
        monkeypatch.setattr(m, "LIB_PATH", str(tmp_path / "libgdr2.so"))
        monkeypatch.setattr(m, "_lib", None)
        with pytest.raises(RuntimeError, match="build"):
            m.lib()
    finally:
        importlib.reload(gdr2)
