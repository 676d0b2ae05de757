"""Operand precision a tensor-core backward needs (CPU emulation): the chunk
form with every matrix-product operand truncated to tf32 and fp32 accumulation
stays within the bf16-input bound (5e-3) on every gradient, with room left for
the bf16 rounding of the outputs. (With bf16 operands instead, the decay and
erase-gate gradients reach about 6.7e-3 and 5.1e-3, over the bound: run
`python tests/chunk_bwd_form.py` for the table.)"""
from chunk_bwd_form import bf16, operand_precision_errors, tf32


def test_tf32_operands_stay_within_the_bf16_bound():
    errs = operand_precision_errors(T=256, rnd=tf32)
    assert max(errs.values()) < 4e-3, errs


def test_bf16_operands_leave_no_margin_on_the_gate_gradients():
    errs = operand_precision_errors(T=256, rnd=bf16)
    assert max(errs["dlog_alpha"], errs["db"]) > 4e-3, errs
