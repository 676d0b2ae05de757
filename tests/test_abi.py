"""The C-ABI library loads, exports what include/gdr2.h declares, and rejects
bad arguments on the host before any launch (no GPU needed)."""
import ctypes
import os
import re

import pytest

import linear_attention_recurrence_gdr2_b200 as gdr2

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADERS = [os.path.join(ROOT, "include", f) for f in os.listdir(os.path.join(ROOT, "include"))
           if f.endswith(".h")]

OK, INVALID, UNSUPPORTED, WORKSPACE = 0, 1, 2, 3
FAKE = 0x10000  # 16-byte aligned, never dereferenced: validation fails first


def declared_functions():
    names = set()
    for h in HEADERS:
        src = open(h).read()
        src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
        for m in re.finditer(r"^[A-Za-z_][\w \*]*?\b(gdr2_\w+)\s*\(", src, flags=re.M):
            names.add(m.group(1))
    return sorted(names)


def test_header_declares_the_boundary():
    names = declared_functions()
    for fn in ("gdr2_chunk_fwd", "gdr2_recurrent_step", "gdr2_chunk_fwd_workspace_size",
               "gdr2_status_string", "gdr2_version"):
        assert fn in names


@pytest.mark.parametrize("name", declared_functions())
def test_library_exports_declared_symbol(name):
    lib = ctypes.CDLL(gdr2.LIB_PATH)
    assert hasattr(lib, name), f"{name} declared in include/ but not exported"


def test_status_strings_and_version():
    assert gdr2.status_string(0) == "ok"
    for s in range(1, 6):
        assert gdr2.status_string(s) not in ("ok", "unknown status")
    assert gdr2.status_string(99) == "unknown status"
    assert gdr2.version() >= 100


def test_workspace_size_query():
    assert gdr2.workspace_size(4, 2048, 16, 128, 128, 4, gdr2.GDR2_BF16) >= 0
    with pytest.raises(gdr2.GDR2Error) as e:
        gdr2.workspace_size(4, 2048, 16, 96, 96, 4, gdr2.GDR2_BF16)
    assert e.value.status == UNSUPPORTED
    with pytest.raises(gdr2.GDR2Error) as e:
        gdr2.workspace_size(4, 2048, 0, 128, 128, 4, gdr2.GDR2_BF16)
    assert e.value.status == INVALID


def _chunk(**over):
    a = dict(q=FAKE, k=FAKE, v=FAKE, la=FAKE, b=FAKE, w=FAKE, s0=None, cu=None,
             B=2, T=128, H=4, dk=128, dv=128, N=2, dtype=1, o=FAKE, sf=FAKE,
             ws=None, wsb=0, stream=None)
    a.update(over)
    return gdr2.lib().gdr2_chunk_fwd(a["q"], a["k"], a["v"], a["la"], a["b"], a["w"], a["s0"],
                                     a["cu"], a["B"], a["T"], a["H"], a["dk"], a["dv"], a["N"],
                                     a["dtype"], a["o"], a["sf"], a["ws"], a["wsb"], a["stream"])


@pytest.mark.parametrize("over,expect", [
    (dict(q=None), INVALID),
    (dict(o=None), INVALID),
    (dict(la=FAKE + 4), INVALID),          # misaligned
    (dict(v=FAKE + 2), INVALID),
    (dict(H=0), INVALID),
    (dict(T=-1), INVALID),
    (dict(dtype=7), INVALID),
    (dict(N=3), INVALID),                  # num_seqs != B without cu_seqlens
    (dict(cu=FAKE, B=2), INVALID),         # packed batch needs B == 1
    (dict(dk=96, dv=96), UNSUPPORTED),
    (dict(dk=128, dv=64), UNSUPPORTED),
    (dict(dk=0, dv=128), INVALID),
    (dict(s0=FAKE + 8), INVALID),
    (dict(sf=FAKE + 8), INVALID),
    (dict(H=70000), UNSUPPORTED),
])
def test_chunk_fwd_rejects_bad_arguments(over, expect):
    assert _chunk(**over) == expect


def _step(**over):
    a = dict(q=FAKE, k=FAKE, v=FAKE, la=FAKE, b=FAKE, w=FAKE, s=FAKE, N=4, H=2, dk=64, dv=64,
             dtype=0, o=FAKE, stream=None)
    a.update(over)
    return gdr2.lib().gdr2_recurrent_step(a["q"], a["k"], a["v"], a["la"], a["b"], a["w"],
                                          a["s"], a["N"], a["H"], a["dk"], a["dv"], a["dtype"],
                                          a["o"], a["stream"])


@pytest.mark.parametrize("over,expect", [
    (dict(s=None), INVALID),
    (dict(k=FAKE + 1), INVALID),
    (dict(N=-1), INVALID),
    (dict(H=0), INVALID),
    (dict(dtype=3), INVALID),
    (dict(dk=32, dv=32), UNSUPPORTED),
])
def test_recurrent_step_rejects_bad_arguments(over, expect):
    assert _step(**over) == expect


def test_packed_batch_needs_workspace():
    need = gdr2.workspace_size(1, 1000, 4, 128, 128, 3, gdr2.GDR2_BF16)
    assert need >= 3 * 4 and need % 256 == 0
    # fixed-length batches need none; many (sequence, head) units get no split
    assert gdr2.workspace_size(4, 2048, 16, 128, 128, 4, gdr2.GDR2_BF16) == 0
    assert gdr2.workspace_size(2, 1000, 4, 128, 128, 2, gdr2.GDR2_FP32) == 0
    assert _chunk(B=1, N=3, cu=FAKE) == WORKSPACE
    assert _chunk(B=1, N=3, cu=FAKE, ws=FAKE, wsb=need - 1) == WORKSPACE
    assert _chunk(B=1, N=3, cu=FAKE, ws=FAKE + 8, wsb=need) == INVALID  # misaligned workspace


def test_segment_split_workspace():
    """Few long bf16 sequences report room for the segment-parallel scan: o-sized
    psi (bf16) plus two [N][segments][H][128][128] fp32 state arrays."""
    B, T, H = 1, 32768, 16
    need = gdr2.workspace_size(B, T, H, 128, 128, B, gdr2.GDR2_BF16)
    psi = B * T * H * 128 * 2
    assert need >= psi + 2 * 2 * B * H * 128 * 128 * 4  # at least two segments
    assert need % 256 == 0
    # no split for d = 64, fp32, or sequences too short for two 8-chunk segments
    assert gdr2.workspace_size(B, T, H, 64, 64, B, gdr2.GDR2_BF16) == 0
    assert gdr2.workspace_size(B, T, H, 128, 128, B, gdr2.GDR2_FP32) == 0
    assert gdr2.workspace_size(1, 64 * 15, 1, 128, 128, 1, gdr2.GDR2_BF16) == 0
    assert gdr2.workspace_size(1, 64 * 16, 1, 128, 128, 1, gdr2.GDR2_BF16) > 0


def test_empty_problems_return_ok_without_launch():
    assert _chunk(B=0, N=0, q=None, o=None) == OK
    assert _chunk(B=1, T=0, N=0, cu=FAKE) == OK
    assert _step(N=0, q=None, s=None) == OK


def test_prologue_flags_validated():
    """The *_preact entry points reject unknown prologue bits before anything else."""
    L = gdr2.lib()
    assert L.gdr2_chunk_fwd_preact(*([None] * 8), 1, 64, 1, 64, 64, 1, 0, None, None, None, 0, 8,
                                   None) == INVALID
    assert L.gdr2_recurrent_step_preact(*([None] * 7), 1, 1, 64, 64, 0, None, 8, None) == INVALID
    # known bits pass the flag check and reach the usual validation (null pointers)
    assert L.gdr2_chunk_fwd_preact(*([None] * 8), 1, 64, 1, 64, 64, 1, 0, None, None, None, 0, 7,
                                   None) == INVALID
    assert gdr2.GDR2_PROLOGUE_ALL == 7


def _bwd(**over):
    a = dict(q=FAKE, k=FAKE, v=FAKE, la=FAKE, b=FAKE, w=FAKE, s0=None, cu=None, do=FAKE, dsf=None,
             B=2, T=128, H=4, dk=64, dv=64, N=2, dtype=0, dq=FAKE, dkk=FAKE, dvv=FAKE, dla=FAKE,
             db=FAKE, dw=FAKE, ds0=None, ws=None, wsb=0, stream=None)
    a.update(over)
    return gdr2.lib().gdr2_chunk_bwd(
        a["q"], a["k"], a["v"], a["la"], a["b"], a["w"], a["s0"], a["cu"], a["do"], a["dsf"],
        a["B"], a["T"], a["H"], a["dk"], a["dv"], a["N"], a["dtype"], a["dq"], a["dkk"], a["dvv"],
        a["dla"], a["db"], a["dw"], a["ds0"], a["ws"], a["wsb"], a["stream"])


def test_bwd_workspace_size():
    """Two fp32 checkpoint arrays of (tokens/64 + N) slots and two per-token fp32 vectors."""
    for B, T, H, d, N, cu in ((4, 2048, 16, 128, 4, False), (1, 1000, 3, 64, 5, True),
                              (2, 1, 1, 64, 2, False), (1, 0, 2, 128, 3, True)):
        need = gdr2.bwd_workspace_size(B, T, H, d, d, N, gdr2.GDR2_BF16)
        slots = (B * T) // 64 + N
        expect = 2 * slots * H * d * d * 4 + 2 * B * T * H * d * 4
        assert need % 256 == 0 and expect <= need < expect + 256
    with pytest.raises(gdr2.GDR2Error) as e:
        gdr2.bwd_workspace_size(1, 64, 1, 96, 96, 1, gdr2.GDR2_FP32)
    assert e.value.status == UNSUPPORTED


@pytest.mark.parametrize("over,expect", [
    (dict(do=None), INVALID),
    (dict(dla=None), INVALID),
    (dict(dw=FAKE + 4), INVALID),
    (dict(dsf=FAKE + 8), INVALID),
    (dict(ds0=FAKE + 8), INVALID),
    (dict(H=0), INVALID),
    (dict(N=3), INVALID),
    (dict(cu=FAKE, B=2), INVALID),
    (dict(dtype=5), INVALID),
    (dict(dk=128, dv=64), UNSUPPORTED),
    ({}, WORKSPACE),                        # the workspace is required
    (dict(ws=FAKE, wsb=1024), WORKSPACE),
    (dict(ws=FAKE + 8, wsb=1 << 30), INVALID),
    (dict(B=0, N=0, q=None, dq=None), OK),  # nothing to do
])
def test_chunk_bwd_rejects_bad_arguments(over, expect):
    assert _bwd(**over) == expect


def _qed(**over):
    a = dict(q=FAKE, k=FAKE, v=FAKE, la=FAKE, b=FAKE, w=FAKE, lam=FAKE, dirs=None, flags=3, s0=None,
             cu=None, B=2, T=64, H=4, dk=64, dv=64, N=2, dtype=0, o=FAKE, sf=None, stream=None)
    a.update(over)
    return gdr2.lib().gdr2_qed_fwd(a["q"], a["k"], a["v"], a["la"], a["b"], a["w"], a["lam"], a["dirs"],
                                    a["flags"], a["s0"], a["cu"], a["B"], a["T"], a["H"], a["dk"], a["dv"],
                                    a["N"], a["dtype"], a["o"], a["sf"], a["stream"])


def test_qed_arguments_validated_on_the_host():
    assert _qed(flags=4) == INVALID           # unknown flag bit
    assert _qed(lam=None) == INVALID          # the strength is required
    assert _qed(lam=FAKE + 2) == INVALID      # misaligned fp32 array
    assert _qed(dirs=FAKE + 1) == INVALID
    assert _qed(q=None) == INVALID
    assert _qed(o=FAKE + 8) == INVALID        # token tensors 16-byte aligned
    assert _qed(dk=96, dv=96) == UNSUPPORTED
    assert _qed(dk=64, dv=128) == UNSUPPORTED
    assert _qed(N=3) == INVALID               # num_seqs must equal B without cu_seqlens
    assert _qed(cu=FAKE, B=2) == INVALID      # packed batches have B = 1
    assert _qed(dtype=7) == INVALID
    assert _qed(B=0, N=0, q=None, o=None) == OK
