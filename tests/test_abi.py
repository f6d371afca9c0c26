"""The C ABI on a machine without a GPU: the library loads, exports every
entry point include/dsc.h declares, and rejects bad arguments before any CUDA
call (so these checks make no compute call)."""

import ctypes as C
import os
import re
import subprocess

import pytest

from input_dependent_short_b200 import _lib

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADERS = [os.path.join(ROOT, "include", f) for f in os.listdir(os.path.join(ROOT, "include")) if f.endswith(".h")]


def declared():
    names = set()
    for h in HEADERS:
        src = open(h).read()
        names |= set(re.findall(r"DSC_API\s+[\w\s\*]+?\b(dsc_\w+)\s*\(", src))
    return names


def test_header_declares_the_entry_points():
    d = declared()
    for n in ["dsc_fwd_headwise", "dsc_bwd_headwise", "dsc_fwd_lowrank", "dsc_bwd_lowrank", "dsc_fwd_static",
              "dsc_bwd_static", "dsc_check", "dsc_status_string"]:
        assert n in d


def test_library_exports_every_declared_symbol():
    L = _lib.lib()
    out = subprocess.run(["nm", "-D", "--defined-only", _lib.LIB_PATH], capture_output=True, text=True, check=True).stdout
    exported = {l.split()[-1] for l in out.splitlines() if " T " in l}
    for n in declared():
        assert n in exported, n
        assert getattr(L, n) is not None
    # nothing but the declared C ABI is exported
    assert {e for e in exported if e.startswith("dsc_")} == declared()


def test_every_binding_signature_is_declared():
    assert set(_lib._SIGS) == declared()


def test_version_and_status_strings():
    assert _lib.lib().dsc_version() >= 100
    assert _lib.status_string(_lib.DSC_OK) == "ok"
    assert "aligned" in _lib.status_string(_lib.DSC_ERR_MISALIGNED)
    assert "timed out" in _lib.status_string(_lib.DSC_ERR_TIMEOUT)
    assert _lib.status_string(99) == "unknown status"


def P(B=1, T=8, D=16, W=4, H=1, R=0, dtype=1, residual=1):
    return _lib.DscProblem(B, T, D, W, H, R, dtype, residual)


GOOD = 0x10000  # a 16-byte aligned, never dereferenced address


@pytest.mark.parametrize("bad", [dict(B=0), dict(T=0), dict(D=0), dict(W=0), dict(W=9), dict(H=0), dict(D=10, H=4),
                                 dict(dtype=7)])
def test_invalid_problem_rejected(bad):
    L = _lib.lib()
    p = P(**bad)
    assert L.dsc_fwd_headwise(C.byref(p), GOOD, GOOD, GOOD, None) == _lib.DSC_ERR_INVALID_ARG
    assert L.dsc_bwd_headwise(C.byref(p), GOOD, GOOD, GOOD, GOOD, GOOD, None) == _lib.DSC_ERR_INVALID_ARG
    assert L.dsc_fwd_static(C.byref(p), GOOD, GOOD, GOOD, None) == _lib.DSC_ERR_INVALID_ARG
    assert L.dsc_bwd_static_workspace_bytes(C.byref(p)) == 0


@pytest.mark.parametrize("R", [0, 257])
def test_invalid_rank_rejected(R):
    L = _lib.lib()
    p = P(R=R)
    assert L.dsc_fwd_lowrank(C.byref(p), GOOD, GOOD, GOOD, GOOD, None, 0, None) == _lib.DSC_ERR_INVALID_ARG
    assert L.dsc_bwd_lowrank(C.byref(p), GOOD, GOOD, GOOD, GOOD, GOOD, GOOD, GOOD, None, 0, None) == _lib.DSC_ERR_INVALID_ARG
    assert L.dsc_fwd_lowrank_workspace_bytes(C.byref(p)) == 0


def test_null_problem_and_pointers_rejected():
    L = _lib.lib()
    assert L.dsc_fwd_headwise(None, GOOD, GOOD, GOOD, None) == _lib.DSC_ERR_INVALID_ARG
    p = P()
    assert L.dsc_fwd_headwise(C.byref(p), None, GOOD, GOOD, None) == _lib.DSC_ERR_INVALID_ARG
    assert L.dsc_bwd_headwise(C.byref(p), GOOD, GOOD, GOOD, GOOD, None, None) == _lib.DSC_ERR_INVALID_ARG
    assert L.dsc_bwd_static(C.byref(p), GOOD, GOOD, GOOD, GOOD, GOOD, None, 0, None) == _lib.DSC_ERR_INVALID_ARG


def test_misaligned_pointers_rejected():
    L = _lib.lib()
    p = P()
    assert L.dsc_fwd_headwise(C.byref(p), GOOD + 2, GOOD, GOOD, None) == _lib.DSC_ERR_MISALIGNED
    assert L.dsc_fwd_static(C.byref(p), GOOD, GOOD, GOOD + 8, None) == _lib.DSC_ERR_MISALIGNED
    p.R = 4
    assert L.dsc_fwd_lowrank(C.byref(p), GOOD, GOOD + 4, GOOD, GOOD, None, 0, None) == _lib.DSC_ERR_MISALIGNED


def test_binding_rejects_cpu_tensors():
    import torch

    from input_dependent_short_b200 import ops

    x = torch.zeros(1, 4, 8, dtype=torch.bfloat16)
    w = torch.zeros(1, 4, 8, 4, dtype=torch.bfloat16)
    with pytest.raises(ValueError):
        ops.dsc_fwd_headwise(x, w)


# (B, T, D, W, H, R) -> kernel family of the bf16 forward and backward
# (0 tensor cores, 1 fused on CUDA cores); the plan runs on the host.
KERNEL_CHOICE = [
    ((8, 2048, 6144, 4, 1, 32), 0, 0),      # Q/K/V low-rank workload
    ((4, 4096, 8192, 4, 64, 64), 0, 0),     # all-linear low-rank workload
    ((1, 16384, 4096, 3, 1, 16), 0, 0),     # W = 3: 32-group blocks, 96 filter columns
    ((1, 16384, 4096, 3, 1, 64), 0, 0),
    ((2, 500, 4096, 3, 64, 64), 0, 0),
    ((1, 200, 2048, 2, 64, 32), 0, 0),      # block narrowed to 32 groups so that it divides D
    ((1, 16384, 4096, 2, 1, 64), 0, 0),     # backward with one dw tile
    ((1, 16384, 4096, 8, 1, 16), 0, 0),     # W = 8, H = 1: 16-channel blocks and sub-tiles
    ((1, 16384, 4096, 8, 1, 64), 0, 0),
    ((2, 100, 4096, 5, 2, 16), 0, 0),       # W = 5 .. 7: 16-group blocks
    ((2, 100, 4096, 7, 1, 32), 0, 0),
    ((2, 100, 4096, 6, 16, 64), 0, 0),
    ((2, 100, 4096, 6, 64, 64), 0, 1),      # W >= 5, H = 64, R = 64: the backward's tiles overflow shared memory
    ((2, 100, 4096, 4, 1, 5), 1, 1),        # R not a multiple of 8
    ((2, 100, 4096, 4, 1, 72), 1, 1),       # R above 64
]


@pytest.mark.parametrize("shape,fwd,bwd", KERNEL_CHOICE, ids=lambda v: str(v))
def test_lowrank_kernel_choice(shape, fwd, bwd):
    L = _lib.lib()
    p = P(*shape, dtype=1)
    assert L.dsc_lowrank_kernels(C.byref(p), 0) == fwd
    assert L.dsc_lowrank_kernels(C.byref(p), 1) == bwd
    p32 = P(*shape, dtype=0)
    assert L.dsc_lowrank_kernels(C.byref(p32), 0) == 1
    assert L.dsc_lowrank_kernels(C.byref(p32), 1) == 1
    bad = P(*shape[:5], R=0)
    assert L.dsc_lowrank_kernels(C.byref(bad), 0) == -1


def test_decode_argument_checks():
    """Decode calls take one token per sequence and reject bad arguments
    before any CUDA call."""
    L = _lib.lib()
    p2 = P(T=2)
    assert L.dsc_decode_headwise(C.byref(p2), GOOD, GOOD, GOOD, GOOD, None) == _lib.DSC_ERR_INVALID_ARG
    assert L.dsc_decode_static(C.byref(p2), GOOD, GOOD, GOOD, GOOD, None) == _lib.DSC_ERR_INVALID_ARG
    p = P(T=1)
    assert L.dsc_decode_headwise(C.byref(p), GOOD, GOOD, None, GOOD, None) == _lib.DSC_ERR_INVALID_ARG  # W > 1: state
    assert L.dsc_decode_headwise(C.byref(p), GOOD, GOOD, GOOD + 8, GOOD, None) == _lib.DSC_ERR_MISALIGNED
    fused = P(B=3, T=1, D=16, W=4, H=2, R=4)  # filters formed in registers: no scratch
    assert L.dsc_decode_lowrank_workspace_bytes(C.byref(fused)) == 0
    lr = P(B=3, T=1, D=18, W=4, H=3, R=4)  # D not a multiple of 8: the token's filters through a scratch
    assert L.dsc_decode_lowrank_workspace_bytes(C.byref(lr)) == 3 * 6 * 4 * 4
    assert L.dsc_decode_lowrank(C.byref(lr), GOOD, GOOD, GOOD, GOOD, GOOD, GOOD, 16, None) == _lib.DSC_ERR_INVALID_ARG
    assert L.dsc_decode_lowrank(C.byref(lr), GOOD, GOOD, GOOD, GOOD, GOOD, None, 0, None) == _lib.DSC_ERR_INVALID_ARG
    assert L.dsc_decode_lowrank_workspace_bytes(C.byref(P(T=2, R=4))) == 0
    assert L.dsc_decode_state(C.byref(P(T=5)), None, GOOD, None) == _lib.DSC_ERR_INVALID_ARG
    # decode kernel family: tensor cores for the Q/K/V decode shape, CUDA cores in fp32, a scratch for ragged D
    assert L.dsc_lowrank_kernels(C.byref(P(B=2048, T=1, D=6144, W=4, H=1, R=32)), 2) == 0
    assert L.dsc_lowrank_kernels(C.byref(P(B=2048, T=1, D=6144, W=4, H=1, R=32, dtype=0)), 2) == 1
    assert L.dsc_lowrank_kernels(C.byref(P(B=3, T=1, D=18, W=4, H=3, R=4)), 2) == 2
    assert L.dsc_lowrank_kernels(C.byref(P(B=3, T=2, D=64, W=4, H=1, R=8)), 2) == -1


def test_noalloc_backward_reports_the_regular_backwards_argument_errors():
    """dsc_bwd_static_noalloc returns the same status codes as dsc_bwd_static
    for rejected arguments, before touching any device state: an unsupported
    length (T > 2^30), an invalid shape, a NULL or misaligned pointer."""
    L = _lib.lib()

    def both(p, ptrs):
        a = L.dsc_bwd_static(C.byref(p) if p is not None else None, *ptrs, GOOD, 1 << 40, None)
        b = L.dsc_bwd_static_noalloc(C.byref(p) if p is not None else None, *ptrs, None)
        return a, b

    good = [GOOD] * 5
    assert both(P(T=(1 << 30) + 1), good) == (_lib.DSC_ERR_UNSUPPORTED, _lib.DSC_ERR_UNSUPPORTED)
    assert both(P(B=(1 << 30) + 1), good) == (_lib.DSC_ERR_UNSUPPORTED, _lib.DSC_ERR_UNSUPPORTED)
    assert both(P(W=9), good) == (_lib.DSC_ERR_INVALID_ARG, _lib.DSC_ERR_INVALID_ARG)
    assert both(None, good) == (_lib.DSC_ERR_INVALID_ARG, _lib.DSC_ERR_INVALID_ARG)
    assert both(P(), [GOOD, GOOD, None, GOOD, GOOD]) == (_lib.DSC_ERR_INVALID_ARG, _lib.DSC_ERR_INVALID_ARG)
    assert both(P(), [GOOD, GOOD, GOOD, GOOD + 4, GOOD]) == (_lib.DSC_ERR_MISALIGNED, _lib.DSC_ERR_MISALIGNED)
