"""dsc_bwd_static_noalloc: the static-filter backward for callers that cannot
allocate device memory or pass a workspace (plugin interfaces that hand an
operator only its inputs and outputs; services that must not call cudaMalloc
after start-up).  Its scratch is an array built into the library.

Checked through the C ABI against the regular dsc_bwd_static on two calls in
a row with different inputs (the shared array keeps the previous call's
contents, which must not leak into the next result), for the vectorised and
the generic kernel paths: the two run the same deterministic kernels, so the
results must be equal bit for bit.  The size limit is checked to be enforced
before anything is launched.  This file is collected last on purpose.
"""

import ctypes as C

import pytest
import torch

from input_dependent_short_b200 import _lib
from synth import workloads as wls

from helpers import to_dev

pytestmark = pytest.mark.gpu

LIMIT = 16 << 20  # DSC_NOALLOC_SCRATCH_BYTES


def _problem(wl):
    return _lib.DscProblem(wl.B, wl.T, wl.D, wl.W, 1, 0, _lib.DSC_BF16 if wl.dtype == "bf16" else _lib.DSC_F32,
                           wl.residual)


def _inputs(wl):
    t = wls.make_inputs(wl)
    return {k: to_dev(v, wl.dtype) for k, v in t.items()}


def _regular(wl, p, d):
    L = _lib.lib()
    dx = torch.empty_like(d["x"])
    dws = torch.empty(d["ws"].shape, dtype=torch.float32, device="cuda")
    n = L.dsc_bwd_static_workspace_bytes(C.byref(p))
    scratch = torch.empty(n, dtype=torch.uint8, device="cuda")
    s = torch.cuda.current_stream().cuda_stream
    _lib.call("dsc_bwd_static", p, d["x"].data_ptr(), d["ws"].data_ptr(), d["dy"].data_ptr(), dx.data_ptr(),
              dws.data_ptr(), scratch.data_ptr(), n, s)
    torch.cuda.synchronize()
    return dx, dws


def _noalloc(p, d):
    dx = torch.empty_like(d["x"])
    dws = torch.empty(d["ws"].shape, dtype=torch.float32, device="cuda")
    s = torch.cuda.current_stream().cuda_stream
    _lib.call("dsc_bwd_static_noalloc", p, d["x"].data_ptr(), d["ws"].data_ptr(), d["dy"].data_ptr(),
              dx.data_ptr(), dws.data_ptr(), s)
    torch.cuda.synchronize()
    return dx, dws


@pytest.mark.parametrize("shape", [
    ("bf16", 2, 1000, 1024, 4),   # vectorised kernels
    ("f32", 1, 300, 20, 3),       # generic kernels (D not a multiple of the vector)
])
def test_noalloc_matches_regular_backward_twice(shape):
    if not torch.cuda.is_available():
        pytest.fail("needs a CUDA device")
    dtype, B, T, D, W = shape
    L = _lib.lib()
    for seed in (11, 12):  # two calls in a row, different inputs
        wl = wls.Workload("noalloc", wls.STATIC, B, T, D, W, dtype=dtype, residual=1, seed=seed)
        p = _problem(wl)
        assert 0 < L.dsc_bwd_static_workspace_bytes(C.byref(p)) <= LIMIT
        d = _inputs(wl)
        dx_ref, dws_ref = _regular(wl, p, d)
        dx, dws = _noalloc(p, d)
        # The same deterministic kernels with a fixed-order reduction of the
        # same partials: the results are identical bit for bit.  Stale
        # contents of the shared array would show as any difference at all.
        assert torch.equal(dx, dx_ref)
        assert torch.equal(dws, dws_ref)


def test_noalloc_rejects_problems_beyond_its_scratch():
    if not torch.cuda.is_available():
        pytest.fail("needs a CUDA device")
    L = _lib.lib()
    # 128 one-tile sequences of 8192 channels at W = 8: 128 partials of 256 KiB.
    wl = wls.Workload("too-big", wls.STATIC, 128, 32, 8192, 8, dtype="bf16")
    p = _problem(wl)
    assert L.dsc_bwd_static_workspace_bytes(C.byref(p)) > LIMIT  # rejected before any launch
    x = torch.zeros(wl.B, wl.T, wl.D, dtype=torch.bfloat16, device="cuda")
    ws = torch.zeros(wl.D, wl.W, dtype=torch.bfloat16, device="cuda")
    dx = torch.empty_like(x)
    dws = torch.empty(wl.D, wl.W, dtype=torch.float32, device="cuda")
    st = L.dsc_bwd_static_noalloc(C.byref(p), x.data_ptr(), ws.data_ptr(), x.data_ptr(), dx.data_ptr(),
                                  dws.data_ptr(), torch.cuda.current_stream().cuda_stream)
    assert st == _lib.DSC_ERR_UNSUPPORTED
