"""Failure detection on the device: a bounded on-chip wait that runs out.

The tensor-core kernels wait on mbarriers with a time limit; when a wait
gives up they record DSC_ERR_TIMEOUT in a device status word and return.
dsc_selftest_timeout launches one kernel whose barrier nothing completes
(the wait limit is a few milliseconds), so the path is exercised without a
fault or a hang: the status must reach the host through dsc_check, be
cleared by that read, and leave the context usable for the next call.
"""

import pytest
import torch

import oracle
from input_dependent_short_b200 import _lib, ops
from synth import workloads as wls

from helpers import TOL, rel_err, to_dev, to_host64

pytestmark = pytest.mark.gpu


def test_device_wait_timeout_is_reported_and_cleared():
    if not torch.cuda.is_available():
        pytest.fail("needs a CUDA device")
    L = _lib.lib()
    s = torch.cuda.current_stream().cuda_stream
    assert L.dsc_check(s) == _lib.DSC_OK
    n0 = L.dsc_launch_count()
    assert L.dsc_selftest_timeout(s) == _lib.DSC_OK
    assert L.dsc_launch_count() == n0 + 1
    assert L.dsc_check(s) == _lib.DSC_ERR_TIMEOUT
    assert L.dsc_check(s) == _lib.DSC_OK  # read and cleared
    # the context is still usable: a tensor-core low-rank forward after it is correct
    wl = wls.Workload("after-timeout", wls.LOWRANK, 1, 130, 256, 4, H=8, R=16, dtype="bf16")
    t = wls.make_inputs(wl)
    x, z, U = (to_dev(t[k], "bf16") for k in ("x", "z", "U"))
    y = ops.dsc_fwd_lowrank(x, z, U, H=wl.H)
    torch.cuda.synchronize()
    assert L.dsc_check(s) == _lib.DSC_OK
    ref = oracle.forward_lowrank(oracle.problem_of(wl), t["x"], t["z"], t["U"])
    assert rel_err(to_host64(y), ref) <= TOL["bf16"]
