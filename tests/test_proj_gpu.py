"""The low-rank calls with the first projection (z = hV formed by the
library: dsc_fwd_lowrank_proj / dsc_bwd_lowrank_proj), through the C ABI,
against the fp64 oracle (oracle.forward_lowrank_proj / backward_lowrank_proj).
Shapes cover the tensor-core path (bf16, R a multiple of 8 up to 64 with and
without padding to 16, d_model a multiple of 128, ragged last token tile) and
the CUDA-core GEMMs (fp32, and d_model not a multiple of 128)."""

import pytest
import torch

import oracle
from synth import workloads as wls
from synth.workloads import LOWRANK, Workload

from helpers import assert_close, bound, to_dev, to_host64

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.fail("no CUDA device: the -m gpu tests need a B200")
    import input_dependent_short_b200  # noqa: F401


CASES = [
    # B, T, D, W, H, R, d_model, dtype
    (2, 300, 256, 4, 1, 32, 512, "bf16"),
    (1, 200, 2048, 4, 64, 64, 256, "bf16"),
    (2, 129, 1024, 3, 1, 8, 128, "bf16"),     # R = 8: rank padded to 16 in the MMA
    (1, 130, 512, 4, 16, 24, 384, "bf16"),    # R = 24: padded to 32; d_model not a multiple of 256
    (2, 256, 6144, 4, 1, 32, 2048, "bf16"),   # the Q/K/V widths (d_model 2048, D = 3 * 2048)
    (1, 70, 64, 4, 1, 8, 96, "f32"),          # CUDA-core GEMMs
    (1, 90, 256, 4, 2, 16, 200, "bf16"),      # d_model not a multiple of 128: CUDA-core GEMMs
]


@pytest.mark.parametrize("case", CASES, ids=lambda c: "B{}-T{}-D{}-W{}-H{}-R{}-d{}-{}".format(*c))
def test_projection_calls_match_oracle(case):
    from input_dependent_short_b200 import ops

    B, T, D, W, H, R, dm, dtype = case
    wl = Workload("proj", LOWRANK, B, T, D, W, H=H, R=R, dtype=dtype, seed=8)
    t = wls.make_inputs(wl)
    t.update(wls.projection_inputs(wl, dm))
    x, dy, U, h, V = (to_dev(t[k], dtype) for k in ("x", "dy", "U", "h", "V"))
    y, z = ops.dsc_fwd_lowrank_proj(x, h, V, U, H)
    dx, dh, dV, dU = ops.dsc_bwd_lowrank_proj(x, h, V, z, U, dy, H)
    torch.cuda.synchronize()
    P = oracle.problem_of(wl)
    ry, rz = oracle.forward_lowrank_proj(P, t["x"], t["h"], t["V"], t["U"])
    rdx, rdh, rdV, rdU, _ = oracle.backward_lowrank_proj(P, t["x"], t["h"], t["V"], t["U"], t["dy"])
    name = f"proj B{B} T{T} D{D} W{W} H{H} R{R} d{dm} {dtype}"
    assert_close(name + ":z", to_host64(z), rz, dtype, bound("y", dtype))
    assert_close(name + ":y", to_host64(y), ry, dtype, bound("y", dtype))
    assert_close(name + ":dx", to_host64(dx), rdx, dtype, bound("dx", dtype))
    assert_close(name + ":dh", to_host64(dh), rdh, dtype, bound("dz", dtype))
    assert_close(name + ":dV", to_host64(dV), rdV, dtype, bound("dU", dtype))
    assert_close(name + ":dU", to_host64(dU), rdU, dtype, bound("dU", dtype))
    ops.dsc_check()


def test_projection_z_equals_a_separate_projection_then_the_plain_call():
    """z from the projection call, fed to the plain low-rank calls, gives the
    projection calls' y and dx bit for bit (the same kernels on the same z)."""
    from input_dependent_short_b200 import ops

    wl = Workload("proj-eq", LOWRANK, 2, 300, 1024, 4, H=1, R=32, seed=9)
    t = wls.make_inputs(wl)
    t.update(wls.projection_inputs(wl, 256))
    x, dy, U, h, V = (to_dev(t[k], "bf16") for k in ("x", "dy", "U", "h", "V"))
    y, z = ops.dsc_fwd_lowrank_proj(x, h, V, U)
    assert torch.equal(y, ops.dsc_fwd_lowrank(x, z, U))
    dx, dh, dV, dU = ops.dsc_bwd_lowrank_proj(x, h, V, z, U, dy)
    dx2, dz2, dU2 = ops.dsc_bwd_lowrank(x, z, U, dy)
    assert torch.equal(dx, dx2) and torch.equal(dU, dU2)
    # dh = dz V^T and dV = h^T dz against torch's fp32 matmul on the dz of the
    # plain call.  On this shape the backward adds dz over channel blocks with
    # atomic fp32 adds, so the two calls' bf16 dz can differ by one rounding
    # in a few elements: hence the bounds (dh also carries its own bf16 output
    # rounding).
    ref_dh = dz2.float().reshape(-1, 32) @ V.float().t()
    err = (dh.float().reshape(-1, 256) - ref_dh).abs().max() / ref_dh.abs().max()
    assert err.item() < 8e-3
    ref_dV = h.float().reshape(-1, 256).t() @ dz2.float().reshape(-1, 32)
    err = (dV - ref_dV).abs().max() / ref_dV.abs().max()
    assert err.item() < 2e-3
