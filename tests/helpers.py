"""Shared helpers of the parity tests: device transfer and the error measure.

Error measure (per output tensor): max_i |gpu_i - ref_i| / max_i |ref_i|,
the normwise-max relative error.  Bounds: 1e-5 for fp32 inputs and 1.5e-2
for bf16 inputs with fp32 accumulation.
"""

import numpy as np

import synth

TOL = {"f32": 1e-5, "bf16": 1.5e-2}


def to_dev(arr, dtype, device="cuda"):
    return synth.to_torch(arr, dtype).to(device)


def to_host64(t):
    import torch

    return t.detach().to(torch.float64).cpu().numpy()


def rel_err(got, ref):
    got = np.asarray(got, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    scale = np.max(np.abs(ref)) if ref.size else 0.0
    if scale == 0.0:
        return float(np.max(np.abs(got))) if got.size else 0.0
    return float(np.max(np.abs(got - ref)) / scale)


def assert_close(name, got, ref, dtype):
    e = rel_err(got, ref)
    assert e <= TOL[dtype], f"{name}: normwise relative error {e:.3e} > {TOL[dtype]:.1e}"
    return e
