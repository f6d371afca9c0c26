"""Parity past 2^31 elements: one row of T = 262400 tokens x D = 8192
channels (2,149,580,800 elements per activation tensor, 4.3 GB in bf16), so
that every offset beyond element 2^31 must be formed in 64-bit arithmetic.

The inputs are seeded normals drawn on the device (torch's generator); the
oracle receives the same values, copied back as bf16 bits.  Each sampled
output is checked against the fp64 oracle run on a crop of the inputs that
holds everything the output depends on: tokens t-(W-1) .. t+(W-1) (the
causal taps of y and dw, the later filters and dy of dx), clipped to the
sequence, and the channels of the sampled channel's filter group (all
channels for dz, which sums over them).  Cropping is exact: the definition
("Dynamic Short Convolutions Improve Transformers", technical summary,
Methodology, "Mechanism") reads nothing further away, and a crop that
starts at token 0 or ends at token T keeps the sequence's zero padding.
"""

import numpy as np
import pytest

import oracle
from helpers import assert_close

pytestmark = pytest.mark.gpu

B, T, D, W = 1, 262400, 8192, 4
assert B * T * D > 2 ** 31


def _bits(t):
    """bf16 device tensor -> host uint16 bits (the oracle's bf16 input form)."""
    import torch

    return t.contiguous().view(torch.int16).cpu().numpy().view(np.uint16)


def _samples(n, seed):
    rng = np.random.default_rng(seed)
    t = rng.integers(T - 4096, T, n)  # element offsets past 2^31
    c = rng.integers(0, D, n)
    t[:6] = [T - 1, T - 1, T - 2, T - W, (2 ** 31) // D, (2 ** 31) // D + 1]
    c[:6] = [D - 1, 0, D // 2, 1, (2 ** 31) % D, 0]
    return t, c


def _crop(t):
    return max(0, t - (W - 1)), min(T, t + W)


def _device_inputs(kind, H=1, R=0):
    import torch

    g = torch.Generator(device="cuda").manual_seed(20260)
    x = torch.randn(B, T, D, device="cuda", generator=g, dtype=torch.float32).to(torch.bfloat16)
    dy = torch.randn(B, T, D, device="cuda", generator=g, dtype=torch.float32).to(torch.bfloat16)
    f = {}
    if kind == oracle.HEADWISE:
        f["w"] = (torch.randn(B, T, D // H, W, device="cuda", generator=g) / W ** 0.5).to(torch.bfloat16)
    elif kind == oracle.STATIC:
        f["ws"] = (torch.randn(D, W, device="cuda", generator=g) / W ** 0.5).to(torch.bfloat16)
    else:
        f["z"] = torch.randn(B, T, R, device="cuda", generator=g).to(torch.bfloat16)
        f["U"] = (torch.randn(R, (D // H) * W, device="cuda", generator=g) / (R * W) ** 0.5).to(torch.bfloat16)
    return x, dy, f


def _free():
    import gc

    import torch

    gc.collect()
    torch.cuda.empty_cache()


@pytest.fixture(autouse=True)
def _needs_memory():
    import torch

    if torch.cuda.get_device_properties(0).total_memory < 40 * 2 ** 30:
        pytest.skip("needs about 30 GB of device memory")
    yield
    _free()


def test_headwise_past_2_31_elements():
    from input_dependent_short_b200 import ops

    H = 64
    x, dy, f = _device_inputs(oracle.HEADWISE, H=H)
    y = ops.dsc_fwd_headwise(x, f["w"])
    dx, dw = ops.dsc_bwd_headwise(x, f["w"], dy)
    ts, cs = _samples(48, 1)
    got = {"y": [], "dx": [], "dw": []}
    ref = {"y": [], "dx": [], "dw": []}
    for t, c in zip(ts, cs):
        s0, e0 = _crop(int(t))
        g = int(c) // H
        c0 = g * H
        P = oracle.problem(1, e0 - s0, H, W, H, 0, 1)
        kw = dict(x=_bits(x[:, s0:e0, c0:c0 + H]), dy=_bits(dy[:, s0:e0, c0:c0 + H]),
                  w=_bits(f["w"][:, s0:e0, g:g + 1, :]))
        k = int(t) % W
        for name, what, idx, gv in (("y", oracle.Y, [0, t - s0, c - c0], y[0, t, c]),
                                    ("dx", oracle.DX, [0, t - s0, c - c0], dx[0, t, c]),
                                    ("dw", oracle.DW, [0, t - s0, 0, k], dw[0, t, g, k])):
            ref[name].append(oracle.sample(P, oracle.HEADWISE, what, np.array([idx]), **kw)[0])
            got[name].append(float(gv))
    for name in got:
        assert_close(f"past-2^31 head-wise:{name}", np.array(got[name]), np.array(ref[name]), "bf16")


def test_static_past_2_31_elements():
    from input_dependent_short_b200 import ops

    x, dy, f = _device_inputs(oracle.STATIC)
    y = ops.dsc_fwd_static(x, f["ws"])
    dx, _ = ops.dsc_bwd_static(x, f["ws"], dy)
    ts, cs = _samples(48, 2)
    got = {"y": [], "dx": []}
    ref = {"y": [], "dx": []}
    for t, c in zip(ts, cs):
        s0, e0 = _crop(int(t))
        P = oracle.problem(1, e0 - s0, 1, W, 1, 0, 0)  # the static calls' default: no residual
        kw = dict(x=_bits(x[:, s0:e0, c:c + 1]), dy=_bits(dy[:, s0:e0, c:c + 1]), w=_bits(f["ws"][c:c + 1]))
        for name, what, gv in (("y", oracle.Y, y[0, t, c]), ("dx", oracle.DX, dx[0, t, c])):
            ref[name].append(oracle.sample(P, oracle.STATIC, what, np.array([[0, t - s0, 0]]), **kw)[0])
            got[name].append(float(gv))
    for name in got:
        assert_close(f"past-2^31 static:{name}", np.array(got[name]), np.array(ref[name]), "bf16")


def test_lowrank_past_2_31_elements():
    from input_dependent_short_b200 import ops

    H, R = 1, 16
    x, dy, f = _device_inputs(oracle.LOWRANK, H=H, R=R)
    y = ops.dsc_fwd_lowrank(x, f["z"], f["U"], H)
    dx, dz, _ = ops.dsc_bwd_lowrank(x, f["z"], f["U"], dy, H)
    ts, cs = _samples(32, 3)
    Ub = _bits(f["U"])
    got = {"y": [], "dx": [], "dz": []}
    ref = {"y": [], "dx": [], "dz": []}
    for i, (t, c) in enumerate(zip(ts, cs)):
        s0, e0 = _crop(int(t))
        zw = _bits(f["z"][:, s0:e0, :])
        # y and dx of channel c need its own filter columns only
        P1 = oracle.problem(1, e0 - s0, 1, W, 1, R, 1)
        kw1 = dict(x=_bits(x[:, s0:e0, c:c + 1]), dy=_bits(dy[:, s0:e0, c:c + 1]), z=zw,
                   U=np.ascontiguousarray(Ub[:, c * W:(c + 1) * W]))
        for name, what, gv in (("y", oracle.Y, y[0, t, c]), ("dx", oracle.DX, dx[0, t, c])):
            ref[name].append(oracle.sample(P1, oracle.LOWRANK, what, np.array([[0, t - s0, 0]]), **kw1)[0])
            got[name].append(float(gv))
        if i < 8:  # dz sums over every channel: crop the tokens only
            r = int(c) % R
            PD = oracle.problem(1, e0 - s0, D, W, 1, R, 1)
            kwd = dict(x=_bits(x[:, s0:e0, :]), dy=_bits(dy[:, s0:e0, :]), z=zw, U=Ub)
            ref["dz"].append(oracle.sample(PD, oracle.LOWRANK, oracle.DZ, np.array([[0, t - s0, r]]), **kwd)[0])
            got["dz"].append(float(dz[0, t, r]))
    for name in got:
        assert_close(f"past-2^31 low-rank:{name}", np.array(got[name]), np.array(ref[name]), "bf16")
