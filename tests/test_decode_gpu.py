"""Parity of the decode step (one new token per sequence, rolling state of the
last W-1 inputs) with the fp64 oracle, through the C ABI.

* one step from a random state, every filter kind, both dtypes, the vector
  and the per-channel paths (D not a multiple of the vector width), W = 1..8:
  y within the tolerance, the shifted state bit-exact (it is a copy);
* many steps from a zero state, and steps after a prompt whose state comes
  from dsc_decode_state, against the oracle's training forward over the whole
  sequence (the oracle's decode is itself pinned to that forward);
* canary bands around y and the state.
"""

import numpy as np
import pytest
import torch

import oracle
import synth

from helpers import TOL, rel_err, to_dev, to_host64

pytestmark = pytest.mark.gpu

KINDS = {"headwise": oracle.HEADWISE, "lowrank": oracle.LOWRANK, "static": oracle.STATIC}


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.fail("no CUDA device: the -m gpu tests need a B200")
    import input_dependent_short_b200  # noqa: F401


def ops():
    from input_dependent_short_b200 import ops as o

    return o


def inputs(kind, B, T, D, W, H, R, dtype, seed=7):
    """Seeded storage-form tensors: x [B,T,D] and the filters of every token."""
    G = D // H
    t = {"x": synth.make_tensor(seed, 1, (B, T, D), 1.0, dtype)}
    if kind == "headwise":
        t["w"] = synth.make_tensor(seed, 2, (B, T, G, W), 1.0 / np.sqrt(W), dtype)
    elif kind == "lowrank":
        t["z"] = synth.make_tensor(seed, 3, (B, T, R), 1.0, dtype)
        t["U"] = synth.make_tensor(seed, 4, (R, G * W), 1.0 / np.sqrt(R * W), dtype)
    else:
        t["ws"] = synth.make_tensor(seed, 6, (D, W), 1.0 / np.sqrt(W), dtype)
    return t


def step(kind, x, t, tok, state, H, residual, dtype):
    """One GPU decode step at token `tok` of the stored inputs `t`."""
    o = ops()
    if kind == "headwise":
        return o.dsc_decode_headwise(x, to_dev(np.ascontiguousarray(t["w"][:, tok]), dtype), state, residual)
    if kind == "lowrank":
        return o.dsc_decode_lowrank(x, to_dev(np.ascontiguousarray(t["z"][:, tok]), dtype), to_dev(t["U"], dtype),
                                    state, H, residual)
    return o.dsc_decode_static(x, to_dev(t["ws"], dtype), state, residual)


def oracle_step(kind, x, t, tok, state, B, D, W, H, R, residual):
    P = oracle.problem(B, 1, D, W, H if kind != "static" else 1, R, residual)
    if kind == "headwise":
        return oracle.decode(P, KINDS[kind], x, state, w=np.ascontiguousarray(t["w"][:, tok]))
    if kind == "lowrank":
        return oracle.decode(P, KINDS[kind], x, state, z=np.ascontiguousarray(t["z"][:, tok]), U=t["U"])
    return oracle.decode(P, KINDS[kind], x, state, ws=t["ws"])


SHAPES = [
    # (B, D, W, H, R)
    (3, 64, 4, 16, 8),
    (2, 20, 3, 4, 5),       # D not a multiple of 8: per-channel path in bf16
    (4, 96, 1, 1, 16),      # W = 1: no state
    (1, 6144, 4, 16, 32),
    (5, 40, 8, 5, 3),
    (2, 256, 2, 256, 64),   # one group
    (17, 136, 5, 8, 24),
    (3, 30, 7, 3, 2),       # D not a multiple of 4 or 8
    (200, 4096, 4, 64, 64), # tiles too large for the tensor-core decode's shared memory: CUDA cores
    # bf16 low-rank on the tensor-core decode (tiles of 128 sequences, ragged last tile)
    (300, 512, 4, 1, 32),
    (129, 2048, 3, 2, 16),
    (64, 1024, 8, 1, 8),
    (200, 4096, 4, 64, 32),
    (5, 256, 1, 8, 16),
    (130, 1024, 2, 4, 24),
]

TC_DECODE = SHAPES[9:]


@pytest.mark.parametrize("dtype", ["bf16", "f32"])
@pytest.mark.parametrize("kind", ["headwise", "lowrank", "static"])
@pytest.mark.parametrize("shape", SHAPES, ids=lambda s: "B{}D{}W{}H{}R{}".format(*s))
def test_decode_step_matches_oracle(shape, kind, dtype):
    B, D, W, H, R = shape
    if kind == "lowrank" and dtype == "bf16" and shape in TC_DECODE:
        import ctypes as C

        from input_dependent_short_b200 import _lib

        p = _lib.DscProblem(B, 1, D, W, H, R, _lib.DSC_BF16, 1)
        assert _lib.lib().dsc_lowrank_kernels(C.byref(p), 2) == 0  # the tensor-core decode
    residual = 1 if kind != "static" else 0
    t = inputs(kind, B, 1, D, W, H, R, dtype)
    x0 = np.ascontiguousarray(t["x"][:, 0])
    st0 = synth.make_tensor(11, 5, (B, W - 1, D), 1.0, dtype)
    x = to_dev(x0, dtype)
    state = to_dev(st0, dtype) if W > 1 else None
    y = step(kind, x, t, 0, state, H, residual, dtype)
    torch.cuda.synchronize()
    y_ref, st_ref = oracle_step(kind, x0, t, 0, st0, B, D, W, H, R, residual)
    assert rel_err(to_host64(y), y_ref) <= TOL[dtype]
    if W > 1:
        assert np.array_equal(to_host64(state), st_ref)


@pytest.mark.parametrize("dtype", ["bf16", "f32"])
@pytest.mark.parametrize("kind", ["headwise", "lowrank", "static"])
@pytest.mark.parametrize("shape", [(2, 12, 64, 4, 16, 8), (3, 5, 24, 8, 2, 16), (1, 9, 4096, 3, 1, 32),
                                   (130, 6, 1024, 4, 1, 16)],
                         ids=lambda s: "B{}T{}D{}W{}H{}R{}".format(*s))
def test_decode_steps_and_prompt_match_forward(shape, kind, dtype):
    """A prompt of T0 tokens (its state from dsc_decode_state), then T - T0
    decode steps; and all T tokens decoded from a zero state.  Both agree with
    the oracle's training forward over the T tokens."""
    B, T, D, W, H, R = shape
    residual = 1 if kind != "static" else 0
    t = inputs(kind, B, T, D, W, H, R, dtype)
    Hk = H if kind != "static" else 1
    P = oracle.problem(B, T, D, W, Hk, R, residual)
    if kind == "headwise":
        y_ref = oracle.forward_headwise(P, t["x"], t["w"])
    elif kind == "lowrank":
        y_ref = oracle.forward_lowrank(P, t["x"], t["z"], t["U"])
    else:
        y_ref = oracle.forward_static(P, t["x"], t["ws"])
    o = ops()
    xd = to_dev(t["x"], dtype)
    for T0 in (0, T // 2):
        if T0 == 0:
            state = torch.zeros(B, W - 1, D, dtype=xd.dtype, device="cuda") if W > 1 else None
        else:
            state = o.dsc_decode_state(xd[:, :T0].contiguous(), W)
        ys = [step(kind, xd[:, tok].contiguous(), t, tok, state, H, residual, dtype) for tok in range(T0, T)]
        got = to_host64(torch.stack(ys, dim=1))
        assert rel_err(got, y_ref[:, T0:]) <= TOL[dtype], f"prompt of {T0} tokens"


@pytest.mark.parametrize("T", [1, 2, 6])
def test_decode_state_from_prompt_exact(T):
    """Rows before the prompt's start are zero; the rest copy the last inputs."""
    B, D, W = 3, 40, 4
    x0 = synth.make_tensor(3, 1, (B, T, D), 1.0, "bf16")
    st = ops().dsc_decode_state(to_dev(x0, "bf16"), W)
    torch.cuda.synchronize()
    xv = to_host64(to_dev(x0, "bf16"))
    expect = np.zeros((B, W - 1, D))
    for j in range(W - 1):
        if T - (W - 1) + j >= 0:
            expect[:, j] = xv[:, T - (W - 1) + j]
    assert np.array_equal(to_host64(st), expect)


def test_decode_outputs_do_not_touch_neighbouring_memory():
    """Canary bands around y and the state (per-channel path, ragged D)."""
    import ctypes as C

    from input_dependent_short_b200 import _lib

    B, D, W, H = 3, 20, 4, 4
    t = inputs("headwise", B, 1, D, W, H, 0, "bf16")
    x = to_dev(np.ascontiguousarray(t["x"][:, 0]), "bf16")
    w = to_dev(np.ascontiguousarray(t["w"][:, 0]), "bf16")
    pad = 4096
    buf_y = torch.full((B * D + 2 * pad,), 7.0, device="cuda", dtype=torch.bfloat16)
    buf_s = torch.full((B * (W - 1) * D + 2 * pad,), 7.0, device="cuda", dtype=torch.bfloat16)
    buf_s[pad:pad + B * (W - 1) * D] = 0.0
    p = _lib.DscProblem(B, 1, D, W, H, 0, _lib.DSC_BF16, 1)
    s = torch.cuda.current_stream().cuda_stream
    _lib.call("dsc_decode_headwise", p, x.data_ptr(), w.data_ptr(), buf_s[pad:].data_ptr(), buf_y[pad:].data_ptr(), s)
    torch.cuda.synchronize()
    for b, n in [(buf_y, B * D), (buf_s, B * (W - 1) * D)]:
        assert torch.all(b[:pad] == 7.0) and torch.all(b[pad + n:] == 7.0)
    assert torch.equal(buf_s[pad + B * (W - 1) * D - D:pad + B * (W - 1) * D].view(1, D), x[-1:].view(1, D))
