"""Pins of the fp64 oracle to things other than itself.

Each check below would catch a plausible slip in the oracle (a dropped term,
a wrong sign, a wrong tap/lag index, a transposed operand, a wrong channel to
group mapping):

* hand-worked values (tests/golden/handworked.json);
* the convolution written as a banded T x T matrix per (batch, channel):
  y = (rI + A) x, hence dx = (rI + A)^T dy by linear algebra;
* exact central differences of L = <dy, y>, which is linear in each of x, w,
  z and U separately, so the difference quotient is exact up to rounding;
* the static filter against torch.nn.functional.conv1d (a library routine)
  and its autograd gradients in fp64;
* the equivalences between the parameterisations (head-wise H vs per-channel,
  constant-in-time vs static, full-rank identity U vs head-wise);
* special cases (zero filter, delta filter, W = 1, T = 1, T < W).
"""

import itertools
import json
import os

import numpy as np
import pytest
import torch

import oracle

HERE = os.path.dirname(os.path.abspath(__file__))
RNG = np.random.default_rng(1234)


def rand(*shape):
    return RNG.standard_normal(shape)


def P(B, T, D, W, H=1, R=0, residual=1):
    return oracle.problem(B, T, D, W, H, R, residual)


def banded(wch, T, W):
    """A[t, t-k] = wch[t, k] for one (batch, channel): the causal conv as a matrix."""
    A = np.zeros((T, T))
    for t in range(T):
        for k in range(W):
            if t - k >= 0:
                A[t, t - k] = wch[t, k]
    return A


# ---------------------------------------------------------------- golden ---

def _golden_cases():
    with open(os.path.join(HERE, "golden", "handworked.json")) as f:
        return json.load(f)["cases"]


@pytest.mark.parametrize("case", _golden_cases(), ids=lambda c: c["name"])
def test_handworked_golden(case):
    c = case
    p = P(c["B"], c["T"], c["D"], c["W"], c["H"], c["R"], c["residual"])
    x = np.array(c["x"], dtype=np.float64)
    dy = np.array(c["dy"], dtype=np.float64)
    if c["variant"] == "headwise":
        w = np.array(c["w"], dtype=np.float64)
        np.testing.assert_array_equal(oracle.forward_headwise(p, x, w), c["y"])
        dx, dw = oracle.backward_headwise(p, x, w, dy)
        np.testing.assert_array_equal(dx, c["dx"])
        np.testing.assert_array_equal(dw, c["dw"])
    elif c["variant"] == "lowrank":
        z = np.array(c["z"], dtype=np.float64)
        U = np.array(c["U"], dtype=np.float64)
        np.testing.assert_array_equal(oracle.forward_lowrank(p, x, z, U), c["y"])
        dx, dz, dU, _ = oracle.backward_lowrank(p, x, z, U, dy)
        np.testing.assert_array_equal(dx, c["dx"])
        np.testing.assert_array_equal(dz, c["dz"])
        np.testing.assert_array_equal(dU, c["dU"])
    else:
        ws = np.array(c["ws"], dtype=np.float64)
        np.testing.assert_array_equal(oracle.forward_static(p, x, ws), c["y"])
        dx, dws = oracle.backward_static(p, x, ws, dy)
        np.testing.assert_array_equal(dx, c["dx"])
        np.testing.assert_array_equal(dws, c["dws"])


# ----------------------------------------------------------- matrix form ---

def _shapes():
    out = []
    for T, D, W in [(1, 1, 1), (1, 3, 4), (2, 4, 3), (3, 2, 5), (5, 6, 2), (9, 4, 4), (16, 8, 3), (7, 6, 5)]:
        for H in [h for h in range(1, D + 1) if D % h == 0]:
            out.append((T, D, W, H))
    return out


@pytest.mark.parametrize("T,D,W,H", _shapes())
@pytest.mark.parametrize("residual", [0, 1])
def test_matrix_form_headwise(T, D, W, H, residual):
    B, G = 2, D // H
    p = P(B, T, D, W, H, 0, residual)
    x, w, dy = rand(B, T, D), rand(B, T, G, W), rand(B, T, D)
    y = oracle.forward_headwise(p, x, w)
    dx, _ = oracle.backward_headwise(p, x, w, dy)
    for b, c in itertools.product(range(B), range(D)):
        M = residual * np.eye(T) + banded(w[b, :, c // H, :], T, W)
        np.testing.assert_allclose(y[b, :, c], M @ x[b, :, c], rtol=0, atol=1e-12)
        np.testing.assert_allclose(dx[b, :, c], M.T @ dy[b, :, c], rtol=0, atol=1e-12)


# -------------------------------------------- exact central differences ---

def _loss_grad_check(f, arg, grad, eps=0.5, n_probe=None):
    """f is linear in `arg`: (f(a+eps e) - f(a-eps e)) / 2eps = grad . e exactly."""
    flat = arg.reshape(-1)
    gflat = grad.reshape(-1)
    idx = range(flat.size) if n_probe is None else RNG.choice(flat.size, n_probe, replace=False)
    for i in idx:
        old = flat[i]
        flat[i] = old + eps
        lp = f()
        flat[i] = old - eps
        lm = f()
        flat[i] = old
        assert abs((lp - lm) / (2 * eps) - gflat[i]) <= 1e-9 * (1 + abs(gflat[i])), i


@pytest.mark.parametrize("T,D,W,H", [(6, 4, 3, 2), (5, 6, 4, 3), (3, 2, 5, 1), (8, 8, 2, 8)])
def test_fd_headwise(T, D, W, H):
    B = 2
    p = P(B, T, D, W, H)
    x, w, dy = rand(B, T, D), rand(B, T, D // H, W), rand(B, T, D)
    dx, dw = oracle.backward_headwise(p, x, w, dy)
    f = lambda: float(np.sum(dy * oracle.forward_headwise(p, x, w)))
    _loss_grad_check(f, x, dx)
    _loss_grad_check(f, w, dw)


@pytest.mark.parametrize("T,D,W,H,R", [(6, 4, 3, 2, 3), (5, 6, 4, 1, 2), (4, 8, 2, 4, 5), (3, 3, 4, 3, 1)])
def test_fd_lowrank(T, D, W, H, R):
    B = 2
    p = P(B, T, D, W, H, R)
    x, z, U, dy = rand(B, T, D), rand(B, T, R), rand(R, (D // H) * W), rand(B, T, D)
    dx, dz, dU, _ = oracle.backward_lowrank(p, x, z, U, dy)
    f = lambda: float(np.sum(dy * oracle.forward_lowrank(p, x, z, U)))
    _loss_grad_check(f, x, dx)
    _loss_grad_check(f, z, dz)
    _loss_grad_check(f, U, dU)


def test_adjoint_dw():
    """<dy, conv(x; v)> = <dw(x, dy), v> for a random filter direction v."""
    B, T, D, W, H = 3, 11, 12, 4, 3
    p0 = P(B, T, D, W, H, 0, residual=0)
    p1 = P(B, T, D, W, H, 0, residual=1)
    x, dy, w = rand(B, T, D), rand(B, T, D), rand(B, T, D // H, W)
    _, dw = oracle.backward_headwise(p1, x, w, dy)
    for _ in range(5):
        v = rand(B, T, D // H, W)
        lhs = np.sum(dy * oracle.forward_headwise(p0, x, v))
        assert abs(lhs - np.sum(dw * v)) < 1e-10 * (1 + abs(lhs))


# ------------------------------------------ static filter vs torch conv1d ---

@pytest.mark.parametrize("T,D,W,residual", [(1, 3, 4, 1), (3, 5, 4, 0), (17, 8, 4, 1), (9, 6, 2, 1), (12, 4, 8, 0), (6, 2, 1, 1)])
def test_static_vs_torch_conv1d(T, D, W, residual):
    B = 2
    p = P(B, T, D, W, 1, 0, residual)
    x, ws, dy = rand(B, T, D), rand(D, W), rand(B, T, D)
    y = oracle.forward_static(p, x, ws)
    dx, dws = oracle.backward_static(p, x, ws, dy)

    xt = torch.tensor(x, requires_grad=True)
    wt = torch.tensor(ws, requires_grad=True)
    # conv1d is a cross-correlation: reversed taps make weight[..., W-1-k] hit x_{t-k}.
    ref = torch.nn.functional.conv1d(xt.transpose(1, 2), wt.flip(-1)[:, None, :], groups=D, padding=W - 1)
    ref = ref[..., :T].transpose(1, 2) + residual * xt
    ref.backward(torch.tensor(dy))
    np.testing.assert_allclose(y, ref.detach().numpy(), rtol=0, atol=1e-12)
    np.testing.assert_allclose(dx, xt.grad.numpy(), rtol=0, atol=1e-12)
    np.testing.assert_allclose(dws, wt.grad.numpy(), rtol=0, atol=1e-11)


# ------------------------------------------------------- equivalences ---

@pytest.mark.parametrize("H", [1, 2, 3, 6])
def test_constant_filters_equal_static(H):
    B, T, D, W = 2, 10, 6, 4
    G = D // H
    p = P(B, T, D, W, H)
    wg = rand(G, W)
    w = np.broadcast_to(wg, (B, T, G, W)).copy()
    ws = np.repeat(wg, H, axis=0)  # channel c uses group c // H
    x, dy = rand(B, T, D), rand(B, T, D)
    np.testing.assert_allclose(oracle.forward_headwise(p, x, w), oracle.forward_static(P(B, T, D, W), x, ws), atol=1e-12)
    dx_h, dw_h = oracle.backward_headwise(p, x, w, dy)
    dx_s, dws = oracle.backward_static(P(B, T, D, W), x, ws, dy)
    np.testing.assert_allclose(dx_h, dx_s, atol=1e-12)
    np.testing.assert_allclose(dw_h.sum(axis=(0, 1)), dws.reshape(G, H, W).sum(axis=1), atol=1e-10)


@pytest.mark.parametrize("D,H", [(6, 2), (6, 3), (8, 4), (4, 4)])
def test_headwise_equals_replicated_per_channel(D, H):
    B, T, W = 2, 9, 3
    G = D // H
    x, dy, w = rand(B, T, D), rand(B, T, D), rand(B, T, G, W)
    w1 = np.repeat(w, H, axis=2)  # per-channel filters: channel c takes group c // H
    pH, p1 = P(B, T, D, W, H), P(B, T, D, W, 1)
    np.testing.assert_allclose(oracle.forward_headwise(pH, x, w), oracle.forward_headwise(p1, x, w1), atol=1e-12)
    dxH, dwH = oracle.backward_headwise(pH, x, w, dy)
    dx1, dw1 = oracle.backward_headwise(p1, x, w1, dy)
    np.testing.assert_allclose(dxH, dx1, atol=1e-12)
    np.testing.assert_allclose(dwH, dw1.reshape(B, T, G, H, W).sum(axis=3), atol=1e-12)


@pytest.mark.parametrize("D,H,W", [(4, 1, 3), (6, 2, 2), (6, 3, 4)])
def test_lowrank_full_rank_identity_equals_headwise(D, H, W):
    B, T = 2, 7
    G = D // H
    R = G * W
    w = rand(B, T, G, W)
    z = w.reshape(B, T, R).copy()
    U = np.eye(R)
    x, dy = rand(B, T, D), rand(B, T, D)
    p = P(B, T, D, W, H, R)
    np.testing.assert_allclose(oracle.lowrank_filters(p, z, U), w, atol=1e-14)
    np.testing.assert_allclose(oracle.forward_lowrank(p, x, z, U), oracle.forward_headwise(p, x, w), atol=1e-12)
    dx, dz, dU, dwl = oracle.backward_lowrank(p, x, z, U, dy)
    dxh, dwh = oracle.backward_headwise(p, x, w, dy)
    np.testing.assert_allclose(dx, dxh, atol=1e-12)
    np.testing.assert_allclose(dz, dwh.reshape(B, T, R), atol=1e-12)
    # with U = I, dU[r, j] = sum over tokens of w[., r] * dw[., j]
    np.testing.assert_allclose(dU, np.einsum("nr,nj->rj", w.reshape(-1, R), dwh.reshape(-1, R)), atol=1e-10)


# ---------------------------------------------------------- special cases ---

def test_zero_filter_is_identity():
    B, T, D, W, H = 2, 8, 6, 4, 2
    p = P(B, T, D, W, H)
    x, dy = rand(B, T, D), rand(B, T, D)
    w = np.zeros((B, T, D // H, W))
    np.testing.assert_array_equal(oracle.forward_headwise(p, x, w), x)
    np.testing.assert_array_equal(oracle.backward_headwise(p, x, w, dy)[0], dy)


@pytest.mark.parametrize("j", [0, 1, 3])
def test_delta_filter_shifts(j):
    B, T, D, W = 1, 9, 3, 4
    p = P(B, T, D, W, 1)
    x = rand(B, T, D)
    w = np.zeros((B, T, D, W))
    w[..., j] = 1.0
    shifted = np.zeros_like(x)
    shifted[:, j:] = x[:, :T - j]
    np.testing.assert_allclose(oracle.forward_headwise(p, x, w), x + shifted, atol=1e-15)


def test_width_one_is_scaling():
    B, T, D = 2, 5, 4
    p = P(B, T, D, 1, 1)
    x, w, dy = rand(B, T, D), rand(B, T, D, 1), rand(B, T, D)
    np.testing.assert_allclose(oracle.forward_headwise(p, x, w), (1 + w[..., 0]) * x, atol=1e-14)
    dx, dw = oracle.backward_headwise(p, x, w, dy)
    np.testing.assert_allclose(dx, (1 + w[..., 0]) * dy, atol=1e-14)
    np.testing.assert_allclose(dw[..., 0], dy * x, atol=1e-14)


@pytest.mark.parametrize("T", [1, 2])
def test_short_sequences_only_reach_back_to_zero(T):
    B, D, W = 2, 4, 5
    p = P(B, T, D, W, 2)
    x, w, dy = rand(B, T, D), rand(B, T, 2, W), rand(B, T, D)
    y = oracle.forward_headwise(p, x, w)
    wc = np.repeat(w, 2, axis=2)
    np.testing.assert_allclose(y[:, 0], x[:, 0] * (1 + wc[:, 0, :, 0]), atol=1e-14)
    _, dw = oracle.backward_headwise(p, x, w, dy)
    for t in range(T):
        assert np.all(dw[:, t, :, t + 1:] == 0)


def test_batches_are_independent():
    B, T, D, W, H = 3, 6, 4, 3, 2
    p = P(B, T, D, W, H)
    x, w, dy = rand(B, T, D), rand(B, T, D // H, W), rand(B, T, D)
    y = oracle.forward_headwise(p, x, w)
    for b in range(B):
        yb = oracle.forward_headwise(P(1, T, D, W, H), x[b:b + 1].copy(), w[b:b + 1].copy())
        np.testing.assert_array_equal(y[b:b + 1], yb)


# ------------------------------------------ storage dtypes and sampling ---

def test_bf16_and_f32_inputs_read_exactly():
    import synth

    B, T, D, W, H = 1, 6, 8, 4, 2
    p = P(B, T, D, W, H)
    x32 = rand(B, T, D).astype(np.float32)
    w32 = rand(B, T, D // H, W).astype(np.float32)
    xb, wb = synth.f32_to_bf16_bits(x32), synth.f32_to_bf16_bits(w32)
    ref = oracle.forward_headwise(p, synth.to_f64(xb, "bf16"), synth.to_f64(wb, "bf16"))
    np.testing.assert_array_equal(oracle.forward_headwise(p, xb, wb), ref)
    np.testing.assert_array_equal(oracle.forward_headwise(p, x32, w32),
                                  oracle.forward_headwise(p, x32.astype(np.float64), w32.astype(np.float64)))


def test_sample_matches_full():
    B, T, D, W, H, R = 2, 7, 6, 3, 2, 4
    p = P(B, T, D, W, H, R)
    x, z, U, dy = rand(B, T, D), rand(B, T, R), rand(R, (D // H) * W), rand(B, T, D)
    y = oracle.forward_lowrank(p, x, z, U)
    dx, dz, dU, dw = oracle.backward_lowrank(p, x, z, U, dy)
    wf = oracle.lowrank_filters(p, z, U)
    kw = dict(x=x, dy=dy, z=z, U=U)
    bt = np.array(list(itertools.product(range(B), range(T))))
    pts = np.array([(b, t, c) for b, t in bt for c in range(D)])
    np.testing.assert_allclose(oracle.sample(p, oracle.LOWRANK, oracle.Y, pts, **kw), y.reshape(-1), atol=1e-12)
    np.testing.assert_allclose(oracle.sample(p, oracle.LOWRANK, oracle.DX, pts, **kw), dx.reshape(-1), atol=1e-12)
    pg = np.array([(b, t, g, k) for b, t in bt for g in range(D // H) for k in range(W)])
    np.testing.assert_allclose(oracle.sample(p, oracle.LOWRANK, oracle.DW, pg, **kw), dw.reshape(-1), atol=1e-12)
    np.testing.assert_allclose(oracle.sample(p, oracle.LOWRANK, oracle.W_TAP, pg, **kw), wf.reshape(-1), atol=1e-12)
    pr = np.array([(b, t, r) for b, t in bt for r in range(R)])
    np.testing.assert_allclose(oracle.sample(p, oracle.LOWRANK, oracle.DZ, pr, **kw), dz.reshape(-1), atol=1e-12)
    pu = np.array([(r, g, k) for r in range(R) for g in range(D // H) for k in range(W)])
    np.testing.assert_allclose(oracle.sample(p, oracle.LOWRANK, oracle.DU, pu, **kw), dU.reshape(-1), atol=1e-11)
    ws = rand(D, W)
    _, dws = oracle.backward_static(p, x, ws, dy)
    pc = np.array([(c, k) for c in range(D) for k in range(W)])
    np.testing.assert_allclose(oracle.sample(p, oracle.STATIC, oracle.DWS, pc, x=x, dy=dy, w=ws), dws.reshape(-1), atol=1e-11)


# ---------------------------------------------------------------- decode ---

DECODE_CASES = [
    (oracle.HEADWISE, 7, 12, 4, 3, 0, 1),
    (oracle.HEADWISE, 2, 8, 4, 1, 0, 0),   # T < W: the state still holds zero rows
    (oracle.HEADWISE, 5, 6, 1, 2, 0, 1),   # W = 1: no state
    (oracle.LOWRANK, 6, 8, 3, 2, 5, 1),
    (oracle.LOWRANK, 9, 16, 8, 4, 3, 0),
    (oracle.STATIC, 6, 5, 4, 1, 0, 1),
    (oracle.STATIC, 3, 4, 8, 1, 0, 0),
]


@pytest.mark.parametrize("kind,T,D,W,H,R,residual", DECODE_CASES)
def test_decode_steps_equal_forward(kind, T, D, W, H, R, residual):
    """T decode steps from a zero state reproduce the (pinned) forward over the
    T tokens token by token, and the final state holds the last W-1 inputs
    (zero rows for positions before the start)."""
    B, G = 2, D // H
    x = rand(B, T, D)
    Pf = P(B, T, D, W, H, R, residual)
    if kind == oracle.HEADWISE:
        w = rand(B, T, G, W)
        yref = oracle.forward_headwise(Pf, x, w)
        filt = lambda t: dict(w=np.ascontiguousarray(w[:, t]))
    elif kind == oracle.LOWRANK:
        z, U = rand(B, T, R), rand(R, G * W)
        yref = oracle.forward_lowrank(Pf, x, z, U)
        filt = lambda t: dict(z=np.ascontiguousarray(z[:, t]), U=U)
    else:
        ws = rand(D, W)
        yref = oracle.forward_static(Pf, x, ws)
        filt = lambda t: dict(ws=ws)
    Pd = P(B, 1, D, W, H, R, residual)
    state = np.zeros((B, W - 1, D))
    for t in range(T):
        y, state = oracle.decode(Pd, kind, np.ascontiguousarray(x[:, t]), state, **filt(t))
        np.testing.assert_allclose(y, yref[:, t], rtol=0, atol=1e-12)
    expect = np.zeros((B, W - 1, D))
    for j in range(W - 1):
        if T - (W - 1) + j >= 0:
            expect[:, j] = x[:, T - (W - 1) + j]
    assert np.array_equal(state, expect)


@pytest.mark.parametrize("j", [0, 1, 3])
def test_decode_delta_filter_reads_the_right_state_row(j):
    """w_k = delta(k, j): y = x + x_{t-j}, x_{t-j} being state row W-1-j (j >= 1)."""
    B, D, W = 2, 5, 4
    x, state = rand(B, D), rand(B, W - 1, D)
    w = np.zeros((B, D, W))
    w[:, :, j] = 1.0
    y, st = oracle.decode(P(B, 1, D, W, 1, 0, 1), oracle.HEADWISE, x, state, w=w)
    np.testing.assert_array_equal(y, x + (x if j == 0 else state[:, W - 1 - j]))
    np.testing.assert_array_equal(st[:, :-1], state[:, 1:])
    np.testing.assert_array_equal(st[:, -1], x)


# ------------------------------------------------- variable-length (packed) ---

VARLEN_CASES = [
    # (kind, document lengths, D, W, H, R, residual)
    (oracle.HEADWISE, (5, 1, 7, 3), 6, 4, 2, 0, 1),
    (oracle.HEADWISE, (2, 9), 4, 3, 1, 0, 0),
    (oracle.LOWRANK, (4, 6, 2), 8, 3, 4, 3, 1),
    (oracle.STATIC, (3, 3, 5), 5, 4, 1, 0, 1),
    (oracle.STATIC, (1, 1, 1, 6), 3, 8, 1, 0, 0),
]


def _varlen_inputs(kind, T, D, W, H, R):
    G = D // H
    f = {}
    if kind == oracle.HEADWISE:
        f["w"] = rand(1, T, G, W)
    elif kind == oracle.LOWRANK:
        f["z"], f["U"] = rand(1, T, R), rand(R, G * W)
    else:
        f["ws"] = rand(D, W)
    return rand(1, T, D), rand(1, T, D), f


def _plain(kind, P_, x, dy, f):
    """The (pinned) oracle on one sequence: (y, gradients)."""
    if kind == oracle.HEADWISE:
        return oracle.forward_headwise(P_, x, f["w"]), oracle.backward_headwise(P_, x, f["w"], dy)
    if kind == oracle.LOWRANK:
        return oracle.forward_lowrank(P_, x, f["z"], f["U"]), oracle.backward_lowrank(P_, x, f["z"], f["U"], dy)
    return oracle.forward_static(P_, x, f["ws"]), oracle.backward_static(P_, x, f["ws"], dy)


@pytest.mark.parametrize("kind,lens,D,W,H,R,residual", VARLEN_CASES)
def test_varlen_equals_documents_run_separately(kind, lens, D, W, H, R, residual):
    """Packed documents give, token by token, what each document gives as a
    sequence of its own; the token reductions (static dws, low-rank dU) are the
    sums over the documents."""
    T = sum(lens)
    cu = np.concatenate([[0], np.cumsum(lens)])
    x, dy, f = _varlen_inputs(kind, T, D, W, H, R)
    Pp = P(1, T, D, W, H, R, residual)
    y = oracle.forward_varlen(Pp, kind, x, cu, **f)
    g = oracle.backward_varlen(Pp, kind, x, dy, cu, **f)
    total = None
    for d in range(len(lens)):
        sl = slice(cu[d], cu[d + 1])
        fd = {k: (np.ascontiguousarray(v[:, sl]) if k in ("w", "z") else v) for k, v in f.items()}
        yd, gd = _plain(kind, P(1, lens[d], D, W, H, R, residual), np.ascontiguousarray(x[:, sl]),
                        np.ascontiguousarray(dy[:, sl]), fd)
        np.testing.assert_allclose(y[:, sl], yd, rtol=0, atol=1e-12)
        np.testing.assert_allclose(g[0][:, sl], gd[0], rtol=0, atol=1e-12)  # dx
        if kind == oracle.HEADWISE:
            np.testing.assert_allclose(g[1][:, sl], gd[1], rtol=0, atol=1e-12)  # dw
        elif kind == oracle.LOWRANK:
            np.testing.assert_allclose(g[1][:, sl], gd[1], rtol=0, atol=1e-12)  # dz
            total = gd[2] if total is None else total + gd[2]
        else:
            total = gd[1] if total is None else total + gd[1]
    if kind == oracle.LOWRANK:
        np.testing.assert_allclose(g[2], total, rtol=0, atol=1e-11)  # dU
    elif kind == oracle.STATIC:
        np.testing.assert_allclose(g[1], total, rtol=0, atol=1e-11)  # dws


@pytest.mark.parametrize("kind", [oracle.HEADWISE, oracle.LOWRANK, oracle.STATIC])
def test_varlen_empty_documents_change_nothing(kind):
    """A document of no tokens (equal consecutive offsets: at the start, twice
    in a row inside, at the end) has no outputs and no taps, so the packed
    result is the one without it, exactly; and each non-empty document is
    still the plain op on its own tokens."""
    lens = (3, 1, 5, 4)
    T, D, W, H, R = sum(lens), 6, 4, 3, 2
    x, dy, f = _varlen_inputs(kind, T, D, W, H, R)
    Pp = P(1, T, D, W, H, R, 1)
    cu = np.concatenate([[0], np.cumsum(lens)])
    cu_e = np.array([0, 0, 3, 4, 4, 4, 9, 13, 13])
    np.testing.assert_array_equal(oracle.forward_varlen(Pp, kind, x, cu_e, **f), oracle.forward_varlen(Pp, kind, x, cu, **f))
    for a, b in zip(oracle.backward_varlen(Pp, kind, x, dy, cu_e, **f), oracle.backward_varlen(Pp, kind, x, dy, cu, **f)):
        np.testing.assert_array_equal(a, b)
    yd, _ = _plain(kind, P(1, 5, D, W, H, R, 1), np.ascontiguousarray(x[:, 4:9]), np.ascontiguousarray(dy[:, 4:9]),
                   {k: (np.ascontiguousarray(v[:, 4:9]) if k in ("w", "z") else v) for k, v in f.items()})
    np.testing.assert_allclose(oracle.forward_varlen(Pp, kind, x, cu_e, **f)[:, 4:9], yd, rtol=0, atol=1e-12)


@pytest.mark.parametrize("kind", [oracle.HEADWISE, oracle.LOWRANK, oracle.STATIC])
def test_varlen_one_document_is_the_plain_op(kind):
    T, D, W, H, R = 9, 6, 4, 3, 2
    x, dy, f = _varlen_inputs(kind, T, D, W, H, R)
    Pp = P(1, T, D, W, H, R, 1)
    y, g = _plain(kind, Pp, x, dy, f)
    np.testing.assert_array_equal(oracle.forward_varlen(Pp, kind, x, [0, T], **f), y)
    for a, b in zip(oracle.backward_varlen(Pp, kind, x, dy, [0, T], **f), g):
        np.testing.assert_array_equal(a, b)


# ------------------------------------------------- sequence chunks (halos) ---
# Context parallelism splits each sequence along time; a chunk's result needs
# the W-1 inputs before it (x_prev) and, in the backward, dy and the filters
# of the W-1 tokens after it.  Pinned against the whole-sequence oracle: the
# chunks, each with its neighbours' rows as halos, give the whole sequence's
# outputs row for row, and their token reductions sum to its dU / dws.

CHUNK_CASES = [
    # kind, B, chunk lengths, D, W, H, R, residual
    (oracle.HEADWISE, 2, (5, 4, 6), 6, 4, 2, 0, 1),
    (oracle.HEADWISE, 1, (2, 1, 3, 5), 4, 5, 1, 0, 0),   # chunks shorter than W-1: halos span several chunks
    (oracle.HEADWISE, 2, (7, 7), 8, 1, 4, 0, 1),         # W = 1: no halo at all
    (oracle.LOWRANK, 2, (4, 6, 3), 8, 3, 4, 3, 1),
    (oracle.LOWRANK, 1, (1, 2, 6), 6, 4, 1, 2, 1),
    (oracle.STATIC, 2, (3, 5, 4), 5, 4, 1, 0, 1),
    (oracle.STATIC, 1, (2, 2, 2, 3), 3, 6, 1, 0, 0),
]


def _chunk_inputs(kind, B, L, D, W, H, R):
    G = D // H
    f = {}
    if kind == oracle.HEADWISE:
        f["w"] = rand(B, L, G, W)
    elif kind == oracle.LOWRANK:
        f["z"], f["U"] = rand(B, L, R), rand(R, G * W)
    else:
        f["ws"] = rand(D, W)
    return rand(B, L, D), rand(B, L, D), f


def _rows(a, lo, hi):
    """Rows lo .. hi-1 of a [B, L, ...] array, zero where outside [0, L)."""
    B, L = a.shape[:2]
    out = np.zeros((B, hi - lo) + a.shape[2:])
    s, e = max(lo, 0), min(hi, L)
    if s < e:
        out[:, s - lo:e - lo] = a[:, s:e]
    return out


@pytest.mark.parametrize("kind,B,lens,D,W,H,R,residual", CHUNK_CASES)
def test_chunks_with_halos_equal_the_whole_sequence(kind, B, lens, D, W, H, R, residual):
    L = sum(lens)
    x, dy, f = _chunk_inputs(kind, B, L, D, W, H, R)
    Pl = P(B, L, D, W, H, R, residual)
    y_full, g_full = _plain(kind, Pl, x, dy, f)
    starts = np.concatenate([[0], np.cumsum(lens)])
    total = None
    for i, n in enumerate(lens):
        t0, t1 = starts[i], starts[i + 1]
        Pc = P(B, n, D, W, H, R, residual)
        xc, dyc = np.ascontiguousarray(x[:, t0:t1]), np.ascontiguousarray(dy[:, t0:t1])
        first, last = i == 0, i == len(lens) - 1
        x_prev = None if first else _rows(x, t0 - (W - 1), t0)
        dy_next = None if last else _rows(dy, t1, t1 + W - 1)
        kw = {}
        if kind == oracle.HEADWISE:
            kw = dict(w=np.ascontiguousarray(f["w"][:, t0:t1]),
                      w_next=None if last else _rows(f["w"], t1, t1 + W - 1))
        elif kind == oracle.LOWRANK:
            kw = dict(z=np.ascontiguousarray(f["z"][:, t0:t1]), U=f["U"],
                      z_next=None if last else _rows(f["z"], t1, t1 + W - 1))
        else:
            kw = dict(ws=f["ws"])
        fwd_kw = {k: v for k, v in kw.items() if k not in ("w_next", "z_next")}
        yc = oracle.forward_chunk(Pc, kind, xc, x_prev, **fwd_kw)
        gc = oracle.backward_chunk(Pc, kind, xc, dyc, x_prev, dy_next, **kw)
        np.testing.assert_array_equal(yc, y_full[:, t0:t1])
        np.testing.assert_array_equal(gc[0], g_full[0][:, t0:t1])  # dx
        if kind == oracle.HEADWISE:
            np.testing.assert_array_equal(gc[1], g_full[1][:, t0:t1])  # dw
        elif kind == oracle.LOWRANK:
            np.testing.assert_allclose(gc[1], g_full[1][:, t0:t1], rtol=0, atol=1e-12)  # dz
            np.testing.assert_array_equal(gc[3], g_full[3][:, t0:t1])  # dw
            total = gc[2] if total is None else total + gc[2]
        else:
            total = gc[1] if total is None else total + gc[1]
    if kind == oracle.LOWRANK:
        np.testing.assert_allclose(total, g_full[2], rtol=0, atol=1e-11)  # dU
    elif kind == oracle.STATIC:
        np.testing.assert_allclose(total, g_full[1], rtol=0, atol=1e-11)  # dws


@pytest.mark.parametrize("kind", [oracle.HEADWISE, oracle.LOWRANK, oracle.STATIC])
def test_chunk_without_halos_is_the_plain_op(kind):
    B, T, D, W, H, R = 2, 9, 6, 4, 3, 2
    x, dy, f = _chunk_inputs(kind, B, T, D, W, H, R)
    Pp = P(B, T, D, W, H, R, 1)
    y, g = _plain(kind, Pp, x, dy, f)
    np.testing.assert_array_equal(oracle.forward_chunk(Pp, kind, x, None, **f), y)
    for a, b in zip(oracle.backward_chunk(Pp, kind, x, dy, None, None, **f), g):
        np.testing.assert_array_equal(a, b)


def test_chunk_halo_rows_are_read_at_their_positions():
    """A delta filter on tap j makes y_t = x_t + x_{t-j}: at the chunk's first
    tokens that reads halo row W-1-j+t, and dx at its last tokens reads dy_next
    row t+j-T (checked by hand-indexing, W = 4, one channel)."""
    W, T = 4, 3
    for j in range(1, W):
        w = np.zeros((1, T, 1, W))
        w[..., j] = 1.0
        x, xp = rand(1, T, 1), rand(1, W - 1, 1)
        y = oracle.forward_chunk(P(1, T, 1, W), oracle.HEADWISE, x, xp, w=w)
        for t in range(T):
            src = x[0, t - j, 0] if t - j >= 0 else xp[0, W - 1 + t - j, 0]
            assert y[0, t, 0] == x[0, t, 0] + src
        dy, dyn = rand(1, T, 1), rand(1, W - 1, 1)
        wn = np.zeros((1, W - 1, 1, W))
        wn[..., j] = 1.0
        dx, _ = oracle.backward_chunk(P(1, T, 1, W), oracle.HEADWISE, x, dy, xp, dyn, w=w, w_next=wn)
        for s in range(T):
            src = dy[0, s + j, 0] if s + j < T else dyn[0, s + j - T, 0]
            assert dx[0, s, 0] == dy[0, s, 0] + src


# ------------------------------------------------ first projection z = hV ---

@pytest.mark.parametrize("B,T,D,W,H,R,dm", [(1, 6, 4, 3, 1, 2, 5), (2, 5, 6, 2, 3, 3, 4)])
def test_projection_gradients_by_exact_differences(B, T, D, W, H, R, dm):
    """L = <dy, y> is linear in h and in V separately (z = hV, y linear in z),
    so central differences give dh and dV exactly (up to fp64 rounding)."""
    G = D // H
    x, dy, h = rand(B, T, D), rand(B, T, D), rand(B, T, dm)
    V, U = rand(dm, R), rand(R, G * W)
    Pp = P(B, T, D, W, H, R)
    dx, dh, dV, dU, dz = oracle.backward_lowrank_proj(Pp, x, h, V, U, dy)
    loss = lambda: float(np.sum(dy * oracle.forward_lowrank_proj(Pp, x, h, V, U)[0]))  # noqa: E731
    _loss_grad_check(loss, h, dh)
    _loss_grad_check(loss, V, dV)
    _loss_grad_check(loss, U, dU)
    _loss_grad_check(loss, x, dx)


def test_projection_with_identity_V_is_the_plain_lowrank_op():
    B, T, D, W, H, R = 2, 7, 6, 3, 2, 4
    G = D // H
    x, dy, h, U = rand(B, T, D), rand(B, T, D), rand(B, T, R), rand(R, G * W)
    Pp = P(B, T, D, W, H, R)
    y, z = oracle.forward_lowrank_proj(Pp, x, h, np.eye(R), U)
    np.testing.assert_array_equal(z, h)
    np.testing.assert_array_equal(y, oracle.forward_lowrank(Pp, x, h, U))
    dx, dh, dV, dU, dz = oracle.backward_lowrank_proj(Pp, x, h, np.eye(R), U, dy)
    dxl, dzl, dUl, _ = oracle.backward_lowrank(Pp, x, h, U, dy)
    np.testing.assert_array_equal(dx, dxl)
    np.testing.assert_array_equal(dh, dzl)
    np.testing.assert_array_equal(dU, dUl)
