"""Plant plausible mistakes in a copy of the oracle and check that the pins
catch every one of them.  Mutations are text edits of a temporary copy of
``oracle/dsc_oracle.c``; the committed oracle is never touched.  Every
mutant stays in bounds (it only changes which in-range element is read or
how terms combine), so a failing pin shows up as a wrong value.
"""

import json
import os

import numpy as np
import pytest
import torch

import oracle

HERE = os.path.dirname(os.path.abspath(__file__))
SRC = os.path.join(os.path.dirname(HERE), "oracle", "dsc_oracle.c")

MUTANTS = {
    "strided groups instead of consecutive": ("int64_t g = c / P->H;", "int64_t g = c % G;"),
    "residual dropped in dx": ("double acc = P->residual ? xval(P, dy, b, s, c) : 0.0;", "double acc = 0.0;"),
    "dx uses w(s) instead of w(s+k)": ("acc += tap(P, F, b, s + k, c, k)", "acc += tap(P, F, b, s, c, k)"),
    "dw ignores the lag": ("++c)\n        s += xval(P, dy, b, t, c) * xval(P, x, b, t - k, c);",
                           "++c)\n        s += xval(P, dy, b, t, c) * xval(P, x, b, t, c);"),
    "U read transposed in zU": ("* P->R + r) * val(F->U, r * GW + g * P->W + k);",
                                "* P->R + r) * val(F->U, (g * P->W + k) * P->R + r);"),
    "causal boundary off by one": ("if (t - k >= 0) s += tap", "if (t - k > 0) s += tap"),
    "conv term sign flipped": ("s += tap(P, F, b, t, c, k) * xval(P, x, b, t - k, c);",
                               "s -= tap(P, F, b, t, c, k) * xval(P, x, b, t - k, c);"),
    "dz drops the rank index of U": ("s += dw[n * GW + j] * val(U, r * GW + j);", "s += dw[n * GW + j] * val(U, j);"),
    "dU skips the first token": ("for (int64_t n = 0; n < NT; ++n) s += val(z,", "for (int64_t n = 1; n < NT; ++n) s += val(z,"),
    "static dw reads the wrong lag": ("for (int64_t t = k; t < P->T; ++t)\n            s += xval(P, dy, b, t, c) * xval(P, x, b, t - k, c);",
                                      "for (int64_t t = k; t < P->T; ++t)\n            s += xval(P, dy, b, t, c) * xval(P, x, b, t - (k > 0), c);"),
    "static taps in reverse order": ("if (F->kind == ORC_STATIC) return val(F->w, c * P->W + k);",
                                     "if (F->kind == ORC_STATIC) return val(F->w, c * P->W + (P->W - 1 - k));"),
    "decode reads the state rows in reverse": ("val(state, (b * S + (S - k)) * P->D + c)",
                                               "val(state, (b * S + (k - 1)) * P->D + c)"),
    "decode does not shift the state": ("= val(state, (b * S + j + 1) * P->D + c);",
                                        "= val(state, (b * S + j) * P->D + c);"),
    "decode drops the residual": ("double s = P->residual ? xt : 0.0;", "double s = 0.0;"),
    "packed forward reaches across a document start": ("if (t - k >= start) s += tap(P, &F, 0, t, c, k)",
                                                       "if (t - k >= 0) s += tap(P, &F, 0, t, c, k)"),
    "packed dx reaches past a document end": ("if (s + k < end) acc += tap(P, &F, 0, s + k, c, k)",
                                              "if (s + k < P->T) acc += tap(P, &F, 0, s + k, c, k)"),
    "packed dw reaches across a document start": ("if (t - k >= start)\n                        for",
                                                  "if (t - k >= 0)\n                        for"),
    "chunk halo rows read in reverse": ("*v = val(h->xp, (b * (P->W - 1) + (u + P->W - 1)) * P->D + c);",
                                        "*v = val(h->xp, (b * (P->W - 1) + (-u - 1)) * P->D + c);"),
    "chunk dx reads dy_next one row late": (
        "*v = val(h->dyn, (b * (P->W - 1) + (u - P->T)) * P->D + c);",
        "*v = val(h->dyn, (b * (P->W - 1) + (u - P->T + 1 < P->W - 1 ? u - P->T + 1 : u - P->T)) * P->D + c);"),
    "chunk dx ignores the next tokens' filters": (
        "if (u < P->T || F->kind == ORC_STATIC) return tap(P, F, b, u, c, k);",
        "if (1) return tap(P, F, b, u < P->T ? u : P->T - 1, c, k);"),
    "chunk dw ignores the halo": (
        "for (int64_t c = g * P->H; c < (g + 1) * P->H; ++c)\n                        if (x_ext(",
        "for (int64_t c = g * P->H; c < (g + 1) * P->H; ++c)\n                        if (t - k >= 0 && x_ext("),
}


def _pins(lib):
    """A compact run of the pins; returns the names of those that fail."""
    rng = np.random.default_rng(5)
    fails = []

    def check(name, ok):
        if not ok:
            fails.append(name)

    with open(os.path.join(HERE, "golden", "handworked.json")) as f:
        cases = json.load(f)["cases"]
    for c in cases:
        p = oracle.problem(c["B"], c["T"], c["D"], c["W"], c["H"], c["R"], c["residual"])
        x, dy = np.array(c["x"], float), np.array(c["dy"], float)
        if c["variant"] == "headwise":
            w = np.array(c["w"], float)
            dx, dw = oracle.backward_headwise(p, x, w, dy, lib=lib)
            check("golden", np.array_equal(oracle.forward_headwise(p, x, w, lib=lib), c["y"])
                  and np.array_equal(dx, c["dx"]) and np.array_equal(dw, c["dw"]))
        elif c["variant"] == "lowrank":
            z, U = np.array(c["z"], float), np.array(c["U"], float)
            dx, dz, dU, _ = oracle.backward_lowrank(p, x, z, U, dy, lib=lib)
            check("golden", np.array_equal(oracle.forward_lowrank(p, x, z, U, lib=lib), c["y"])
                  and np.array_equal(dx, c["dx"]) and np.array_equal(dz, c["dz"]) and np.array_equal(dU, c["dU"]))
        else:
            ws = np.array(c["ws"], float)
            dx, dws = oracle.backward_static(p, x, ws, dy, lib=lib)
            check("golden", np.array_equal(oracle.forward_static(p, x, ws, lib=lib), c["y"])
                  and np.array_equal(dx, c["dx"]) and np.array_equal(dws, c["dws"]))

    # static vs torch conv1d and its autograd
    B, T, D, W = 2, 9, 4, 3
    p = oracle.problem(B, T, D, W, 1, 0, 1)
    x, ws, dy = rng.standard_normal((B, T, D)), rng.standard_normal((D, W)), rng.standard_normal((B, T, D))
    xt, wt = torch.tensor(x, requires_grad=True), torch.tensor(ws, requires_grad=True)
    ref = torch.nn.functional.conv1d(xt.transpose(1, 2), wt.flip(-1)[:, None, :], groups=D, padding=W - 1)
    ref = ref[..., :T].transpose(1, 2) + xt
    ref.backward(torch.tensor(dy))
    dx, dws = oracle.backward_static(p, x, ws, dy, lib=lib)
    check("static-conv1d", np.allclose(oracle.forward_static(p, x, ws, lib=lib), ref.detach().numpy(), atol=1e-12)
          and np.allclose(dx, xt.grad.numpy(), atol=1e-12) and np.allclose(dws, wt.grad.numpy(), atol=1e-11))

    # matrix form and exact differences, head-wise and low-rank
    B, T, D, W, H, R = 2, 7, 6, 3, 2, 4
    G = D // H
    p = oracle.problem(B, T, D, W, H, R, 1)
    x, dy = rng.standard_normal((B, T, D)), rng.standard_normal((B, T, D))
    w, z, U = rng.standard_normal((B, T, G, W)), rng.standard_normal((B, T, R)), rng.standard_normal((R, G * W))
    y = oracle.forward_headwise(p, x, w, lib=lib)
    dx, dw = oracle.backward_headwise(p, x, w, dy, lib=lib)
    ok = True
    for b in range(B):
        for c in range(D):
            A = np.eye(T)
            for t in range(T):
                for k in range(W):
                    if t - k >= 0:
                        A[t, t - k] += w[b, t, c // H, k]
            ok &= np.allclose(y[b, :, c], A @ x[b, :, c], atol=1e-12)
            ok &= np.allclose(dx[b, :, c], A.T @ dy[b, :, c], atol=1e-12)
    check("matrix-form", ok)

    def fd(f, arg, grad):
        a, g = arg.reshape(-1), grad.reshape(-1)
        for i in range(a.size):
            o = a[i]
            a[i] = o + 0.5
            lp = f()
            a[i] = o - 0.5
            lm = f()
            a[i] = o
            if abs(lp - lm - g[i]) > 1e-9 * (1 + abs(g[i])):
                return False
        return True

    check("fd-headwise", fd(lambda: np.sum(dy * oracle.forward_headwise(p, x, w, lib=lib)), w, dw))
    dxl, dz, dU, _ = oracle.backward_lowrank(p, x, z, U, dy, lib=lib)
    fl = lambda: np.sum(dy * oracle.forward_lowrank(p, x, z, U, lib=lib))
    check("fd-lowrank", fd(fl, z, dz) and fd(fl, U, dU) and fd(fl, x, dxl))

    # decode steps from a zero state against the forward over the sequence
    pd = oracle.problem(B, 1, D, W, H, 0, 1)
    state, ok = np.zeros((B, W - 1, D)), True
    for t in range(T):
        yt, state = oracle.decode(pd, oracle.HEADWISE, np.ascontiguousarray(x[:, t]), state,
                                  w=np.ascontiguousarray(w[:, t]), lib=lib)
        ok &= np.allclose(yt, y[:, t], atol=1e-12)
    check("decode", ok and np.array_equal(state[:, -1], x[:, -1]))

    # packed documents against the documents run one by one
    lens = (3, 1, 3)
    cu = np.concatenate([[0], np.cumsum(lens)])
    pp = oracle.problem(1, T, D, W, H, 0, 1)
    yp = oracle.forward_varlen(pp, oracle.HEADWISE, x[:1], cu, w=w[:1], lib=lib)
    dxp, dwp = oracle.backward_varlen(pp, oracle.HEADWISE, x[:1], dy[:1], cu, w=w[:1], lib=lib)
    ok = True
    for d in range(len(lens)):
        sl = slice(cu[d], cu[d + 1])
        pd = oracle.problem(1, lens[d], D, W, H, 0, 1)
        xs, ws_, dys = (np.ascontiguousarray(a[:1, sl]) for a in (x, w, dy))
        dxd, dwd = oracle.backward_headwise(pd, xs, ws_, dys, lib=lib)
        ok &= np.allclose(yp[:, sl], oracle.forward_headwise(pd, xs, ws_, lib=lib), atol=1e-12)
        ok &= np.allclose(dxp[:, sl], dxd, atol=1e-12) and np.allclose(dwp[:, sl], dwd, atol=1e-12)
    check("varlen", ok)

    # time chunks with their neighbours' rows as halos against the whole sequence
    # (a chunk shorter than W-1 makes the halo span two chunks)
    Wc, lens = 3, (1, 4, 2)
    pw = oracle.problem(B, T, D, Wc, H, 0, 1)
    wc = rng.standard_normal((B, T, G, Wc))
    yw = oracle.forward_headwise(pw, x, wc, lib=lib)
    dxw, dww = oracle.backward_headwise(pw, x, wc, dy, lib=lib)

    def rows(a, lo, hi):
        out = np.zeros((B, hi - lo) + a.shape[2:])
        s_, e_ = max(lo, 0), min(hi, T)
        if s_ < e_:
            out[:, s_ - lo:e_ - lo] = a[:, s_:e_]
        return out

    ok, t0 = True, 0
    for i, n in enumerate(lens):
        t1 = t0 + n
        pc = oracle.problem(B, n, D, Wc, H, 0, 1)
        xc, dyc, wcc = (np.ascontiguousarray(a[:, t0:t1]) for a in (x, dy, wc))
        xp = None if i == 0 else rows(x, t0 - Wc + 1, t0)
        last = i == len(lens) - 1
        dyn, wn = (None, None) if last else (rows(dy, t1, t1 + Wc - 1), rows(wc, t1, t1 + Wc - 1))
        yc = oracle.forward_chunk(pc, oracle.HEADWISE, xc, xp, w=wcc, lib=lib)
        dxc, dwc = oracle.backward_chunk(pc, oracle.HEADWISE, xc, dyc, xp, dyn, w=wcc, w_next=wn, lib=lib)
        ok &= np.allclose(yc, yw[:, t0:t1], atol=1e-12) and np.allclose(dxc, dxw[:, t0:t1], atol=1e-12)
        ok &= np.allclose(dwc, dww[:, t0:t1], atol=1e-12)
        t0 = t1
    check("chunks", ok)
    return fails


def test_unmutated_copy_passes(tmp_path):
    lib = oracle.load(oracle.build(force=True, out=str(tmp_path / "ok.so")))
    assert _pins(lib) == []


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_pins_catch_mutant(name, tmp_path):
    old, new = MUTANTS[name]
    src = open(SRC).read()
    assert src.count(old) == 1, f"mutation site not unique/present: {old!r}"
    path = tmp_path / "mutant.c"
    path.write_text(src.replace(old, new))
    lib = oracle.load(oracle.build(force=True, src=str(path), out=str(tmp_path / "mutant.so")))
    assert _pins(lib), f"no pin caught the mutant '{name}'"


# The first projection's oracle is numpy (oracle.forward_lowrank_proj /
# backward_lowrank_proj); its planted mistakes are swapped-in functions.
PROJ_MUTANTS = {
    "projection reads V's rows in reverse": lambda h, V: np.einsum("btd,dr->btr", oracle._f64(h), oracle._f64(V)[::-1]),
    "projection drops the last model dimension": lambda h, V: np.einsum("btd,dr->btr", oracle._f64(h)[..., :-1],
                                                                        oracle._f64(V)[:-1]),
}


def _proj_pins_pass(monkeypatch, mutant):
    if mutant is not None:
        monkeypatch.setattr(oracle, "projection", mutant)
    rng = np.random.default_rng(9)
    B, T, D, W, H, R, dm = 1, 5, 4, 3, 1, 3, 3
    x, dy, h = rng.standard_normal((B, T, D)), rng.standard_normal((B, T, D)), rng.standard_normal((B, T, dm))
    V, U = rng.standard_normal((dm, R)), rng.standard_normal((R, (D // H) * W))
    p = oracle.problem(B, T, D, W, H, R, 1)
    dx, dh, dV, dU, _ = oracle.backward_lowrank_proj(p, x, h, V, U, dy)
    ok = True
    for arg, grad in ((h, dh), (V, dV)):
        a, g = arg.reshape(-1), grad.reshape(-1)
        for i in range(a.size):
            o = a[i]
            a[i] = o + 0.5
            lp = np.sum(dy * oracle.forward_lowrank_proj(p, x, h, V, U)[0])
            a[i] = o - 0.5
            lm = np.sum(dy * oracle.forward_lowrank_proj(p, x, h, V, U)[0])
            a[i] = o
            ok &= abs(lp - lm - g[i]) <= 1e-9 * (1 + abs(g[i]))
    # identity V reduces to the plain low-rank op
    y, z = oracle.forward_lowrank_proj(p, x, h, np.eye(dm), U)  # dm == R here
    ok &= np.array_equal(z, h)
    return ok


def test_projection_pins_pass_unmutated(monkeypatch):
    assert _proj_pins_pass(monkeypatch, None)


@pytest.mark.parametrize("name", sorted(PROJ_MUTANTS))
def test_projection_pins_catch_mutant(name, monkeypatch):
    assert not _proj_pins_pass(monkeypatch, PROJ_MUTANTS[name])
