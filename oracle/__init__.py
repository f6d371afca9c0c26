"""fp64 CPU oracle of the dynamic short convolution (test infrastructure).

Only the tests, ``__graft_entry__.smoke()`` and the benchmark's CPU-baseline
leg may import this package.  It shares no code with the CUDA library; the
arithmetic lives in ``dsc_oracle.c`` (plain loops over the definitions, see
that file's header for the formulas and their sources), and this module only
compiles it, marshals numpy arrays and returns fp64 results.

Inputs are numpy arrays in storage form: ``float32`` (fp32), ``uint16``
(bf16 bit patterns) or ``float64``.  Every output is fp64.
"""

from __future__ import annotations

import ctypes as C
import os
import subprocess
import threading

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "dsc_oracle.c")
_LIB = os.path.join(_HERE, "liboracle.so")

F32, BF16, F64 = 0, 1, 2
HEADWISE, LOWRANK, STATIC = 0, 1, 2
Y, DX, DW, DZ, DU, DWS, W_TAP = 0, 1, 2, 3, 4, 5, 6

_lock = threading.Lock()
_lib = None


class Problem(C.Structure):
    _fields_ = [("B", C.c_int64), ("T", C.c_int64), ("D", C.c_int64), ("W", C.c_int64),
                ("H", C.c_int64), ("R", C.c_int64), ("residual", C.c_int64)]

    @property
    def G(self):
        return self.D // self.H


class _In(C.Structure):
    _fields_ = [("p", C.c_void_p), ("dt", C.c_int64)]


class _Filter(C.Structure):
    _fields_ = [("kind", C.c_int64), ("w", _In), ("z", _In), ("U", _In)]


def problem(B, T, D, W, H=1, R=0, residual=1) -> Problem:
    if D % H:
        raise ValueError("D must be a multiple of H")
    return Problem(B, T, D, W, H, R, residual)


def problem_of(wl) -> Problem:
    """Problem of a ``synth.workloads.Workload``."""
    return problem(wl.B, wl.T, wl.D, wl.W, wl.H, wl.R, wl.residual)


def build(force: bool = False, src: str = _SRC, out: str = _LIB) -> str:
    """Compile the oracle with gcc (plain IEEE fp64: no fast-math, no contraction)."""
    if force or not os.path.exists(out) or os.path.getmtime(out) < os.path.getmtime(src):
        tmp = out + f".tmp{os.getpid()}"
        subprocess.run(["gcc", "-O2", "-std=c11", "-fopenmp", "-ffp-contract=off", "-fno-fast-math",
                        "-shared", "-fPIC", src, "-o", tmp, "-lm"], check=True)
        os.replace(tmp, out)
    return out


def load(path: str | None = None):
    """Load (building if needed) the oracle library; ``path`` selects another build."""
    global _lib
    if path is not None:
        return _bind(C.CDLL(path))
    with _lock:
        if _lib is None:
            _lib = _bind(C.CDLL(build()))
    return _lib


def _bind(lib):
    P = C.POINTER(Problem)
    d = C.POINTER(C.c_double)
    lib.orc_max_threads.restype = C.c_int
    lib.orc_lowrank_filters.argtypes = [P, _In, _In, d]
    lib.orc_forward.argtypes = [P, C.c_int64, _In, _In, d]
    lib.orc_backward.argtypes = [P, C.c_int64, _In, _In, _In, d, d]
    lib.orc_lowrank_grads.argtypes = [P, _In, _In, d, d, d]
    lib.orc_sample.argtypes = [P, C.POINTER(_Filter), _In, _In, C.c_int64, C.c_int64,
                               C.POINTER(C.c_int64), d]
    lib.orc_decode.argtypes = [P, C.POINTER(_Filter), _In, _In, d, d]
    i64 = C.POINTER(C.c_int64)
    lib.orc_forward_varlen.argtypes = [P, C.c_int64, _In, _In, i64, C.c_int64, d]
    lib.orc_backward_varlen.argtypes = [P, C.c_int64, _In, _In, _In, i64, C.c_int64, d, d]
    lib.orc_forward_chunk.argtypes = [P, C.c_int64, _In, _In, _In, d]
    lib.orc_backward_chunk.argtypes = [P, C.c_int64, _In, _In, _In, _In, _In, _In, d, d]
    for f in ("orc_lowrank_filters", "orc_forward", "orc_backward", "orc_lowrank_grads", "orc_sample", "orc_decode",
              "orc_forward_varlen", "orc_backward_varlen", "orc_forward_chunk", "orc_backward_chunk"):
        getattr(lib, f).restype = None
    return lib


def max_threads() -> int:
    return load().orc_max_threads()


def _in(a: np.ndarray | None) -> _In:
    if a is None:
        return _In(None, F64)
    if not a.flags.c_contiguous:
        raise ValueError("oracle inputs must be C-contiguous")
    dt = {np.dtype(np.float32): F32, np.dtype(np.uint16): BF16, np.dtype(np.float64): F64}[a.dtype]
    return _In(a.ctypes.data, dt)


def _out(shape) -> np.ndarray:
    return np.empty(shape, dtype=np.float64)


def _dp(a: np.ndarray):
    return a.ctypes.data_as(C.POINTER(C.c_double))


def forward_headwise(P: Problem, x, w, lib=None) -> np.ndarray:
    lib = lib or load()
    y = _out((P.B, P.T, P.D))
    lib.orc_forward(C.byref(P), HEADWISE, _in(w), _in(x), _dp(y))
    return y


def backward_headwise(P: Problem, x, w, dy, lib=None):
    """Returns (dx [B,T,D], dw [B,T,G,W])."""
    lib = lib or load()
    dx = _out((P.B, P.T, P.D))
    dw = _out((P.B, P.T, P.G, P.W))
    lib.orc_backward(C.byref(P), HEADWISE, _in(w), _in(x), _in(dy), _dp(dx), _dp(dw))
    return dx, dw


def forward_static(P: Problem, x, ws, lib=None) -> np.ndarray:
    lib = lib or load()
    y = _out((P.B, P.T, P.D))
    lib.orc_forward(C.byref(P), STATIC, _in(ws), _in(x), _dp(y))
    return y


def backward_static(P: Problem, x, ws, dy, lib=None):
    """Returns (dx [B,T,D], dws [D,W])."""
    lib = lib or load()
    dx = _out((P.B, P.T, P.D))
    dws = _out((P.D, P.W))
    lib.orc_backward(C.byref(P), STATIC, _in(ws), _in(x), _in(dy), _dp(dx), _dp(dws))
    return dx, dws


def lowrank_filters(P: Problem, z, U, lib=None) -> np.ndarray:
    """w [B,T,G,W] = z . U, materialised in fp64."""
    lib = lib or load()
    w = _out((P.B, P.T, P.G, P.W))
    lib.orc_lowrank_filters(C.byref(P), _in(z), _in(U), _dp(w))
    return w


def forward_lowrank(P: Problem, x, z, U, lib=None) -> np.ndarray:
    """Filters w = zU, then the head-wise forward with them."""
    lib = lib or load()
    w = lowrank_filters(P, z, U, lib)
    return forward_headwise(P, x, w, lib)


def backward_lowrank(P: Problem, x, z, U, dy, lib=None):
    """Returns (dx [B,T,D], dz [B,T,R], dU [R,G*W], dw [B,T,G,W])."""
    lib = lib or load()
    w = lowrank_filters(P, z, U, lib)
    dx, dw = backward_headwise(P, x, w, dy, lib)
    dz = _out((P.B, P.T, P.R))
    dU = _out((P.R, P.G * P.W))
    lib.orc_lowrank_grads(C.byref(P), _in(z), _in(U), _dp(dw), _dp(dz), _dp(dU))
    return dx, dz, dU, dw


def sample(P: Problem, kind: int, what: int, idx, *, x=None, dy=None, w=None, z=None, U=None, lib=None):
    """Evaluate single output elements; ``idx`` is an int64 array [n, <=4]."""
    lib = lib or load()
    idx = np.asarray(idx, dtype=np.int64)
    q = np.zeros((idx.shape[0], 4), dtype=np.int64)
    q[:, :idx.shape[1]] = idx
    F = _Filter(kind, _in(w), _in(z), _in(U))
    out = _out((idx.shape[0],))
    lib.orc_sample(C.byref(P), C.byref(F), _in(x), _in(dy), what, idx.shape[0],
                   q.ctypes.data_as(C.POINTER(C.c_int64)), _dp(out))
    return out


def decode(P: Problem, kind: int, x, state, *, w=None, z=None, U=None, ws=None, lib=None):
    """One decode step (P.T must be 1): x [B,D], state [B,W-1,D] (row j holds
    x_{t-W+1+j}); head-wise w [B,G,W], low-rank z [B,R] and U [R,G*W], or
    static ws [D,W].  Returns (y [B,D], the state after the step [B,W-1,D])."""
    if P.T != 1:
        raise ValueError("a decode step has T = 1")
    lib = lib or load()
    y = _out((P.B, P.D))
    st = _out((P.B, P.W - 1, P.D))
    F = _Filter(kind, _in(ws if kind == STATIC else w), _in(z), _in(U))
    lib.orc_decode(C.byref(P), C.byref(F), _in(x), _in(state), _dp(y), _dp(st))
    return y, st


def _cu(P: Problem, cu_seqlens):
    cu = np.ascontiguousarray(cu_seqlens, dtype=np.int64)
    if P.B != 1 or cu[0] != 0 or cu[-1] != P.T or np.any(np.diff(cu) < 0):
        raise ValueError("packed sequences: B = 1 and cu_seqlens non-decreasing from 0 to T")
    return cu, cu.ctypes.data_as(C.POINTER(C.c_int64)), len(cu) - 1


def forward_varlen(P: Problem, kind: int, x, cu_seqlens, *, w=None, z=None, U=None, ws=None, lib=None):
    """Packed documents (B = 1, document d = tokens cu[d] .. cu[d+1]-1), no tap
    crossing a document start.  Head-wise w [1,T,G,W], low-rank z and U (the
    filters materialised as w = zU), or static ws [D,W].  Returns y [1,T,D]."""
    lib = lib or load()
    cu, cp, n = _cu(P, cu_seqlens)
    if kind == LOWRANK:
        w, kind = lowrank_filters(P, z, U, lib), HEADWISE
    y = _out((P.B, P.T, P.D))
    lib.orc_forward_varlen(C.byref(P), kind, _in(ws if kind == STATIC else w), _in(x), cp, n, _dp(y))
    return y


def backward_varlen(P: Problem, kind: int, x, dy, cu_seqlens, *, w=None, z=None, U=None, ws=None, lib=None):
    """Gradients of forward_varlen: (dx, dw) for head-wise, (dx, dws) for
    static, (dx, dz, dU, dw) for low-rank."""
    lib = lib or load()
    cu, cp, n = _cu(P, cu_seqlens)
    lowrank = kind == LOWRANK
    if lowrank:
        w, kind = lowrank_filters(P, z, U, lib), HEADWISE
    dx = _out((P.B, P.T, P.D))
    dw = _out((P.D, P.W)) if kind == STATIC else _out((P.B, P.T, P.G, P.W))
    lib.orc_backward_varlen(C.byref(P), kind, _in(ws if kind == STATIC else w), _in(x), _in(dy), cp, n, _dp(dx),
                            _dp(dw))
    if not lowrank:
        return dx, dw
    dz = _out((P.B, P.T, P.R))
    dU = _out((P.R, P.G * P.W))
    lib.orc_lowrank_grads(C.byref(P), _in(z), _in(U), _dp(dw), _dp(dz), _dp(dU))
    return dx, dz, dU, dw


def _halo(a, B, W, D):
    if a is None:
        return None
    a = np.ascontiguousarray(a)
    if a.shape[0] != B or a.shape[1] != W - 1 or a.shape[-1] != D and a.ndim == 3:
        raise ValueError("halo rows must be [B, W-1, ...]")
    return a


def forward_chunk(P: Problem, kind: int, x, x_prev=None, *, w=None, z=None, U=None, ws=None, lib=None):
    """One time chunk of longer sequences (context parallelism): x [B,T,D]
    holds tokens t0 .. t0+T-1, x_prev [B,W-1,D] the W-1 tokens before t0
    (row j = position t0-W+1+j; None when t0 = 0).  Filters as in
    forward_varlen (low-rank: materialised w = zU).  Returns y [B,T,D]."""
    lib = lib or load()
    if kind == LOWRANK:
        w, kind = lowrank_filters(P, z, U, lib), HEADWISE
    y = _out((P.B, P.T, P.D))
    xp = _halo(x_prev, P.B, P.W, P.D) if P.W > 1 else None
    lib.orc_forward_chunk(C.byref(P), kind, _in(ws if kind == STATIC else w), _in(x), _in(xp), _dp(y))
    return y


def backward_chunk(P: Problem, kind: int, x, dy, x_prev=None, dy_next=None, *, w=None, w_next=None, z=None,
                   z_next=None, U=None, ws=None, lib=None):
    """Gradients of forward_chunk.  dy_next [B,W-1,D] holds dy at positions
    t0+T .. t0+T+W-2 and w_next [B,W-1,G,W] (head-wise) or z_next [B,W-1,R]
    (low-rank) the filters of those tokens; None for the last chunk.
    Returns (dx, dw) head-wise, (dx, dws) static, (dx, dz, dU, dw) low-rank;
    dU and dws sum over this chunk's tokens only."""
    lib = lib or load()
    lowrank = kind == LOWRANK
    if lowrank:
        w = lowrank_filters(P, z, U, lib)
        if dy_next is not None and P.W > 1:
            Pn = problem(P.B, P.W - 1, P.D, P.W, P.H, P.R, P.residual)
            w_next = lowrank_filters(Pn, np.ascontiguousarray(z_next), U, lib)
        kind = HEADWISE
    xp = _halo(x_prev, P.B, P.W, P.D) if P.W > 1 else None
    dyn = _halo(dy_next, P.B, P.W, P.D) if P.W > 1 else None
    wn = np.ascontiguousarray(w_next) if (dyn is not None and kind == HEADWISE) else None
    if dyn is not None and kind == HEADWISE and wn is None:
        raise ValueError("dy_next needs the filters of the same tokens")
    dx = _out((P.B, P.T, P.D))
    dw = _out((P.D, P.W)) if kind == STATIC else _out((P.B, P.T, P.G, P.W))
    lib.orc_backward_chunk(C.byref(P), kind, _in(ws if kind == STATIC else w), _in(x), _in(dy), _in(xp), _in(dyn),
                           _in(wn), _dp(dx), _dp(dw))
    if not lowrank:
        return dx, dw
    dz = _out((P.B, P.T, P.R))
    dU = _out((P.R, P.G * P.W))
    lib.orc_lowrank_grads(C.byref(P), _in(z), _in(U), _dp(dw), _dp(dz), _dp(dU))
    return dx, dz, dU, dw


# ------------------------------------------------ the first projection z = hV ---
# Technical summary, Methodology, "Parameterisation" 1: the filter is a linear
# map of the current hidden state, factorised at rank R, w(t) = h_t V U with
# V [d_model, R] and U [R, G*W].  The library's projection calls take h
# [B,T,d_model] and V and form z = hV themselves; the oracle evaluates the
# same composition in fp64: z = hV (a plain matrix product), then the pinned
# low-rank oracle with that z, and the gradients of h and V through the chain
# rule, dh = dz V^T and dV = sum over tokens of h^T dz.

def _f64(a, dtype_hint=None):
    import synth

    a = np.asarray(a)
    if a.dtype == np.uint16:
        return synth.bf16_bits_to_f32(a).astype(np.float64)
    return a.astype(np.float64)


def projection(h, V) -> np.ndarray:
    """z [B,T,R] = h [B,T,d_model] . V [d_model,R] in fp64."""
    return np.einsum("btd,dr->btr", _f64(h), _f64(V))


def forward_lowrank_proj(P: Problem, x, h, V, U, lib=None):
    """Returns (y [B,T,D], z [B,T,R]) with z = hV exact in fp64."""
    z = np.ascontiguousarray(projection(h, V))
    return forward_lowrank(P, x, z, U, lib), z


def backward_lowrank_proj(P: Problem, x, h, V, U, dy, lib=None):
    """Returns (dx, dh [B,T,d_model], dV [d_model,R], dU [R,G*W], dz)."""
    z = np.ascontiguousarray(projection(h, V))
    dx, dz, dU, _ = backward_lowrank(P, x, z, U, dy, lib)
    dh = np.einsum("btr,dr->btd", dz, _f64(V))
    dV = np.einsum("btd,btr->dr", _f64(h), dz)
    return dx, dh, dV, dU, dz
