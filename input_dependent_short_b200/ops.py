"""PyTorch-facing binding of libdsc.so.

Each function has the name of the C entry point it calls and only marshals
arguments: it checks shapes/dtypes/devices, allocates the outputs (and any
scratch the library asks for) with torch on the tensors' device, and passes
raw device pointers plus torch's current CUDA stream.  Every step of the
computation runs in the library's CUDA kernels.

Layouts (row-major, contiguous): x, dy, y, dx [B,T,D]; head-wise w, dw
[B,T,G,W] with G = D/H; low-rank z, dz [B,T,R] and U [R,G*W]; static
ws [D,W].  dtypes: all bf16 or all fp32; dU and dws are fp32.
"""

from __future__ import annotations

import torch

from ._lib import DSC_BF16, DSC_F32, DscProblem, call, lib

_DT = {torch.bfloat16: DSC_BF16, torch.float32: DSC_F32}


def _ptr(t: torch.Tensor | None):
    return None if t is None else t.data_ptr()


def _stream(dev: torch.device):
    return torch.cuda.current_stream(dev).cuda_stream


def _check(*ts: torch.Tensor, dtype=None):
    dev = ts[0].device
    if dev.type != "cuda":
        raise ValueError("libdsc operates on CUDA tensors")
    for t in ts:
        if t.device != dev:
            raise ValueError("all tensors must be on the same device")
        if not t.is_contiguous():
            raise ValueError("tensors must be contiguous")
        if dtype is not None and t.dtype != dtype:
            raise ValueError(f"expected {dtype}, got {t.dtype}")
    return dev


def problem(x: torch.Tensor, W: int, H: int, R: int = 0, residual: bool = True) -> DscProblem:
    B, T, D = x.shape
    if x.dtype not in _DT:
        raise ValueError(f"unsupported dtype {x.dtype}")
    return DscProblem(B, T, D, W, H, R, _DT[x.dtype], int(bool(residual)))


# ----------------------------------------------------------------- head-wise ---

def dsc_fwd_headwise(x, w, residual=True):
    """y = r*x + causal per-token conv of x with head-wise filters w [B,T,G,W]."""
    dev = _check(x, w, dtype=x.dtype)
    B, T, D = x.shape
    G, W = w.shape[2], w.shape[3]
    if w.shape[:2] != (B, T) or D % G:
        raise ValueError("w must be [B,T,G,W] with G dividing D")
    p = problem(x, W, D // G, 0, residual)
    y = torch.empty_like(x)
    with torch.cuda.device(dev):
        call("dsc_fwd_headwise", p, _ptr(x), _ptr(w), _ptr(y), _stream(dev))
    return y


def dsc_bwd_headwise(x, w, dy, residual=True):
    """Returns (dx, dw)."""
    dev = _check(x, w, dy, dtype=x.dtype)
    B, T, D = x.shape
    G, W = w.shape[2], w.shape[3]
    p = problem(x, W, D // G, 0, residual)
    dx = torch.empty_like(x)
    dw = torch.empty_like(w)
    with torch.cuda.device(dev):
        call("dsc_bwd_headwise", p, _ptr(x), _ptr(w), _ptr(dy), _ptr(dx), _ptr(dw), _stream(dev))
    return dx, dw


# ------------------------------------------------------------------ low-rank ---

def _lr_problem(x, z, U, H, residual):
    B, T, D = x.shape
    R = z.shape[-1]
    if z.shape != (B, T, R) or U.shape[0] != R or D % H or U.shape[1] % (D // H):
        raise ValueError("expected z [B,T,R] and U [R,(D/H)*W]")
    W = U.shape[1] // (D // H)
    return problem(x, W, H, R, residual)


def dsc_fwd_lowrank(x, z, U, H=1, residual=True):
    """y with filters w(t) = z_t U formed on chip (U is [R, (D/H)*W])."""
    dev = _check(x, z, U, dtype=x.dtype)
    p = _lr_problem(x, z, U, H, residual)
    y = torch.empty_like(x)
    n = lib().dsc_fwd_lowrank_workspace_bytes(p)
    ws = torch.empty(n, dtype=torch.uint8, device=dev) if n else None
    with torch.cuda.device(dev):
        call("dsc_fwd_lowrank", p, _ptr(x), _ptr(z), _ptr(U), _ptr(y), _ptr(ws), n, _stream(dev))
    return y


def dsc_bwd_lowrank(x, z, U, dy, H=1, residual=True):
    """Returns (dx, dz, dU); dU is fp32."""
    dev = _check(x, z, U, dy, dtype=x.dtype)
    p = _lr_problem(x, z, U, H, residual)
    dx = torch.empty_like(x)
    dz = torch.empty_like(z)
    dU = torch.empty(U.shape, dtype=torch.float32, device=dev)
    n = lib().dsc_bwd_lowrank_workspace_bytes(p)
    ws = torch.empty(n, dtype=torch.uint8, device=dev) if n else None
    with torch.cuda.device(dev):
        call("dsc_bwd_lowrank", p, _ptr(x), _ptr(z), _ptr(U), _ptr(dy), _ptr(dx), _ptr(dz), _ptr(dU),
             _ptr(ws), n, _stream(dev))
    return dx, dz, dU


# -------------------------------------------------------------------- static ---

def dsc_fwd_static(x, ws, residual=False):
    """Depthwise causal conv with one fixed filter per channel, ws [D,W]."""
    dev = _check(x, ws, dtype=x.dtype)
    p = problem(x, ws.shape[1], 1, 0, residual)
    y = torch.empty_like(x)
    with torch.cuda.device(dev):
        call("dsc_fwd_static", p, _ptr(x), _ptr(ws), _ptr(y), _stream(dev))
    return y


def dsc_bwd_static(x, ws, dy, residual=False):
    """Returns (dx, dws); dws is fp32."""
    dev = _check(x, ws, dy, dtype=x.dtype)
    p = problem(x, ws.shape[1], 1, 0, residual)
    dx = torch.empty_like(x)
    dws = torch.empty(ws.shape, dtype=torch.float32, device=dev)
    with torch.cuda.device(dev):
        n = lib().dsc_bwd_static_workspace_bytes(p)
        scratch = torch.empty(max(n, 16), dtype=torch.uint8, device=dev)
        call("dsc_bwd_static", p, _ptr(x), _ptr(ws), _ptr(dy), _ptr(dx), _ptr(dws), _ptr(scratch), n,
             _stream(dev))
    return dx, dws


# -------------------------------------------------------------------- decode ---

def _dec_problem(x, state, W, H, R, residual):
    B, D = x.shape
    if x.dtype not in _DT:
        raise ValueError(f"unsupported dtype {x.dtype}")
    if W > 1 and (state is None or state.shape != (B, W - 1, D) or state.dtype != x.dtype):
        raise ValueError("state must be [B, W-1, D] in the dtype of x")
    return DscProblem(B, 1, D, W, H, R, _DT[x.dtype], int(bool(residual)))


def dsc_decode_headwise(x, w, state, residual=True):
    """One decode step: x [B,D], the new token's filters w [B,G,W], state
    [B,W-1,D] (last W-1 inputs, oldest first; updated in place).  Returns y."""
    dev = _check(x, w, *([state] if state is not None else []), dtype=x.dtype)
    B, D = x.shape
    G, W = w.shape[1], w.shape[2]
    if w.shape[0] != B or D % G:
        raise ValueError("w must be [B,G,W] with G dividing D")
    p = _dec_problem(x, state, W, D // G, 0, residual)
    y = torch.empty_like(x)
    with torch.cuda.device(dev):
        call("dsc_decode_headwise", p, _ptr(x), _ptr(w), _ptr(state), _ptr(y), _stream(dev))
    return y


def dsc_decode_static(x, ws, state, residual=False):
    """One decode step with static filters ws [D,W]; state updated in place."""
    dev = _check(x, ws, *([state] if state is not None else []), dtype=x.dtype)
    W = ws.shape[1]
    if ws.shape[0] != x.shape[1]:
        raise ValueError("ws must be [D,W]")
    p = _dec_problem(x, state, W, 1, 0, residual)
    y = torch.empty_like(x)
    with torch.cuda.device(dev):
        call("dsc_decode_static", p, _ptr(x), _ptr(ws), _ptr(state), _ptr(y), _stream(dev))
    return y


def dsc_decode_lowrank(x, z, U, state, H=1, residual=True):
    """One decode step with low-rank filters w = z U (z [B,R], U [R,G*W]);
    state updated in place."""
    dev = _check(x, z, U, *([state] if state is not None else []), dtype=x.dtype)
    B, D = x.shape
    R = z.shape[1]
    if z.shape != (B, R) or U.shape[0] != R or D % H or U.shape[1] % (D // H):
        raise ValueError("expected z [B,R] and U [R,(D/H)*W]")
    W = U.shape[1] // (D // H)
    p = _dec_problem(x, state, W, H, R, residual)
    n = lib().dsc_decode_lowrank_workspace_bytes(p)
    ws = torch.empty(n, dtype=torch.uint8, device=dev) if n else None
    y = torch.empty_like(x)
    with torch.cuda.device(dev):
        call("dsc_decode_lowrank", p, _ptr(x), _ptr(z), _ptr(U), _ptr(state), _ptr(y), _ptr(ws), n, _stream(dev))
    return y


def dsc_decode_state(x, W):
    """The decode state [B,W-1,D] after a prompt x [B,T,D]."""
    dev = _check(x)
    B, T, D = x.shape
    state = torch.empty(B, W - 1, D, dtype=x.dtype, device=dev) if W > 1 else None
    p = problem(x, W, 1, 0, False)
    with torch.cuda.device(dev):
        call("dsc_decode_state", p, _ptr(x), _ptr(state), _stream(dev))
    return state


def dsc_check(device=None):
    """Synchronise the current stream and raise if a kernel recorded a timeout."""
    dev = torch.device("cuda", torch.cuda.current_device() if device is None else torch.device(device).index)
    with torch.cuda.device(dev):
        call("dsc_check", _stream(dev))


# ---------------------------------------------------------- packed documents ---
# Variable-length batches: x [1, T, D] holds several documents back to back,
# cu_seqlens (int32, on the device) their offsets; no tap crosses a document
# boundary.

def _cu(cu_seqlens, dev):
    if cu_seqlens.dtype != torch.int32 or cu_seqlens.device != dev or cu_seqlens.dim() != 1:
        raise ValueError("cu_seqlens must be a 1-D int32 tensor on the tensors' device")
    return cu_seqlens.contiguous(), cu_seqlens.numel() - 1


def dsc_fwd_headwise_varlen(x, w, cu_seqlens, residual=True):
    dev = _check(x, w, dtype=x.dtype)
    cu, n = _cu(cu_seqlens, dev)
    p = problem(x, w.shape[3], x.shape[2] // w.shape[2], 0, residual)
    y = torch.empty_like(x)
    with torch.cuda.device(dev):
        call("dsc_fwd_headwise_varlen", p, _ptr(cu), n, _ptr(x), _ptr(w), _ptr(y), _stream(dev))
    return y


def dsc_bwd_headwise_varlen(x, w, dy, cu_seqlens, residual=True):
    """Returns (dx, dw)."""
    dev = _check(x, w, dy, dtype=x.dtype)
    cu, n = _cu(cu_seqlens, dev)
    p = problem(x, w.shape[3], x.shape[2] // w.shape[2], 0, residual)
    dx, dw = torch.empty_like(x), torch.empty_like(w)
    with torch.cuda.device(dev):
        call("dsc_bwd_headwise_varlen", p, _ptr(cu), n, _ptr(x), _ptr(w), _ptr(dy), _ptr(dx), _ptr(dw), _stream(dev))
    return dx, dw


def dsc_fwd_lowrank_varlen(x, z, U, cu_seqlens, H=1, residual=True):
    dev = _check(x, z, U, dtype=x.dtype)
    cu, n = _cu(cu_seqlens, dev)
    p = _lr_problem(x, z, U, H, residual)
    y = torch.empty_like(x)
    nb = lib().dsc_fwd_lowrank_workspace_bytes(p)
    ws = torch.empty(nb, dtype=torch.uint8, device=dev) if nb else None
    with torch.cuda.device(dev):
        call("dsc_fwd_lowrank_varlen", p, _ptr(cu), n, _ptr(x), _ptr(z), _ptr(U), _ptr(y), _ptr(ws), nb, _stream(dev))
    return y


def dsc_bwd_lowrank_varlen(x, z, U, dy, cu_seqlens, H=1, residual=True):
    """Returns (dx, dz, dU); dU is fp32."""
    dev = _check(x, z, U, dy, dtype=x.dtype)
    cu, n = _cu(cu_seqlens, dev)
    p = _lr_problem(x, z, U, H, residual)
    dx, dz = torch.empty_like(x), torch.empty_like(z)
    dU = torch.empty(U.shape, dtype=torch.float32, device=dev)
    nb = lib().dsc_bwd_lowrank_varlen_workspace_bytes(p, n)
    ws = torch.empty(nb, dtype=torch.uint8, device=dev) if nb else None
    with torch.cuda.device(dev):
        call("dsc_bwd_lowrank_varlen", p, _ptr(cu), n, _ptr(x), _ptr(z), _ptr(U), _ptr(dy), _ptr(dx), _ptr(dz),
             _ptr(dU), _ptr(ws), nb, _stream(dev))
    return dx, dz, dU


def dsc_fwd_static_varlen(x, ws, cu_seqlens, residual=False):
    dev = _check(x, ws, dtype=x.dtype)
    cu, n = _cu(cu_seqlens, dev)
    p = problem(x, ws.shape[1], 1, 0, residual)
    y = torch.empty_like(x)
    with torch.cuda.device(dev):
        call("dsc_fwd_static_varlen", p, _ptr(cu), n, _ptr(x), _ptr(ws), _ptr(y), _stream(dev))
    return y


def dsc_bwd_static_varlen(x, ws, dy, cu_seqlens, residual=False):
    """Returns (dx, dws); dws is fp32."""
    dev = _check(x, ws, dy, dtype=x.dtype)
    cu, n = _cu(cu_seqlens, dev)
    p = problem(x, ws.shape[1], 1, 0, residual)
    dx = torch.empty_like(x)
    dws = torch.empty(ws.shape, dtype=torch.float32, device=dev)
    with torch.cuda.device(dev):
        nb = lib().dsc_bwd_static_workspace_bytes(p)
        scratch = torch.empty(max(nb, 16), dtype=torch.uint8, device=dev)
        call("dsc_bwd_static_varlen", p, _ptr(cu), n, _ptr(x), _ptr(ws), _ptr(dy), _ptr(dx), _ptr(dws),
             _ptr(scratch), nb, _stream(dev))
    return dx, dws


# ----------------------------------------------------------- sequence chunks ---
# Context parallelism: x [B, T, D] is one time chunk of longer sequences.
# x_prev [B, W-1, D] holds the W-1 inputs before it (None for the first
# chunk); dy_next [B, W-1, D] and the next tokens' filters (w_next
# [B, W-1, G, W] or z_next [B, W-1, R]) the W-1 after it (None for the last).
# edges_only=True recomputes only the outputs next to the chunk's edges in
# tensors that already hold the plain call's results (passed as `out`).

def _halo_ok(dev, dtype, *hs):
    for h in hs:
        if h is not None:
            _check(h, dtype=dtype)
            if h.device != dev:
                raise ValueError("halos must be on the tensors' device")


def dsc_fwd_headwise_chunk(x, w, x_prev=None, residual=True, out=None):
    dev = _check(x, w, dtype=x.dtype)
    _halo_ok(dev, x.dtype, x_prev)
    p = problem(x, w.shape[3], x.shape[2] // w.shape[2], 0, residual)
    y = out if out is not None else torch.empty_like(x)
    with torch.cuda.device(dev):
        call("dsc_fwd_headwise_chunk", p, _ptr(x_prev), _ptr(x), _ptr(w), _ptr(y), int(out is not None),
             _stream(dev))
    return y


def dsc_bwd_headwise_chunk(x, w, dy, x_prev=None, dy_next=None, w_next=None, residual=True, out=None):
    """Returns (dx, dw)."""
    dev = _check(x, w, dy, dtype=x.dtype)
    _halo_ok(dev, x.dtype, x_prev, dy_next, w_next)
    p = problem(x, w.shape[3], x.shape[2] // w.shape[2], 0, residual)
    dx, dw = out if out is not None else (torch.empty_like(x), torch.empty_like(w))
    with torch.cuda.device(dev):
        call("dsc_bwd_headwise_chunk", p, _ptr(x_prev), _ptr(dy_next), _ptr(w_next), _ptr(x), _ptr(w), _ptr(dy),
             _ptr(dx), _ptr(dw), int(out is not None), _stream(dev))
    return dx, dw


def dsc_fwd_lowrank_chunk(x, z, U, x_prev=None, H=1, residual=True, out=None):
    dev = _check(x, z, U, dtype=x.dtype)
    _halo_ok(dev, x.dtype, x_prev)
    p = _lr_problem(x, z, U, H, residual)
    y = out if out is not None else torch.empty_like(x)
    nb = lib().dsc_fwd_lowrank_workspace_bytes(p)
    ws = torch.empty(nb, dtype=torch.uint8, device=dev) if nb else None
    with torch.cuda.device(dev):
        call("dsc_fwd_lowrank_chunk", p, _ptr(x_prev), _ptr(x), _ptr(z), _ptr(U), _ptr(y), _ptr(ws), nb,
             int(out is not None), _stream(dev))
    return y


def dsc_bwd_lowrank_chunk(x, z, U, dy, x_prev=None, dy_next=None, z_next=None, H=1, residual=True, out=None):
    """Returns (dx, dz, dU); dU (fp32) sums over this chunk's tokens."""
    dev = _check(x, z, U, dy, dtype=x.dtype)
    _halo_ok(dev, x.dtype, x_prev, dy_next, z_next)
    p = _lr_problem(x, z, U, H, residual)
    if out is not None:
        dx, dz, dU = out
    else:
        dx, dz = torch.empty_like(x), torch.empty_like(z)
        dU = torch.empty(U.shape, dtype=torch.float32, device=dev)
    nb = lib().dsc_bwd_lowrank_chunk_workspace_bytes(p)
    ws = torch.empty(nb, dtype=torch.uint8, device=dev) if nb else None
    with torch.cuda.device(dev):
        call("dsc_bwd_lowrank_chunk", p, _ptr(x_prev), _ptr(dy_next), _ptr(z_next), _ptr(x), _ptr(z), _ptr(U),
             _ptr(dy), _ptr(dx), _ptr(dz), _ptr(dU), _ptr(ws), nb, int(out is not None), _stream(dev))
    return dx, dz, dU


def dsc_fwd_static_chunk(x, ws, x_prev=None, residual=False, out=None):
    dev = _check(x, ws, dtype=x.dtype)
    _halo_ok(dev, x.dtype, x_prev)
    p = problem(x, ws.shape[1], 1, 0, residual)
    y = out if out is not None else torch.empty_like(x)
    with torch.cuda.device(dev):
        call("dsc_fwd_static_chunk", p, _ptr(x_prev), _ptr(x), _ptr(ws), _ptr(y), int(out is not None),
             _stream(dev))
    return y


def dsc_bwd_static_chunk(x, ws, dy, x_prev=None, dy_next=None, residual=False, out=None):
    """Returns (dx, dws); dws (fp32) sums over this chunk's tokens."""
    dev = _check(x, ws, dy, dtype=x.dtype)
    _halo_ok(dev, x.dtype, x_prev, dy_next)
    p = problem(x, ws.shape[1], 1, 0, residual)
    if out is not None:
        dx, dws = out
    else:
        dx = torch.empty_like(x)
        dws = torch.empty(ws.shape, dtype=torch.float32, device=dev)
    with torch.cuda.device(dev):
        nb = lib().dsc_bwd_static_workspace_bytes(p)
        scratch = torch.empty(max(nb, 16), dtype=torch.uint8, device=dev)
        call("dsc_bwd_static_chunk", p, _ptr(x_prev), _ptr(dy_next), _ptr(x), _ptr(ws), _ptr(dy), _ptr(dx),
             _ptr(dws), _ptr(scratch), nb, int(out is not None), _stream(dev))
    return dx, dws


# ---------------------------------------------------- first projection z = hV ---

def _proj_problem(x, h, V, U, H, residual):
    B, T, D = x.shape
    dm, R = V.shape
    if h.shape != (B, T, dm) or U.shape[0] != R or D % H or U.shape[1] % (D // H):
        raise ValueError("expected h [B,T,d_model], V [d_model,R], U [R,(D/H)*W]")
    return problem(x, U.shape[1] // (D // H), H, R, residual), dm


def dsc_fwd_lowrank_proj(x, h, V, U, H=1, residual=True):
    """z = hV formed by the library, then y as dsc_fwd_lowrank.  Returns (y, z)."""
    dev = _check(x, h, V, U, dtype=x.dtype)
    p, dm = _proj_problem(x, h, V, U, H, residual)
    y = torch.empty_like(x)
    z = torch.empty(x.shape[0], x.shape[1], V.shape[1], dtype=x.dtype, device=dev)
    n = lib().dsc_fwd_lowrank_proj_workspace_bytes(p, dm)
    ws = torch.empty(n, dtype=torch.uint8, device=dev) if n else None
    with torch.cuda.device(dev):
        call("dsc_fwd_lowrank_proj", p, dm, _ptr(x), _ptr(h), _ptr(V), _ptr(U), _ptr(z), _ptr(y), _ptr(ws), n,
             _stream(dev))
    return y, z


def dsc_bwd_lowrank_proj(x, h, V, z, U, dy, H=1, residual=True):
    """Returns (dx, dh, dV, dU); dV and dU are fp32."""
    dev = _check(x, h, V, z, U, dy, dtype=x.dtype)
    p, dm = _proj_problem(x, h, V, U, H, residual)
    dx, dh = torch.empty_like(x), torch.empty_like(h)
    dV = torch.empty(V.shape, dtype=torch.float32, device=dev)
    dU = torch.empty(U.shape, dtype=torch.float32, device=dev)
    n = lib().dsc_bwd_lowrank_proj_workspace_bytes(p, dm)
    ws = torch.empty(n, dtype=torch.uint8, device=dev)
    with torch.cuda.device(dev):
        call("dsc_bwd_lowrank_proj", p, dm, _ptr(x), _ptr(h), _ptr(V), _ptr(z), _ptr(U), _ptr(dy), _ptr(dx), _ptr(dh),
             _ptr(dV), _ptr(dU), _ptr(ws), n, _stream(dev))
    return dx, dh, dV, dU


# ------------------------------------------------------------------ autograd ---

class DynamicShortConvHeadwise(torch.autograd.Function):
    """Autograd wrapper: forward and backward are the library's kernels."""

    @staticmethod
    def forward(ctx, x, w, residual=True):
        ctx.save_for_backward(x, w)
        ctx.residual = residual
        return dsc_fwd_headwise(x, w, residual)

    @staticmethod
    def backward(ctx, dy):
        x, w = ctx.saved_tensors
        dx, dw = dsc_bwd_headwise(x, w, dy.contiguous(), ctx.residual)
        return dx, dw, None


class DynamicShortConvLowRank(torch.autograd.Function):
    @staticmethod
    def forward(ctx, x, z, U, H=1, residual=True):
        ctx.save_for_backward(x, z, U)
        ctx.H, ctx.residual = H, residual
        return dsc_fwd_lowrank(x, z, U, H, residual)

    @staticmethod
    def backward(ctx, dy):
        x, z, U = ctx.saved_tensors
        dx, dz, dU = dsc_bwd_lowrank(x, z, U, dy.contiguous(), ctx.H, ctx.residual)
        return dx, dz, dU.to(U.dtype), None, None
