"""Context parallelism: the sequences are split along time, one chunk per
rank, and the convolution's W-1-token reach across a chunk edge is served by
exchanging halo rows with the neighbouring ranks.

The forward needs x of the W-1 tokens before the chunk (from rank - 1); the
backward needs dy and the filters of the W-1 tokens after it (from rank + 1).
Those are small point-to-point messages, B * (W-1) * D elements, sent with
``torch.distributed`` (NCCL over NVLink between GPUs; gloo on CPU).  The
calls below start the exchange, run the library's plain call on the chunk
while the halos travel, then let the library recompute only the outputs
next to the chunk edges (the ``edges_only`` form of the ``dsc_*_chunk``
entry points).  Token reductions (dU, dws) are per-rank sums; in training
they join the ordinary gradient all-reduce.

Every rank must call the same functions in the same order (they pair up
sends and receives); chunks must hold at least W-1 tokens, so that a halo
comes from one neighbour.
"""

from __future__ import annotations

import torch
import torch.distributed as dist


def _ranks(group):
    rank = dist.get_rank(group)
    world = dist.get_world_size(group)

    def glob(r):
        return r if group is None else dist.get_global_rank(group, r)

    return rank, world, glob


def _start(sends, recvs, group):
    ops = [dist.P2POp(dist.isend, t, peer, group) for t, peer in sends]
    ops += [dist.P2POp(dist.irecv, t, peer, group) for t, peer in recvs]
    return dist.batch_isend_irecv(ops) if ops else []


def start_prev_halo(x: torch.Tensor, W: int, group=None):
    """Send this chunk's last W-1 rows of x [B, T, D] to the next rank and
    receive the previous rank's.  Returns (requests, x_prev [B, W-1, D] or
    None on the first rank); wait on the requests before reading x_prev."""
    if W < 2:
        return [], None
    B, T = x.shape[:2]
    if T < W - 1:
        raise ValueError("a chunk must hold at least W-1 tokens")
    rank, world, glob = _ranks(group)
    sends, recvs, x_prev = [], [], None
    if rank + 1 < world:
        sends.append((x[:, T - (W - 1):].contiguous(), glob(rank + 1)))
    if rank > 0:
        x_prev = torch.empty((B, W - 1) + tuple(x.shape[2:]), dtype=x.dtype, device=x.device)
        recvs.append((x_prev, glob(rank - 1)))
    return _start(sends, recvs, group), x_prev


def start_next_halo(tensors, W: int, group=None):
    """Send the first W-1 rows of each tensor (dy and the filters, all
    [B, T, ...]) to the previous rank and receive the next rank's.  Returns
    (requests, list of [B, W-1, ...] tensors, or None on the last rank)."""
    if W < 2:
        return [], None
    rank, world, glob = _ranks(group)
    sends, recvs, nxt = [], [], None
    for t in tensors:
        if t.shape[1] < W - 1:
            raise ValueError("a chunk must hold at least W-1 tokens")
    if rank > 0:
        sends = [(t[:, :W - 1].contiguous(), glob(rank - 1)) for t in tensors]
    if rank + 1 < world:
        nxt = [torch.empty((t.shape[0], W - 1) + tuple(t.shape[2:]), dtype=t.dtype, device=t.device) for t in tensors]
        recvs = [(h, glob(rank + 1)) for h in nxt]
    return _start(sends, recvs, group), nxt


def wait(reqs):
    for r in reqs:
        r.wait()


# ------------------------------------------------------- the chunked calls ---

def fwd_headwise(x, w, residual=True, group=None):
    from . import ops

    reqs, x_prev = start_prev_halo(x, w.shape[3], group)
    y = ops.dsc_fwd_headwise(x, w, residual)
    wait(reqs)
    return y if x_prev is None else ops.dsc_fwd_headwise_chunk(x, w, x_prev, residual, out=y)


def bwd_headwise(x, w, dy, residual=True, group=None):
    """Returns (dx, dw) of this rank's chunk."""
    from . import ops

    W = w.shape[3]
    r1, x_prev = start_prev_halo(x, W, group)
    r2, nxt = start_next_halo([dy, w], W, group)
    dx, dw = ops.dsc_bwd_headwise(x, w, dy, residual)
    wait(r1 + r2)
    if x_prev is None and nxt is None:
        return dx, dw
    dy_next, w_next = nxt if nxt is not None else (None, None)
    return ops.dsc_bwd_headwise_chunk(x, w, dy, x_prev, dy_next, w_next, residual, out=(dx, dw))


def fwd_lowrank(x, z, U, H=1, residual=True, group=None):
    from . import ops

    W = U.shape[1] // (x.shape[2] // H)
    reqs, x_prev = start_prev_halo(x, W, group)
    y = ops.dsc_fwd_lowrank(x, z, U, H, residual)
    wait(reqs)
    return y if x_prev is None else ops.dsc_fwd_lowrank_chunk(x, z, U, x_prev, H, residual, out=y)


def bwd_lowrank(x, z, U, dy, H=1, residual=True, group=None):
    """Returns (dx, dz, dU); dU sums over this rank's tokens."""
    from . import ops

    W = U.shape[1] // (x.shape[2] // H)
    r1, x_prev = start_prev_halo(x, W, group)
    r2, nxt = start_next_halo([dy, z], W, group)
    out = ops.dsc_bwd_lowrank(x, z, U, dy, H, residual)
    wait(r1 + r2)
    if x_prev is None and nxt is None:
        return out
    dy_next, z_next = nxt if nxt is not None else (None, None)
    return ops.dsc_bwd_lowrank_chunk(x, z, U, dy, x_prev, dy_next, z_next, H, residual, out=out)


def fwd_static(x, ws, residual=False, group=None):
    from . import ops

    reqs, x_prev = start_prev_halo(x, ws.shape[1], group)
    y = ops.dsc_fwd_static(x, ws, residual)
    wait(reqs)
    return y if x_prev is None else ops.dsc_fwd_static_chunk(x, ws, x_prev, residual, out=y)


def bwd_static(x, ws, dy, residual=False, group=None):
    """Returns (dx, dws); dws sums over this rank's tokens."""
    from . import ops

    W = ws.shape[1]
    r1, x_prev = start_prev_halo(x, W, group)
    r2, nxt = start_next_halo([dy], W, group)
    out = ops.dsc_bwd_static(x, ws, dy, residual)
    wait(r1 + r2)
    if x_prev is None and nxt is None:
        return out
    return ops.dsc_bwd_static_chunk(x, ws, dy, x_prev, None if nxt is None else nxt[0], residual, out=out)
