"""Context parallelism on CPU: three gloo ranks each hold one time chunk of
the same sequences and exchange halo rows with their neighbours
(``input_dependent_short_b200.context_parallel``).  Checked: every rank
receives exactly its neighbours' edge rows (none at the sequence ends), and
the fp64 oracle run on each chunk with the exchanged halos reproduces the
whole sequences' outputs, with the chunks' dU summing to the whole dU.
The GPU side of the same calls (the dsc_*_chunk entry points) is checked in
tests/test_edges_gpu.py."""

import os
import socket

import numpy as np
import pytest
import torch
import torch.multiprocessing as mp

LENS = (5, 4, 6)
B, D, W, H, R = 2, 6, 4, 2, 3


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    p = s.getsockname()[1]
    s.close()
    return p


def _full_inputs():
    rng = np.random.default_rng(11)
    L, G = sum(LENS), D // H
    f32 = lambda *s: rng.standard_normal(s).astype(np.float32)  # noqa: E731
    return dict(x=f32(B, L, D), dy=f32(B, L, D), w=f32(B, L, G, W), z=f32(B, L, R), U=f32(R, G * W))


def _rank(rank, world, port, q):
    import torch.distributed as dist

    import oracle
    from input_dependent_short_b200 import context_parallel as cp

    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        full = _full_inputs()
        starts = np.concatenate([[0], np.cumsum(LENS)])
        t0, t1 = starts[rank], starts[rank + 1]
        mine = {k: torch.from_numpy(np.ascontiguousarray(v[:, t0:t1])) for k, v in full.items() if k != "U"}
        # halos over the process group
        r1, x_prev = cp.start_prev_halo(mine["x"], W)
        r2, nxt = cp.start_next_halo([mine["dy"], mine["w"], mine["z"]], W)
        cp.wait(r1 + r2)
        ok = {}
        ok["x_prev"] = (x_prev is None) if rank == 0 else np.array_equal(x_prev.numpy(), full["x"][:, t0 - W + 1:t0])
        if rank == world - 1:
            ok["next"] = nxt is None
        else:
            ok["next"] = all(np.array_equal(h.numpy(), full[k][:, t1:t1 + W - 1]) for h, k in zip(nxt, ("dy", "w", "z")))
        # the oracle on this chunk with the exchanged halos
        xp = None if x_prev is None else x_prev.numpy()
        dyn, wn, zn = (None, None, None) if nxt is None else (h.numpy() for h in nxt)
        P = oracle.problem(B, t1 - t0, D, W, H, R, 1)
        xs, dys = mine["x"].numpy(), mine["dy"].numpy()
        y = oracle.forward_chunk(P, oracle.HEADWISE, xs, xp, w=mine["w"].numpy())
        dx, dw = oracle.backward_chunk(P, oracle.HEADWISE, xs, dys, xp, dyn, w=mine["w"].numpy(), w_next=wn)
        dxl, dz, dU, _ = oracle.backward_chunk(P, oracle.LOWRANK, xs, dys, xp, dyn, z=mine["z"].numpy(), U=full["U"],
                                               z_next=zn)
        Pf = oracle.problem(B, sum(LENS), D, W, H, R, 1)
        yf = oracle.forward_headwise(Pf, full["x"], full["w"])
        dxf, dwf = oracle.backward_headwise(Pf, full["x"], full["w"], full["dy"])
        dxlf, dzf, _, _ = oracle.backward_lowrank(Pf, full["x"], full["z"], full["U"], full["dy"])
        sl = slice(t0, t1)
        ok["rows"] = (np.array_equal(y, yf[:, sl]) and np.array_equal(dx, dxf[:, sl]) and np.array_equal(dw, dwf[:, sl])
                      and np.allclose(dxl, dxlf[:, sl], rtol=0, atol=1e-12)
                      and np.allclose(dz, dzf[:, sl], rtol=0, atol=1e-12))
        # the chunks' dU sum to the whole sequences' (the gradient all-reduce)
        dU_t = torch.from_numpy(dU)
        dist.all_reduce(dU_t)
        ok["dU"] = np.allclose(dU_t.numpy(), oracle.backward_lowrank(Pf, full["x"], full["z"], full["U"],
                                                                        full["dy"])[2], rtol=0, atol=1e-10)
        q.put((rank, ok))
    finally:
        dist.barrier()
        dist.destroy_process_group()


def test_three_ranks_exchange_halos_and_reproduce_the_whole_sequence():
    world, port = len(LENS), _free_port()
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    procs = [ctx.Process(target=_rank, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    out = dict(q.get(timeout=180) for _ in range(world))
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    for rank, ok in sorted(out.items()):
        assert all(ok.values()), (rank, ok)


def test_chunks_shorter_than_the_halo_are_refused_before_any_exchange():
    from input_dependent_short_b200 import context_parallel as cp

    with pytest.raises(ValueError):
        cp.start_prev_halo(torch.zeros(1, 2, 8), 4)
    with pytest.raises(ValueError):
        cp.start_next_halo([torch.zeros(1, 2, 8)], 4)
    assert cp.start_prev_halo(torch.zeros(1, 2, 8), 1) == ([], None)
