"""The N>1 path of bench.py on CPU: two gloo ranks, each with its own batch,
the timing reduced as the max over ranks and the job value aggregated over
ranks (data parallel; the path has no exchange step)."""

import os
import socket

import torch.multiprocessing as mp

import bench
from synth import workloads as wls


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    p = s.getsockname()[1]
    s.close()
    return p


def _rank(rank, world, port, q):
    import torch.distributed as dist

    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world),
                      LOCAL_RANK=str(rank))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    wl = bench.rank_workload(wls.TINY_F32, rank)
    t = wls.make_inputs(wl)
    ms = 10.0 + 5.0 * rank  # rank 1 is the slow one
    mx = bench.max_over_ranks(ms, world, "cpu")
    q.put((rank, wl.seed, float(t["x"].reshape(-1)[0]), mx, bench.dist_env()))
    dist.barrier()
    dist.destroy_process_group()


def test_two_ranks_shard_batches_and_take_the_max_time():
    world, port = 2, _free_port()
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    procs = [ctx.Process(target=_rank, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    out = sorted(q.get(timeout=120) for _ in range(world))
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    (r0, s0, x0, m0, env0), (r1, s1, x1, m1, env1) = out
    assert (s0, s1) == (0, 1)          # each rank draws its own batch
    assert x0 != x1
    assert m0 == m1 == 15.0            # max over ranks
    assert env0 == (2, 0, 0) and env1 == (2, 1, 1)
    # whole-job tokens/s = all ranks' tokens / the slowest rank's time
    assert bench.job_tokens_per_s(1000, 2, 10, 15.0) == 1000 * 2 * 10 / 0.015


def test_algorithmic_bytes_of_the_headline_workload():
    fb, bb = bench.step_bytes(wls.QKV_HEADWISE)
    N, D, GW = 8 * 2048, 6144, 384 * 4
    assert fb == N * (4 * D + 2 * GW)
    assert bb == N * (6 * D + 4 * GW)
    assert fb + bb == 1_157_627_904


def test_algorithmic_bytes_of_the_decode_workloads():
    """x and y, the state read and written (W-1 rows each), and the filters."""
    B, D, W, s = 2048, 6144, 4, 2
    base = B * D * s * (2 + 2 * (W - 1))
    assert bench.decode_bytes(wls.DECODE_QKV_HEADWISE) == base + B * 384 * W * s
    assert bench.decode_bytes(wls.DECODE_QKV_LOWRANK) == base + B * 32 * s + 32 * 6144 * W * s
    assert bench.decode_bytes(wls.DECODE_STATIC) == base + D * W * s
    assert bench.decode_bytes(wls.DECODE_QKV_HEADWISE) > 126 * 2 ** 20  # one step's bytes exceed L2


def test_decode_reference_arm_runs_the_oracle_on_a_sample():
    """The CPU arm of the decode workloads: the oracle's decode step on a
    bounded sample of sequences."""
    wl = wls.DECODE_QKV_LOWRANK.with_(B=8, D=256)
    n, B, el = bench.decode_reference(wl, steps=2, warmup=1, sequences=4)
    assert n == 2 and B == 4 and el > 0


def _dp_rank(rank, world, port, q):
    """Data parallel: rank r holds batch rows r, r+world, ...; the per-rank
    token reductions (low-rank dU, static dws), all-reduced, are the whole
    batch's."""
    import numpy as np
    import torch
    import torch.distributed as dist

    import oracle

    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        rng = np.random.default_rng(3)
        B, T, D, W, H, R = 4, 9, 6, 3, 2, 3
        x, dy, z = rng.standard_normal((B, T, D)), rng.standard_normal((B, T, D)), rng.standard_normal((B, T, R))
        U, ws = rng.standard_normal((R, (D // H) * W)), rng.standard_normal((D, W))
        rows = list(range(rank, B, world))
        mine = lambda a: np.ascontiguousarray(a[rows])  # noqa: E731
        P = oracle.problem(len(rows), T, D, W, H, R, 1)
        dU = torch.from_numpy(oracle.backward_lowrank(P, mine(x), mine(z), U, mine(dy))[2])
        dws = torch.from_numpy(oracle.backward_static(oracle.problem(len(rows), T, D, W, 1, 0, 1), mine(x), ws,
                                                      mine(dy))[1])
        dist.all_reduce(dU)
        dist.all_reduce(dws)
        Pf = oracle.problem(B, T, D, W, H, R, 1)
        ok = np.allclose(dU.numpy(), oracle.backward_lowrank(Pf, x, z, U, dy)[2], rtol=0, atol=1e-11)
        ok &= np.allclose(dws.numpy(), oracle.backward_static(oracle.problem(B, T, D, W, 1, 0, 1), x, ws, dy)[1],
                          rtol=0, atol=1e-11)
        q.put((rank, bool(ok)))
    finally:
        dist.barrier()
        dist.destroy_process_group()


def test_data_parallel_token_reductions_all_reduce_to_the_whole_batch():
    world, port = 2, _free_port()
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    procs = [ctx.Process(target=_dp_rank, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    out = dict(q.get(timeout=120) for _ in range(world))
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    assert out == {0: True, 1: True}


def test_reference_arm_prints_one_contract_line():
    """`bench.py --impl reference` (the oracle on the host cores, a bounded
    sample) prints one JSON line carrying the keys of the bench contract,
    with its own value repeated as the CPU baseline and as e2e (no copies)."""
    import json
    import subprocess
    import sys

    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    r = subprocess.run([sys.executable, "bench.py", "--impl", "reference", "--steps", "1", "--warmup", "3",
                        "--ref-tokens", "32"], cwd=root, capture_output=True, text=True, timeout=600)
    assert r.returncode == 0, r.stderr[-2000:]
    lines = [ln for ln in r.stdout.splitlines() if ln.startswith("{")]
    assert len(lines) == 1
    d = json.loads(lines[0])
    for k in ("impl", "metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step", "higher_is_better",
              "scaling", "vs_baseline", "dtype", "data", "config", "cpu_baseline", "e2e"):
        assert k in d, k
    assert d["impl"] == "reference" and d["n_gpus"] == 1 and d["steps"] == 1 and d["warmup"] == 3
    assert d["value"] > 0 and d["higher_is_better"] is True and d["vs_baseline"] is None
    assert d["config"]["workload"] == wls.QKV_HEADWISE.name
    cb = d["cpu_baseline"]
    assert cb["kind"] == "oracle" and cb["cores"] >= 1 and cb["sample"] and cb["value"] == d["value"]
    assert d["e2e"]["value"] == d["value"] and d["e2e"]["h2d_bytes_per_step"] == 0 and d["e2e"]["d2h_bytes_per_step"] == 0
