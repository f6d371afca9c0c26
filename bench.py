#!/usr/bin/env python
"""Throughput of the dynamic short convolution's training hot path on B200.

One step = the forward and the backward of the convolution over one batch of
the named workload (default: the Q/K/V placement with head-wise filters,
B=8, T=2048, D=6144, W=4, H=16, bf16 with fp32 accumulation), called through
the C ABI of libdsc.so on torch's current stream with inputs resident in HBM.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME]
    python bench.py --impl reference ...     # the fp64 CPU oracle, same line

Prints ONE JSON line (rank 0).  `value` is whole-job tokens/s: every rank
processes its own batch (data parallel, no exchange on this path: "weak"
scaling), the time is the max over ranks of the device-measured time of K
steps.  Also reported: the roofline of the dominant kernel (the backward)
against the measured HBM copy bandwidth, the oracle on the host cores as a
CPU baseline, the same metric end to end with host buffers (H2D of the
inputs and D2H of all outputs inside the timed region; head-wise batches
pipelined row by row over three streams), SM clocks sampled during the timed
region, and the number of library kernels launched.  The default run also
times the other three training workloads (Q/K/V low-rank, all-linear
head-wise and low-rank) and reports each under `workloads` with its own
roofline; `--workloads none` skips them.
"""

from __future__ import annotations

import argparse
import datetime
import hashlib
import json
import os
import statistics
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

METRIC = "tokens/s and achieved HBM GB/s (fwd+bwd, bf16, W=4) vs B200 roofline"
FALLBACK_HBM_GBS = 6650.0
L2_BYTES = 126 * 2 ** 20


# ------------------------------------------------------------ rank helpers ---

def dist_env():
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return world, rank, local


def rank_workload(wl, rank: int):
    """Each rank draws its own batch (seed = base seed + rank)."""
    return wl.with_(seed=wl.seed + rank)


def max_over_ranks(x: float, world: int, device=None) -> float:
    if world == 1:
        return x
    import torch
    import torch.distributed as dist

    t = torch.tensor([x], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def job_tokens_per_s(tokens_per_rank_step: int, world: int, steps: int, max_ms: float) -> float:
    return tokens_per_rank_step * world * steps / (max_ms / 1e3)


# ------------------------------------------------------- algorithmic bytes ---

def step_bytes(wl):
    """Algorithmic HBM bytes of one forward and one backward launch (each
    tensor read or written once; w/z never materialised for low-rank)."""
    s = 2 if wl.dtype == "bf16" else 4
    N, D, GW, R = wl.B * wl.T, wl.D, (wl.D // wl.H) * wl.W, wl.R
    if wl.variant == "headwise":
        fb, bb = N * (2 * D + GW) * s, N * (3 * D + 2 * GW) * s
    elif wl.variant == "lowrank":
        u = R * GW * s
        fb, bb = N * (2 * D + R) * s + u, N * (3 * D + 2 * R) * s + u + 4 * R * GW
    else:
        fb, bb = N * 2 * D * s + D * wl.W * s, N * 3 * D * s + D * wl.W * s + 4 * D * wl.W
    if wl.mode == "proj":  # + h read and z written (forward); h read and dh written, V and dV (backward)
        dm = wl.d_model
        fb += N * (dm + R) * s + dm * R * s
        bb += 2 * N * dm * s + dm * R * (s + 4)
    elif wl.mode == "chunk":  # + the halo rows
        S = wl.W - 1
        fb += wl.B * S * D * s
        bb += wl.B * S * (2 * D + (wl.G * wl.W if wl.variant == "headwise" else R)) * s
    return fb, bb


def hbm_peak():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            return float(json.load(f)["hbm_gbs"]), "measured"
    except (OSError, KeyError, ValueError):
        return FALLBACK_HBM_GBS, "fallback"


KERNEL_SOURCES = {
    "decode": ("decode.cu", "lowrank_tc_dec.cu", "generic.cu", "lowrank_tc.cuh", "tc.cuh", "common.cuh",
               "kernels.cuh"),
    "headwise": ("conv_stream.cu", "common.cuh", "kernels.cuh"),
    "static": ("conv_stream.cu", "common.cuh", "kernels.cuh"),
    "lowrank": ("lowrank_tc_fwd.cu", "lowrank_tc_bwd.cu", "lowrank_tc.cuh", "tc.cuh", "lowrank.cu", "common.cuh",
                "kernels.cuh"),
}


def source_digest(variant: str) -> str:
    """sha256 of the sources of a variant's kernels, to match ncu traffic
    figures (profiles/traffic.txt) to the build they were taken on."""
    h = hashlib.sha256()
    for name in KERNEL_SOURCES[variant]:
        with open(os.path.join(ROOT, "input_dependent_short_b200", "csrc", name), "rb") as f:
            h.update(name.encode() + f.read())
    return h.hexdigest()[:16]


def ncu_traffic(kernel: str, workload: str, digest: str):
    """DRAM bytes per launch from profiles/traffic.txt, if taken on this source."""
    path = os.path.join(ROOT, "profiles", "traffic.txt")
    try:
        with open(path) as f:
            for line in f:
                parts = line.split("|")
                if len(parts) >= 4 and not line.startswith("#"):
                    k, w, d, b = (p.strip() for p in parts[:4])
                    if k == kernel and w == workload and d == digest:
                        return float(b)
    except OSError:
        pass
    return None


# ------------------------------------------------------------------ clocks ---

class ClockSampler:
    """SM clock and throttle reasons via NVML, sampled every 5 ms (read only)."""

    REASONS = {
        "hw_slowdown": 0x8, "sw_thermal_slowdown": 0x20, "hw_thermal_slowdown": 0x40, "sw_power_cap": 0x4,
        "hw_power_brake_slowdown": 0x80,
    }

    def __init__(self, index: int):
        self.samples, self.reasons, self.max_mhz = [], set(), None
        self._stop = threading.Event()
        try:
            import pynvml

            pynvml.nvmlInit()
            self.nv = pynvml
            self.h = pynvml.nvmlDeviceGetHandleByIndex(index)
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self.h, pynvml.NVML_CLOCK_SM)
        except Exception:  # noqa: BLE001
            self.nv = None

    def _run(self):
        while not self._stop.is_set():
            try:
                self.samples.append(self.nv.nvmlDeviceGetClockInfo(self.h, self.nv.NVML_CLOCK_SM))
                r = self.nv.nvmlDeviceGetCurrentClocksEventReasons(self.h)
                for name, bit in self.REASONS.items():
                    if r & bit:
                        self.reasons.add(name)
            except Exception:  # noqa: BLE001
                pass
            time.sleep(0.005)

    def __enter__(self):
        if self.nv:
            self.t = threading.Thread(target=self._run, daemon=True)
            self.t.start()
        return self

    def __exit__(self, *a):
        self._stop.set()
        if self.nv:
            self.t.join()

    def summary(self):
        if not self.samples:
            return {"sm_mhz": None, "sm_max_mhz": self.max_mhz, "reasons": sorted(self.reasons), "samples": 0}
        return {"sm_mhz": statistics.median(self.samples), "sm_max_mhz": self.max_mhz,
                "reasons": sorted(self.reasons), "samples": len(self.samples)}


# ---------------------------------------------------------------- the step ---

class Step:
    """Pre-allocated device buffers and the two C-ABI calls of one step."""

    def __init__(self, wl, host, device):
        import torch

        from input_dependent_short_b200 import _lib, ops

        self.wl, self.L = wl, _lib
        self.dev = device
        td = torch.bfloat16 if wl.dtype == "bf16" else torch.float32
        import synth

        host = dict(host)
        if wl.mode == "proj":  # the filters come from h and V: z is an output
            from synth import workloads as wls

            host.pop("z", None)
            host.update(wls.projection_inputs(wl, wl.d_model))
        self.h = {k: synth.to_torch(v, wl.dtype).pin_memory() for k, v in host.items()}
        self.d = {k: v.to(device) for k, v in self.h.items()}
        x = self.d["x"]
        if wl.mode == "varlen":
            import numpy as np

            from synth import workloads as wls

            lens = wls.doc_lengths(wl.T, wl.doc_mean, wl.seed)
            self.n_docs = len(lens)
            self.cu = torch.tensor(np.concatenate([[0], np.cumsum(lens)]), dtype=torch.int32, device=device)
        if wl.mode == "chunk":
            from synth import workloads as wls

            self.halo = {k: synth.to_torch(v, wl.dtype).to(device) for k, v in wls.chunk_halos(wl).items()}
        self.out = {"y": torch.empty_like(x), "dx": torch.empty_like(x)}
        if wl.variant == "headwise":
            self.out["dw"] = torch.empty_like(self.d["w"])
            self.p = ops.problem(x, wl.W, wl.H, 0, bool(wl.residual))
        elif wl.variant == "lowrank":
            if wl.mode == "proj":
                self.z = torch.empty(wl.B, wl.T, wl.R, dtype=x.dtype, device=device)
                self.out["dh"] = torch.empty_like(self.d["h"])
                self.out["dV"] = torch.empty(self.d["V"].shape, dtype=torch.float32, device=device)
            else:
                self.out["dz"] = torch.empty_like(self.d["z"])
            self.out["dU"] = torch.empty(self.d["U"].shape, dtype=torch.float32, device=device)
            self.p = ops.problem(x, wl.W, wl.H, wl.R, bool(wl.residual))
        else:
            self.out["dws"] = torch.empty(self.d["ws"].shape, dtype=torch.float32, device=device)
            self.p = ops.problem(x, wl.W, 1, 0, bool(wl.residual))
        lib = _lib.lib()
        self.nfw = self.nbw = 0
        if wl.variant == "lowrank" and wl.mode == "proj":
            self.nfw = lib.dsc_fwd_lowrank_proj_workspace_bytes(self.p, wl.d_model)
            self.nbw = lib.dsc_bwd_lowrank_proj_workspace_bytes(self.p, wl.d_model)
        elif wl.variant == "lowrank" and wl.mode == "varlen":
            self.nfw = lib.dsc_fwd_lowrank_workspace_bytes(self.p)
            self.nbw = lib.dsc_bwd_lowrank_varlen_workspace_bytes(self.p, self.n_docs)
        elif wl.variant == "lowrank" and wl.mode == "chunk":
            self.nfw = lib.dsc_fwd_lowrank_workspace_bytes(self.p)
            self.nbw = lib.dsc_bwd_lowrank_chunk_workspace_bytes(self.p)
        elif wl.variant == "lowrank":
            self.nfw = lib.dsc_fwd_lowrank_workspace_bytes(self.p)
            self.nbw = lib.dsc_bwd_lowrank_workspace_bytes(self.p)
        elif wl.variant == "static":
            self.nbw = lib.dsc_bwd_static_workspace_bytes(self.p)
        self.fws = torch.empty(max(self.nfw, 16), dtype=torch.uint8, device=device)
        self.bws = torch.empty(max(self.nbw, 16), dtype=torch.uint8, device=device)
        self.out_h = {k: torch.empty(v.shape, dtype=v.dtype).pin_memory() for k, v in self.out.items()}
        self.td = td

    def fwd(self, stream):
        d, o, L = self.d, self.out, self.L
        if self.wl.mode:
            return self.fwd_mode(stream)
        if self.wl.variant == "headwise":
            L.call("dsc_fwd_headwise", self.p, d["x"].data_ptr(), d["w"].data_ptr(), o["y"].data_ptr(), stream)
        elif self.wl.variant == "lowrank":
            L.call("dsc_fwd_lowrank", self.p, d["x"].data_ptr(), d["z"].data_ptr(), d["U"].data_ptr(),
                   o["y"].data_ptr(), self.fws.data_ptr(), self.nfw, stream)
        else:
            L.call("dsc_fwd_static", self.p, d["x"].data_ptr(), d["ws"].data_ptr(), o["y"].data_ptr(), stream)

    def bwd(self, stream):
        d, o, L = self.d, self.out, self.L
        if self.wl.mode:
            return self.bwd_mode(stream)
        if self.wl.variant == "headwise":
            L.call("dsc_bwd_headwise", self.p, d["x"].data_ptr(), d["w"].data_ptr(), d["dy"].data_ptr(),
                   o["dx"].data_ptr(), o["dw"].data_ptr(), stream)
        elif self.wl.variant == "lowrank":
            L.call("dsc_bwd_lowrank", self.p, d["x"].data_ptr(), d["z"].data_ptr(), d["U"].data_ptr(),
                   d["dy"].data_ptr(), o["dx"].data_ptr(), o["dz"].data_ptr(), o["dU"].data_ptr(),
                   self.bws.data_ptr(), self.nbw, stream)
        else:
            L.call("dsc_bwd_static", self.p, d["x"].data_ptr(), d["ws"].data_ptr(), d["dy"].data_ptr(),
                   o["dx"].data_ptr(), o["dws"].data_ptr(), self.bws.data_ptr(), self.nbw, stream)

    # ---- the next rows: packed documents, middle chunks, first projection
    def fwd_mode(self, stream):
        d, o, L, wl, P = self.d, self.out, self.L, self.wl, lambda t: t.data_ptr()
        if wl.mode == "varlen":
            if wl.variant == "headwise":
                L.call("dsc_fwd_headwise_varlen", self.p, P(self.cu), self.n_docs, P(d["x"]), P(d["w"]), P(o["y"]), stream)
            elif wl.variant == "lowrank":
                L.call("dsc_fwd_lowrank_varlen", self.p, P(self.cu), self.n_docs, P(d["x"]), P(d["z"]), P(d["U"]),
                       P(o["y"]), P(self.fws), self.nfw, stream)
            else:
                L.call("dsc_fwd_static_varlen", self.p, P(self.cu), self.n_docs, P(d["x"]), P(d["ws"]), P(o["y"]), stream)
        elif wl.mode == "chunk":
            xp = P(self.halo["x_prev"])
            if wl.variant == "headwise":
                L.call("dsc_fwd_headwise_chunk", self.p, xp, P(d["x"]), P(d["w"]), P(o["y"]), 0, stream)
            elif wl.variant == "lowrank":
                L.call("dsc_fwd_lowrank_chunk", self.p, xp, P(d["x"]), P(d["z"]), P(d["U"]), P(o["y"]), P(self.fws),
                       self.nfw, 0, stream)
            else:
                L.call("dsc_fwd_static_chunk", self.p, xp, P(d["x"]), P(d["ws"]), P(o["y"]), 0, stream)
        else:  # proj
            L.call("dsc_fwd_lowrank_proj", self.p, wl.d_model, P(d["x"]), P(d["h"]), P(d["V"]), P(d["U"]), P(self.z),
                   P(o["y"]), P(self.fws), self.nfw, stream)

    def bwd_mode(self, stream):
        d, o, L, wl, P = self.d, self.out, self.L, self.wl, lambda t: t.data_ptr()
        if wl.mode == "varlen":
            if wl.variant == "headwise":
                L.call("dsc_bwd_headwise_varlen", self.p, P(self.cu), self.n_docs, P(d["x"]), P(d["w"]), P(d["dy"]),
                       P(o["dx"]), P(o["dw"]), stream)
            elif wl.variant == "lowrank":
                L.call("dsc_bwd_lowrank_varlen", self.p, P(self.cu), self.n_docs, P(d["x"]), P(d["z"]), P(d["U"]),
                       P(d["dy"]), P(o["dx"]), P(o["dz"]), P(o["dU"]), P(self.bws), self.nbw, stream)
            else:
                L.call("dsc_bwd_static_varlen", self.p, P(self.cu), self.n_docs, P(d["x"]), P(d["ws"]), P(d["dy"]),
                       P(o["dx"]), P(o["dws"]), P(self.bws), self.nbw, stream)
        elif wl.mode == "chunk":
            h = self.halo
            if wl.variant == "headwise":
                L.call("dsc_bwd_headwise_chunk", self.p, P(h["x_prev"]), P(h["dy_next"]), P(h["w_next"]), P(d["x"]),
                       P(d["w"]), P(d["dy"]), P(o["dx"]), P(o["dw"]), 0, stream)
            elif wl.variant == "lowrank":
                L.call("dsc_bwd_lowrank_chunk", self.p, P(h["x_prev"]), P(h["dy_next"]), P(h["z_next"]), P(d["x"]),
                       P(d["z"]), P(d["U"]), P(d["dy"]), P(o["dx"]), P(o["dz"]), P(o["dU"]), P(self.bws), self.nbw, 0,
                       stream)
            else:
                L.call("dsc_bwd_static_chunk", self.p, P(h["x_prev"]), P(h["dy_next"]), P(d["x"]), P(d["ws"]),
                       P(d["dy"]), P(o["dx"]), P(o["dws"]), P(self.bws), self.nbw, 0, stream)
        else:  # proj
            L.call("dsc_bwd_lowrank_proj", self.p, wl.d_model, P(d["x"]), P(d["h"]), P(d["V"]), P(self.z), P(d["U"]),
                   P(d["dy"]), P(o["dx"]), P(o["dh"]), P(o["dV"]), P(o["dU"]), P(self.bws), self.nbw, stream)

    def h2d(self):
        for k, v in self.h.items():
            self.d[k].copy_(v, non_blocking=True)

    def d2h(self):
        for k, v in self.out.items():
            self.out_h[k].copy_(v, non_blocking=True)

    # ---- end to end by batch row: rows are independent sequences, so a row's
    # copies and kernels can overlap another row's.  Only for head-wise filters:
    # the low-rank dU and the static dws sum over every row of the batch.
    def row_chunks(self):
        plain = self.wl.variant == "headwise" and not self.wl.mode
        return self.wl.B if plain and self.wl.B > 1 else 1

    def run_row(self, i, stream):
        """H2D of row i's inputs, its forward and backward (one C-ABI call
        each, B = 1), D2H of its outputs; all on `stream` (a torch stream)."""
        import torch

        from input_dependent_short_b200 import ops

        if not hasattr(self, "p1"):
            x = self.d["x"]
            self.p1 = ops.problem(x[:1], self.wl.W, self.wl.H, 0, bool(self.wl.residual))
        with torch.cuda.stream(stream):
            for k, v in self.h.items():
                self.d[k][i].copy_(v[i], non_blocking=True)
            d, o, L, sp = self.d, self.out, self.L, stream.cuda_stream
            L.call("dsc_fwd_headwise", self.p1, d["x"][i].data_ptr(), d["w"][i].data_ptr(), o["y"][i].data_ptr(), sp)
            L.call("dsc_bwd_headwise", self.p1, d["x"][i].data_ptr(), d["w"][i].data_ptr(), d["dy"][i].data_ptr(),
                   o["dx"][i].data_ptr(), o["dw"][i].data_ptr(), sp)
            for k, v in self.out.items():
                self.out_h[k][i].copy_(v[i], non_blocking=True)

    def bytes_in(self):
        return sum(v.numel() * v.element_size() for v in self.h.values())

    def bytes_out(self):
        return sum(v.numel() * v.element_size() for v in self.out.values())


# ----------------------------------------------------------------- our arm ---

def run_dsc(args, wl0):
    import torch
    import torch.distributed as dist

    import synth  # noqa: F401
    from synth import workloads as wls

    world, rank, local = dist_env()
    if world > 1:
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=180))
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    wl = rank_workload(wl0, rank)
    host = wls.make_inputs(wl)
    step = Step(wl, host, dev)
    stream = torch.cuda.current_stream(dev).cuda_stream

    for _ in range(args.warmup):
        step.fwd(stream)
        step.bwd(stream)
    torch.cuda.synchronize(dev)

    K = args.steps
    ev = [[torch.cuda.Event(enable_timing=True) for _ in range(3)] for _ in range(K)]
    start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize(dev)
    lib = step.L.lib()
    n0 = lib.dsc_launch_count()
    with ClockSampler(local) as clocks:
        start.record()
        for i in range(K):
            ev[i][0].record()
            step.fwd(stream)
            ev[i][1].record()
            step.bwd(stream)
            ev[i][2].record()
        end.record()
        end.synchronize()
    torch.cuda.synchronize(dev)
    launches = lib.dsc_launch_count() - n0
    if world > 1:
        dist.barrier()
    ms_local = start.elapsed_time(end)
    fwd_ms = statistics.mean(ev[i][0].elapsed_time(ev[i][1]) for i in range(K))
    bwd_ms = statistics.mean(ev[i][1].elapsed_time(ev[i][2]) for i in range(K))
    ms = max_over_ranks(ms_local, world, dev)

    # end to end: inputs from pinned host memory, every output back to the host
    Ke = max(3, min(args.e2e_steps, K))
    e2e_ms, e2e_mode = time_e2e(step, Ke, stream, dev, world)
    tokens = wl.B * wl.T
    fb, bb = step_bytes(wl)
    peak, peak_src = hbm_peak()
    digest = source_digest(wl.variant)
    bwd_gbs = bb / (bwd_ms / 1e3) / 1e9
    fwd_gbs = fb / (fwd_ms / 1e3) / 1e9
    step_gbs = (fb + bb) / (ms / K / 1e3) / 1e9
    kname = {"headwise": "k_stream_bwd", "static": "k_stream_bwd",
             "lowrank": "k_lr_tc_bwd" if wl.dtype == "bf16" else "k_lr_bwd"}[wl.variant]
    traffic = ncu_traffic(kname, wl0.name, digest)

    result = None
    if rank == 0:
        result = {
            "metric": METRIC,
            "value": job_tokens_per_s(tokens, world, K, ms),
            "unit": "tokens/s",
            "n_gpus": world,
            "steps": K,
            "warmup": args.warmup,
            "ms_per_step": ms / K,
            "higher_is_better": True,
            "scaling": "weak",
            "vs_baseline": None,
            "dtype": "bf16" if wl.dtype == "bf16" else "f32",
            "accumulate": "f32",
            "data": "synthetic (seeded normals, seed = rank)",
            "config": {
                "workload": wl0.name, "variant": wl.variant, "B": wl.B, "T": wl.T, "D": wl.D, "W": wl.W,
                "H": wl.H, "R": wl.R, "residual": wl.residual, "pass": "forward + backward",
                "global_batch": wl.B * world, "seq_len": wl.T, "parallelism": f"dp{world}",
                "l2": "inputs larger than L2 (x, dy, y, dx are %.0f MB each; L2 126 MB), no flush"
                      % (tokens * wl.D * (2 if wl.dtype == "bf16" else 4) / 1e6),
            },
            "hbm_gbs_step": step_gbs,
            "kernels": {
                "fwd": {"us": fwd_ms * 1e3, "alg_bytes": fb, "gbs": fwd_gbs, "frac": fwd_gbs / peak},
                "bwd": {"us": bwd_ms * 1e3, "alg_bytes": bb, "gbs": bwd_gbs, "frac": bwd_gbs / peak},
            },
            "roofline": {
                "kernel": kname, "bound": "hbm", "achieved": bwd_gbs, "peak": peak, "unit": "GB/s",
                "frac": bwd_gbs / peak, "traffic": traffic, "peak_source": peak_src + " (hbm_gbs, copy)",
                "frac_of_8000": bwd_gbs / 8000.0, "step_frac": step_gbs / peak,
            },
            "e2e": {"value": job_tokens_per_s(tokens, world, Ke, e2e_ms), "unit": "tokens/s",
                    "h2d_bytes_per_step": step.bytes_in(), "d2h_bytes_per_step": step.bytes_out(),
                    "steps": Ke, "ms_per_step": e2e_ms / Ke, "pipeline": e2e_mode},
            "gpu_launches": launches,
            "clocks": clocks.summary(),
            "source_digest": digest,
        }
    # the other training workloads, each timed the same way (fewer steps), with
    # the oracle on a bounded sample of the same workload beside it (N = 1)
    others = {}
    if args.workloads:
        del step
        torch.cuda.empty_cache()
        for name in args.workloads.split(","):
            other = rank_workload(wls.NAMED[name], rank)
            others[name] = time_workload(other, args.other_steps, args.warmup, dev, world, peak)
            if world == 1 and not args.no_cpu_baseline:
                others[name]["cpu_baseline"] = cpu_baseline(other, wls.make_inputs(other.with_(B=1, T=min(other.T, 256))),
                                                            seconds=args.other_cpu_seconds, tokens=256)
            torch.cuda.empty_cache()
    if result is not None and others:
        result["workloads"] = others
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()
    return result, host, wl


def time_e2e(step, K, stream, dev, world):
    """Device time of K end-to-end steps: every step copies its inputs from
    pinned host memory and every output back.  Head-wise batches run row by
    row, round-robin over three streams, so that one row's H2D, another's
    kernels and a third's D2H overlap (both copy directions at once)."""
    import torch
    import torch.distributed as dist

    n = step.row_chunks()
    streams = [torch.cuda.Stream(dev) for _ in range(3)] if n > 1 else []

    def one():
        if n == 1:
            step.h2d(); step.fwd(stream); step.bwd(stream); step.d2h()
            return
        for i in range(n):
            step.run_row(i, streams[i % 3])

    for _ in range(2):
        one()
    torch.cuda.synchronize(dev)
    if world > 1:
        dist.barrier()
    main = torch.cuda.current_stream(dev)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(main)
    for s in streams:
        s.wait_event(e0)
    for _ in range(K):
        one()
    for s in streams:
        ev = torch.cuda.Event()
        ev.record(s)
        main.wait_event(ev)
    e1.record(main)
    e1.synchronize()
    mode = f"{n} batch rows over 3 streams (H2D, kernels and D2H of different rows overlap)" if n > 1 else "serial"
    return max_over_ranks(e0.elapsed_time(e1), world, dev), mode


def time_workload(wl, steps, warmup, dev, world, peak):
    """Forward + backward of another workload: device time per step, the two
    calls' HBM fractions and the roofline of its dominant kernel."""
    import torch

    from synth import workloads as wls

    step = Step(wl, wls.make_inputs(wl), dev)
    stream = torch.cuda.current_stream(dev).cuda_stream
    for _ in range(warmup):
        step.fwd(stream)
        step.bwd(stream)
    torch.cuda.synchronize(dev)
    ev = [[torch.cuda.Event(enable_timing=True) for _ in range(3)] for _ in range(steps)]
    lib = step.L.lib()
    n0 = lib.dsc_launch_count()
    for i in range(steps):
        ev[i][0].record()
        step.fwd(stream)
        ev[i][1].record()
        step.bwd(stream)
        ev[i][2].record()
    torch.cuda.synchronize(dev)
    launches = lib.dsc_launch_count() - n0
    fwd_ms = statistics.mean(ev[i][0].elapsed_time(ev[i][1]) for i in range(steps))
    bwd_ms = statistics.mean(ev[i][1].elapsed_time(ev[i][2]) for i in range(steps))
    ms = max_over_ranks(statistics.mean(ev[i][0].elapsed_time(ev[i][2]) for i in range(steps)), world, dev)
    fb, bb = step_bytes(wl)
    fg, bg = fb / (fwd_ms / 1e3) / 1e9, bb / (bwd_ms / 1e3) / 1e9
    kname = {"headwise": "k_stream_bwd", "static": "k_stream_bwd",
             "lowrank": "k_lr_tc_bwd" if wl.dtype == "bf16" else "k_lr_bwd"}[wl.variant]
    digest = source_digest(wl.variant)
    out = {
        "config": {"workload": wl.name, "variant": wl.variant, "B": wl.B, "T": wl.T, "D": wl.D, "W": wl.W,
                   "H": wl.H, "R": wl.R, **({"mode": wl.mode} if wl.mode else {}),
                   **({"d_model": wl.d_model} if wl.d_model else {}),
                   **({"documents": step.n_docs} if wl.mode == "varlen" else {})},
        "value": job_tokens_per_s(wl.B * wl.T, world, 1, ms), "unit": "tokens/s", "ms_per_step": ms,
        "steps": steps, "warmup": warmup, "gpu_launches": launches,
        "kernels": {"fwd": {"us": fwd_ms * 1e3, "alg_bytes": fb, "gbs": fg, "frac": fg / peak},
                    "bwd": {"us": bwd_ms * 1e3, "alg_bytes": bb, "gbs": bg, "frac": bg / peak}},
        "roofline": {"kernel": kname, "bound": "hbm", "achieved": bg, "peak": peak, "unit": "GB/s", "frac": bg / peak,
                     "traffic": ncu_traffic(kname, wl.name, digest), "step_frac": (fb + bb) / (ms / 1e3) / 1e9 / peak},
        "source_digest": digest,
    }
    del step
    return out


# ------------------------------------------------------------------ decode ---

DECODE_METRIC = "decode tokens/s and achieved HBM GB/s (one token per sequence, bf16, W=4) vs B200 roofline"


def decode_bytes(wl):
    """Algorithmic HBM bytes of one decode step: x, y, the state read and
    written (W-1 rows each), and the filters of the new tokens (head-wise w,
    low-rank z plus U once, static ws once)."""
    s = 2 if wl.dtype == "bf16" else 4
    B, D, W, G, R = wl.B, wl.D, wl.W, wl.G, wl.R
    base = B * D * s * (2 + 2 * (W - 1))
    if wl.variant == "headwise":
        return base + B * G * W * s
    if wl.variant == "lowrank":
        return base + B * R * s + R * G * W * s
    return base + D * W * s


class DecodeStep:
    """Device buffers and the C-ABI call of one decode step."""

    def __init__(self, wl, device):
        import torch

        import synth
        from input_dependent_short_b200 import _lib
        from synth import workloads as wls

        self.wl, self.L = wl, _lib
        host = wls.make_inputs(wl)
        B, D, W = wl.B, wl.D, wl.W
        h = {"x": host["x"].reshape(B, D)}
        if wl.variant == "headwise":
            h["w"] = host["w"].reshape(B, wl.G, W)
        elif wl.variant == "lowrank":
            h["z"], h["U"] = host["z"].reshape(B, wl.R), host["U"]
        else:
            h["ws"] = host["ws"]
        self.h = {k: synth.to_torch(v, wl.dtype).pin_memory() for k, v in h.items()}
        self.d = {k: v.to(device) for k, v in self.h.items()}
        self.state = synth.to_torch(wls.decode_state(wl), wl.dtype).to(device)
        self.y = torch.empty_like(self.d["x"])
        self.y_h = torch.empty(self.y.shape, dtype=self.y.dtype).pin_memory()
        self.p = _lib.DscProblem(B, 1, D, W, wl.H if wl.variant != "static" else 1, wl.R,
                                 _lib.DSC_BF16 if wl.dtype == "bf16" else _lib.DSC_F32, int(wl.residual))
        self.nws = _lib.lib().dsc_decode_lowrank_workspace_bytes(self.p) if wl.variant == "lowrank" else 0
        self.ws = torch.empty(max(self.nws, 16), dtype=torch.uint8, device=device)

    def run(self, stream):
        d, L = self.d, self.L
        if self.wl.variant == "headwise":
            L.call("dsc_decode_headwise", self.p, d["x"].data_ptr(), d["w"].data_ptr(), self.state.data_ptr(),
                   self.y.data_ptr(), stream)
        elif self.wl.variant == "lowrank":
            L.call("dsc_decode_lowrank", self.p, d["x"].data_ptr(), d["z"].data_ptr(), d["U"].data_ptr(),
                   self.state.data_ptr(), self.y.data_ptr(), self.ws.data_ptr(), self.nws, stream)
        else:
            L.call("dsc_decode_static", self.p, d["x"].data_ptr(), d["ws"].data_ptr(), self.state.data_ptr(),
                   self.y.data_ptr(), stream)

    def h2d(self):  # the new tokens' inputs and filters (U and ws are weights: resident)
        for k, v in self.h.items():
            if k not in ("U", "ws"):
                self.d[k].copy_(v, non_blocking=True)

    def bytes_in(self):
        return sum(v.numel() * v.element_size() for k, v in self.h.items() if k not in ("U", "ws"))


def run_decode(args, wl0):
    import torch
    import torch.distributed as dist

    world, rank, local = dist_env()
    if world > 1:
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=180))
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    wl = rank_workload(wl0, rank)
    st = DecodeStep(wl, dev)
    stream = torch.cuda.current_stream(dev).cuda_stream
    for _ in range(args.warmup):
        st.run(stream)
    torch.cuda.synchronize(dev)
    K = args.steps
    ev = [[torch.cuda.Event(enable_timing=True) for _ in range(2)] for _ in range(K)]
    start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize(dev)
    lib = st.L.lib()
    n0 = lib.dsc_launch_count()
    with ClockSampler(local) as clocks:
        start.record()
        for i in range(K):
            ev[i][0].record()
            st.run(stream)
            ev[i][1].record()
        end.record()
        end.synchronize()
    torch.cuda.synchronize(dev)
    launches = lib.dsc_launch_count() - n0
    if world > 1:
        dist.barrier()
    ms = max_over_ranks(start.elapsed_time(end), world, dev)
    call_ms = statistics.mean(ev[i][0].elapsed_time(ev[i][1]) for i in range(K))
    # end to end: the new tokens' inputs from pinned host memory, y back to the host
    Ke = max(3, min(args.e2e_steps, K))
    for _ in range(2):
        st.h2d(); st.run(stream); st.y_h.copy_(st.y, non_blocking=True)
    torch.cuda.synchronize(dev)
    if world > 1:
        dist.barrier()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record()
    for _ in range(Ke):
        st.h2d()
        st.run(stream)
        st.y_h.copy_(st.y, non_blocking=True)
    e1.record()
    e1.synchronize()
    e2e_ms = max_over_ranks(e0.elapsed_time(e1), world, dev)
    nb = decode_bytes(wl)
    peak, peak_src = hbm_peak()
    gbs = nb / (call_ms / 1e3) / 1e9
    digest = source_digest("decode")
    kname = ("k_lr_tc_dec" if wl.dtype == "bf16" else "k_decode_lr") if wl.variant == "lowrank" else "k_decode"
    traffic = ncu_traffic(kname, wl0.name, digest)
    result = None
    if rank == 0:
        result = {
            "metric": DECODE_METRIC, "value": job_tokens_per_s(wl.B, world, K, ms), "unit": "tokens/s",
            "n_gpus": world, "steps": K, "warmup": args.warmup, "ms_per_step": ms / K, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "bf16" if wl.dtype == "bf16" else "f32",
            "accumulate": "f32", "data": "synthetic (seeded normals, seed = rank)",
            "config": {"workload": wl0.name, "variant": wl.variant, "B": wl.B, "D": wl.D, "W": wl.W, "H": wl.H,
                       "R": wl.R, "residual": wl.residual, "pass": "decode step (one token per sequence)",
                       "global_batch": wl.B * world, "parallelism": f"dp{world}",
                       "l2": "step bytes %.0f MB > L2 126 MB, no flush" % (nb / 1e6)},
            "kernels": {"decode": {"us": call_ms * 1e3, "alg_bytes": nb, "gbs": gbs, "frac": gbs / peak}},
            "roofline": {"kernel": kname, "bound": "hbm", "achieved": gbs, "peak": peak, "unit": "GB/s",
                         "frac": gbs / peak, "traffic": traffic, "peak_source": peak_src + " (hbm_gbs, copy)"},
            "e2e": {"value": job_tokens_per_s(wl.B, world, Ke, e2e_ms), "unit": "tokens/s",
                    "h2d_bytes_per_step": st.bytes_in(), "d2h_bytes_per_step": st.y.numel() * st.y.element_size(),
                    "steps": Ke, "ms_per_step": e2e_ms / Ke},
            "gpu_launches": launches, "clocks": clocks.summary(), "source_digest": digest,
        }
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()
    return result


def decode_reference(wl, seconds=None, steps=None, warmup=0, sequences=64):
    """The oracle's decode step on `sequences` sequences of the workload: either
    for about `seconds`, or for `steps` timed steps after `warmup`."""
    import oracle
    from synth import workloads as wls

    sub = wl.with_(B=min(wl.B, sequences))
    host = wls.make_inputs(sub)
    B, D, W = sub.B, sub.D, sub.W
    P = oracle.problem(B, 1, D, W, sub.H if sub.variant != "static" else 1, sub.R, sub.residual)
    kind = {"headwise": oracle.HEADWISE, "lowrank": oracle.LOWRANK, "static": oracle.STATIC}[sub.variant]
    x, state = host["x"].reshape(B, D), wls.decode_state(sub)
    kw = {"headwise": lambda: dict(w=host["w"].reshape(B, sub.G, W)),
          "lowrank": lambda: dict(z=host["z"].reshape(B, sub.R), U=host["U"]),
          "static": lambda: dict(ws=host["ws"])}[sub.variant]()
    for _ in range(warmup):
        oracle.decode(P, kind, x, state, **kw)
    n, t0 = 0, time.perf_counter()
    while True:
        oracle.decode(P, kind, x, state, **kw)
        n += 1
        el = time.perf_counter() - t0
        if (steps is not None and n >= steps) or (seconds is not None and el >= seconds):
            break
    return n, B, el


# ----------------------------------------------------------- CPU baselines ---

def oracle_pass(wl, t):
    import oracle

    if wl.mode:
        return oracle_pass_mode(wl, t)
    if wl.variant == "headwise":
        P = oracle.problem_of(wl)
        oracle.forward_headwise(P, t["x"], t["w"])
        oracle.backward_headwise(P, t["x"], t["w"], t["dy"])
    elif wl.variant == "lowrank":
        P = oracle.problem_of(wl)
        oracle.forward_lowrank(P, t["x"], t["z"], t["U"])
        oracle.backward_lowrank(P, t["x"], t["z"], t["U"], t["dy"])
    else:
        P = oracle.problem(wl.B, wl.T, wl.D, wl.W, 1, 0, wl.residual)
        oracle.forward_static(P, t["x"], t["ws"])
        oracle.backward_static(P, t["x"], t["ws"], t["dy"])


def oracle_pass_mode(wl, t):
    """The oracle's forward + backward of the next rows' workloads (packed
    documents, a middle chunk with halos, the first projection)."""
    import numpy as np

    import oracle
    from synth import workloads as wls

    kind = {"headwise": oracle.HEADWISE, "lowrank": oracle.LOWRANK, "static": oracle.STATIC}[wl.variant]
    P = oracle.problem(wl.B, wl.T, wl.D, wl.W, wl.H if wl.variant != "static" else 1, wl.R, wl.residual)
    f = {k: t[k] for k in ("w", "z", "U", "ws") if k in t}
    if wl.mode == "proj":
        hv = wls.projection_inputs(wl, wl.d_model)
        oracle.forward_lowrank_proj(P, t["x"], hv["h"], hv["V"], t["U"])
        oracle.backward_lowrank_proj(P, t["x"], hv["h"], hv["V"], t["U"], t["dy"])
    elif wl.mode == "varlen":
        cu = np.concatenate([[0], np.cumsum(wls.doc_lengths(wl.T, wl.doc_mean, wl.seed))])
        oracle.forward_varlen(P, kind, t["x"], cu, **f)
        oracle.backward_varlen(P, kind, t["x"], t["dy"], cu, **f)
    else:  # chunk
        h = wls.chunk_halos(wl)
        nxt = {"headwise": {"w_next": h.get("w_next")}, "lowrank": {"z_next": h.get("z_next")}, "static": {}}
        oracle.forward_chunk(P, kind, t["x"], h["x_prev"], **f)
        oracle.backward_chunk(P, kind, t["x"], t["dy"], h["x_prev"], h["dy_next"], **f, **nxt[wl.variant])


def sample_of(wl, host, tokens):
    """The first `tokens` tokens of batch row 0 (a causal prefix: the same
    per-token work as the full workload)."""
    T = max(1, min(wl.T, tokens))
    sub = wl.with_(B=1, T=T)
    t = {}
    for k, v in host.items():
        if k in ("x", "dy", "w", "z"):
            t[k] = v[:1, :T].copy()
        else:
            t[k] = v
    return sub, t


def cpu_baseline(wl, host, seconds=10.0, tokens=2048):
    import oracle

    sub, t = sample_of(wl, host, tokens)
    n = 0
    t0 = time.perf_counter()
    while True:
        oracle_pass(sub, t)
        n += 1
        el = time.perf_counter() - t0
        if el >= seconds:
            break
    return {"value": n * sub.B * sub.T / el, "unit": "tokens/s", "cores": oracle.max_threads(), "kind": "oracle",
            "sample": f"{n} passes of fwd+bwd over the first {sub.T} tokens of batch row 0 "
                      f"({sub.D} channels, fp64 oracle, {el:.1f} s)"}


def run_reference(args, wl0):
    """The fp64 oracle on the host cores, same metric and config."""
    world, rank, _ = dist_env()
    if rank != 0:
        return None
    import oracle
    from synth import workloads as wls

    oracle.build()
    tokens = args.ref_tokens
    sub0 = wl0.with_(B=1, T=min(wl0.T, tokens))
    host = wls.make_inputs(sub0)
    sub, t = sample_of(sub0, host, tokens)
    for _ in range(args.warmup):
        oracle_pass(sub, t)
    t0 = time.perf_counter()
    for _ in range(args.steps):
        oracle_pass(sub, t)
    el = time.perf_counter() - t0
    v = args.steps * sub.T / el
    cores = oracle.max_threads()
    return {
        "impl": "reference", "metric": METRIC, "value": v, "unit": "tokens/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": el / args.steps * 1e3,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": {"workload": wl0.name, "variant": wl0.variant, "pass": "forward + backward",
                   "sample_tokens_per_step": sub.T},
        "cpu_baseline": {"value": v, "unit": "tokens/s", "cores": cores, "kind": "oracle",
                         "sample": f"each step: fwd+bwd over the first {sub.T} tokens of one sequence"},
        "e2e": {"value": v, "unit": "tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }


def main():
    ap = argparse.ArgumentParser(description=__doc__, formatter_class=argparse.RawDescriptionHelpFormatter)
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=500)
    ap.add_argument("--warmup", type=int, default=10)
    ap.add_argument("--impl", choices=["dsc", "reference"], default="dsc")
    ap.add_argument("--workload", default="qkv-headwise")
    ap.add_argument("--e2e-steps", type=int, default=10)
    ap.add_argument("--ref-tokens", type=int, default=256)
    ap.add_argument("--cpu-seconds", type=float, default=10.0)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--workloads", default=None,
                    help="comma-separated named workloads also timed in the same run (default: the other three "
                         "training workloads when --workload is the headline one; 'none' for none)")
    ap.add_argument("--other-steps", type=int, default=20)
    ap.add_argument("--other-cpu-seconds", type=float, default=3.0)
    args = ap.parse_args()
    if args.warmup < 3:
        ap.error("--warmup must be at least 3")
    from synth import workloads as wls

    if args.workload in wls.DECODE:
        wl0 = wls.DECODE[args.workload]
        if args.impl == "reference":
            world, rank, _ = dist_env()
            if rank == 0:
                import oracle

                oracle.build()
                n, B, el = decode_reference(wl0, steps=args.steps, warmup=args.warmup)
                v = n * B / el
                print(json.dumps({
                    "impl": "reference", "metric": DECODE_METRIC, "value": v, "unit": "tokens/s", "n_gpus": world,
                    "steps": args.steps, "warmup": args.warmup, "ms_per_step": el / n * 1e3,
                    "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
                    "data": "synthetic", "config": {"workload": wl0.name, "variant": wl0.variant,
                                                   "pass": "decode step", "sample_sequences": B},
                    "cpu_baseline": {"value": v, "unit": "tokens/s", "cores": oracle.max_threads(), "kind": "oracle",
                                     "sample": f"each step: one decode step of {B} sequences"},
                    "e2e": {"value": v, "unit": "tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}),
                    flush=True)
            return
        res = run_decode(args, wl0)
        if res is not None:
            if res["n_gpus"] == 1 and not args.no_cpu_baseline:
                import oracle

                n, B, el = decode_reference(wl0, seconds=args.cpu_seconds)
                res["cpu_baseline"] = {"value": n * B / el, "unit": "tokens/s", "cores": oracle.max_threads(),
                                       "kind": "oracle", "sample": f"{n} decode steps of {B} sequences "
                                                                   f"(fp64 oracle, {el:.1f} s)"}
            else:
                res["cpu_baseline"] = None
            print(json.dumps(res), flush=True)
        return
    if args.workload in wls.NAMED:
        wl0 = wls.NAMED[args.workload]
    else:
        matches = [w for w in wls.sweep_workloads() if w.name.replace(" ", "-") == args.workload]
        if not matches:
            ap.error(f"unknown workload {args.workload}")
        wl0 = matches[0]

    if args.workloads is None:
        args.workloads = ("qkv-lowrank,all-linear-headwise,all-linear-lowrank,qkv-headwise-varlen,"
                          "qkv-headwise-chunk,qkv-lowrank-proj" if args.workload == "qkv-headwise" else "none")
    if args.workloads == "none":
        args.workloads = ""
    for name in filter(None, args.workloads.split(",")):
        if name not in wls.NAMED:
            ap.error(f"unknown workload {name}")
    if args.impl == "reference":
        res = run_reference(args, wl0)
    else:
        res, host, wl = run_dsc(args, wl0)
        if res is not None:
            world = res["n_gpus"]
            if world == 1 and not args.no_cpu_baseline:
                res["cpu_baseline"] = cpu_baseline(wl, host, args.cpu_seconds)
            else:
                res["cpu_baseline"] = None
    if res is not None:
        print(json.dumps(res), flush=True)


if __name__ == "__main__":
    main()
