"""Workload shapes and the input recipe for the dynamic short convolution.

Shapes follow the placements the pages describe ("Dynamic Short Convolutions
Improve Transformers", summary pages, section Methodology / Placement): the
convolution on the concatenated Q, K, V projections of a d_model = 2048
Transformer (D = 3 * 2048 = 6144) and after every linear layer at ~2B scale
(MLP width D = 8192).  Values are synthetic: the pages' activations come from
models trained on Nemotron-CC, which are not available, so seeded normals of
the stated shapes stand in for them.

Recipe (all tensors are seeded by ``synth.make_tensor``):
  x, z, dy ~ N(0, 1)
  w (head-wise filters [B, T, D/H, W]) and static filters [D, W] ~ N(0, 1/W)
  U ([R, (D/H) * W]) ~ N(0, 1/(R * W))
The second parameter of N(.,.) is the variance.
"""

from __future__ import annotations

import math
from dataclasses import dataclass, replace

from . import BF16, F32, TID_DY, TID_H, TID_STATE, TID_U, TID_V, TID_W, TID_WS, TID_X, TID_Z, make_tensor

HEADWISE = "headwise"
LOWRANK = "lowrank"
STATIC = "static"


@dataclass(frozen=True)
class Workload:
    name: str
    variant: str
    B: int
    T: int
    D: int
    W: int
    H: int = 1
    R: int = 0
    dtype: str = BF16
    residual: int = 1
    seed: int = 0
    # "": plain batch rows; "varlen": one row of packed documents (mean length
    # doc_mean); "chunk": each row a middle time chunk of longer sequences
    # (halos on both sides); "proj": low-rank filters from h [B,T,d_model] and V
    mode: str = ""
    doc_mean: int = 0
    d_model: int = 0

    @property
    def G(self) -> int:
        return self.D // self.H

    @property
    def tokens(self) -> int:
        return self.B * self.T

    def with_(self, **kw) -> "Workload":
        return replace(self, **kw)


def make_inputs(wl: Workload) -> dict:
    """Seeded inputs of a workload, in storage form (fp32 arrays or bf16 bits)."""
    dt = wl.dtype
    out = {
        "x": make_tensor(wl.seed, TID_X, (wl.B, wl.T, wl.D), 1.0, dt),
        "dy": make_tensor(wl.seed, TID_DY, (wl.B, wl.T, wl.D), 1.0, dt),
    }
    if wl.variant == HEADWISE:
        out["w"] = make_tensor(wl.seed, TID_W, (wl.B, wl.T, wl.G, wl.W), 1.0 / math.sqrt(wl.W), dt)
    elif wl.variant == LOWRANK:
        out["z"] = make_tensor(wl.seed, TID_Z, (wl.B, wl.T, wl.R), 1.0, dt)
        out["U"] = make_tensor(wl.seed, TID_U, (wl.R, wl.G * wl.W), 1.0 / math.sqrt(wl.R * wl.W), dt)
    elif wl.variant == STATIC:
        out["ws"] = make_tensor(wl.seed, TID_WS, (wl.D, wl.W), 1.0 / math.sqrt(wl.W), dt)
    else:
        raise ValueError(wl.variant)
    return out


# The five workloads the dynamic-conv kernels are measured and checked on.
TINY_F32 = Workload("tiny-f32 B1 T64 D64 W4 H1", HEADWISE, 1, 64, 64, 4, H=1, dtype=F32)
QKV_HEADWISE = Workload("qkv-headwise B8 T2048 D6144 W4 H16", HEADWISE, 8, 2048, 6144, 4, H=16)
QKV_LOWRANK = Workload("qkv-lowrank B8 T2048 D6144 W4 H1 R32", LOWRANK, 8, 2048, 6144, 4, H=1, R=32)
ALL_LINEAR_HEADWISE = Workload("all-linear-headwise B4 T4096 D8192 W4 H64", HEADWISE, 4, 4096, 8192, 4, H=64)
ALL_LINEAR_LOWRANK = Workload("all-linear-lowrank B4 T4096 D8192 W4 H64 R64", LOWRANK, 4, 4096, 8192, 4, H=64, R=64)


def sweep_workloads() -> list:
    """Width/length sweep: B=1, T=16384, D=4096, bf16; each dynamic variant
    next to the static-filter conv on the same shapes.  Low-rank uses H=1."""
    out = []
    for W in (2, 3, 4, 8):
        for H in (1, 16, 128):
            out.append(Workload(f"sweep-headwise W{W} H{H}", HEADWISE, 1, 16384, 4096, W, H=H))
        for R in (16, 64):
            out.append(Workload(f"sweep-lowrank W{W} R{R}", LOWRANK, 1, 16384, 4096, W, H=1, R=R))
        out.append(Workload(f"sweep-static W{W}", STATIC, 1, 16384, 4096, W))
    return out


# Decode: one new token for each of B sequences (T = 1), the Q/K/V width;
# the inputs, outputs and state of one step (~200 MB) exceed L2.
DECODE_QKV_HEADWISE = Workload("decode-qkv-headwise B2048 D6144 W4 H16", HEADWISE, 2048, 1, 6144, 4, H=16)
DECODE_QKV_LOWRANK = Workload("decode-qkv-lowrank B2048 D6144 W4 H1 R32", LOWRANK, 2048, 1, 6144, 4, H=1, R=32)
DECODE_STATIC = Workload("decode-static B2048 D6144 W4", STATIC, 2048, 1, 6144, 4)

DECODE = {
    "decode-qkv-headwise": DECODE_QKV_HEADWISE,
    "decode-qkv-lowrank": DECODE_QKV_LOWRANK,
    "decode-static": DECODE_STATIC,
}


def decode_state(wl):
    """A seeded decode state [B, W-1, D] (the last W-1 inputs of each sequence)."""
    return make_tensor(wl.seed, TID_STATE, (wl.B, wl.W - 1, wl.D), 1.0, wl.dtype)


# The next rows on the same Q/K/V shapes: the same tokens as packed
# documents (variable-length batch), as middle time chunks of longer
# sequences (context parallelism), and the low-rank filters with their first
# projection from a d_model = 2048 hidden state.
QKV_HEADWISE_VARLEN = Workload("qkv-headwise-varlen B1 T16384 D6144 W4 H16 docs~1024", HEADWISE, 1, 16384, 6144, 4,
                               H=16, mode="varlen", doc_mean=1024)
QKV_HEADWISE_CHUNK = Workload("qkv-headwise-chunk B8 T2048 D6144 W4 H16 halos", HEADWISE, 8, 2048, 6144, 4, H=16,
                              mode="chunk")
QKV_LOWRANK_PROJ = Workload("qkv-lowrank-proj B8 T2048 D6144 W4 H1 R32 d2048", LOWRANK, 8, 2048, 6144, 4, H=1, R=32,
                            mode="proj", d_model=2048)

NAMED = {
    "tiny": TINY_F32,
    "qkv-headwise": QKV_HEADWISE,
    "qkv-lowrank": QKV_LOWRANK,
    "all-linear-headwise": ALL_LINEAR_HEADWISE,
    "all-linear-lowrank": ALL_LINEAR_LOWRANK,
    "qkv-headwise-varlen": QKV_HEADWISE_VARLEN,
    "qkv-headwise-chunk": QKV_HEADWISE_CHUNK,
    "qkv-lowrank-proj": QKV_LOWRANK_PROJ,
}


def projection_inputs(wl: Workload, d_model: int) -> dict:
    """The hidden state and first projection of the low-rank filter generator
    (w(t) = h_t V U): h [B, T, d_model] ~ N(0, 1) and V [d_model, R] ~
    N(0, 1/d_model), so that z = hV has unit variance like the z of the
    recipe above."""
    return {
        "h": make_tensor(wl.seed, TID_H, (wl.B, wl.T, d_model), 1.0, wl.dtype),
        "V": make_tensor(wl.seed, TID_V, (d_model, wl.R), 1.0 / math.sqrt(d_model), wl.dtype),
    }


def doc_lengths(T: int, mean: int, seed: int = 0) -> list:
    """Seeded document lengths summing to T: geometric with the given mean
    (a long-tailed mix of short and long documents, as in web text), the
    last one cut to fit.  The pages' documents (Nemotron-CC) are not
    available; this stands in for their length mix."""
    import numpy as np

    rng = np.random.default_rng(1000003 * seed + 17)
    out, left = [], T
    while left > 0:
        n = int(min(left, max(1, rng.geometric(1.0 / mean))))
        out.append(n)
        left -= n
    return out


def chunk_halos(wl: Workload) -> dict:
    """Seeded halo rows of a middle time chunk: x of the W-1 tokens before it,
    dy and the filters (head-wise w or low-rank z) of the W-1 after it."""
    dt, S = wl.dtype, max(wl.W - 1, 1)
    out = {"x_prev": make_tensor(wl.seed + 7919, TID_X, (wl.B, S, wl.D), 1.0, dt),
           "dy_next": make_tensor(wl.seed + 7919, TID_DY, (wl.B, S, wl.D), 1.0, dt)}
    if wl.variant == HEADWISE:
        out["w_next"] = make_tensor(wl.seed + 7919, TID_W, (wl.B, S, wl.G, wl.W), 1.0 / math.sqrt(wl.W), dt)
    elif wl.variant == LOWRANK:
        out["z_next"] = make_tensor(wl.seed + 7919, TID_Z, (wl.B, S, wl.R), 1.0, dt)
    return out
