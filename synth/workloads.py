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


NAMED = {
    "tiny": TINY_F32,
    "qkv-headwise": QKV_HEADWISE,
    "qkv-lowrank": QKV_LOWRANK,
    "all-linear-headwise": ALL_LINEAR_HEADWISE,
    "all-linear-lowrank": ALL_LINEAR_LOWRANK,
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
