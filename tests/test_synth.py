"""The seeded input generator: determinism, distribution and rounding."""

import numpy as np
import torch

import synth
from synth import workloads


def test_splitmix64_reference_values():
    # SplitMix64 started at state 0: the published first outputs
    # (Steele, Lea & Flood 2014; also the seeding generator of xoshiro).
    out = synth.splitmix_outputs(0, 0, 3)
    assert [int(v) for v in out] == [0xE220A8397B1DCDAF, 0x6E789E6AA1B965F4, 0x06C45D188009454F]


def test_counter_based_and_deterministic():
    a = synth.normals_f64(0, 1, 1000)
    b = synth.normals_f64(0, 1, 400, start=600)
    np.testing.assert_array_equal(a[600:], b)
    np.testing.assert_array_equal(a, synth.normals_f64(0, 1, 1000))
    assert not np.array_equal(a, synth.normals_f64(0, 2, 1000))
    assert not np.array_equal(a, synth.normals_f64(1, 1, 1000))


def test_normal_moments():
    a = synth.normals_f64(7, 3, 1 << 20)
    assert abs(a.mean()) < 5e-3
    assert abs(a.var() - 1) < 5e-3
    assert abs(np.mean(a ** 4) - 3) < 5e-2


def test_bf16_rounding_matches_torch():
    a = (synth.normals_f64(0, 9, 100000) * 3).astype(np.float32)
    ours = synth.f32_to_bf16_bits(a)
    ref = torch.from_numpy(a).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    np.testing.assert_array_equal(ours, ref)
    back = synth.bf16_bits_to_f32(ours)
    np.testing.assert_array_equal(back, torch.from_numpy(a).to(torch.bfloat16).float().numpy())


def test_make_inputs_shapes_and_scales():
    wl = workloads.Workload("t", workloads.LOWRANK, 2, 64, 32, 4, H=2, R=8)
    t = workloads.make_inputs(wl)
    assert t["x"].shape == (2, 64, 32) and t["x"].dtype == np.uint16
    assert t["z"].shape == (2, 64, 8)
    assert t["U"].shape == (8, 16 * 4)
    u = synth.to_f64(t["U"], "bf16")
    assert abs(u.std() - 1 / np.sqrt(32)) < 0.03
    wh = workloads.make_inputs(workloads.TINY_F32)
    assert wh["w"].dtype == np.float32 and wh["w"].shape == (1, 64, 64, 4)
    assert abs(wh["w"].std() - 0.5) < 0.03
