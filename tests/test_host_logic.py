"""Host-side invariants the CUDA kernels rely on (no GPU needed)."""

from math import gcd

import pytest


def fast_path_mapping(D, H, V):
    """Groups per thread (GPT) or None, for the vectorised streaming kernels:
    a thread owns V channels; either H divides V, or H is a multiple of V with
    at most 32 lanes per group."""
    if D % V:
        return None
    if V % H == 0:
        return V // H
    if H % V == 0 and H // V <= 32:
        return 1
    return None


@pytest.mark.parametrize("elem,V", [(2, 8), (4, 4)], ids=["bf16", "f32"])
def test_filter_rows_are_aligned_to_their_compile_time_alignment(elem, V):
    """Every per-thread filter row w[b,t,g0:g0+GPT,:] starts at a multiple of
    gcd(16, GPT*W*elem) bytes, for a 16-byte aligned base: the token stride
    G*W*elem and each thread's group offset are multiples of that."""
    for D in range(V, 1025, V):
        for H in range(1, D + 1):
            if D % H:
                continue
            gpt = fast_path_mapping(D, H, V)
            if gpt is None:
                continue
            G = D // H
            for W in range(1, 9):
                A = gcd(16, gpt * W * elem)
                assert (G * W * elem) % A == 0, (D, H, W)
                for c0 in range(0, D, V):
                    assert ((c0 // H) * W * elem) % A == 0, (D, H, W, c0)


def test_fast_path_covers_the_measured_workloads():
    for D, H in [(6144, 16), (8192, 64), (6144, 1), (8192, 64), (4096, 1), (4096, 16), (4096, 128)]:
        assert fast_path_mapping(D, H, 8) is not None
    assert fast_path_mapping(24, 3, 8) is None   # generic kernels
    assert fast_path_mapping(20, 5, 8) is None
