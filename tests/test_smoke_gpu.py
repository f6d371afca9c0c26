"""The entry point's smoke run (one small forward + backward of every variant,
the tensor-core low-rank kernels included) against the oracle on cuda:0."""

import pytest


@pytest.mark.gpu
def test_smoke_entry_point():
    import __graft_entry__

    __graft_entry__.smoke()
