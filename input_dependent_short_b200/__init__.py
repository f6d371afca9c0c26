"""B200-native dynamic short convolution (sm_100a CUDA kernels behind a C ABI).

The computation is a causal depthwise convolution whose width-W filter is
chosen per token, with head-wise tied, low-rank (w = zU formed on chip) and
static filters, forward and backward.  ``ops`` holds the PyTorch-facing
binding; ``_lib`` the ctypes view of ``libdsc.so``; ``build`` compiles it.
"""

from ._lib import DscError, DscProblem  # noqa: F401
from .ops import (  # noqa: F401
    DynamicShortConvHeadwise,
    DynamicShortConvLowRank,
    dsc_bwd_headwise,
    dsc_bwd_lowrank,
    dsc_bwd_static,
    dsc_check,
    dsc_fwd_headwise,
    dsc_fwd_lowrank,
    dsc_fwd_static,
)
