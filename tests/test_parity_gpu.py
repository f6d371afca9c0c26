"""Parity of the CUDA kernels (called through the C ABI) with the fp64 oracle.

Inputs are the seeded synthetic tensors of ``synth``; both sides see the
same bits.  Small shapes are compared element by element over whole tensors;
they span several tiles, ragged tails, T < W, every H regime (groups inside a
thread, groups across 2..32 lanes, non-power-of-two lanes per group, groups
wider than a warp, D not a multiple of the vector width), W = 1..8 and both
dtypes.  The full-size workloads are compared on sampled outputs that the
oracle evaluates one by one (always including the first and last tokens).
"""

import functools

import numpy as np
import pytest
import torch

import oracle
import synth
from synth import workloads as wls
from synth.workloads import HEADWISE, LOWRANK, STATIC, Workload

from helpers import TOL, assert_close, bound, rel_err, to_dev, to_host64

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.fail("no CUDA device: the -m gpu tests need a B200")
    import input_dependent_short_b200  # noqa: F401  (loads libdsc.so, fails loudly if missing)


def ops():
    from input_dependent_short_b200 import ops as o

    return o


# ------------------------------------------------------------ runners ---

def run_gpu(wl: Workload, t: dict):
    o = ops()
    dt = wl.dtype
    x, dy = to_dev(t["x"], dt), to_dev(t["dy"], dt)
    res = bool(wl.residual)
    out = {}
    if wl.variant == HEADWISE:
        w = to_dev(t["w"], dt)
        out["y"] = o.dsc_fwd_headwise(x, w, res)
        out["dx"], out["dw"] = o.dsc_bwd_headwise(x, w, dy, res)
    elif wl.variant == LOWRANK:
        z, U = to_dev(t["z"], dt), to_dev(t["U"], dt)
        out["y"] = o.dsc_fwd_lowrank(x, z, U, wl.H, res)
        out["dx"], out["dz"], out["dU"] = o.dsc_bwd_lowrank(x, z, U, dy, wl.H, res)
    else:
        ws = to_dev(t["ws"], dt)
        out["y"] = o.dsc_fwd_static(x, ws, res)
        out["dx"], out["dws"] = o.dsc_bwd_static(x, ws, dy, res)
    torch.cuda.synchronize()
    return out


def run_oracle(wl: Workload, t: dict):
    P = oracle.problem_of(wl)
    if wl.variant == HEADWISE:
        y = oracle.forward_headwise(P, t["x"], t["w"])
        dx, dw = oracle.backward_headwise(P, t["x"], t["w"], t["dy"])
        return dict(y=y, dx=dx, dw=dw)
    if wl.variant == LOWRANK:
        y = oracle.forward_lowrank(P, t["x"], t["z"], t["U"])
        dx, dz, dU, _ = oracle.backward_lowrank(P, t["x"], t["z"], t["U"], t["dy"])
        return dict(y=y, dx=dx, dz=dz, dU=dU)
    P = oracle.problem(wl.B, wl.T, wl.D, wl.W, 1, 0, wl.residual)
    y = oracle.forward_static(P, t["x"], t["ws"])
    dx, dws = oracle.backward_static(P, t["x"], t["ws"], t["dy"])
    return dict(y=y, dx=dx, dws=dws)


def check_full(wl: Workload):
    t = wls.make_inputs(wl)
    got = run_gpu(wl, t)
    ref = run_oracle(wl, t)
    errs = {}
    for k, r in ref.items():
        g = to_host64(got[k])
        assert g.shape == r.shape, k
        assert np.all(np.isfinite(g)), k
        errs[k] = assert_close(f"{wl.name}:{k}", g, r, wl.dtype, bound(k, wl.dtype))
    return errs


# ------------------------------------------------------- small shapes ---

def W_(name, variant, B, T, D, W, H=1, R=0, dtype="bf16", residual=1):
    return Workload(name, variant, B, T, D, W, H=H, R=R, dtype=dtype, residual=residual)


HEADWISE_SHAPES = [
    # (B, T, D, W, H): comment = regime for bf16 (V=8) / fp32 (V=4)
    (2, 37, 64, 4, 1),      # 8 / 4 groups per thread
    (2, 100, 256, 3, 16),   # 2 / 4 lanes per group
    (1, 300, 512, 4, 64),   # 8 / 16 lanes per group, many tiles, ragged tail
    (2, 70, 384, 2, 128),   # 16 / 32 lanes per group
    (1, 50, 1024, 4, 256),  # 32 lanes / generic (group wider than a warp)
    (2, 33, 96, 5, 24),     # 3 / 6 lanes per group (not a power of two)
    (1, 17, 48, 8, 2),      # 4 / 2 groups per thread, W = 8
    (1, 9, 24, 4, 3),       # generic: H neither divides nor is a multiple of V
    (3, 5, 20, 4, 5),       # generic: D not a multiple of the vector
    (2, 2, 64, 4, 16),      # T < W
    (1, 1, 64, 4, 1),       # T = 1
    (2, 40, 64, 1, 8),      # W = 1
    (1, 129, 256, 8, 1),    # W = 8 per-channel
    (1, 200, 128, 6, 32),
    (1, 77, 40, 7, 8),      # D = 40: 5 vectors of 8
    # groups of 16 or more lanes: the backward's reduce-scatter of dw (taps padded to 4 or 8)
    (1, 90, 256, 5, 128),   # 16 / 32 lanes, W = 5
    (1, 60, 256, 8, 128),   # 16 / 32 lanes, W = 8
    (2, 40, 512, 7, 256),   # 32 lanes / generic, W = 7
    (1, 70, 256, 3, 64),    # 8 / 16 lanes, W = 3
]


@pytest.mark.parametrize("dtype", ["bf16", "f32"])
@pytest.mark.parametrize("shape", HEADWISE_SHAPES, ids=lambda s: "B{}T{}D{}W{}H{}".format(*s))
def test_headwise_small(shape, dtype):
    B, T, D, W, H = shape
    check_full(W_("hw", HEADWISE, B, T, D, W, H, dtype=dtype))


@pytest.mark.parametrize("dtype", ["bf16", "f32"])
def test_headwise_no_residual(dtype):
    check_full(W_("hw-nores", HEADWISE, 2, 90, 128, 4, 16, dtype=dtype, residual=0))


STATIC_SHAPES = [(2, 100, 64, 4), (1, 50, 20, 3), (1, 300, 256, 1), (2, 64, 512, 2), (1, 130, 96, 8), (1, 3, 32, 5)]


@pytest.mark.parametrize("dtype", ["bf16", "f32"])
@pytest.mark.parametrize("residual", [0, 1])
@pytest.mark.parametrize("shape", STATIC_SHAPES, ids=lambda s: "B{}T{}D{}W{}".format(*s))
def test_static_small(shape, dtype, residual):
    B, T, D, W = shape
    check_full(W_("st", STATIC, B, T, D, W, dtype=dtype, residual=residual))


LOWRANK_SHAPES = [
    # (B, T, D, W, H, R)
    (1, 64, 64, 4, 1, 8),
    (2, 50, 96, 3, 4, 5),
    (1, 130, 256, 4, 16, 32),
    (2, 33, 128, 2, 64, 64),
    (1, 40, 48, 8, 1, 3),
    (2, 3, 64, 4, 8, 1),
    (1, 70, 40, 5, 5, 7),
    # shapes the tensor-core kernels take in bf16 (W in {1,2,3,4,8}, H | 64, D % 32H == 0)
    (2, 300, 256, 4, 8, 16),
    (1, 200, 2048, 2, 64, 32),
    (2, 129, 64, 8, 2, 48),
    (1, 128, 32, 1, 1, 20),
    (1, 131, 1024, 4, 32, 64),
    (1, 140, 512, 4, 16, 16),
    (2, 150, 2048, 4, 64, 32),
    (1, 260, 256, 8, 8, 24),
    # enough tiles that each tensor-core CTA walks several items: operand and
    # TMEM double buffers and the sub-tile ring wrap, items split between CTAs
    (4, 1024, 4096, 4, 1, 32),
    (2, 1000, 8192, 4, 64, 64),
    (2, 700, 2048, 8, 2, 48),
    (2, 600, 1024, 8, 1, 16),
    (2, 500, 4096, 2, 1, 32),
    # W = 3 (blocks of 32 groups: 96 of the 128 filter columns in use)
    (2, 300, 256, 3, 8, 16),
    (1, 200, 2048, 3, 1, 32),
    (2, 700, 2048, 3, 2, 48),
    (2, 500, 4096, 3, 64, 64),
    (1, 130, 512, 3, 16, 8),
    # W = 2, R = 64, H = 1: the backward plan that falls back to one dw tile
    (2, 600, 1024, 2, 1, 64),
    # W = 8, H = 1: blocks of 16 channels, sub-tiles of 16 (4 channels a thread)
    (2, 300, 512, 8, 1, 64),
    (1, 200, 2048, 8, 1, 8),
    # W = 5 .. 7: blocks of 16 groups (80 .. 112 filter columns)
    (2, 300, 512, 5, 1, 16),
    (1, 260, 1024, 6, 2, 32),
    (2, 140, 2048, 7, 8, 24),
    (1, 200, 4096, 6, 64, 32),
    (1, 150, 1024, 7, 1, 64),
]


LOWRANK_TC = LOWRANK_SHAPES[7:]  # the shapes from the tensor-core comment on


@pytest.mark.parametrize("dtype", ["bf16", "f32"])
@pytest.mark.parametrize("shape", LOWRANK_SHAPES, ids=lambda s: "B{}T{}D{}W{}H{}R{}".format(*s))
def test_lowrank_small(shape, dtype):
    B, T, D, W, H, R = shape
    if dtype == "bf16" and shape in LOWRANK_TC and R % 8 == 0:
        # these run on the tensor-core kernels
        import ctypes as C

        from input_dependent_short_b200 import _lib

        p = _lib.DscProblem(B, T, D, W, H, R, 1, 1)
        assert _lib.lib().dsc_lowrank_kernels(C.byref(p), 0) == 0
        assert _lib.lib().dsc_lowrank_kernels(C.byref(p), 1) == 0
    check_full(W_("lr", LOWRANK, B, T, D, W, H, R, dtype=dtype))


def test_lowrank_full_rank_identity_matches_headwise():
    """R = G*W with U = I: the low-rank op is the head-wise op with w = z."""
    B, T, D, W, H = 2, 45, 64, 4, 16
    G = D // H
    R = G * W
    t = wls.make_inputs(W_("hw", HEADWISE, B, T, D, W, H))
    z = t["w"].reshape(B, T, R).copy()
    U = synth.f32_to_bf16_bits(np.eye(R, dtype=np.float32))
    o = ops()
    x, dy = to_dev(t["x"], "bf16"), to_dev(t["dy"], "bf16")
    y_lr = o.dsc_fwd_lowrank(x, to_dev(z, "bf16"), to_dev(U, "bf16"), H)
    y_hw = o.dsc_fwd_headwise(x, to_dev(t["w"], "bf16"))
    dx_lr, dz, _ = o.dsc_bwd_lowrank(x, to_dev(z, "bf16"), to_dev(U, "bf16"), dy, H)
    dx_hw, dw = o.dsc_bwd_headwise(x, to_dev(t["w"], "bf16"), dy)
    assert rel_err(to_host64(y_lr), to_host64(y_hw)) <= TOL["bf16"]
    assert rel_err(to_host64(dx_lr), to_host64(dx_hw)) <= TOL["bf16"]
    assert rel_err(to_host64(dz).reshape(-1), to_host64(dw).reshape(-1)) <= TOL["bf16"]


def test_tiny_f32_workload_all_variants():
    """The tiny fp32 workload (B=1, T=64, D=64, W=4, H=1), element by element,
    and the same shape for the low-rank and static variants."""
    errs = check_full(wls.TINY_F32)
    assert max(errs.values()) < TOL["f32"]
    check_full(wls.TINY_F32.with_(variant=LOWRANK, R=8))
    check_full(wls.TINY_F32.with_(variant=STATIC))


def test_zero_filter_is_identity_exactly():
    o = ops()
    x = torch.randn(2, 50, 256, device="cuda").to(torch.bfloat16)
    w = torch.zeros(2, 50, 16, 4, device="cuda", dtype=torch.bfloat16)
    assert torch.equal(o.dsc_fwd_headwise(x, w), x)
    dx, dw = o.dsc_bwd_headwise(x, w, x)
    assert torch.equal(dx, x)


def test_outputs_do_not_touch_neighbouring_memory():
    """Canary bands around every output stay intact (ragged shapes)."""
    o = ops()
    from input_dependent_short_b200 import _lib
    import ctypes as C

    wl = W_("canary", HEADWISE, 2, 37, 96, 5, 24)
    t = wls.make_inputs(wl)
    x, w, dy = (to_dev(t[k], "bf16") for k in ("x", "w", "dy"))
    pad = 4096
    n_y, n_w = x.numel(), w.numel()
    buf_y = torch.full((n_y + 2 * pad,), 7.0, device="cuda", dtype=torch.bfloat16)
    buf_dx = torch.full((n_y + 2 * pad,), 7.0, device="cuda", dtype=torch.bfloat16)
    buf_dw = torch.full((n_w + 2 * pad,), 7.0, device="cuda", dtype=torch.bfloat16)
    p = o.problem(x, 5, 24)
    s = torch.cuda.current_stream().cuda_stream
    _lib.call("dsc_fwd_headwise", p, x.data_ptr(), w.data_ptr(), buf_y[pad:].data_ptr(), s)
    _lib.call("dsc_bwd_headwise", p, x.data_ptr(), w.data_ptr(), dy.data_ptr(), buf_dx[pad:].data_ptr(),
              buf_dw[pad:].data_ptr(), s)
    torch.cuda.synchronize()
    for b, n in [(buf_y, n_y), (buf_dx, n_y), (buf_dw, n_w)]:
        assert torch.all(b[:pad] == 7.0) and torch.all(b[pad + n:] == 7.0)
    ref = run_oracle(wl, t)
    assert rel_err(to_host64(buf_y[pad:pad + n_y]).reshape(ref["y"].shape), ref["y"]) <= TOL["bf16"]


@pytest.mark.parametrize("shape", [(2, 150, 2048, 4, 64, 32), (1, 200, 256, 4, 1, 16), (2, 70, 512, 8, 8, 24)],
                         ids=lambda s: "B{}T{}D{}W{}H{}R{}".format(*s))
def test_lowrank_outputs_do_not_touch_neighbouring_memory(shape):
    """Canary bands around y, dx, dz and dU of the tensor-core low-rank kernels
    (TMA loads, ragged last tile, partial-sum workspaces)."""
    from input_dependent_short_b200 import _lib

    o = ops()
    B, T, D, W, H, R = shape
    wl = W_("canary-lr", LOWRANK, B, T, D, W, H, R)
    t = wls.make_inputs(wl)
    x, z, U, dy = (to_dev(t[k], "bf16") for k in ("x", "z", "U", "dy"))
    pad = 4096
    L = _lib.lib()

    def band(n, dtype):
        return torch.full((n + 2 * pad,), 7.0, device="cuda", dtype=dtype)

    buf = {"y": band(x.numel(), torch.bfloat16), "dx": band(x.numel(), torch.bfloat16),
           "dz": band(z.numel(), torch.bfloat16), "dU": band(U.numel(), torch.float32)}
    p = o.problem(x, W, H, R)
    s = torch.cuda.current_stream().cuda_stream
    nf, nb = L.dsc_fwd_lowrank_workspace_bytes(p), L.dsc_bwd_lowrank_workspace_bytes(p)
    wsf = torch.empty(max(nf, 16), dtype=torch.uint8, device="cuda")
    wsb = torch.empty(max(nb, 16), dtype=torch.uint8, device="cuda")
    _lib.call("dsc_fwd_lowrank", p, x.data_ptr(), z.data_ptr(), U.data_ptr(), buf["y"][pad:].data_ptr(),
              wsf.data_ptr(), nf, s)
    _lib.call("dsc_bwd_lowrank", p, x.data_ptr(), z.data_ptr(), U.data_ptr(), dy.data_ptr(),
              buf["dx"][pad:].data_ptr(), buf["dz"][pad:].data_ptr(), buf["dU"][pad:].data_ptr(),
              wsb.data_ptr(), nb, s)
    torch.cuda.synchronize()
    assert L.dsc_check(s) == _lib.DSC_OK
    ref = run_oracle(wl, t)
    for k, b in buf.items():
        n = ref[k].size
        assert torch.all(b[:pad] == 7.0) and torch.all(b[pad + n:] == 7.0), k
        assert rel_err(to_host64(b[pad:pad + n]).reshape(ref[k].shape), ref[k]) <= TOL["bf16"], k


# ------------------------------------------------- full-size workloads ---

@functools.lru_cache(maxsize=2)
def _inputs(wl: Workload):
    return wls.make_inputs(wl)


def _sample_points(rng, wl, n):
    B, T, D = wl.B, wl.T, wl.D
    b = rng.integers(0, B, n)
    t = rng.integers(0, T, n)
    t[:8] = [0, 1, 2, wl.W - 1, T - 1, T - 2, T // 2, T // 2 + 1]
    c = rng.integers(0, D, n)
    c[:4] = [0, D - 1, D // 2, 1]
    return b, t, c


def sampled_check(wl: Workload, n=384, seed=0):
    t = _inputs(wl)
    got = run_gpu(wl, t)
    rng = np.random.default_rng(seed)
    P = oracle.problem_of(wl)
    kind = {HEADWISE: oracle.HEADWISE, LOWRANK: oracle.LOWRANK, STATIC: oracle.STATIC}[wl.variant]
    if wl.variant == STATIC:
        P = oracle.problem(wl.B, wl.T, wl.D, wl.W, 1, 0, wl.residual)
    kw = dict(x=t["x"], dy=t["dy"], w=t.get("w", t.get("ws")), z=t.get("z"), U=t.get("U"))
    b, tt, c = _sample_points(rng, wl, n)
    errs = {}
    for name, what in (("y", oracle.Y), ("dx", oracle.DX)):
        ref = oracle.sample(P, kind, what, np.stack([b, tt, c], 1), **kw)
        g = got[name][torch.as_tensor(b), torch.as_tensor(tt), torch.as_tensor(c)].double().cpu().numpy()
        errs[name] = assert_close(f"{wl.name}:{name}", g, ref, wl.dtype, bound(name, wl.dtype))
    G = wl.D // wl.H
    if wl.variant == HEADWISE or wl.variant == LOWRANK:
        g_ = rng.integers(0, G, n)
        k_ = rng.integers(0, wl.W, n)
        if wl.variant == HEADWISE:
            ref = oracle.sample(P, kind, oracle.DW, np.stack([b, tt, g_, k_], 1), **kw)
            gv = got["dw"][torch.as_tensor(b), torch.as_tensor(tt), torch.as_tensor(g_), torch.as_tensor(k_)]
            errs["dw"] = assert_close(f"{wl.name}:dw", gv.double().cpu().numpy(), ref, wl.dtype, bound("dw", wl.dtype))
        else:
            r_ = rng.integers(0, wl.R, n)
            ref = oracle.sample(P, kind, oracle.DZ, np.stack([b, tt, r_], 1)[:128], **kw)
            gv = got["dz"][torch.as_tensor(b[:128]), torch.as_tensor(tt[:128]), torch.as_tensor(r_[:128])]
            errs["dz"] = assert_close(f"{wl.name}:dz", gv.double().cpu().numpy(), ref, wl.dtype, bound("dz", wl.dtype))
            ref = oracle.sample(P, kind, oracle.DU, np.stack([r_, g_, k_], 1)[:128], **kw)
            gv = got["dU"][torch.as_tensor(r_[:128]), torch.as_tensor(g_[:128] * wl.W + k_[:128])]
            errs["dU"] = assert_close(f"{wl.name}:dU", gv.double().cpu().numpy(), ref, wl.dtype, bound("dU", wl.dtype))
    else:
        k_ = rng.integers(0, wl.W, n)
        ref = oracle.sample(P, kind, oracle.DWS, np.stack([c, k_], 1)[:128], **kw)
        gv = got["dws"][torch.as_tensor(c[:128]), torch.as_tensor(k_[:128])]
        errs["dws"] = assert_close(f"{wl.name}:dws", gv.double().cpu().numpy(), ref, wl.dtype, bound("dws", wl.dtype))
    for name, v in got.items():
        assert torch.isfinite(v.float()).all(), name
    return errs


@pytest.mark.parametrize("name", ["qkv-headwise", "qkv-lowrank", "all-linear-headwise", "all-linear-lowrank"])
def test_full_size_workloads_sampled(name):
    sampled_check(wls.NAMED[name])


# Every variant of the width and length sweep (B=1, T=16384, D=4096, bf16):
# W in {2,3,4,8} x (head-wise H in {1,16,128}, low-rank R in {16,64}, static).
# The tensor-core plans (CTA ranges, blocks per CTA, the one-dw-tile fallback)
# depend on the shape, so each is checked at its own configuration.
SWEEP = wls.sweep_workloads()


@pytest.mark.parametrize("wl", SWEEP, ids=lambda w: w.name.replace(" ", "-"))
def test_sweep_workloads_sampled(wl):
    sampled_check(wl, n=256)


@pytest.mark.parametrize("shape", [(4, 4096, 8192, 4, 64, 64), (2, 2048, 6144, 4, 1, 32)],
                         ids=["all-linear-shape", "qkv-shape"])
def test_lowrank_fused_materialises_no_filters(shape):
    """The fused low-rank kernels never hold w = zU or dw in device memory: the
    forward's workspace is at most a copy of U, the backward's workspace (operand images of z
    and U, per-range dU partials and an fp32 dz accumulator: O(B*T*R +
    ranges*R*G*W), not O(B*T*G*W)) stays well below the fp32 filter tensor,
    and the peak allocation grows by the outputs and that workspace only.  On
    the all-linear shape G*W = 512 is small, so the bound there is half the
    filter tensor; on the Q/K/V-like shape (G*W = 24576) it is about 12 MB
    against a 400 MB filter tensor."""
    import ctypes as C

    from input_dependent_short_b200 import _lib

    B, T, D, W, H, R = shape
    o = ops()
    wl = W_("lr-mem", LOWRANK, B, T, D, W, H, R)
    t = wls.make_inputs(wl)
    x, dy, z, U = (to_dev(t[k], "bf16") for k in ("x", "dy", "z", "U"))
    p = o.problem(x, W, H, R)
    L = _lib.lib()
    filters = B * T * (D // H) * W * 4
    ws = L.dsc_bwd_lowrank_workspace_bytes(C.byref(p))
    wsf = L.dsc_fwd_lowrank_workspace_bytes(C.byref(p))
    assert wsf <= R * (D // H) * W * 2 + 256  # at most a tap-ordered copy of U
    assert ws < filters / 2
    if (D // H) * W > 4096:
        assert ws < filters / 20
    torch.cuda.synchronize()
    base = torch.cuda.memory_allocated()
    torch.cuda.reset_peak_memory_stats()
    y = o.dsc_fwd_lowrank(x, z, U, H)
    dx, dz, dU = o.dsc_bwd_lowrank(x, z, U, dy, H)
    torch.cuda.synchronize()
    outputs = sum(v.numel() * v.element_size() for v in (y, dx, dz, dU))
    assert torch.cuda.max_memory_allocated() - base <= outputs + ws + wsf + (1 << 20)
