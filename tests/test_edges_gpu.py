"""Packed documents (variable-length batches) and sequence chunks (context
parallelism) on the GPU, through the C ABI, against the fp64 oracle.

Packed documents: one row of T tokens holding several documents; the oracle
is ``oracle.forward_varlen`` / ``backward_varlen`` (pinned against the
documents run one by one).  Document-length mixes include documents of one
token, documents shorter than W-1, boundaries inside and at the edges of the
tensor-core kernels' 128-token tiles, and a seeded mix of long documents.

Chunks: sequences split along time, each chunk called with its neighbours'
rows as halos; each chunk's outputs are compared with the rows of the oracle
run on the whole sequences, and its dU / dws summed over the chunks with the
whole sequences' reductions.
"""

import numpy as np
import pytest
import torch

import oracle
from synth import workloads as wls
from synth.workloads import HEADWISE, LOWRANK, STATIC, Workload

from helpers import TOL, assert_close, bound, to_dev, to_host64

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.fail("no CUDA device: the -m gpu tests need a B200")
    import input_dependent_short_b200  # noqa: F401


def ops():
    from input_dependent_short_b200 import ops as o

    return o


KIND = {HEADWISE: oracle.HEADWISE, LOWRANK: oracle.LOWRANK, STATIC: oracle.STATIC}


def _filters(wl, t, dev=True):
    f = {}
    for k in ("w", "z", "U", "ws"):
        if k in t:
            f[k] = to_dev(t[k], wl.dtype) if dev else t[k]
    return f


# -------------------------------------------------------- packed documents ---

def doc_lengths(T, mix, seed=0):
    """Document lengths summing to T: a named mix or an explicit tuple."""
    if isinstance(mix, tuple):
        assert sum(mix) == T
        return list(mix)
    rng = np.random.default_rng(seed)
    out, left = [], T
    while left > 0:
        n = int(min(left, max(1, rng.geometric(1.0 / mix))))
        out.append(n)
        left -= n
    return out


VARLEN_CASES = [
    # variant, T, D, W, H, R, dtype, lengths (tuple) or mean length (int)
    (HEADWISE, 300, 256, 4, 16, 0, "bf16", (1, 2, 3, 50, 127, 1, 116)),
    (HEADWISE, 300, 256, 4, 16, 0, "f32", (1, 2, 3, 50, 127, 1, 116)),
    (HEADWISE, 1000, 512, 8, 1, 0, "bf16", 37),
    (HEADWISE, 200, 96, 5, 24, 0, "bf16", (3, 4, 5, 188)),
    (HEADWISE, 130, 40, 3, 8, 0, "f32", (128, 2)),            # generic kernels (D not a multiple of 8)
    (STATIC, 300, 256, 4, 1, 0, "bf16", (1, 2, 3, 50, 127, 1, 116)),
    (STATIC, 500, 64, 7, 1, 0, "f32", 23),
    (LOWRANK, 600, 1024, 4, 1, 32, "bf16", (127, 1, 128, 2, 3, 339)),  # tensor-core kernels
    (LOWRANK, 2048, 1024, 4, 1, 32, "bf16", 300),
    (LOWRANK, 500, 2048, 4, 64, 64, "bf16", (100, 1, 399)),
    (LOWRANK, 300, 512, 8, 1, 16, "bf16", (5, 7, 288)),
    (LOWRANK, 200, 96, 3, 4, 5, "f32", (1, 1, 198)),               # CUDA-core fused kernels
    (LOWRANK, 90, 40, 5, 5, 7, "bf16", (40, 50)),                  # unfused path
    # empty documents (a padded list of documents): at the start, twice in a row, at the end
    (HEADWISE, 300, 256, 4, 16, 0, "bf16", (0, 1, 2, 0, 0, 3, 50, 127, 1, 116, 0)),
    (STATIC, 300, 256, 4, 1, 0, "bf16", (0, 60, 0, 0, 240, 0)),
    (LOWRANK, 600, 1024, 4, 1, 32, "bf16", (0, 127, 0, 1, 128, 0, 0, 2, 3, 339, 0)),
]


def _varlen_run(wl, t, lens):
    o = ops()
    dt = wl.dtype
    cu = np.concatenate([[0], np.cumsum(lens)]).astype(np.int64)
    cu_d = torch.tensor(cu, dtype=torch.int32, device="cuda")
    x, dy = to_dev(t["x"], dt), to_dev(t["dy"], dt)
    f = _filters(wl, t)
    P = oracle.problem(1, wl.T, wl.D, wl.W, wl.H if wl.variant != STATIC else 1, wl.R, wl.residual)
    of = _filters(wl, t, dev=False)
    ref_y = oracle.forward_varlen(P, KIND[wl.variant], t["x"], cu, **of)
    ref_g = oracle.backward_varlen(P, KIND[wl.variant], t["x"], t["dy"], cu, **of)
    res = bool(wl.residual)
    if wl.variant == HEADWISE:
        got = {"y": o.dsc_fwd_headwise_varlen(x, f["w"], cu_d, res)}
        got["dx"], got["dw"] = o.dsc_bwd_headwise_varlen(x, f["w"], dy, cu_d, res)
        ref = {"y": ref_y, "dx": ref_g[0], "dw": ref_g[1]}
    elif wl.variant == LOWRANK:
        got = {"y": o.dsc_fwd_lowrank_varlen(x, f["z"], f["U"], cu_d, wl.H, res)}
        got["dx"], got["dz"], got["dU"] = o.dsc_bwd_lowrank_varlen(x, f["z"], f["U"], dy, cu_d, wl.H, res)
        ref = {"y": ref_y, "dx": ref_g[0], "dz": ref_g[1], "dU": ref_g[2]}
    else:
        got = {"y": o.dsc_fwd_static_varlen(x, f["ws"], cu_d, res)}
        got["dx"], got["dws"] = o.dsc_bwd_static_varlen(x, f["ws"], dy, cu_d, res)
        ref = {"y": ref_y, "dx": ref_g[0], "dws": ref_g[1]}
    torch.cuda.synchronize()
    return got, ref


@pytest.mark.parametrize("case", VARLEN_CASES, ids=lambda c: "{}-T{}-D{}-W{}-H{}-R{}-{}".format(*c[:7]))
def test_varlen_matches_oracle(case):
    variant, T, D, W, H, R, dtype, mix = case
    wl = Workload("varlen", variant, 1, T, D, W, H=H, R=R, dtype=dtype, seed=3)
    lens = doc_lengths(T, mix)
    t = wls.make_inputs(wl)
    got, ref = _varlen_run(wl, t, lens)
    for k, r in ref.items():
        assert_close(f"varlen {variant} T{T} D{D} W{W} {dtype}:{k}", to_host64(got[k]).reshape(r.shape), r, dtype,
                     bound(k, dtype))
    ops().dsc_check()


def test_varlen_one_document_equals_the_plain_call():
    """A single document is the plain op: the fix-up pass has nothing to do
    and the results are the plain call's bits."""
    o = ops()
    wl = Workload("one-doc", HEADWISE, 1, 500, 512, 4, H=16, seed=4)
    t = wls.make_inputs(wl)
    x, w, dy = (to_dev(t[k], "bf16") for k in ("x", "w", "dy"))
    cu = torch.tensor([0, 500], dtype=torch.int32, device="cuda")
    assert torch.equal(o.dsc_fwd_headwise_varlen(x, w, cu), o.dsc_fwd_headwise(x, w))
    a, b = o.dsc_bwd_headwise_varlen(x, w, dy, cu), o.dsc_bwd_headwise(x, w, dy)
    assert torch.equal(a[0], b[0]) and torch.equal(a[1], b[1])


def test_varlen_documents_equal_separate_sequences_on_the_gpu():
    """Packed documents give what the plain calls give on each document as a
    batch row of its own (tensor-core low-rank kernels, bf16)."""
    o = ops()
    lens = [300, 1, 211, 512]
    T, D, W, R = sum(lens), 1024, 4, 32
    wl = Workload("docs", LOWRANK, 1, T, D, W, H=1, R=R, seed=5)
    t = wls.make_inputs(wl)
    x, z, U, dy = (to_dev(t[k], "bf16") for k in ("x", "z", "U", "dy"))
    cu = torch.tensor(np.concatenate([[0], np.cumsum(lens)]), dtype=torch.int32, device="cuda")
    y = o.dsc_fwd_lowrank_varlen(x, z, U, cu)
    dx, dz, dU = o.dsc_bwd_lowrank_varlen(x, z, U, dy, cu)
    dU_sum = torch.zeros_like(dU)
    s = 0
    for n in lens:
        sl = slice(s, s + n)
        yd = o.dsc_fwd_lowrank(x[:, sl].contiguous(), z[:, sl].contiguous(), U)
        dxd, dzd, dUd = o.dsc_bwd_lowrank(x[:, sl].contiguous(), z[:, sl].contiguous(), U, dy[:, sl].contiguous())
        for a, b in ((y[:, sl], yd), (dx[:, sl], dxd), (dz[:, sl], dzd)):
            err = (a.double() - b.double()).abs().max().item() / max(b.double().abs().max().item(), 1e-30)
            assert err <= TOL["bf16"]
        dU_sum += dUd
        s += n
    err = (dU - dU_sum).abs().max().item() / dU_sum.abs().max().item()
    assert err <= 1e-3


def test_varlen_rejects_bad_arguments():
    import ctypes as C

    from input_dependent_short_b200 import _lib

    L = _lib.lib()
    x = torch.zeros(2, 8, 16, dtype=torch.bfloat16, device="cuda")
    w = torch.zeros(2, 8, 16, 4, dtype=torch.bfloat16, device="cuda")
    cu = torch.tensor([0, 8], dtype=torch.int32, device="cuda")
    p = _lib.DscProblem(2, 8, 16, 4, 1, 0, 1, 1)  # B = 2: packed documents need one row
    s = torch.cuda.current_stream().cuda_stream
    assert L.dsc_fwd_headwise_varlen(C.byref(p), cu.data_ptr(), 1, x.data_ptr(), w.data_ptr(), x.data_ptr(),
                                     s) == _lib.DSC_ERR_INVALID_ARG
    p.B = 1
    assert L.dsc_fwd_headwise_varlen(C.byref(p), cu.data_ptr() + 2, 1, x.data_ptr(), w.data_ptr(), x.data_ptr(),
                                     s) == _lib.DSC_ERR_MISALIGNED
    assert L.dsc_fwd_headwise_varlen(C.byref(p), cu.data_ptr(), 0, x.data_ptr(), w.data_ptr(), x.data_ptr(),
                                     s) == _lib.DSC_ERR_INVALID_ARG
    # more documents than tokens is allowed (empty documents); a count whose fix-up
    # grid would not fit is refused before anything is read or launched
    assert L.dsc_fwd_headwise_varlen(C.byref(p), cu.data_ptr(), 1 << 31, x.data_ptr(), w.data_ptr(), x.data_ptr(),
                                     s) == _lib.DSC_ERR_UNSUPPORTED


# --------------------------------------------------------- sequence chunks ---

CHUNK_CASES = [
    # variant, B, chunk lengths, D, W, H, R, dtype
    (HEADWISE, 2, (300, 129, 2, 200), 256, 4, 16, 0, "bf16"),
    (HEADWISE, 2, (100, 3, 77), 96, 8, 24, 0, "f32"),
    (STATIC, 2, (300, 1, 256), 256, 4, 1, 0, "bf16"),
    (STATIC, 1, (64, 2, 64), 40, 5, 1, 0, "f32"),
    (LOWRANK, 2, (256, 128, 300), 1024, 4, 1, 32, "bf16"),  # tensor-core kernels
    (LOWRANK, 1, (500, 2, 300), 2048, 4, 64, 64, "bf16"),
    (LOWRANK, 2, (90, 1, 40), 96, 3, 4, 5, "f32"),
]


def _rows(a, lo, hi):
    """Rows lo .. hi-1 (dim 1) of a device tensor, zero outside [0, L)."""
    B, L = a.shape[:2]
    out = torch.zeros((B, hi - lo) + tuple(a.shape[2:]), dtype=a.dtype, device=a.device)
    s, e = max(lo, 0), min(hi, L)
    if s < e:
        out[:, s - lo:e - lo] = a[:, s:e]
    return out


@pytest.mark.parametrize("case", CHUNK_CASES, ids=lambda c: "{}-B{}-{}-D{}-W{}-{}".format(c[0], c[1], len(c[2]), c[3],
                                                                                          c[4], c[7]))
@pytest.mark.parametrize("edges_only", [False, True])
def test_chunks_match_the_whole_sequence(case, edges_only):
    variant, B, lens, D, W, H, R, dtype = case
    L = sum(lens)
    o = ops()
    wl = Workload("chunks", variant, B, L, D, W, H=H, R=R, dtype=dtype, seed=6)
    t = wls.make_inputs(wl)
    P = oracle.problem(B, L, D, W, H if variant != STATIC else 1, R, 1)
    of = _filters(wl, t, dev=False)
    k = KIND[variant]
    if variant == HEADWISE:
        ref_y = oracle.forward_headwise(P, t["x"], t["w"])
        ref = dict(zip(("dx", "dw"), oracle.backward_headwise(P, t["x"], t["w"], t["dy"])))
    elif variant == LOWRANK:
        ref_y = oracle.forward_lowrank(P, t["x"], t["z"], t["U"])
        ref = dict(zip(("dx", "dz", "dU"), oracle.backward_lowrank(P, t["x"], t["z"], t["U"], t["dy"])[:3]))
    else:
        ref_y = oracle.forward_static(P, t["x"], t["ws"])
        ref = dict(zip(("dx", "dws"), oracle.backward_static(P, t["x"], t["ws"], t["dy"])))
    del k, of
    x, dy = to_dev(t["x"], dtype), to_dev(t["dy"], dtype)
    f = _filters(wl, t)
    red = None
    s = 0
    for i, n in enumerate(lens):
        sl = slice(s, s + n)
        xc, dyc = x[:, sl].contiguous(), dy[:, sl].contiguous()
        first, last = i == 0, i == len(lens) - 1
        x_prev = None if first or W == 1 else _rows(x, s - W + 1, s)
        dy_next = None if last or W == 1 else _rows(dy, s + n, s + n + W - 1)
        if variant == HEADWISE:
            wc = f["w"][:, sl].contiguous()
            w_next = None if dy_next is None else _rows(f["w"], s + n, s + n + W - 1)
            if edges_only:
                y = o.dsc_fwd_headwise_chunk(xc, wc, x_prev, out=o.dsc_fwd_headwise(xc, wc))
                g = o.dsc_bwd_headwise_chunk(xc, wc, dyc, x_prev, dy_next, w_next, out=o.dsc_bwd_headwise(xc, wc, dyc))
            else:
                y = o.dsc_fwd_headwise_chunk(xc, wc, x_prev)
                g = o.dsc_bwd_headwise_chunk(xc, wc, dyc, x_prev, dy_next, w_next)
            got = {"dx": g[0], "dw": g[1]}
        elif variant == LOWRANK:
            zc = f["z"][:, sl].contiguous()
            z_next = None if dy_next is None else _rows(f["z"], s + n, s + n + W - 1)
            if edges_only:
                y = o.dsc_fwd_lowrank_chunk(xc, zc, f["U"], x_prev, H, out=o.dsc_fwd_lowrank(xc, zc, f["U"], H))
                g = o.dsc_bwd_lowrank_chunk(xc, zc, f["U"], dyc, x_prev, dy_next, z_next, H,
                                            out=o.dsc_bwd_lowrank(xc, zc, f["U"], dyc, H))
            else:
                y = o.dsc_fwd_lowrank_chunk(xc, zc, f["U"], x_prev, H)
                g = o.dsc_bwd_lowrank_chunk(xc, zc, f["U"], dyc, x_prev, dy_next, z_next, H)
            got = {"dx": g[0], "dz": g[1]}
            red = g[2].double() if red is None else red + g[2].double()
        else:
            if edges_only:
                y = o.dsc_fwd_static_chunk(xc, f["ws"], x_prev, True, out=o.dsc_fwd_static(xc, f["ws"], True))
                g = o.dsc_bwd_static_chunk(xc, f["ws"], dyc, x_prev, dy_next, True,
                                           out=o.dsc_bwd_static(xc, f["ws"], dyc, True))
            else:
                y = o.dsc_fwd_static_chunk(xc, f["ws"], x_prev, True)
                g = o.dsc_bwd_static_chunk(xc, f["ws"], dyc, x_prev, dy_next, True)
            got = {"dx": g[0]}
            red = g[1].double() if red is None else red + g[1].double()
        torch.cuda.synchronize()
        name = f"chunk {variant} {dtype} W{W} [{s},{s + n})"
        assert_close(name + ":y", to_host64(y), ref_y[:, sl], dtype, bound("y", dtype))
        for kk, v in got.items():
            assert_close(f"{name}:{kk}", to_host64(v), ref[kk][:, sl], dtype, bound(kk, dtype))
        s += n
    if variant == LOWRANK:
        assert_close(f"chunk {variant} {dtype}:dU", red.cpu().numpy(), ref["dU"], dtype, bound("dU", dtype))
    elif variant == STATIC:
        assert_close(f"chunk {variant} {dtype}:dws", red.cpu().numpy(), ref["dws"], dtype, bound("dws", dtype))
    ops().dsc_check()


def test_edges_only_waits_for_the_kernel_that_wrote_its_halos():
    """The edges-only form may follow, on the same stream, the kernel that
    wrote its halos; here x_prev and dy_next are the last rows of a long
    forward's output, launched just before the fix-ups.  The fix-ups must read
    them only once that kernel is done: each result equals the one-call form
    run after a synchronize."""
    o = ops()
    B, L, D, W, H = 1, 256, 1024, 4, 16
    G, Tbig = D // H, 1 << 17
    g = torch.Generator(device="cuda").manual_seed(11)

    def rnd(*shape, scale=1.0):
        return (torch.randn(*shape, device="cuda", generator=g) * scale).to(torch.bfloat16)

    xc, dyc = rnd(B, L, D), rnd(B, L, D)
    wc, w_next = rnd(B, L, G, W, scale=0.5), rnd(B, W - 1, G, W, scale=0.5)
    for _ in range(3):
        a, wa = rnd(B, Tbig, D), rnd(B, Tbig, G, W, scale=0.5)
        y = o.dsc_fwd_headwise(xc, wc)
        x_prev = o.dsc_fwd_headwise(a, wa)[:, Tbig - (W - 1):]
        y = o.dsc_fwd_headwise_chunk(xc, wc, x_prev, out=y)
        gr = o.dsc_bwd_headwise(xc, wc, dyc)
        dy_next = o.dsc_fwd_headwise(a, wa, False)[:, Tbig - (W - 1):]
        gr = o.dsc_bwd_headwise_chunk(xc, wc, dyc, x_prev, dy_next, w_next, out=gr)
        torch.cuda.synchronize()
        assert torch.equal(y, o.dsc_fwd_headwise_chunk(xc, wc, x_prev))
        full = o.dsc_bwd_headwise_chunk(xc, wc, dyc, x_prev, dy_next, w_next)
        assert torch.equal(gr[0], full[0]) and torch.equal(gr[1], full[1])
    ops().dsc_check()


@pytest.mark.parametrize("variant", ["headwise", "static"])
def test_full_size_chunks_are_bit_exact_with_the_whole_call(variant):
    """At the Q/K/V size (B=8, T=2048, D=6144, W=4; H=16 head-wise) the whole
    call and four chunk calls of 512 tokens tile time differently: the whole
    head-wise call runs several waves of tiles of about 40 tokens, the chunks
    one wave of shorter ones.  The streaming kernels compute every output
    element by the same arithmetic in the same order whatever the tiling
    (the token's taps summed tap by tap), so away from the chunk edges y, dx
    and the head-wise dw must agree bit for bit at every element, which
    checks the tile and wave boundaries of the full-size launch.  The W-1
    rows next to a chunk edge come from the fix-up kernels, which sum in
    another order: they are compared within the bf16 tolerance, as is the
    static dws (a sum over tiles, whose order differs)."""
    o = ops()
    B, T, D, W, H = 8, 2048, 6144, 4, 16
    g = torch.Generator(device="cuda").manual_seed(31)

    def rnd(*shape, scale=1.0):
        return (torch.randn(*shape, device="cuda", generator=g) * scale).to(torch.bfloat16)

    x, dy = rnd(B, T, D), rnd(B, T, D)
    if variant == "headwise":
        w = rnd(B, T, D // H, W, scale=0.5)
        y = o.dsc_fwd_headwise(x, w)
        dx, dw = o.dsc_bwd_headwise(x, w, dy)
    else:
        ws = rnd(D, W, scale=0.5)
        y = o.dsc_fwd_static(x, ws, True)
        dx, dws = o.dsc_bwd_static(x, ws, dy, True)
        dws_sum = torch.zeros_like(dws)
    n = T // 4
    for c in range(4):
        sl = slice(c * n, (c + 1) * n)
        xc, dyc = x[:, sl].contiguous(), dy[:, sl].contiguous()
        x_prev = None if c == 0 else x[:, c * n - (W - 1):c * n].contiguous()
        dy_next = None if c == 3 else dy[:, (c + 1) * n:(c + 1) * n + W - 1].contiguous()
        lo = 0 if c == 0 else W - 1      # rows after a left edge (fixed up: y, dw)
        hi = n if c == 3 else n - (W - 1)  # rows before a right edge (fixed up: dx)

        def same(name, got, ref, a, b):
            assert torch.equal(got[:, a:b], ref[:, a:b]), f"{name} differs in chunk {c}"
            if a > 0:
                assert_close(f"{name} chunk {c} left edge", to_host64(got[:, :a]), to_host64(ref[:, :a]), "bf16")
            if b < n:
                assert_close(f"{name} chunk {c} right edge", to_host64(got[:, b:]), to_host64(ref[:, b:]), "bf16")

        if variant == "headwise":
            w_next = None if c == 3 else w[:, (c + 1) * n:(c + 1) * n + W - 1].contiguous()
            yc = o.dsc_fwd_headwise_chunk(xc, w[:, sl].contiguous(), x_prev)
            dxc, dwc = o.dsc_bwd_headwise_chunk(xc, w[:, sl].contiguous(), dyc, x_prev, dy_next, w_next)
            same("dw", dwc, dw[:, sl], lo, n)
        else:
            yc = o.dsc_fwd_static_chunk(xc, ws, x_prev, True)
            dxc, dwsc = o.dsc_bwd_static_chunk(xc, ws, dyc, x_prev, dy_next, True)
            dws_sum += dwsc
        same("y", yc, y[:, sl], lo, n)
        same("dx", dxc, dx[:, sl], 0, hi)
    if variant == "static":
        assert_close("full-size static dws, chunked", to_host64(dws_sum), to_host64(dws), "bf16", bound("dws", "bf16"))
    ops().dsc_check()


def test_chunk_without_halos_is_the_plain_call():
    o = ops()
    wl = Workload("first-last", HEADWISE, 2, 300, 256, 4, H=16, seed=7)
    t = wls.make_inputs(wl)
    x, w, dy = (to_dev(t[k], "bf16") for k in ("x", "w", "dy"))
    assert torch.equal(o.dsc_fwd_headwise_chunk(x, w, None), o.dsc_fwd_headwise(x, w))
    a, b = o.dsc_bwd_headwise_chunk(x, w, dy), o.dsc_bwd_headwise(x, w, dy)
    assert torch.equal(a[0], b[0]) and torch.equal(a[1], b[1])
