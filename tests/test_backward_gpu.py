"""GPU parity of the backward kernels against the float64 oracle's gradients.

Both sides get the same seeded, dtype-rounded inputs and upstream gradient;
every gradient element is compared with the tolerances of tests/parity.py
(grad_x / grad_value are float32 sums rounded once, like a forward output).
Full-size workloads are run whole on the GPU, in the launch configuration
the benchmark times, and checked image by image on sampled batch items (the
gradients of one image depend on that image alone).
"""
import numpy as np
import pytest
import torch

import deformable_attention_sampling_b200 as dcnb
import gen
import oracle
from tests.parity import compare
from tests.test_parity_gpu import SMALL

pytestmark = pytest.mark.gpu
DEV = "cuda:0"


def dcn_problem(w, seed):
    inp = gen.dcn_inputs(w, seed=seed)
    inp["grad_out"] = gen.grad_out((w.N, w.Ho, w.Wo, w.C), w.dtype, seed)
    return inp


def run_dcn_bwd(inp, w, workspace=None):
    d = {k: v.to(DEV) for k, v in inp.items()}
    g = dcnb.dcn_grad(d["x"], d["offset"], d["mask"], d["grad_out"], w.kh, w.kw, w.stride,
                      w.pad, w.dil, w.softmax_flag, workspace=workspace)
    torch.cuda.synchronize()
    return g


def ref_dcn_bwd(inp, w, n=None):
    sel = (lambda t: t[n:n + 1]) if n is not None else (lambda t: t)
    return oracle.dcn_backward_ref(sel(inp["x"]), sel(inp["offset"]), sel(inp["mask"]),
                                   sel(inp["grad_out"]), w.kh, w.kw, w.stride, w.pad, w.dil,
                                   w.softmax_flag)


def check_dcn(got, ref, label, n=None):
    sel = (lambda t: t[n:n + 1]) if n is not None else (lambda t: t)
    for name, g, r in zip(("grad_x", "grad_offset", "grad_mask"), got, ref):
        compare(sel(g), r, f"{label} {name}")


# ------------------------------------------------------------ full workloads

DCN_WORKLOADS = [n for n, w in gen.WORKLOADS.items() if isinstance(w, gen.DcnWorkload)]


@pytest.mark.parametrize("name", DCN_WORKLOADS)
def test_dcn_backward_workload_full_size(name):
    w = gen.WORKLOADS[name]
    inp = dcn_problem(w, seed=0)
    got = run_dcn_bwd(inp, w)
    # first, middle (where the persistent CTAs' ranges meet) and last image
    for n in sorted({0, w.N // 2, w.N - 1}):
        check_dcn(got, ref_dcn_bwd(inp, w, n), f"{name} image {n}", n)


def msda_problem(w, seed):
    inp = gen.msda_inputs(w, seed=seed)
    inp["grad_out"] = gen.grad_out((w.N, w.queries, w.M * w.D), w.dtype, seed)
    return inp


def run_msda_bwd(inp):
    d = {k: (v.to(DEV) if torch.is_tensor(v) else v) for k, v in inp.items()}
    g = dcnb.msda_grad(d["value"], d["spatial_shapes"], d["level_start"], d["loc"], d["attn"],
                       d["grad_out"])
    torch.cuda.synchronize()
    return g


def ref_msda_bwd(inp):
    return oracle.msda_backward_ref(inp["value"], inp["spatial_shapes"], inp["level_start"],
                                    inp["loc"], inp["attn"], inp["grad_out"])


def check_msda(got, ref, label):
    for name, g, r in zip(("grad_value", "grad_loc", "grad_attn"), got, ref):
        compare(g, r, f"{label} {name}")


def test_msda_backward_workload_full_size():
    w = gen.WORKLOADS["msda_f32_2x4lvl_m8_d32_k4"]
    inp = msda_problem(w, seed=0)
    check_msda(run_msda_bwd(inp), ref_msda_bwd(inp), w.name)


# ------------------------------------------------------------ small shapes

@pytest.mark.parametrize("case", SMALL, ids=[f"case{i}" for i in range(len(SMALL))])
def test_dcn_backward_small_shapes(case):
    N, H, W, C, G, kh, kw, stride, pad, dil, dt, sm, sigma = case
    w = gen.DcnWorkload("small", N=N, H=H, W=W, C=C, G=G, kh=kh, kw=kw, stride=stride, pad=pad,
                        dil=dil, dtype=dt, offset_sigma=sigma, softmax_flag=sm)
    inp = dcn_problem(w, seed=5)
    check_dcn(run_dcn_bwd(inp, w), ref_dcn_bwd(inp, w), str(case))


@pytest.mark.parametrize("dt", ["f32", "f16", "bf16"])
@pytest.mark.parametrize("sm", [0, 1])
def test_dcn_backward_ragged_tail_and_many_tiles(dt, sm):
    w = gen.DcnWorkload("ragged", N=3, H=37, W=41, C=64, G=4, dtype=dt, offset_sigma=2.0,
                        softmax_flag=sm)
    inp = dcn_problem(w, seed=11)
    check_dcn(run_dcn_bwd(inp, w), ref_dcn_bwd(inp, w), f"ragged {dt} softmax {sm}")


@pytest.mark.parametrize("dt", ["f32", "f16"])
def test_dcn_backward_non_power_of_two_threads_per_item(dt):
    """D = 48 fp16 (96 bytes: 3 threads of 32 bytes) and D = 24 fp32 (3 x 32
    bytes): the per-tap sums are reduced over 3 lanes, and 2 lanes of every
    warp serve no item."""
    C = 96 if dt == "f16" else 48
    w = gen.DcnWorkload("tpi3", N=2, H=9, W=13, C=C, G=2, dtype=dt, offset_sigma=2.0)
    inp = dcn_problem(w, seed=4)
    check_dcn(run_dcn_bwd(inp, w), ref_dcn_bwd(inp, w), f"tpi3 {dt}")


@pytest.mark.parametrize("dt", ["f32", "f16", "bf16"])
def test_dcn_backward_extreme_offsets(dt):
    """Huge, infinite and NaN offsets: such taps get zero gradients and add
    nothing to grad_x.  The oracle agrees on huge offsets; where it yields NaN
    (NaN or infinite positions) the expected gradient of that tap is 0."""
    w = gen.DcnWorkload("extreme", N=2, H=6, W=7, C=32, G=2, dtype=dt, offset_sigma=1.0)
    inp = dcn_problem(w, seed=3)
    off = inp["offset"].double()
    big = 1e30 if dt == "f32" else 6e4
    off[0, 0, 0, 0, :, 0] = big
    off[0, 1, 2, 1, :, 1] = -big
    off[1, 2, 3, 0, 4, 0] = float("inf")
    off[1, 3, 3, 1, 2, 1] = float("nan")
    inp["offset"] = off.to(gen.DTYPES[dt])
    gx, goff, gmask = ref_dcn_bwd(inp, w)
    bad = ~np.isfinite(goff).all(axis=-1)               # taps with a non-finite position
    goff[bad] = 0.0
    gmask[bad] = 0.0
    assert bad.sum() == 2 and np.isfinite(gx).all()
    check_dcn(run_dcn_bwd(inp, w), (gx, goff, gmask), f"extreme {dt}")


def test_dcn_backward_misaligned_bases():
    """x and grad_out one element past a 32-byte boundary (narrower vectors),
    float32 grad_x one element past 16 bytes (scalar reductions)."""
    w = gen.DcnWorkload("mis", N=2, H=10, W=12, C=32, G=2, dtype="f32", offset_sigma=2.0)
    inp = dcn_problem(w, seed=8)
    ref = ref_dcn_bwd(inp, w)

    def shifted(t):
        buf = torch.empty(t.numel() + 8, dtype=t.dtype, device=DEV)
        view = buf[1:1 + t.numel()].view(t.shape)
        view.copy_(t.to(DEV))
        return view

    x, go = shifted(inp["x"]), shifted(inp["grad_out"])
    off, mask = inp["offset"].to(DEV), inp["mask"].to(DEV)
    gx = shifted(torch.zeros_like(inp["x"]))
    goff = torch.empty_like(off)
    gmask = torch.empty_like(mask)
    dcnb.dcn_backward(x, off, mask, go, gx, goff, gmask, None, 0, w.N, w.H, w.W, w.C, w.G, w.kh,
                      w.kw, w.stride, w.pad, w.dil, 0, 0)
    torch.cuda.synchronize()
    check_dcn((gx, goff, gmask), ref, "misaligned")


@pytest.mark.parametrize("dt", ["f16", "bf16"])
def test_dcn_backward_reuses_a_dirty_workspace(dt):
    """Two calls in a row with one caller-owned workspace, filled with garbage
    before the first: the zero fill is part of every call."""
    w = gen.DcnWorkload("ws", N=2, H=11, W=9, C=64, G=4, dtype=dt, offset_sigma=2.0)
    inp = dcn_problem(w, seed=9)
    ref = ref_dcn_bwd(inp, w)
    nbytes = dcnb.dcn_backward_workspace_size(w.N, w.H, w.W, w.C, gen.DTYPE_CODES[dt])
    ws = torch.full((nbytes // 4,), 12345.0, device=DEV)
    first = run_dcn_bwd(inp, w, workspace=ws)
    second = run_dcn_bwd(inp, w, workspace=ws)
    check_dcn(first, ref, f"ws first {dt}")
    check_dcn(second, ref, f"ws second {dt}")
    # grad_offset and grad_mask are deterministic; grad_x may differ in the
    # order of its float32 additions only
    assert torch.equal(first[1], second[1]) and torch.equal(first[2], second[2])


def test_dcn_backward_launches_and_side_stream():
    w = gen.DcnWorkload("ls", N=2, H=8, W=8, C=64, G=4, dtype="f16", offset_sigma=1.0)
    inp = dcn_problem(w, seed=2)
    d = {k: v.to(DEV) for k, v in inp.items()}
    side = torch.cuda.Stream()
    torch.cuda.synchronize()
    before = dcnb.dcn_launch_count()
    with torch.cuda.stream(side):
        got = dcnb.dcn_grad(d["x"], d["offset"], d["mask"], d["grad_out"], stream=side)
    side.synchronize()
    assert dcnb.dcn_launch_count() - before == 3          # zero fill, gradients, rounding
    check_dcn(got, ref_dcn_bwd(inp, w), "side stream")
    w32 = gen.scaled(w, dtype="f32")
    inp32 = dcn_problem(w32, seed=2)
    before = dcnb.dcn_launch_count()
    got32 = run_dcn_bwd(inp32, w32)
    assert dcnb.dcn_launch_count() - before == 2          # float32: no rounding pass
    check_dcn(got32, ref_dcn_bwd(inp32, w32), "f32 launches")


def test_dcn_backward_empty_batch():
    w = gen.DcnWorkload("empty", N=0, H=5, W=5, C=16, G=1, dtype="f16")
    x = torch.empty((0, 5, 5, 16), dtype=torch.float16, device=DEV)
    off = torch.empty((0, 5, 5, 1, 9, 2), dtype=torch.float16, device=DEV)
    mask = torch.empty((0, 5, 5, 1, 9), dtype=torch.float16, device=DEV)
    before = dcnb.dcn_launch_count()
    gx, goff, gmask = dcnb.dcn_grad(x, off, mask, torch.empty_like(x))
    assert dcnb.dcn_launch_count() == before and gx.shape == x.shape
    assert w.N == 0


# ------------------------------------------------------------ MSDA

MSDA_SMALL = [
    # N, shapes, M, D, K, dtype, sigma
    (1, ((5, 7),), 1, 8, 1, "f32", 1.0),
    (2, ((6, 9), (3, 5)), 2, 16, 3, "f16", 2.0),
    (1, ((10, 12), (5, 6), (3, 3)), 4, 32, 4, "bf16", 2.0),
    (2, ((7, 11), (4, 6), (2, 3), (1, 2)), 8, 32, 4, "f32", 3.0),
    (1, ((9, 9), (4, 4)), 3, 6, 2, "f32", 1.5),          # D = 6 fp32: 3 x 8-byte lanes
    (1, ((8, 8),), 2, 64, 8, "f16", 20.0),               # most samples far outside
    (1, ((12, 5), (6, 3)), 2, 24, 2, "f16", 2.0),        # D = 24 fp16: 3 lanes
]


@pytest.mark.parametrize("case", MSDA_SMALL, ids=[f"case{i}" for i in range(len(MSDA_SMALL))])
def test_msda_backward_small_shapes(case):
    N, shapes, M, D, K, dt, sigma = case
    w = gen.MsdaWorkload("small", N=N, M=M, D=D, shapes=shapes, K=K, dtype=dt,
                         offset_sigma=sigma)
    inp = msda_problem(w, seed=6)
    check_msda(run_msda_bwd(inp), ref_msda_bwd(inp), str(case))


def test_msda_backward_launches_and_repeat():
    w = gen.MsdaWorkload("rep", N=2, M=4, D=16, shapes=((9, 13), (5, 7)), K=4, dtype="f16",
                         offset_sigma=2.0)
    inp = msda_problem(w, seed=12)
    ref = ref_msda_bwd(inp)
    before = dcnb.dcn_launch_count()
    first = run_msda_bwd(inp)
    assert dcnb.dcn_launch_count() - before == 3
    second = run_msda_bwd(inp)
    check_msda(first, ref, "first")
    check_msda(second, ref, "second")
    assert torch.equal(first[1], second[1]) and torch.equal(first[2], second[2])


def test_msda_backward_far_and_nan_locations():
    """Locations far outside every level, and NaN ones, get zero location and
    weight gradients and add nothing to grad_value; the rest match the oracle."""
    w = gen.MsdaWorkload("far", N=1, M=2, D=16, shapes=((6, 8), (3, 4)), K=2, Lq=9,
                         dtype="f32", offset_sigma=2.0)
    inp = msda_problem(w, seed=14)
    loc = inp["loc"].clone()
    loc[0, 0, 0, 0, 0] = torch.tensor([40.0, -35.0])
    loc[0, 1, 1, 1, 1, 0] = float("nan")
    inp["loc"] = loc
    gv, gl, ga = ref_msda_bwd(inp)
    bad = ~np.isfinite(gl).all(axis=-1)
    gl[bad] = 0.0
    ga[bad] = 0.0
    assert bad.sum() == 1 and np.isfinite(gv).all()
    check_msda(run_msda_bwd(inp), (gv, gl, ga), "far / nan")
