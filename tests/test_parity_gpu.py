"""GPU parity: the CUDA path through the C interface against the float64 oracle.

Every test feeds both sides the same seeded, dtype-rounded inputs and compares
every output element (tests/parity.py states the tolerances).  The workloads
run at their full sizes, in the launch configuration the benchmark times, plus
small shapes that span several blocks and a ragged tail, and the edge cases:
odd sizes, every vector width, strided / dilated / padded windows, offsets far
outside the map, huge and non-finite offsets, misaligned bases, empty batches.
"""
import numpy as np
import pytest
import torch

import deformable_attention_sampling_b200 as dcnb
import gen
import oracle
from tests.parity import compare

pytestmark = pytest.mark.gpu
DEV = "cuda:0"
DT = {"f32": torch.float32, "f16": torch.float16, "bf16": torch.bfloat16}


def run_dcn(inp, w, **kw):
    d = {k: v.to(DEV) for k, v in inp.items()}
    out = dcnb.dcn(d["x"], d["offset"], d["mask"], w.kh, w.kw, w.stride, w.pad, w.dil,
                   w.softmax_flag, **kw)
    torch.cuda.synchronize()
    return out


def ref_dcn(inp, w):
    return oracle.dcn_forward_ref(inp["x"], inp["offset"], inp["mask"], w.kh, w.kw, w.stride,
                                  w.pad, w.dil, w.softmax_flag)


def run_msda(inp):
    d = {k: (v.to(DEV) if torch.is_tensor(v) else v) for k, v in inp.items()}
    out = dcnb.msda(d["value"], d["spatial_shapes"], d["level_start"], d["loc"], d["attn"])
    torch.cuda.synchronize()
    return out


def ref_msda(inp):
    return oracle.msda_forward_ref(inp["value"], inp["spatial_shapes"], inp["level_start"],
                                   inp["loc"], inp["attn"])


# ------------------------------------------------------------ full workloads

DCN_WORKLOADS = [n for n, w in gen.WORKLOADS.items() if isinstance(w, gen.DcnWorkload)]


@pytest.mark.parametrize("name", DCN_WORKLOADS)
def test_dcn_workload_full_size(name):
    w = gen.WORKLOADS[name]
    inp = gen.dcn_inputs(w, seed=0)
    compare(run_dcn(inp, w), ref_dcn(inp, w), name)


def test_msda_workload_full_size():
    w = gen.WORKLOADS["msda_f32_2x4lvl_m8_d32_k4"]
    inp = gen.msda_inputs(w, seed=0)
    compare(run_msda(inp), ref_msda(inp), w.name)


@pytest.mark.parametrize("seed", [1, 2])
def test_headline_workload_other_seeds(seed):
    w = gen.WORKLOADS[gen.HEADLINE]
    inp = gen.dcn_inputs(w, seed=seed)
    compare(run_dcn(inp, w), ref_dcn(inp, w), f"{w.name} seed {seed}")


# ------------------------------------------------------------ small shapes

SMALL = [
    # N, H, W, C, G, kh, kw, stride, pad, dil, dtype, softmax, sigma
    (1, 1, 1, 8, 1, 1, 1, 1, 0, 1, "f32", 0, 0.5),
    (2, 2, 3, 16, 1, 3, 3, 1, 1, 1, "f16", 0, 1.0),
    (1, 3, 5, 32, 2, 3, 3, 1, 1, 1, "bf16", 1, 2.0),
    (3, 5, 7, 64, 4, 3, 3, 1, 1, 1, "f16", 0, 2.0),
    (2, 9, 11, 48, 2, 3, 3, 2, 1, 1, "f16", 0, 1.5),     # D = 24: 16-byte vectors
    (1, 8, 8, 6, 3, 3, 3, 1, 2, 2, "f32", 1, 1.0),       # D = 2, dilation 2
    (2, 7, 6, 5, 5, 2, 3, 1, 1, 1, "f16", 0, 1.0),       # D = 1: 2-byte vectors
    (1, 6, 9, 12, 3, 5, 5, 1, 2, 1, "bf16", 1, 2.5),     # D = 4, 5x5
    (2, 10, 4, 128, 2, 1, 3, 1, 0, 1, "f32", 0, 3.0),    # D = 64 fp32: 8 threads/item
    (1, 13, 17, 256, 2, 3, 3, 2, 0, 3, "f16", 0, 4.0),   # D = 128 fp16
    (1, 12, 12, 64, 4, 7, 7, 1, 3, 1, "f16", 1, 3.0),    # 7x7 window, softmax
    (4, 14, 14, 64, 4, 3, 3, 1, 1, 1, "f32", 1, 1.0),    # DCNv3 fp32 shape, N = 4
    (2, 16, 16, 32, 4, 3, 3, 1, 1, 1, "bf16", 0, 20.0),  # offsets mostly far outside
    (1, 5, 40, 40, 5, 3, 3, 1, 1, 1, "f16", 0, 2.0),     # D = 8: 16-byte vectors
]


@pytest.mark.parametrize("case", SMALL, ids=[f"case{i}" for i in range(len(SMALL))])
def test_dcn_small_shapes(case):
    N, H, W, C, G, kh, kw, stride, pad, dil, dt, sm, sigma = case
    w = gen.DcnWorkload("small", N=N, H=H, W=W, C=C, G=G, kh=kh, kw=kw, stride=stride, pad=pad,
                        dil=dil, dtype=dt, offset_sigma=sigma, softmax_flag=sm)
    inp = gen.dcn_inputs(w, seed=7)
    compare(run_dcn(inp, w), ref_dcn(inp, w), str(case))


@pytest.mark.parametrize("dt", ["f32", "f16", "bf16"])
def test_dcn_ragged_tail_and_many_blocks(dt):
    """An item count that is no multiple of the block size, large enough that
    every resident CTA loops over several blocks."""
    w = gen.DcnWorkload("ragged", N=3, H=37, W=41, C=64, G=4, dtype=dt, offset_sigma=2.0)
    inp = gen.dcn_inputs(w, seed=11)
    compare(run_dcn(inp, w), ref_dcn(inp, w), f"ragged {dt}")


@pytest.mark.parametrize("dt", ["f32", "f16", "bf16"])
def test_dcn_extreme_offsets(dt):
    """Huge, infinite and NaN offsets: such taps contribute 0, like the oracle."""
    w = gen.DcnWorkload("extreme", N=2, H=6, W=7, C=32, G=2, dtype=dt, offset_sigma=1.0)
    inp = gen.dcn_inputs(w, seed=3)
    off = inp["offset"].double()
    big = 1e30 if dt == "f32" else 6e4
    off[0, 0, 0, 0, :, 0] = big
    off[0, 1, 1, 1, :, 1] = -big
    off[1, 2, 2, 0, 4, 0] = float("nan")
    off[1, 3, 3, 1, 2, 1] = float("inf")
    off[1, 4, 4, 0, 7, 0] = -float("inf")
    off[0, 5, 6, 1, :, :] = -1.0 - 2 ** -8     # just outside the top-left corner
    inp["offset"] = off.to(DT[dt])
    compare(run_dcn(inp, w), ref_dcn(inp, w), f"extreme {dt}")


@pytest.mark.parametrize("dt", ["f32", "f16"])
def test_dcn_misaligned_bases_use_narrower_vectors(dt):
    """x and out one element past an aligned address: the library picks a
    narrower vector width and the result is unchanged."""
    w = gen.DcnWorkload("mis", N=2, H=9, W=10, C=64, G=4, dtype=dt)
    inp = gen.dcn_inputs(w, seed=5)
    ref = ref_dcn(inp, w)
    xs = torch.empty(inp["x"].numel() + 1, dtype=DT[dt], device=DEV)
    xs[1:] = inp["x"].reshape(-1).to(DEV)
    x = xs[1:].view(inp["x"].shape)
    os_ = torch.empty(ref.size + 1, dtype=DT[dt], device=DEV)
    out = os_[1:].view(ref.shape)
    dcnb.dcn(x, inp["offset"].to(DEV), inp["mask"].to(DEV), out=out)
    torch.cuda.synchronize()
    compare(out, ref, f"misaligned {dt}")


def test_dcn_output_guard_bands_untouched():
    w = gen.DcnWorkload("guard", N=2, H=11, W=13, C=64, G=4, dtype="f16")
    inp = gen.dcn_inputs(w, seed=9)
    ref = ref_dcn(inp, w)
    guard = 4096
    buf = torch.full((ref.size + 2 * guard,), 1234.0, dtype=torch.float16, device=DEV)
    out = buf[guard:guard + ref.size].view(ref.shape)
    dcnb.dcn(inp["x"].to(DEV), inp["offset"].to(DEV), inp["mask"].to(DEV), out=out)
    torch.cuda.synchronize()
    compare(out, ref, "guard")
    assert bool((buf[:guard] == 1234.0).all()) and bool((buf[-guard:] == 1234.0).all())


def test_dcn_empty_batch_launches_nothing():
    x = torch.empty((0, 8, 8, 16), dtype=torch.float16, device=DEV)
    off = torch.empty((0, 8, 8, 2, 9, 2), dtype=torch.float16, device=DEV)
    mask = torch.empty((0, 8, 8, 2, 9), dtype=torch.float16, device=DEV)
    before = dcnb.dcn_launch_count()
    out = dcnb.dcn(x, off, mask)
    assert out.shape == (0, 8, 8, 16) and dcnb.dcn_launch_count() == before


def test_dcn_side_stream_one_launch_per_call_deterministic():
    w = gen.DcnWorkload("stream", N=4, H=20, W=20, C=64, G=4, dtype="f16")
    inp = gen.dcn_inputs(w, seed=13)
    d = {k: v.to(DEV) for k, v in inp.items()}
    s = torch.cuda.Stream()
    torch.cuda.synchronize()
    before = dcnb.dcn_launch_count()
    with torch.cuda.stream(s):
        a = dcnb.dcn(d["x"], d["offset"], d["mask"], stream=s)
        b = dcnb.dcn(d["x"], d["offset"], d["mask"], stream=s)
    s.synchronize()
    assert dcnb.dcn_launch_count() == before + 2
    assert torch.equal(a, b)                       # bitwise reproducible
    compare(a, ref_dcn(inp, w), "side stream")


# ------------------------------------------------------------ MSDA variants

MSDA_SMALL = [
    # N, M, D, shapes, K, Lq, dtype, sigma
    (1, 1, 1, ((3, 4),), 1, 5, "f32", 1.0),
    (2, 2, 8, ((5, 7), (3, 4)), 2, 9, "f32", 2.0),
    (1, 3, 4, ((6, 5), (3, 3), (2, 2)), 3, 17, "f16", 2.0),
    (2, 8, 32, ((20, 30), (10, 15), (5, 8), (3, 4)), 4, 300, "f32", 2.0),
    (1, 4, 64, ((9, 9), (5, 5)), 8, 40, "bf16", 3.0),
    (2, 2, 16, ((4, 4),) * 16, 2, 11, "f32", 1.0),       # 16 levels
    (1, 2, 12, ((7, 3), (2, 9)), 64, 6, "f32", 5.0),     # 64 points per level
]


@pytest.mark.parametrize("case", MSDA_SMALL, ids=[f"msda{i}" for i in range(len(MSDA_SMALL))])
def test_msda_small_shapes(case):
    N, M, D, shapes, K, Lq, dt, sigma = case
    w = gen.MsdaWorkload("small", N=N, M=M, D=D, shapes=shapes, K=K, Lq=Lq, dtype=dt,
                         offset_sigma=sigma)
    inp = gen.msda_inputs(w, seed=21)
    compare(run_msda(inp), ref_msda(inp), str(case))


def test_msda_locations_far_outside_and_nan():
    w = gen.MsdaWorkload("far", N=1, M=2, D=8, shapes=((6, 8), (3, 4)), K=3, Lq=10,
                         dtype="f32")
    inp = gen.msda_inputs(w, seed=4)
    loc = inp["loc"].clone()
    loc[0, 0, 0, 0, :, 0] = 1e30
    loc[0, 1, 1, 1, 0, 1] = -5.0
    loc[0, 2, 0, 0, 1, 0] = float("nan")
    loc[0, 3, 1, 1, 2, :] = 0.0          # the image corner: one quarter of cell (0, 0)
    inp["loc"] = loc
    compare(run_msda(inp), ref_msda(inp), "msda far")
