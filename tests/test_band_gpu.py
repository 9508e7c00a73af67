"""GPU parity of the two DCN forward kernels (dcn_forward_algo).

The band kernel stages the input rows a CTA's output rows can reach in shared
memory and gathers corners there; the gather kernel reads corners through L1.
Both are checked element by element against the float64 oracle on the same
seeded inputs (tests/parity.py tolerances), and against each other: they add
the same float32 products in the same order, so their outputs are equal bit
for bit, including taps that leave the band (read from global memory).

Shapes cover several images per CTA and CTAs that straddle images, bands
clipped by the map, maps shorter than a band, ragged runs, stride 2,
dilation, a 5 x 3 window, the DCNv3 softmax, heavy offsets that leave the band
often, huge / infinite / NaN offsets, and the full-size stage sweep.
"""
import pytest
import torch

import deformable_attention_sampling_b200 as dcnb
import gen
import oracle
from tests.parity import compare

pytestmark = pytest.mark.gpu
DEV = "cuda:0"
DT = {"f32": torch.float32, "f16": torch.float16, "bf16": torch.bfloat16}


def run(inp, w, algo):
    d = {k: v.to(DEV) for k, v in inp.items()}
    out = dcnb.dcn(d["x"], d["offset"], d["mask"], w.kh, w.kw, w.stride, w.pad, w.dil,
                   w.softmax_flag, algo=algo)
    torch.cuda.synchronize()
    return out


def ref(inp, w):
    return oracle.dcn_forward_ref(inp["x"], inp["offset"], inp["mask"], w.kh, w.kw, w.stride,
                                  w.pad, w.dil, w.softmax_flag)


def check_both(inp, w, label):
    band = run(inp, w, "band")
    gather = run(inp, w, "gather")
    expect = ref(inp, w)
    compare(band, expect, f"{label} band")
    compare(gather, expect, f"{label} gather")
    assert torch.equal(band, gather), f"{label}: band and gather kernels differ"


BAND_SMALL = [
    # N, H, W, C, G, kh, kw, stride, pad, dil, dtype, softmax, sigma
    (2, 12, 14, 64, 4, 3, 3, 1, 1, 1, "f16", 0, 2.0),
    (3, 9, 6, 64, 4, 3, 3, 1, 1, 1, "bf16", 0, 3.0),      # several images per CTA
    (5, 3, 8, 64, 4, 3, 3, 1, 1, 1, "f16", 0, 1.0),       # map shorter than a band
    (2, 7, 7, 512, 32, 3, 3, 1, 1, 1, "bf16", 0, 2.0),    # stage-4 shape, whole map staged
    (2, 14, 14, 256, 16, 3, 3, 1, 1, 1, "bf16", 0, 2.0),
    (2, 28, 28, 128, 8, 3, 3, 1, 1, 1, "bf16", 0, 2.0),
    (1, 30, 19, 64, 4, 3, 3, 2, 1, 1, "f16", 0, 2.0),     # stride 2
    (1, 20, 12, 64, 4, 5, 3, 1, 2, 2, "f16", 0, 2.0),     # 5 x 3 window, dilation 2
    (2, 12, 10, 64, 4, 3, 3, 1, 1, 1, "f16", 1, 2.0),     # DCNv3 softmax; 40-item rows
    (2, 16, 16, 192, 12, 3, 3, 1, 1, 1, "bf16", 1, 1.5),  # G = 12: 384-byte pixels
    (1, 40, 8, 64, 4, 3, 3, 1, 1, 1, "f16", 0, 30.0),     # most taps leave the band
    (2, 33, 16, 64, 4, 1, 1, 1, 0, 1, "f16", 0, 5.0),     # 1 x 1 window
    (1, 5, 40, 64, 4, 3, 3, 1, 1, 1, "bf16", 0, 2.0),
    (2, 12, 14, 64, 4, 3, 3, 1, 0, 1, "f16", 0, 1.0),     # no padding: Ho < H
]


@pytest.mark.parametrize("case", BAND_SMALL, ids=[f"band{i}" for i in range(len(BAND_SMALL))])
def test_band_small_shapes(case):
    N, H, W, C, G, kh, kw, stride, pad, dil, dt, sm, sigma = case
    w = gen.DcnWorkload("band", N=N, H=H, W=W, C=C, G=G, kh=kh, kw=kw, stride=stride, pad=pad,
                        dil=dil, dtype=dt, offset_sigma=sigma, softmax_flag=sm)
    inp = gen.dcn_inputs(w, seed=17)
    check_both(inp, w, str(case))


@pytest.mark.parametrize("dt", ["f16", "bf16"])
def test_band_extreme_offsets(dt):
    """Huge, infinite and NaN offsets (taps that contribute 0), offsets just
    past the band margin, and a tap leaving through the map's bottom edge."""
    w = gen.DcnWorkload("extreme", N=2, H=20, W=8, C=64, G=4, dtype=dt, offset_sigma=1.0)
    inp = gen.dcn_inputs(w, seed=3)
    off = inp["offset"].double()
    off[0, 0, 0, 0, :, 0] = 6e4
    off[0, 1, 1, 1, :, 1] = -6e4
    off[1, 2, 2, 0, 4, 0] = float("nan")
    off[1, 3, 3, 1, 2, 1] = float("inf")
    off[1, 4, 4, 0, 7, 1] = -float("inf")
    off[0, 10, 3, 2, :, 1] = 6.0              # exactly the margin: leaves the band
    off[0, 10, 4, 3, :, 1] = -6.0 - 2 ** -6    # just past it, upwards
    off[0, 10, 5, 1, :, 1] = 5.0 + 2 ** -6     # inside
    off[1, 19, 7, 3, :, 1] = 0.75              # bottom row, corner below the map
    inp["offset"] = off.to(DT[dt])
    check_both(inp, w, f"extreme {dt}")


@pytest.mark.parametrize("name", ["dcnv4_f16_64x56x56x64_g4", "dcnv4_bf16_64x28x28x128_g8",
                                  "dcnv4_bf16_64x7x7x512_g32"])
def test_band_full_size_equals_gather(name):
    w = gen.WORKLOADS[name]
    inp = gen.dcn_inputs(w, seed=4)
    band = run(inp, w, "band")
    gather = run(inp, w, "gather")
    assert torch.equal(band, gather), f"{name}: band and gather kernels differ"
    # sampled outputs against the oracle: the first, middle and last image
    for n in (0, w.N // 2, w.N - 1):
        one = {k: v[n:n + 1] for k, v in inp.items()}
        compare(band[n:n + 1], ref(one, w), f"{name} image {n}")


def test_band_is_taken_by_default_and_unsupported_shapes_fall_back():
    w = gen.DcnWorkload("auto", N=2, H=10, W=12, C=64, G=4, dtype="f16")
    inp = gen.dcn_inputs(w, seed=8)
    auto = run(inp, w, "auto")
    assert torch.equal(auto, run(inp, w, "band"))
    # an odd output width (mask rows of 16 * 9 * 2 * odd bytes) is not for the band kernel
    w2 = gen.DcnWorkload("odd", N=2, H=10, W=11, C=64, G=4, dtype="f16")
    inp2 = gen.dcn_inputs(w2, seed=8)
    with pytest.raises(dcnb.DcnError):
        run(inp2, w2, "band")
    compare(run(inp2, w2, "auto"), ref(inp2, w2), "odd width, auto")


def test_band_output_guard_bands_untouched():
    w = gen.DcnWorkload("guard", N=3, H=11, W=14, C=64, G=4, dtype="bf16")
    inp = gen.dcn_inputs(w, seed=9)
    expect = ref(inp, w)
    guard = 4096
    buf = torch.full((expect.size + 2 * guard,), 1234.0, dtype=torch.bfloat16, device=DEV)
    out = buf[guard:guard + expect.size].view(expect.shape)
    dcnb.dcn(inp["x"].to(DEV), inp["offset"].to(DEV), inp["mask"].to(DEV), out=out, algo="band")
    torch.cuda.synchronize()
    compare(out, expect, "guard")
    assert bool((buf[:guard] == 1234.0).all()) and bool((buf[-guard:] == 1234.0).all())


def test_band_no_wait_ran_out():
    """Runs last in this file: no bounded wait of the band kernel's pipeline
    has given up in any of the calls above."""
    assert dcnb.dcn_device_flags() & dcnb.DCN_FLAG_WAIT_TIMEOUT == 0
