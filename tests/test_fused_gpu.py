"""GPU parity of dcnv4_fused_forward (the DCNv4 core fed by its merged
offset / mask linear on the tensor cores) against the float64 oracle: the
merged linear as a float64 matmul, then the DCN oracle.

Both kernels are checked: the band kernel with the linear as one tcgen05
product per step ("band"), and the gather kernel with the linear per warp run
on mma.sync ("gather"); "auto" takes the band kernel where it applies."""
import numpy as np
import pytest
import torch

import deformable_attention_sampling_b200 as dcnb
import gen
import oracle
from tests.parity import compare

pytestmark = pytest.mark.gpu
DEV = "cuda:0"


def run(inp, w, bias=True, algo="auto"):
    d = {k: v.to(DEV) for k, v in inp.items()}
    out = dcnb.dcnv4_fused(d["x"], d["w_om"], d["b_om"] if bias else None, groups=w.G, kh=w.kh,
                           kw=w.kw, pad=w.pad, dil=w.dil, algo=algo)
    torch.cuda.synchronize()
    return out


def ref(inp, w, n=None, bias=True):
    x = inp["x"] if n is None else inp["x"][n:n + 1]
    out, _, _ = oracle.dcnv4_front_end_ref(x, inp["w_om"], inp["b_om"] if bias else None, w.kh,
                                           w.kw, w.pad, w.dil, w.G)
    return out


@pytest.mark.parametrize("algo", ["band", "gather"])
def test_fused_headline_shape_full_size(algo):
    w = gen.WORKLOADS["dcnv4_fused_f16_64x56x56x64_g4"]
    inp = gen.front_end_inputs(w, seed=0)
    out = run(inp, w, algo=algo)
    for n in (0, w.N // 2, w.N - 1):
        compare(out[n:n + 1], ref(inp, w, n), f"{w.name} {algo} image {n}")


CASES = [
    # N, H, W, C, G, k, pad, dil, dtype
    (1, 6, 7, 64, 4, 3, 1, 1, "f16"),
    (2, 9, 13, 32, 2, 3, 1, 1, "bf16"),      # 16 pixels per run: full 16-row tiles
    (1, 5, 11, 128, 8, 3, 1, 1, "f16"),      # 4 pixels per run
    (1, 8, 9, 64, 1, 3, 1, 1, "f16"),        # D = 64: 4 lanes per item
    (1, 7, 40, 16, 1, 3, 1, 1, "bf16"),      # 32 pixels per run: two m-tiles
    (2, 9, 10, 32, 2, 5, 2, 1, "f16"),       # 5 x 5 window
    (1, 10, 12, 64, 4, 3, 2, 2, "bf16"),     # dilation 2
]


@pytest.mark.parametrize("case", CASES, ids=[f"case{i}" for i in range(len(CASES))])
def test_fused_small_shapes(case):
    N, H, W, C, G, k, pad, dil, dt = case
    w = gen.FusedWorkload("small", N=N, H=H, W=W, C=C, G=G, kh=k, kw=k, pad=pad, dil=dil, dtype=dt)
    inp = gen.front_end_inputs(w, seed=4)
    compare(run(inp, w), ref(inp, w), str(case))


BAND_CASES = [
    # N, H, W, C, G, k, pad, dil, dtype
    (2, 12, 14, 64, 4, 3, 1, 1, "f16"),
    (2, 10, 20, 128, 8, 3, 1, 1, "bf16"),    # two 64-channel K slices, 216 outputs
    (2, 9, 32, 64, 4, 1, 0, 1, "f16"),       # 1 x 1 window: 128 pixels per step, the whole M tile
    (3, 5, 9, 64, 4, 1, 0, 1, "bf16"),       # 1 x 1 window: 12 outputs
    (2, 12, 16, 64, 4, 3, 2, 2, "f16"),      # dilation 2
    (5, 3, 8, 64, 4, 3, 1, 1, "f16"),        # several images per CTA
    (1, 12, 8, 256, 16, 1, 0, 1, "bf16"),    # C = 256: four K slices
]


@pytest.mark.parametrize("case", BAND_CASES, ids=[f"band{i}" for i in range(len(BAND_CASES))])
def test_fused_band_kernel_small_shapes(case):
    N, H, W, C, G, k, pad, dil, dt = case
    w = gen.FusedWorkload("band", N=N, H=H, W=W, C=C, G=G, kh=k, kw=k, pad=pad, dil=dil,
                          dtype=dt)
    inp = gen.front_end_inputs(w, seed=6)
    expect = ref(inp, w)
    band = run(inp, w, algo="band")
    compare(band, expect, f"{case} band")
    if C <= 128:   # the gather kernel's per-warp linear holds at most 128 channels
        compare(run(inp, w, algo="gather"), expect, f"{case} gather")
    assert torch.equal(run(inp, w, algo="auto"), band)


def test_fused_band_kernel_rejects_other_shapes():
    w = gen.FusedWorkload("no", N=1, H=6, W=7, C=32, G=2, dtype="f16")   # C not a multiple of 64
    inp = gen.front_end_inputs(w, seed=6)
    with pytest.raises(dcnb.DcnError) as e:
        run(inp, w, algo="band")
    assert e.value.status == dcnb.DCN_ERR_UNSUPPORTED
    compare(run(inp, w, algo="auto"), ref(inp, w), "auto falls back")


def test_fused_no_wait_ran_out():
    assert dcnb.dcn_device_flags() & dcnb.DCN_FLAG_WAIT_TIMEOUT == 0


def test_fused_without_bias_and_one_launch():
    w = gen.FusedWorkload("nb", N=2, H=8, W=8, C=64, G=4)
    inp = gen.front_end_inputs(w, seed=5)
    before = dcnb.dcn_launch_count()
    out = run(inp, w, bias=False)
    assert dcnb.dcn_launch_count() - before == 1
    compare(out, ref(inp, w, bias=False), "no bias")


def test_fused_rejects_float32_and_uneven_windows():
    x = torch.zeros((1, 4, 4, 16), device=DEV)
    wom = torch.zeros((1 * 9 * 3, 16), device=DEV)
    with pytest.raises(dcnb.DcnError) as e:
        dcnb.dcnv4_fused(x, wom, None, groups=1)
    assert e.value.status == dcnb.DCN_ERR_UNSUPPORTED
    xh = x.half()
    with pytest.raises(dcnb.DcnError) as e:
        dcnb.dcnv4_fused(xh, wom.half(), None, groups=1, pad=0)
    assert e.value.status == dcnb.DCN_ERR_UNSUPPORTED
