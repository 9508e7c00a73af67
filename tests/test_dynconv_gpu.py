"""GPU parity of dynconv_forward (the ContMix core) against the float64
oracle (tests/parity.py tolerances), through the C interface: the full-size
workloads in the benchmark's launch configuration (checked on sampled batch
items: an output depends on its own image only), then small shapes across
tile edges, window sizes, group widths, dtypes and both weight modes."""
import numpy as np
import pytest
import torch

import deformable_attention_sampling_b200 as dcnb
import gen
import oracle
from tests.parity import compare

pytestmark = pytest.mark.gpu
DEV = "cuda:0"


def run(inp, w, algo="auto"):
    out = dcnb.dynconv(inp["x"].to(DEV), inp["weights"].to(DEV), w.K, w.softmax_flag, algo=algo)
    torch.cuda.synchronize()
    return out


def ref(inp, w, n=None):
    sel = (lambda t: t[n:n + 1]) if n is not None else (lambda t: t)
    return oracle.dynconv_forward_ref(sel(inp["x"]), sel(inp["weights"]), w.K, w.softmax_flag)


DYN_WORKLOADS = [n for n, w in gen.WORKLOADS.items() if isinstance(w, gen.DynWorkload)]


@pytest.mark.parametrize("algo", ["tensor", "simt"])
@pytest.mark.parametrize("name", DYN_WORKLOADS)
def test_dynconv_workload_full_size(name, algo):
    w = gen.WORKLOADS[name]
    inp = gen.dynconv_inputs(w, seed=0)
    out = run(inp, w, algo)
    for n in sorted({0, w.N // 2, w.N - 1}):
        compare(out[n:n + 1], ref(inp, w, n), f"{name} {algo} image {n}")


TENSOR_SMALL = [
    # N, H, W, C, G, K, dtype, softmax: the tensor-core kernel (16-bit, K = 7 or 13)
    (1, 1, 1, 16, 1, 7, "f16", 1),         # one pixel: every tap but the centre is padding
    (2, 9, 17, 32, 2, 7, "f16", 1),        # second 16-column block holds one column
    (1, 8, 32, 64, 4, 13, "bf16", 1),      # exactly one tile
    (1, 19, 70, 16, 1, 13, "f16", 0),      # weights as given; ragged rows and columns
    (2, 13, 40, 64, 2, 13, "bf16", 1),     # D = 32: two 16-channel chunks per group
    (1, 3, 5, 48, 3, 13, "f16", 1),        # window wider and taller than the map
    (3, 11, 45, 32, 2, 7, "bf16", 0),
]


@pytest.mark.parametrize("case", TENSOR_SMALL, ids=[f"tc{i}" for i in range(len(TENSOR_SMALL))])
def test_dynconv_tensor_small_shapes(case):
    N, H, W, C, G, K, dt, sm = case
    w = gen.DynWorkload("tc", N=N, H=H, W=W, C=C, G=G, K=K, dtype=dt, softmax_flag=sm)
    inp = gen.dynconv_inputs(w, seed=11)
    expect = ref(inp, w)
    tc = run(inp, w, "tensor")
    compare(tc, expect, f"{case} tensor")
    compare(run(inp, w, "simt"), expect, f"{case} simt")
    assert torch.equal(run(inp, w, "auto"), tc), "auto takes the tensor-core kernel"


@pytest.mark.parametrize("dt", ["f16", "bf16"])
def test_dynconv_tensor_large_logits(dt):
    """Logits far from 0 and rising along the rows: the running maximum
    grows from one kernel row to the next, so the accumulators are rescaled."""
    w = gen.DynWorkload("big", N=1, H=12, W=35, C=32, G=2, K=13, dtype=dt)
    inp = gen.dynconv_inputs(w, seed=6)
    ramp = torch.arange(13, dtype=torch.float64).repeat_interleave(13) * 3.0
    inp["weights"] = (inp["weights"].double() * 20.0 + 40.0 + ramp).to(inp["weights"].dtype)
    compare(run(inp, w, "tensor"), ref(inp, w), f"large logits {dt}")


def test_dynconv_tensor_rejects_what_it_does_not_cover():
    for dt, K in (("f32", 7), ("f16", 5), ("bf16", 9)):
        C = 16 if dt != "f32" else 8
        w = gen.DynWorkload("rej", N=1, H=6, W=9, C=C, G=1, K=K, dtype=dt)
        inp = gen.dynconv_inputs(w, seed=2)
        with pytest.raises(dcnb.DcnError) as e:
            run(inp, w, "tensor")
        assert e.value.status == dcnb.DCN_ERR_UNSUPPORTED
        compare(run(inp, w, "auto"), ref(inp, w), f"auto falls back ({dt}, K={K})")
    with pytest.raises(ValueError):
        run(inp, w, "band")


SMALL = [
    # N, H, W, C, G, K, dtype, softmax
    (1, 1, 1, 16, 1, 1, "f16", 1),
    (2, 5, 7, 32, 2, 3, "f16", 1),
    (1, 9, 33, 64, 4, 5, "bf16", 1),       # a second, ragged column tile
    (1, 67, 40, 16, 1, 7, "f16", 1),       # more than 64 rows: 16-row tiles
    (2, 13, 70, 32, 1, 13, "f16", 0),      # D = 32: two 32-byte channel chunks
    (1, 6, 6, 16, 2, 13, "f32", 1),        # D = 8 fp32; window wider than the map
    (1, 20, 24, 48, 3, 17, "bf16", 1),     # more than 16 taps per kernel row
    (1, 5, 5, 16, 1, 31, "f16", 1),        # the largest window on a tiny map
    (3, 8, 12, 24, 3, 9, "f32", 0),        # D = 8 fp32, weights used as given
    (1, 31, 29, 64, 4, 7, "f32", 1),       # D = 16 fp32: two chunks
]


@pytest.mark.parametrize("case", SMALL, ids=[f"case{i}" for i in range(len(SMALL))])
def test_dynconv_small_shapes(case):
    N, H, W, C, G, K, dt, sm = case
    w = gen.DynWorkload("small", N=N, H=H, W=W, C=C, G=G, K=K, dtype=dt, softmax_flag=sm)
    inp = gen.dynconv_inputs(w, seed=3)
    compare(run(inp, w), ref(inp, w), str(case))


def test_dynconv_large_logits_and_one_launch():
    """Logits far from 0 (the max subtraction keeps exp finite), one launch."""
    w = gen.DynWorkload("big", N=2, H=10, W=11, C=32, G=2, K=5, dtype="f32")
    inp = gen.dynconv_inputs(w, seed=4)
    inp["weights"] = inp["weights"] * 40.0 + 60.0
    before = dcnb.dcn_launch_count()
    out = run(inp, w)
    assert dcnb.dcn_launch_count() - before == 1
    compare(out, ref(inp, w), "large logits")


def test_dynconv_x_on_a_16_byte_boundary_and_errors():
    w = gen.DynWorkload("mis", N=1, H=6, W=9, C=16, G=1, K=3, dtype="f16")
    inp = gen.dynconv_inputs(w, seed=5)
    buf = torch.empty(inp["x"].numel() + 8, dtype=torch.float16, device=DEV)
    x = buf[8:].view(inp["x"].shape)          # 16 bytes past a 32-byte boundary
    x.copy_(inp["x"].to(DEV))
    out = dcnb.dynconv(x, inp["weights"].to(DEV), w.K)
    torch.cuda.synchronize()
    compare(out, ref(inp, w), "x at 16 bytes")
    bad = torch.empty(out.numel() + 8, dtype=torch.float16, device=DEV)[8:].view(out.shape)
    with pytest.raises(dcnb.DcnError) as e:
        dcnb.dynconv(x, inp["weights"].to(DEV), w.K, out=bad)
    assert e.value.status == dcnb.DCN_ERR_MISALIGNED


def test_dynconv_empty_batch():
    x = torch.empty((0, 4, 4, 16), dtype=torch.float16, device=DEV)
    wt = torch.empty((0, 4, 4, 1, 9), dtype=torch.float16, device=DEV)
    before = dcnb.dcn_launch_count()
    out = dcnb.dynconv(x, wt, 3)
    assert dcnb.dcn_launch_count() == before and out.shape == x.shape
    assert np.prod(out.shape) == 0


@pytest.mark.parametrize("dt", ["f16", "bf16", "f32"])
def test_dynconv_one_by_one_softmax_is_the_identity(dt):
    """K = 1 with the softmax: every weight is exactly 1, so out == x bit for bit."""
    C = 16 if dt != "f32" else 8
    w = gen.DynWorkload("k1", N=2, H=5, W=37, C=C, G=1, K=1, dtype=dt)
    inp = gen.dynconv_inputs(w, seed=13)
    out = run(inp, w)
    assert torch.equal(out.cpu(), inp["x"])
