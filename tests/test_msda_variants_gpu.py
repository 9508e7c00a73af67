"""GPU parity of the MSDA reference-point variants (locations formed in the
kernel from point / box references and valid ratios) and of the value
masking, against the float64 oracle (tests/parity.py tolerances)."""
import numpy as np
import pytest
import torch

import deformable_attention_sampling_b200 as dcnb
import gen
import oracle
from tests.parity import compare

pytestmark = pytest.mark.gpu
DEV = "cuda:0"


def run_points(inp, use_ratios=True):
    d = {k: v.to(DEV) for k, v in inp.items()}
    out = dcnb.msda_points(d["value"], d["spatial_shapes"], d["level_start"], d["reference"],
                           d["offsets"], d["attn"], d["valid_ratios"] if use_ratios else None)
    torch.cuda.synchronize()
    return out


def ref_points(inp, use_ratios=True):
    return oracle.msda_points_ref(inp["value"], inp["spatial_shapes"], inp["level_start"],
                                  inp["reference"], inp["offsets"], inp["attn"],
                                  inp["valid_ratios"] if use_ratios else None)


def test_box_workload_full_size():
    w = gen.WORKLOADS["msda_f32_2x4lvl_m8_d32_k4_box300"]
    inp = gen.msda_ref_inputs(w, seed=0)
    compare(run_points(inp), ref_points(inp), w.name)


CASES = [
    # N, shapes, M, D, K, Lq, dtype, ref_dim
    (1, ((6, 9),), 1, 8, 2, 5, "f32", 2),
    (2, ((10, 12), (5, 6)), 2, 16, 4, 7, "f16", 4),
    (1, ((12, 15), (6, 8), (3, 4)), 4, 32, 3, 11, "bf16", 2),
    (2, ((7, 11), (4, 6), (2, 3), (1, 2)), 8, 32, 4, 33, "f32", 4),
    (1, ((9, 9), (4, 4)), 3, 6, 2, 9, "f32", 4),          # 3 lanes per head
]


@pytest.mark.parametrize("case", CASES, ids=[f"case{i}" for i in range(len(CASES))])
@pytest.mark.parametrize("use_ratios", [True, False])
def test_reference_variants_small(case, use_ratios):
    N, shapes, M, D, K, Lq, dt, rd = case
    w = gen.MsdaWorkload("small", N=N, M=M, D=D, shapes=shapes, K=K, Lq=Lq, dtype=dt, ref_dim=rd)
    inp = gen.msda_ref_inputs(w, seed=8)
    compare(run_points(inp, use_ratios), ref_points(inp, use_ratios), f"{case} ratios={use_ratios}")


@pytest.mark.parametrize("dt", ["f32", "f16", "bf16"])
def test_mask_value_and_masked_sampling(dt):
    w = gen.MsdaWorkload("mask", N=2, M=4, D=8, shapes=((8, 10), (4, 5)), K=3, Lq=13, dtype=dt,
                         ref_dim=4)
    inp = gen.msda_ref_inputs(w, seed=9)
    v = inp["value"].to(DEV)
    m = inp["mask"].to(DEV)
    before = dcnb.dcn_launch_count()
    masked = dcnb.mask_value(v, m)
    torch.cuda.synchronize()
    assert dcnb.dcn_launch_count() - before == 1
    expect = oracle.mask_value_ref(inp["value"], inp["mask"].numpy())
    assert np.array_equal(masked.double().cpu().numpy(), expect)
    # in place, then the sampler reads the zeros
    dcnb.mask_value(v, m, out=v)
    inp2 = dict(inp)
    inp2["value"] = v.cpu()
    got = run_points(inp2)
    compare(got, oracle.msda_points_ref(expect, inp["spatial_shapes"], inp["level_start"],
                                        inp["reference"], inp["offsets"], inp["attn"],
                                        inp["valid_ratios"]), f"masked {dt}")


def test_reference_variant_validation():
    w = gen.MsdaWorkload("v", N=1, M=2, D=8, shapes=((4, 4),), K=2, Lq=3, ref_dim=2)
    inp = {k: v.to(DEV) for k, v in gen.msda_ref_inputs(w, seed=1).items()}
    out = torch.empty((1, 3, 16), device=DEV)
    with pytest.raises(dcnb.DcnError) as e:
        dcnb.msda_forward_points(inp["value"], inp["spatial_shapes"], inp["level_start"],
                                 inp["reference"], 3, None, inp["offsets"], inp["attn"], out,
                                 1, 3, 2, 8, 1, 2, 0)
    assert e.value.status == dcnb.DCN_ERR_INVALID_ARG


def test_mask_value_rows_not_multiple_of_16_bytes():
    """M * D * 4 = 36 bytes per row: the element-wise path, out of place and in place."""
    N, S, M, D = 2, 11, 3, 3
    value = torch.randn(N, S, M, D, device=DEV)
    mask = torch.rand(N, S, device=DEV) < 0.4
    expect = value.masked_fill(mask[:, :, None, None], 0.0)
    assert torch.equal(dcnb.mask_value(value, mask), expect)
    dcnb.mask_value(value, mask, out=value)
    torch.cuda.synchronize()
    assert torch.equal(value, expect)
