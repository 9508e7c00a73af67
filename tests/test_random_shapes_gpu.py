"""Seeded random small shapes for every forward entry point (the DCN and
MSDA cores, the MSDA reference variants, the fused DCNv4 front end and the
ContMix core) and the two backward calls. Each is checked element by element
against the float64 oracle (tests/parity.py tolerances).

The shapes are drawn once from a fixed generator, so the test set is the same
on every run. They cover the kernels' dispatch decisions between them:
- the band or gather kernel for the DCN core;
- the tensor-core or CUDA-core kernel for the ContMix core;
- staged or unstaged MSDA runs, with odd and even L·K.
They also cover ragged edges: maps narrower than a warp run, channel counts
that split into several 32-byte chunks, and windows wider than the map.
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


def _dcn_cases(count=24, seed=2024):
    rng = np.random.default_rng(seed)
    cases = []
    while len(cases) < count:
        G = int(rng.choice([1, 2, 4, 8]))
        dt = str(rng.choice(["f16", "bf16", "f32"]))
        D = int(rng.choice([16, 32])) if dt != "f32" else int(rng.choice([8, 16]))
        k = int(rng.choice([1, 3, 5]))
        dil = int(rng.choice([1, 2]))
        pad = (k - 1) * dil // 2
        stride = int(rng.choice([1, 1, 2]))
        H, W = int(rng.integers(1, 24)), int(rng.integers(1, 40))
        if gen.DcnWorkload("t", N=1, H=H, W=W, C=D * G, G=G, kh=k, kw=k, stride=stride, pad=pad,
                           dil=dil).Ho <= 0:
            continue
        cases.append(dict(N=int(rng.integers(1, 4)), H=H, W=W, C=D * G, G=G, kh=k, kw=k,
                          stride=stride, pad=pad, dil=dil, dtype=dt,
                          offset_sigma=float(rng.choice([0.5, 2.0, 6.0])),
                          softmax_flag=int(rng.integers(0, 2))))
    return cases


@pytest.mark.parametrize("case", _dcn_cases(), ids=lambda c: "dcn_" + "_".join(
    f"{k}{v}" for k, v in c.items() if k in ("N", "H", "W", "C", "G", "kh", "stride", "dtype")))
def test_dcn_random_shapes(case):
    w = gen.DcnWorkload("rand", **case)
    inp = gen.dcn_inputs(w, seed=5)
    out = dcnb.dcn(inp["x"].to(DEV), inp["offset"].to(DEV), inp["mask"].to(DEV), w.kh, w.kw,
                   w.stride, w.pad, w.dil, w.softmax_flag)
    torch.cuda.synchronize()
    ref = oracle.dcn_forward_ref(inp["x"], inp["offset"], inp["mask"], w.kh, w.kw, w.stride,
                                 w.pad, w.dil, w.softmax_flag)
    compare(out, ref, str(case))


def _msda_cases(count=12, seed=77):
    rng = np.random.default_rng(seed)
    cases = []
    for _ in range(count):
        L = int(rng.integers(1, 5))
        shapes = tuple((int(rng.integers(1, 20)), int(rng.integers(1, 20))) for _ in range(L))
        dt = str(rng.choice(["f32", "f16", "bf16"]))
        cases.append(dict(N=int(rng.integers(1, 3)), M=int(rng.choice([1, 2, 8])),
                          D=int(rng.choice([8, 16, 32])), shapes=shapes,
                          K=int(rng.integers(1, 6)), Lq=int(rng.integers(1, 90)), dtype=dt,
                          offset_sigma=float(rng.choice([1.0, 3.0]))))
    return cases


@pytest.mark.parametrize("case", _msda_cases(), ids=lambda c: "msda_" + "_".join(
    f"{k}{v}" for k, v in c.items() if k in ("N", "M", "D", "K", "Lq", "dtype")))
def test_msda_random_shapes(case):
    m = gen.MsdaWorkload("rand", **case)
    inp = gen.msda_inputs(m, seed=9)
    out = dcnb.msda(inp["value"].to(DEV), inp["spatial_shapes"].to(DEV),
                    inp["level_start"].to(DEV), inp["loc"].to(DEV), inp["attn"].to(DEV))
    torch.cuda.synchronize()
    ref = oracle.msda_forward_ref(inp["value"], inp["spatial_shapes"], inp["level_start"],
                                  inp["loc"], inp["attn"])
    compare(out, ref, str(case))


def _dyn_cases(count=12, seed=31):
    rng = np.random.default_rng(seed)
    cases = []
    for _ in range(count):
        dt = str(rng.choice(["f16", "bf16", "f32"]))
        G = int(rng.choice([1, 2, 4]))
        D = int(rng.choice([16, 32])) if dt != "f32" else int(rng.choice([8, 16]))
        cases.append(dict(N=int(rng.integers(1, 3)), H=int(rng.integers(1, 30)),
                          W=int(rng.integers(1, 50)), C=D * G, G=G,
                          K=int(rng.choice([3, 7, 7, 13, 13])), dtype=dt,
                          softmax_flag=int(rng.choice([0, 1, 1]))))
    return cases


@pytest.mark.parametrize("case", _dyn_cases(), ids=lambda c: "dyn_" + "_".join(
    f"{k}{v}" for k, v in c.items() if k in ("N", "H", "W", "C", "G", "K", "dtype")))
def test_dynconv_random_shapes(case):
    d = gen.DynWorkload("rand", **case)
    inp = gen.dynconv_inputs(d, seed=4)
    out = dcnb.dynconv(inp["x"].to(DEV), inp["weights"].to(DEV), d.K, d.softmax_flag)
    torch.cuda.synchronize()
    ref = oracle.dynconv_forward_ref(inp["x"], inp["weights"], d.K, d.softmax_flag)
    compare(out, ref, str(case))


# ------------------------------------------------------------------ backward

@pytest.mark.parametrize("case", _dcn_cases(count=10, seed=4242), ids=lambda c: "dcnb_" + "_".join(
    f"{k}{v}" for k, v in c.items() if k in ("N", "H", "W", "C", "G", "kh", "stride", "dtype")))
def test_dcn_backward_random_shapes(case):
    w = gen.DcnWorkload("rand", **case)
    inp = gen.dcn_inputs(w, seed=6)
    go = gen.grad_out((w.N, w.Ho, w.Wo, w.C), w.dtype, seed=6)
    got = dcnb.dcn_grad(inp["x"].to(DEV), inp["offset"].to(DEV), inp["mask"].to(DEV),
                        go.to(DEV), w.kh, w.kw, w.stride, w.pad, w.dil, w.softmax_flag)
    torch.cuda.synchronize()
    ref = oracle.dcn_backward_ref(inp["x"], inp["offset"], inp["mask"], go, w.kh, w.kw,
                                  w.stride, w.pad, w.dil, w.softmax_flag)
    for name, g, r in zip(("grad_x", "grad_offset", "grad_mask"), got, ref):
        compare(g, r, f"{case} {name}")


@pytest.mark.parametrize("case", _msda_cases(count=6, seed=99), ids=lambda c: "msdab_" + "_".join(
    f"{k}{v}" for k, v in c.items() if k in ("N", "M", "D", "K", "Lq", "dtype")))
def test_msda_backward_random_shapes(case):
    m = gen.MsdaWorkload("rand", **case)
    inp = gen.msda_inputs(m, seed=10)
    go = gen.grad_out((m.N, m.queries, m.M * m.D), m.dtype, seed=10)
    got = dcnb.msda_grad(inp["value"].to(DEV), inp["spatial_shapes"].to(DEV),
                         inp["level_start"].to(DEV), inp["loc"].to(DEV), inp["attn"].to(DEV),
                         go.to(DEV))
    torch.cuda.synchronize()
    ref = oracle.msda_backward_ref(inp["value"], inp["spatial_shapes"], inp["level_start"],
                                   inp["loc"], inp["attn"], go)
    for name, g, r in zip(("grad_value", "grad_loc", "grad_attn"), got, ref):
        compare(g, r, f"{case} {name}")


# ----------------------------------------------- reference variants, front end

@pytest.mark.parametrize("case", _msda_cases(count=6, seed=123), ids=lambda c: "pts_" + "_".join(
    f"{k}{v}" for k, v in c.items() if k in ("N", "M", "D", "K", "Lq", "dtype")))
@pytest.mark.parametrize("ref_dim", [2, 4])
def test_msda_points_random_shapes(case, ref_dim):
    m = gen.MsdaWorkload("rand", ref_dim=ref_dim, **case)
    inp = gen.msda_ref_inputs(m, seed=12)
    d = {k: v.to(DEV) for k, v in inp.items() if torch.is_tensor(v)}
    out = dcnb.msda_points(d["value"], d["spatial_shapes"], d["level_start"], d["reference"],
                           d["offsets"], d["attn"], d["valid_ratios"])
    torch.cuda.synchronize()
    ref = oracle.msda_points_ref(inp["value"], inp["spatial_shapes"], inp["level_start"],
                                 inp["reference"], inp["offsets"], inp["attn"],
                                 inp["valid_ratios"])
    compare(out, ref, f"{case} ref_dim={ref_dim}")


def _fused_cases(count=8, seed=555):
    rng = np.random.default_rng(seed)
    cases = []
    for _ in range(count):
        G = int(rng.choice([4, 8, 16]))
        k = int(rng.choice([1, 3]))
        cases.append(dict(N=int(rng.integers(1, 3)), H=int(rng.integers(2, 20)),
                          W=int(rng.integers(2, 40)), C=16 * G, G=G, kh=k, kw=k,
                          pad=(k - 1) // 2, dil=1, dtype=str(rng.choice(["f16", "bf16"]))))
    return cases


@pytest.mark.parametrize("case", _fused_cases(), ids=lambda c: "fused_" + "_".join(
    f"{k}{v}" for k, v in c.items() if k in ("N", "H", "W", "C", "kh", "dtype")))
def test_fused_front_end_random_shapes(case):
    f = gen.FusedWorkload("rand", **case)
    inp = gen.front_end_inputs(f, seed=13)
    out = dcnb.dcnv4_fused(inp["x"].to(DEV), inp["w_om"].to(DEV), inp["b_om"].to(DEV),
                           groups=f.G, kh=f.kh, kw=f.kw, pad=f.pad, dil=f.dil)
    torch.cuda.synchronize()
    ref, _, _ = oracle.dcnv4_front_end_ref(inp["x"], inp["w_om"], inp["b_om"], f.kh, f.kw,
                                           f.pad, f.dil, f.G)
    compare(out, ref, str(case))
