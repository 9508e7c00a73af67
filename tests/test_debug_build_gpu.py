"""The debug library (libdcn_b200_debug.so) on the GPU.

It is the forward calls compiled with device-side checks: every gather,
shared-memory and store address against its buffer, and the MSDA level table
on the device. A violation is reported in the status word (dcn_device_flags)
instead of trapping. On valid inputs it must give the release library's
outputs bit for bit and report nothing. A level table with a gap (a broken
precondition of msda_forward, which the release library does not check)
must be reported, and no value row is read.
"""
import ctypes

import pytest
import torch

import deformable_attention_sampling_b200 as dcnb
import gen

pytestmark = pytest.mark.gpu
DEV = "cuda:0"


@pytest.fixture(scope="module")
def dbg():
    lib = dcnb.debug_library()
    assert dcnb.dcn_debug_checks(lib) == 1
    torch.cuda.synchronize()
    dcnb.dcn_device_flags(reset=True, lib=lib)
    return lib


def _stream():
    return int(torch.cuda.current_stream().cuda_stream)


DCN_CASES = [
    # name args, algo: the band kernel, the gather kernel, DCNv3 fp32 (gather)
    (dict(N=2, H=12, W=14, C=64, G=4, dtype="f16", offset_sigma=2.0), 2),
    (dict(N=2, H=12, W=14, C=64, G=4, dtype="bf16", offset_sigma=20.0), 2),
    (dict(N=2, H=12, W=13, C=64, G=4, dtype="f16", offset_sigma=2.0), 1),
    (dict(N=1, H=14, W=14, C=64, G=4, dtype="f32", offset_sigma=1.0, softmax_flag=1), 0),
]


@pytest.mark.parametrize("case", DCN_CASES, ids=[f"dcn{i}" for i in range(len(DCN_CASES))])
def test_debug_dcn_matches_release_and_reports_nothing(dbg, case):
    kw, algo = case
    w = gen.DcnWorkload("dbg", **kw)
    inp = gen.dcn_inputs(w, seed=12)
    off = inp["offset"].double()
    off[0, 0, 0, 0, :, 0] = float("nan")     # taps outside the map and non-finite
    off[0, 1, 1, 1, :, 1] = 1e4
    inp["offset"] = off.to(inp["offset"].dtype)
    d = {k: v.to(DEV) for k, v in inp.items()}
    outs = []
    for lib in (dcnb.library(), dbg):
        out = torch.empty((w.N, w.Ho, w.Wo, w.C), dtype=d["x"].dtype, device=DEV)
        st = lib.dcn_forward_algo(d["x"].data_ptr(), d["offset"].data_ptr(), d["mask"].data_ptr(),
                                  out.data_ptr(), w.N, w.H, w.W, w.C, w.G, w.kh, w.kw, w.stride,
                                  w.pad, w.dil, w.softmax_flag, gen.DTYPE_CODES[w.dtype], algo,
                                  _stream())
        assert st == 0
        outs.append(out)
    torch.cuda.synchronize()
    assert torch.equal(outs[0], outs[1])
    assert dcnb.dcn_device_flags(lib=dbg) == 0


def test_debug_fused_matches_release(dbg):
    w = gen.FusedWorkload("dbg", N=2, H=10, W=14, C=64, G=4)
    inp = gen.front_end_inputs(w, seed=5)
    d = {k: v.to(DEV) for k, v in inp.items()}
    outs = []
    for lib in (dcnb.library(), dbg):
        out = torch.empty_like(d["x"])
        st = lib.dcnv4_fused_forward_algo(d["x"].data_ptr(), d["w_om"].data_ptr(),
                                          d["b_om"].data_ptr(), out.data_ptr(), w.N, w.H, w.W,
                                          w.C, w.G, w.kh, w.kw, w.pad, w.dil,
                                          gen.DTYPE_CODES[w.dtype], 0, _stream())
        assert st == 0
        outs.append(out)
    torch.cuda.synchronize()
    assert torch.equal(outs[0], outs[1])
    assert dcnb.dcn_device_flags(lib=dbg) == 0


def _msda_call(lib, d, w, shapes, starts, out):
    return lib.msda_forward(d["value"].data_ptr(), shapes.data_ptr(), starts.data_ptr(),
                            d["loc"].data_ptr(), d["attn"].data_ptr(), out.data_ptr(), w.N,
                            w.queries, w.M, w.D, w.L, w.K, gen.DTYPE_CODES[w.dtype], _stream())


def test_debug_msda_matches_release_and_flags_a_gapped_level_table(dbg):
    w = gen.MsdaWorkload("dbg", N=2, M=4, D=16, shapes=((9, 12), (5, 6), (3, 3)), K=3, Lq=40)
    inp = gen.msda_inputs(w, seed=6)
    d = {k: (v.to(DEV) if torch.is_tensor(v) else v) for k, v in inp.items() if k != "logits"}
    loc = d["loc"].clone()
    loc[0, 0, 0, 0, :, 0] = float("nan")
    loc[1, 1, 1, 1, 0, :] = 40.0
    d["loc"] = loc
    outs = []
    for lib in (dcnb.library(), dbg):
        out = torch.empty((w.N, w.queries, w.M * w.D), device=DEV)
        assert _msda_call(lib, d, w, d["spatial_shapes"], d["level_start"], out) == 0
        outs.append(out)
    torch.cuda.synchronize()
    assert torch.equal(outs[0], outs[1])
    assert dcnb.dcn_device_flags(lib=dbg) == 0
    # a gap between levels 0 and 1: the table describes rows the value tensor may
    # not have.  Only the debug library is given it; it reports the table and
    # reads nothing, leaving the output as it was.
    bad = d["level_start"].clone()
    bad[1:] += 1000
    out = torch.full((w.N, w.queries, w.M * w.D), 7.0, device=DEV)
    assert _msda_call(dbg, d, w, d["spatial_shapes"], bad, out) == 0
    torch.cuda.synchronize()
    assert dcnb.dcn_device_flags(reset=True, lib=dbg) == dcnb.DCN_FLAG_BAD_LEVELS
    assert bool((out == 7.0).all())
    assert dcnb.dcn_device_flags(lib=dbg) == 0
