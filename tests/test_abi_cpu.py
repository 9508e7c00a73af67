"""The C interface without a GPU: the library builds, loads and exports every
symbol include/dcn.h declares, and host-side validation returns the documented
status before any CUDA call (fake, never-dereferenced pointer values)."""
import ctypes
import os
import re

import pytest

import deformable_attention_sampling_b200 as dcnb
from deformable_attention_sampling_b200 import build as dcn_build
import oracle

HEADER = os.path.join(dcn_build.INCLUDE, "dcn.h")

# plausible, 256-byte aligned fake device addresses; validation never reads them
X, OFF, MASK, OUT = 0x7F0000000000, 0x7F0010000000, 0x7F0020000000, 0x7F0030000000
F16 = 1


@pytest.fixture(scope="module")
def lib():
    dcn_build.build()
    return dcnb.library()


def declared_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return set(re.findall(r"^\s*DCN_API\s+(?:const\s+)?(?:\w+\s+)*?\w+\*?\s+\*?(\w+)\s*\(",
                          text, flags=re.M))


def test_header_declares_the_interface():
    names = declared_functions()
    assert {"dcn_forward", "msda_forward", "dcn_backward", "msda_backward",
            "dcn_backward_workspace_size", "msda_backward_workspace_size",
            "dcn_status_string"} <= names
    assert names == set(dcnb.SIGNATURES), "binding signatures out of sync with dcn.h"


def test_library_exports_every_declared_symbol(lib):
    for name in declared_functions():
        assert hasattr(lib, name), name
    # the library is the in-tree build, not an installed copy
    assert os.path.dirname(dcnb.LIB_PATH).startswith(os.path.dirname(dcn_build.LIB_DIR))


def test_status_strings_and_version(lib):
    assert dcnb.dcn_status_string(0) == "ok"
    for s in (-1, -2, -3, -4, 123):
        assert isinstance(dcnb.dcn_status_string(s), str) and dcnb.dcn_status_string(s)
    assert dcnb.dcn_version() >= 10000
    assert dcnb.dcn_last_cuda_error() == 0
    assert dcnb.dcn_launch_count() == 0


@pytest.mark.parametrize("n_in,k,stride,pad,dil", [
    (56, 3, 1, 1, 1), (7, 3, 2, 1, 1), (10, 5, 1, 2, 2), (4, 3, 1, 0, 2), (1, 1, 1, 0, 1),
    (3, 5, 1, 0, 1), (200, 3, 2, 0, 3)])
def test_output_size_matches_the_oracle(lib, n_in, k, stride, pad, dil):
    expect = oracle.out_size(n_in, k, stride, pad, dil)
    assert dcnb.dcn_output_size(n_in, k, stride, pad, dil) == max(expect, 0)


def call_dcn(lib, **kw):
    args = dict(x=X, offset=OFF, mask=MASK, out=OUT, N=2, H=8, W=8, C=16, G=2, kh=3, kw=3,
                stride=1, pad=1, dil=1, softmax_flag=0, dtype=F16, stream=None)
    args.update(kw)
    return lib.dcn_forward(args["x"], args["offset"], args["mask"], args["out"], args["N"],
                           args["H"], args["W"], args["C"], args["G"], args["kh"], args["kw"],
                           args["stride"], args["pad"], args["dil"], args["softmax_flag"],
                           args["dtype"], args["stream"])


@pytest.mark.parametrize("change,status", [
    (dict(dtype=7), dcnb.DCN_ERR_INVALID_ARG),
    (dict(N=-1), dcnb.DCN_ERR_INVALID_ARG),
    (dict(H=0), dcnb.DCN_ERR_INVALID_ARG),
    (dict(C=15), dcnb.DCN_ERR_INVALID_ARG),            # C % G != 0
    (dict(G=0), dcnb.DCN_ERR_INVALID_ARG),
    (dict(kh=0), dcnb.DCN_ERR_INVALID_ARG),
    (dict(stride=0), dcnb.DCN_ERR_INVALID_ARG),
    (dict(pad=-1), dcnb.DCN_ERR_INVALID_ARG),
    (dict(dil=0), dcnb.DCN_ERR_INVALID_ARG),
    (dict(softmax_flag=2), dcnb.DCN_ERR_INVALID_ARG),
    (dict(H=2, pad=0), dcnb.DCN_ERR_INVALID_ARG),      # Ho <= 0
    (dict(x=None), dcnb.DCN_ERR_INVALID_ARG),
    (dict(out=None), dcnb.DCN_ERR_INVALID_ARG),
    (dict(out=X), dcnb.DCN_ERR_INVALID_ARG),           # out aliases x
    (dict(out=OFF + 64), dcnb.DCN_ERR_INVALID_ARG),    # out overlaps offset
    (dict(x=X + 1), dcnb.DCN_ERR_MISALIGNED),          # not 2-byte aligned
    (dict(mask=MASK + 2, dtype=0), dcnb.DCN_ERR_MISALIGNED),   # f32 needs 4 bytes
    (dict(H=70000), dcnb.DCN_ERR_UNSUPPORTED),
    (dict(kh=33, kw=33, pad=16), dcnb.DCN_ERR_UNSUPPORTED),   # K > 1024
    (dict(C=1026, G=1), dcnb.DCN_ERR_UNSUPPORTED),     # D * 2 bytes > 1024
    (dict(N=0), dcnb.DCN_OK),                          # nothing to do, nothing launched
    (dict(N=0, x=None, out=None), dcnb.DCN_OK),
])
def test_dcn_forward_validation(lib, change, status):
    before = dcnb.dcn_launch_count()
    assert call_dcn(lib, **change) == status
    assert dcnb.dcn_launch_count() == before


def call_dcn_algo(lib, algo, **kw):
    args = dict(x=X, offset=OFF, mask=MASK, out=OUT, N=2, H=8, W=8, C=64, G=4, kh=3, kw=3,
                stride=1, pad=1, dil=1, softmax_flag=0, dtype=F16, stream=None)
    args.update(kw)
    return lib.dcn_forward_algo(args["x"], args["offset"], args["mask"], args["out"],
                                args["N"], args["H"], args["W"], args["C"], args["G"],
                                args["kh"], args["kw"], args["stride"], args["pad"],
                                args["dil"], args["softmax_flag"], args["dtype"], algo,
                                args["stream"])


@pytest.mark.parametrize("algo,change,status", [
    (3, {}, dcnb.DCN_ERR_INVALID_ARG),                           # unknown algo
    (-1, {}, dcnb.DCN_ERR_INVALID_ARG),
    (dcnb.DCN_ALGO_BAND, dict(dtype=0), dcnb.DCN_ERR_UNSUPPORTED),           # float32
    (dcnb.DCN_ALGO_BAND, dict(C=32, G=1), dcnb.DCN_ERR_UNSUPPORTED),         # D = 32
    (dcnb.DCN_ALGO_BAND, dict(C=48, G=3), dcnb.DCN_ERR_UNSUPPORTED),         # 96-byte pixels
    (dcnb.DCN_ALGO_BAND, dict(x=X + 8), dcnb.DCN_ERR_UNSUPPORTED),           # not 16-byte aligned
    (dcnb.DCN_ALGO_BAND, dict(W=7), dcnb.DCN_ERR_UNSUPPORTED),               # mask rows of 504 bytes
    (dcnb.DCN_ALGO_BAND, dict(W=4000), dcnb.DCN_ERR_UNSUPPORTED),            # a band of 500 KB rows
    (dcnb.DCN_ALGO_BAND, dict(pad=9, H=30, W=30), dcnb.DCN_ERR_UNSUPPORTED),  # bands outside the map
    (dcnb.DCN_ALGO_GATHER, dict(C=15), dcnb.DCN_ERR_INVALID_ARG),            # the common checks
    (dcnb.DCN_ALGO_BAND, dict(N=0), dcnb.DCN_OK),
])
def test_dcn_forward_algo_validation(lib, algo, change, status):
    before = dcnb.dcn_launch_count()
    assert call_dcn_algo(lib, algo, **change) == status
    assert dcnb.dcn_launch_count() == before


def call_msda(lib, **kw):
    args = dict(value=X, shapes=OFF, starts=OFF + 1024, loc=MASK, attn=MASK + 2 ** 24, out=OUT,
                N=2, Lq=100, M=8, D=32, L=4, K=4, dtype=0, stream=None)
    args.update(kw)
    return lib.msda_forward(args["value"], args["shapes"], args["starts"], args["loc"],
                            args["attn"], args["out"], args["N"], args["Lq"], args["M"],
                            args["D"], args["L"], args["K"], args["dtype"], args["stream"])


@pytest.mark.parametrize("change,status", [
    (dict(dtype=3), dcnb.DCN_ERR_INVALID_ARG),
    (dict(M=0), dcnb.DCN_ERR_INVALID_ARG),
    (dict(D=-4), dcnb.DCN_ERR_INVALID_ARG),
    (dict(L=0), dcnb.DCN_ERR_INVALID_ARG),
    (dict(K=0), dcnb.DCN_ERR_INVALID_ARG),
    (dict(Lq=-1), dcnb.DCN_ERR_INVALID_ARG),
    (dict(L=17), dcnb.DCN_ERR_UNSUPPORTED),
    (dict(K=65), dcnb.DCN_ERR_UNSUPPORTED),
    (dict(D=260), dcnb.DCN_ERR_UNSUPPORTED),           # D * 4 bytes > 1024
    (dict(shapes=None), dcnb.DCN_ERR_INVALID_ARG),
    (dict(out=MASK), dcnb.DCN_ERR_INVALID_ARG),        # out aliases loc
    (dict(out=X), dcnb.DCN_ERR_INVALID_ARG),           # out aliases value
    (dict(loc=MASK + 2), dcnb.DCN_ERR_MISALIGNED),     # f32 needs 4 bytes
    (dict(starts=OFF + 1028), dcnb.DCN_ERR_MISALIGNED),  # int64 needs 8 bytes
    (dict(Lq=0), dcnb.DCN_OK),
    (dict(N=0, value=None), dcnb.DCN_OK),
])
def test_msda_forward_validation(lib, change, status):
    before = dcnb.dcn_launch_count()
    assert call_msda(lib, **change) == status
    assert dcnb.dcn_launch_count() == before


def test_binding_raises_with_status(lib):
    with pytest.raises(dcnb.DcnError) as e:
        dcnb.dcn_forward(X, OFF, MASK, OUT, 1, 4, 4, 6, 4, 3, 3, 1, 1, 1, 0, F16, stream=0)
    assert e.value.status == dcnb.DCN_ERR_INVALID_ARG
    assert "invalid argument" in str(e.value)


# more fake addresses for the backward's gradients and workspace
GO, GX, GOFF, GMASK, WS = (0x7F0040000000, 0x7F0050000000, 0x7F0060000000, 0x7F0070000000,
                           0x7F0080000000)


def test_backward_workspace_sizes(lib):
    assert dcnb.dcn_backward_workspace_size(2, 8, 8, 16, F16) == 2 * 8 * 8 * 16 * 4
    assert dcnb.dcn_backward_workspace_size(2, 8, 8, 16, 2) == 2 * 8 * 8 * 16 * 4
    assert dcnb.dcn_backward_workspace_size(2, 8, 8, 16, 0) == 0
    assert dcnb.dcn_backward_workspace_size(0, 8, 8, 16, F16) == 0
    assert dcnb.dcn_backward_workspace_size(2, 8, 8, 16, 9) == dcnb.DCN_ERR_INVALID_ARG
    assert dcnb.dcn_backward_workspace_size(2, 0, 8, 16, F16) == dcnb.DCN_ERR_INVALID_ARG
    assert dcnb.msda_backward_workspace_size(2, 100, 8, 32, F16) == 2 * 100 * 8 * 32 * 4
    assert dcnb.msda_backward_workspace_size(2, 100, 8, 32, 0) == 0
    assert dcnb.msda_backward_workspace_size(2, 0, 8, 32, F16) == dcnb.DCN_ERR_INVALID_ARG


def call_dcn_bwd(lib, **kw):
    args = dict(x=X, offset=OFF, mask=MASK, go=GO, gx=GX, goff=GOFF, gmask=GMASK, ws=WS,
                ws_bytes=2 * 8 * 8 * 16 * 4, N=2, H=8, W=8, C=16, G=2, kh=3, kw=3, stride=1,
                pad=1, dil=1, softmax_flag=0, dtype=F16, stream=None)
    args.update(kw)
    a = args
    return lib.dcn_backward(a["x"], a["offset"], a["mask"], a["go"], a["gx"], a["goff"],
                            a["gmask"], a["ws"], a["ws_bytes"], a["N"], a["H"], a["W"], a["C"],
                            a["G"], a["kh"], a["kw"], a["stride"], a["pad"], a["dil"],
                            a["softmax_flag"], a["dtype"], a["stream"])


@pytest.mark.parametrize("change,status", [
    (dict(dtype=7), dcnb.DCN_ERR_INVALID_ARG),
    (dict(N=-1), dcnb.DCN_ERR_INVALID_ARG),
    (dict(C=15), dcnb.DCN_ERR_INVALID_ARG),
    (dict(softmax_flag=3), dcnb.DCN_ERR_INVALID_ARG),
    (dict(go=None), dcnb.DCN_ERR_INVALID_ARG),
    (dict(gx=None), dcnb.DCN_ERR_INVALID_ARG),
    (dict(gmask=None), dcnb.DCN_ERR_INVALID_ARG),
    (dict(ws=None), dcnb.DCN_ERR_INVALID_ARG),                 # 16-bit needs the workspace
    (dict(ws_bytes=100), dcnb.DCN_ERR_INVALID_ARG),            # too small
    (dict(ws=WS + 8), dcnb.DCN_ERR_MISALIGNED),                # not 16-byte aligned
    (dict(gx=X), dcnb.DCN_ERR_INVALID_ARG),                    # grad_x aliases x
    (dict(goff=GO + 64), dcnb.DCN_ERR_INVALID_ARG),            # overlaps grad_out
    (dict(gmask=GOFF + 32), dcnb.DCN_ERR_INVALID_ARG),         # outputs overlap
    (dict(ws=GX), dcnb.DCN_ERR_INVALID_ARG),                   # workspace overlaps grad_x
    (dict(go=GO + 1), dcnb.DCN_ERR_MISALIGNED),
    (dict(kh=25, kw=25, pad=12), dcnb.DCN_ERR_UNSUPPORTED),    # a warp's slice > 200 KiB
    (dict(kh=21, kw=21, pad=10, softmax_flag=1), dcnb.DCN_ERR_UNSUPPORTED),
    (dict(H=70000), dcnb.DCN_ERR_UNSUPPORTED),
    (dict(N=0), dcnb.DCN_OK),
    (dict(N=0, x=None, gx=None, ws=None), dcnb.DCN_OK),
])
def test_dcn_backward_validation(lib, change, status):
    before = dcnb.dcn_launch_count()
    assert call_dcn_bwd(lib, **change) == status
    assert dcnb.dcn_launch_count() == before


def call_msda_bwd(lib, **kw):
    args = dict(value=X, shapes=OFF, starts=OFF + 1024, loc=MASK, attn=MASK + 2 ** 24, go=GO,
                gv=GX, gl=GOFF, ga=GMASK, ws=WS, ws_bytes=2 * 3000 * 8 * 32 * 4, N=2, S=3000,
                Lq=100, M=8, D=32, L=4, K=4, dtype=F16, stream=None)
    args.update(kw)
    a = args
    return lib.msda_backward(a["value"], a["shapes"], a["starts"], a["loc"], a["attn"], a["go"],
                             a["gv"], a["gl"], a["ga"], a["ws"], a["ws_bytes"], a["N"], a["S"],
                             a["Lq"], a["M"], a["D"], a["L"], a["K"], a["dtype"], a["stream"])


@pytest.mark.parametrize("change,status", [
    (dict(dtype=3), dcnb.DCN_ERR_INVALID_ARG),
    (dict(S=0), dcnb.DCN_ERR_INVALID_ARG),
    (dict(K=0), dcnb.DCN_ERR_INVALID_ARG),
    (dict(L=17), dcnb.DCN_ERR_UNSUPPORTED),
    (dict(gv=None), dcnb.DCN_ERR_INVALID_ARG),
    (dict(gl=None), dcnb.DCN_ERR_INVALID_ARG),
    (dict(ws=None), dcnb.DCN_ERR_INVALID_ARG),
    (dict(ws_bytes=64), dcnb.DCN_ERR_INVALID_ARG),
    (dict(ws=WS + 4), dcnb.DCN_ERR_MISALIGNED),
    (dict(gv=X), dcnb.DCN_ERR_INVALID_ARG),                    # grad_value aliases value
    (dict(ga=GOFF + 64), dcnb.DCN_ERR_INVALID_ARG),            # overlaps grad_loc
    (dict(gl=OFF), dcnb.DCN_ERR_INVALID_ARG),                  # overlaps the level table
    (dict(starts=OFF + 1028), dcnb.DCN_ERR_MISALIGNED),
    (dict(N=0, value=None, gv=None), dcnb.DCN_OK),
])
def test_msda_backward_validation(lib, change, status):
    before = dcnb.dcn_launch_count()
    assert call_msda_bwd(lib, **change) == status
    assert dcnb.dcn_launch_count() == before


def call_dyn(lib, **kw):
    args = dict(x=X, w=OFF, out=OUT, N=2, H=8, W=8, C=32, G=2, K=7, softmax_flag=1, dtype=F16,
                stream=None)
    args.update(kw)
    a = args
    return lib.dynconv_forward(a["x"], a["w"], a["out"], a["N"], a["H"], a["W"], a["C"], a["G"],
                               a["K"], a["softmax_flag"], a["dtype"], a["stream"])


@pytest.mark.parametrize("change,status", [
    (dict(dtype=5), dcnb.DCN_ERR_INVALID_ARG),
    (dict(K=4), dcnb.DCN_ERR_INVALID_ARG),              # even window
    (dict(K=0), dcnb.DCN_ERR_INVALID_ARG),
    (dict(C=33), dcnb.DCN_ERR_INVALID_ARG),             # C % G != 0
    (dict(softmax_flag=2), dcnb.DCN_ERR_INVALID_ARG),
    (dict(K=33), dcnb.DCN_ERR_UNSUPPORTED),
    (dict(C=16, G=2), dcnb.DCN_ERR_UNSUPPORTED),        # D * 2 bytes = 16, not a multiple of 32
    (dict(x=None), dcnb.DCN_ERR_INVALID_ARG),
    (dict(out=X), dcnb.DCN_ERR_INVALID_ARG),            # out aliases x
    (dict(x=X + 8), dcnb.DCN_ERR_MISALIGNED),
    (dict(out=OUT + 16), dcnb.DCN_ERR_MISALIGNED),
    (dict(N=0), dcnb.DCN_OK),
])
def test_dynconv_validation(lib, change, status):
    before = dcnb.dcn_launch_count()
    assert call_dyn(lib, **change) == status
    assert dcnb.dcn_launch_count() == before


@pytest.mark.parametrize("algo", [dcnb.DCN_ALGO_SIMT, dcnb.DCN_ALGO_TENSOR])
@pytest.mark.parametrize("change,status", [
    (dict(dtype=5), dcnb.DCN_ERR_INVALID_ARG),
    (dict(K=4), dcnb.DCN_ERR_INVALID_ARG),
    (dict(x=None), dcnb.DCN_ERR_INVALID_ARG),
    (dict(out=X), dcnb.DCN_ERR_INVALID_ARG),
    (dict(out=OUT + 16), dcnb.DCN_ERR_MISALIGNED),
    (dict(N=0), dcnb.DCN_OK),
])
def test_dynconv_forward_algo_validation(lib, algo, change, status):
    args = dict(x=X, w=OFF, out=OUT, N=2, H=8, W=8, C=32, G=2, K=7, softmax_flag=1, dtype=F16)
    args.update(change)
    a = args
    before = dcnb.dcn_launch_count()
    assert lib.dynconv_forward_algo(a["x"], a["w"], a["out"], a["N"], a["H"], a["W"], a["C"],
                                    a["G"], a["K"], a["softmax_flag"], a["dtype"], algo,
                                    None) == status
    assert dcnb.dcn_launch_count() == before


@pytest.mark.parametrize("algo", [-1, 2, 4])
def test_dynconv_forward_algo_rejects_unknown_kernels(lib, algo):
    before = dcnb.dcn_launch_count()
    assert lib.dynconv_forward_algo(X, OFF, OUT, 2, 8, 8, 32, 2, 7, 1, F16, algo,
                                    None) == dcnb.DCN_ERR_INVALID_ARG
    assert dcnb.dcn_launch_count() == before


def test_debug_library_exports_the_forward_and_status_calls(lib):
    dbg = dcnb.debug_library()
    for name in dcnb._binding.DEBUG_SYMBOLS:
        assert hasattr(dbg, name), name
    assert dcnb.dcn_debug_checks(dbg) == 1
    assert dcnb.dcn_debug_checks() == 0
    # host-side validation is the same code in both libraries
    assert dbg.dcn_forward_algo(X, OFF, MASK, OUT, 2, 8, 8, 15, 4, 3, 3, 1, 1, 1, 0, F16, 0,
                                None) == dcnb.DCN_ERR_INVALID_ARG
