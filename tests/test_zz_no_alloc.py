"""dcn_backward_static_scratch: the backward with the library's own static
grad_x accumulator, against dcn_backward with a caller workspace and against
the float64 oracle's gradients.

Collected last on purpose: it must pass both in a fresh process (where its
first call looks up the accumulator's device address) and after every other
test has run.
"""
import os
import re

import pytest
import torch

import deformable_attention_sampling_b200 as dcnb
from deformable_attention_sampling_b200 import build as dcn_build
import gen
import oracle
from tests.parity import compare

DEV = "cuda:0"


def test_header_limit_matches_the_binding():
    text = open(os.path.join(dcn_build.INCLUDE, "dcn.h")).read()
    m = re.search(r"#define\s+DCN_STATIC_SCRATCH_BYTES\s+\((\d+)LL\s*<<\s*(\d+)\)", text)
    assert m and int(m.group(1)) << int(m.group(2)) == dcnb.STATIC_SCRATCH_BYTES


def _args(w, t, grads):
    return (t["x"], t["offset"], t["mask"], t["grad_out"], *grads, w.N, w.H, w.W, w.C, w.G,
            w.kh, w.kw, w.stride, w.pad, w.dil, w.softmax_flag, gen.DTYPE_CODES[w.dtype])


def _empty_grads(t):
    return (torch.empty_like(t["x"]), torch.empty_like(t["offset"]), torch.empty_like(t["mask"]))


@pytest.mark.gpu
@pytest.mark.parametrize("dt,sm", [("f16", 0), ("bf16", 1), ("f32", 0)])
def test_static_scratch_matches_the_workspace_entry(dt, sm):
    w = gen.DcnWorkload("noalloc", N=4, H=28, W=30, C=64, G=4, dtype=dt, offset_sigma=2.0,
                        softmax_flag=sm)
    host = gen.dcn_inputs(w, seed=21)
    host["grad_out"] = gen.grad_out((w.N, w.Ho, w.Wo, w.C), w.dtype, seed=21)
    t = {k: v.to(DEV) for k, v in host.items()}

    exact = oracle.dcn_backward_ref(host["x"], host["offset"], host["mask"], host["grad_out"],
                                    w.kh, w.kw, w.stride, w.pad, w.dil, w.softmax_flag)
    ref = _empty_grads(t)
    code = gen.DTYPE_CODES[dt]
    nbytes = dcnb.dcn_backward_workspace_size(w.N, w.H, w.W, w.C, code)
    ws = torch.empty(max(nbytes // 4, 1), dtype=torch.float32, device=DEV)
    a = _args(w, t, ref)
    dcnb.dcn_backward(*a[:7], ws, nbytes, *a[7:])
    torch.cuda.synchronize()

    for call in range(2):                 # two calls in a row on one accumulator
        got = _empty_grads(t)
        before = dcnb.dcn_launch_count()
        dcnb.dcn_backward_static_scratch(*_args(w, t, got))
        torch.cuda.synchronize()
        assert dcnb.dcn_launch_count() - before == (3 if dt != "f32" else 2)
        for name, g, r, e in zip(("grad_x", "grad_offset", "grad_mask"), got, ref, exact):
            compare(g, r.double().cpu().numpy(), f"{dt} call {call} {name}")
            compare(g, e, f"{dt} call {call} {name} vs the oracle")
        # the per-tap gradients are deterministic: bit for bit the same
        assert torch.equal(got[1], ref[1]) and torch.equal(got[2], ref[2])


@pytest.mark.gpu
def test_static_scratch_rejects_sizes_beyond_its_limit():
    # N * H * W * C * 4 = 16 MiB + 4 KiB > the accumulator: refused, nothing launched
    N, H, W, C = 1, 64, 64, 1025
    assert N * H * W * C * 4 > dcnb.STATIC_SCRATCH_BYTES
    x = torch.zeros((N, H, W, C), dtype=torch.float16, device=DEV)
    off = torch.zeros((N, H, W, 1, 9, 2), dtype=torch.float16, device=DEV)
    mask = torch.zeros((N, H, W, 1, 9), dtype=torch.float16, device=DEV)
    grads = (torch.empty_like(x), torch.empty_like(off), torch.empty_like(mask))
    before = dcnb.dcn_launch_count()
    with pytest.raises(dcnb.DcnError) as e:
        dcnb.dcn_backward_static_scratch(x, off, mask, x, *grads, N, H, W, C, 1, 3, 3, 1, 1, 1,
                                         0, gen.DTYPE_CODES["f16"])
    assert e.value.status == dcnb.DCN_ERR_UNSUPPORTED
    assert dcnb.dcn_launch_count() == before
