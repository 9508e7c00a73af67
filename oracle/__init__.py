"""CPU oracle for the deformable sampling-aggregation path.

TEST INFRASTRUCTURE.  This package is the plain, slow, float64 definition the
CUDA library is checked against.  Only the test suite, the smoke check and the
benchmark's CPU-baseline leg may import it; the product path never does, and
it imports nothing from the product package.

`dcn_forward_ref`, `msda_forward_ref`, their backward twins and
`dynconv_forward_ref` (the ContMix core) call the C loop nests in dcn_oracle.c
through ctypes.  Inputs may be numpy arrays or torch CPU tensors
in any floating dtype; each value is converted exactly to float64 before the
arithmetic (every fp16, bf16 and fp32 value is representable in float64).

Parity status: every function here is pinned by the CPU tests against worked
examples printed on the pages, closed forms, invariants and library routines
(torch grid_sample / conv2d in float64); no function is parity-unpinned.
"""
import ctypes

import numpy as np

from . import build as _build
from . import scalar  # noqa: F401  (re-exported for the tests)

_lib = None


def bind(lib):
    """Declare the C signatures on a loaded oracle library and return it."""
    dp = ctypes.POINTER(ctypes.c_double)
    lp = ctypes.POINTER(ctypes.c_longlong)
    L = ctypes.c_long
    lib.oracle_dcn_forward.argtypes = [dp, dp, dp, dp] + [L] * 10 + [ctypes.c_int]
    lib.oracle_dcn_forward.restype = ctypes.c_int
    lib.oracle_msda_forward.argtypes = [dp, lp, lp, dp, dp, dp] + [L] * 7
    lib.oracle_msda_forward.restype = ctypes.c_int
    lib.oracle_out_size.argtypes = [L] * 5
    lib.oracle_out_size.restype = L
    lib.oracle_dcn_backward.argtypes = [dp] * 7 + [L] * 10 + [ctypes.c_int]
    lib.oracle_dcn_backward.restype = ctypes.c_int
    lib.oracle_msda_backward.argtypes = [dp, lp, lp, dp, dp, dp, dp, dp, dp] + [L] * 7
    lib.oracle_msda_backward.restype = ctypes.c_int
    lib.oracle_dynconv_forward.argtypes = [dp, dp, dp] + [L] * 6 + [ctypes.c_int]
    lib.oracle_dynconv_forward.restype = ctypes.c_int
    lib.oracle_msda_locations.argtypes = [dp, L, dp, dp, lp, dp] + [L] * 5
    lib.oracle_msda_locations.restype = ctypes.c_int
    return lib


def _load():
    global _lib
    if _lib is None:
        _lib = bind(ctypes.CDLL(_build.build()))
    return _lib


def _as_f64(a):
    """Exact float64 copy of a numpy array or torch tensor (any float dtype)."""
    if hasattr(a, "detach"):            # torch tensor (bf16 has no numpy dtype)
        import torch
        a = a.detach().to("cpu", torch.float64).numpy()
    return np.ascontiguousarray(np.asarray(a, dtype=np.float64))


def _ptr(a, ctype=ctypes.c_double):
    return a.ctypes.data_as(ctypes.POINTER(ctype))


def out_size(n_in, k, stride, pad, dil):
    return int(_load().oracle_out_size(n_in, k, stride, pad, dil))


def dcn_forward_ref(x, offset, mask, kh, kw, stride=1, pad=1, dil=1, softmax_flag=0,
                    groups=None):
    """float64 DCNv3/DCNv4 forward.

    x [N, H, W, C], offset [N, Ho, Wo, G, K, 2], mask [N, Ho, Wo, G, K]
    -> out [N, Ho, Wo, C] float64.  G is taken from mask.shape[3] unless given.
    """
    x = _as_f64(x)
    offset = _as_f64(offset)
    mask = _as_f64(mask)
    N, H, W, C = x.shape
    G = groups if groups is not None else mask.shape[3]
    Ho = out_size(H, kh, stride, pad, dil)
    Wo = out_size(W, kw, stride, pad, dil)
    K = kh * kw
    assert offset.size == N * Ho * Wo * G * K * 2, "offset has the wrong size"
    assert mask.size == N * Ho * Wo * G * K, "mask has the wrong size"
    out = np.zeros((N, Ho, Wo, C), dtype=np.float64)
    rc = _load().oracle_dcn_forward(_ptr(x), _ptr(offset), _ptr(mask), _ptr(out),
                                    N, H, W, C, G, kh, kw, stride, pad, dil,
                                    int(softmax_flag))
    if rc != 0:
        raise ValueError("oracle_dcn_forward rejected its arguments")
    return out


def msda_forward_ref(value, spatial_shapes, level_start, loc, attn):
    """float64 MSDeformAttn core forward.

    value [N, S, M, D], spatial_shapes [L, 2] as (H, W), level_start [L],
    loc [N, Lq, M, L, K, 2] as (u, v), attn [N, Lq, M, L, K]
    -> out [N, Lq, M * D] float64.
    """
    value = _as_f64(value)
    loc = _as_f64(loc)
    attn = _as_f64(attn)
    shapes = np.ascontiguousarray(np.asarray(spatial_shapes, dtype=np.int64))
    starts = np.ascontiguousarray(np.asarray(level_start, dtype=np.int64))
    N, S, M, D = value.shape
    _, Lq, _, L, K = attn.shape
    assert loc.shape == (N, Lq, M, L, K, 2), "loc has the wrong shape"
    out = np.zeros((N, Lq, M * D), dtype=np.float64)
    rc = _load().oracle_msda_forward(_ptr(value), _ptr(shapes, ctypes.c_longlong),
                                     _ptr(starts, ctypes.c_longlong), _ptr(loc),
                                     _ptr(attn), _ptr(out), N, S, Lq, M, D, L, K)
    if rc != 0:
        raise ValueError("oracle_msda_forward rejected its arguments")
    return out


def dcn_backward_ref(x, offset, mask, grad_out, kh, kw, stride=1, pad=1, dil=1,
                     softmax_flag=0, groups=None):
    """float64 gradients of dcn_forward_ref for the upstream gradient grad_out.

    Returns (grad_x [N,H,W,C], grad_offset [N,Ho,Wo,G,K,2], grad_mask [N,Ho,Wo,G,K]);
    grad_mask is with respect to the mask argument (the logits when softmax_flag = 1).
    """
    x = _as_f64(x)
    offset = _as_f64(offset)
    mask = _as_f64(mask)
    grad_out = _as_f64(grad_out)
    N, H, W, C = x.shape
    G = groups if groups is not None else mask.shape[3]
    Ho = out_size(H, kh, stride, pad, dil)
    Wo = out_size(W, kw, stride, pad, dil)
    K = kh * kw
    assert offset.size == N * Ho * Wo * G * K * 2 and mask.size == N * Ho * Wo * G * K
    assert grad_out.size == N * Ho * Wo * C, "grad_out has the wrong size"
    gx = np.zeros_like(x)
    goff = np.zeros((N, Ho, Wo, G, K, 2))
    gmask = np.zeros((N, Ho, Wo, G, K))
    rc = _load().oracle_dcn_backward(_ptr(x), _ptr(offset), _ptr(mask), _ptr(grad_out),
                                     _ptr(gx), _ptr(goff), _ptr(gmask), N, H, W, C, G, kh, kw,
                                     stride, pad, dil, int(softmax_flag))
    if rc != 0:
        raise ValueError("oracle_dcn_backward rejected its arguments")
    return gx, goff, gmask


def msda_backward_ref(value, spatial_shapes, level_start, loc, attn, grad_out):
    """float64 gradients of msda_forward_ref for the upstream gradient grad_out.

    Returns (grad_value [N,S,M,D], grad_loc [N,Lq,M,L,K,2], grad_attn [N,Lq,M,L,K]).
    """
    value = _as_f64(value)
    loc = _as_f64(loc)
    attn = _as_f64(attn)
    grad_out = _as_f64(grad_out)
    shapes = np.ascontiguousarray(np.asarray(spatial_shapes, dtype=np.int64))
    starts = np.ascontiguousarray(np.asarray(level_start, dtype=np.int64))
    N, S, M, D = value.shape
    _, Lq, _, L, K = attn.shape
    assert loc.shape == (N, Lq, M, L, K, 2) and grad_out.size == N * Lq * M * D
    gv = np.zeros_like(value)
    gl = np.zeros_like(loc)
    ga = np.zeros_like(attn)
    rc = _load().oracle_msda_backward(_ptr(value), _ptr(shapes, ctypes.c_longlong),
                                      _ptr(starts, ctypes.c_longlong), _ptr(loc), _ptr(attn),
                                      _ptr(grad_out), _ptr(gv), _ptr(gl), _ptr(ga), N, S, Lq,
                                      M, D, L, K)
    if rc != 0:
        raise ValueError("oracle_msda_backward rejected its arguments")
    return gv, gl, ga


def dynconv_forward_ref(x, weights, K, softmax_flag=1, groups=None):
    """float64 dynamic local aggregation (ContMix core).

    x [N, H, W, C], weights [N, H, W, G, K*K] (tap ky * K + kx) -> out
    [N, H, W, C] float64; K odd.  G is taken from weights.shape[3] unless given.
    """
    x = _as_f64(x)
    weights = _as_f64(weights)
    N, H, W, C = x.shape
    G = groups if groups is not None else weights.shape[3]
    assert weights.size == N * H * W * G * K * K, "weights has the wrong size"
    out = np.zeros((N, H, W, C), dtype=np.float64)
    rc = _load().oracle_dynconv_forward(_ptr(x), _ptr(weights), _ptr(out), N, H, W, C, G, K,
                                        int(softmax_flag))
    if rc != 0:
        raise ValueError("oracle_dynconv_forward rejected its arguments")
    return out


def msda_locations_ref(spatial_shapes, reference, offsets, valid_ratios=None):
    """float64 sampling locations of the reference-point variants.

    reference [N, Lq, 2] points or [N, Lq, 4] boxes (cx, cy, w, h) in
    valid-image coordinates; offsets [N, Lq, M, L, K, 2]; valid_ratios
    [N, L, 2] as (W_valid / W, H_valid / H), or None for all 1; spatial_shapes
    [L, 2] as (H, W).  Runs the C loop oracle_msda_locations (point:
    s = p r + dp / (W, H); box: s = c r + (dp / K) (w, h) r / 2)
    -> loc [N, Lq, M, L, K, 2].
    """
    ref = _as_f64(reference)
    off = _as_f64(offsets)
    shapes = np.ascontiguousarray(np.asarray(spatial_shapes, dtype=np.int64))
    N, Lq, M, L, K, _ = off.shape
    ref_dim = ref.shape[-1]
    assert ref.shape == (N, Lq, ref_dim), "reference has the wrong shape"
    assert shapes.shape == (L, 2), "spatial_shapes has the wrong shape"
    loc = np.zeros_like(off)
    if valid_ratios is None:
        vr_ptr = None
    else:
        vr = _as_f64(valid_ratios)
        assert vr.shape == (N, L, 2), "valid_ratios has the wrong shape"
        vr_ptr = _ptr(vr)
    rc = _load().oracle_msda_locations(_ptr(ref), ref_dim, vr_ptr, _ptr(off),
                                       _ptr(shapes, ctypes.c_longlong), _ptr(loc), N, Lq, M,
                                       L, K)
    if rc != 0:
        raise ValueError("oracle_msda_locations rejected its arguments")
    return loc


def mask_value_ref(value, mask):
    """value [N, S, M, D] with every row whose mask [N, S] is set replaced by 0
    (Deformable DETR: the attention module zeroes projected values at masked
    positions)."""
    v = _as_f64(value).copy()
    m = np.asarray(mask).astype(bool)
    v[m] = 0.0
    return v


def msda_points_ref(value, spatial_shapes, level_start, reference, offsets, attn,
                    valid_ratios=None):
    """float64 MSDA core fed from references: the locations of
    msda_locations_ref, then msda_forward_ref."""
    loc = msda_locations_ref(spatial_shapes, reference, offsets, valid_ratios)
    return msda_forward_ref(value, spatial_shapes, level_start, loc, attn)


def dcnv4_front_end_ref(x, w_om, b_om, kh, kw, pad, dil, groups):
    """float64 DCNv4 module core with its merged offset / mask linear.

    "DCNv4" note, "1. Remove Softmax": one linear layer produces every
    location's G*K offset pairs and G*K modulation scalars from the same
    features, which then drive the sampling core (no softmax).  Here
    om = x @ w_om^T + b_om per pixel (a library matmul in float64) with
    w_om [G*K*3, C]; its first G*K*2 outputs are the offsets in [G][K][2]
    order, the last G*K the masks in [G][K] order; stride 1, so the linear is
    applied at every output pixel.  Returns (out, offset, mask).
    """
    x = _as_f64(x)
    w = _as_f64(w_om)
    N, H, W, C = x.shape
    G = groups
    K = kh * kw
    om = x.reshape(-1, C) @ w.T
    if b_om is not None:
        om = om + _as_f64(b_om)[None, :]
    offset = om[:, :G * K * 2].reshape(N, H, W, G, K, 2)
    mask = om[:, G * K * 2:].reshape(N, H, W, G, K)
    out = dcn_forward_ref(x, offset, mask, kh, kw, stride=1, pad=pad, dil=dil, softmax_flag=0,
                          groups=G)
    return out, offset, mask
