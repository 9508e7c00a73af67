"""ctypes binding of libdcn_b200.so (include/dcn.h).

Argument marshalling only: every step of the computation runs in the CUDA
kernels behind the C interface.  Pointer arguments may be integers (device
addresses) or objects with a ``data_ptr()`` method (torch tensors); stream
arguments may be None (torch's current stream), an integer handle, or an object
with a ``cuda_stream`` attribute.  A non-OK status raises DcnError.

There is no fallback: when the shared library is missing the first call
raises RuntimeError naming the build command.
"""
import ctypes
import os

PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(PKG, "_lib", "libdcn_b200.so")
DEBUG_LIB_PATH = os.path.join(PKG, "_lib", "libdcn_b200_debug.so")

DCN_OK = 0
DCN_ERR_INVALID_ARG = -1
DCN_ERR_UNSUPPORTED = -2
DCN_ERR_MISALIGNED = -3
DCN_ERR_CUDA = -4
DTYPE_CODES = {"f32": 0, "f16": 1, "bf16": 2}
DCN_FLAG_WAIT_TIMEOUT = 1
DCN_FLAG_OUT_OF_BOUNDS = 2
DCN_FLAG_BAD_LEVELS = 4
# the entry points the debug library holds (the forward calls and the status calls)
DEBUG_SYMBOLS = ("dcn_forward", "dcn_forward_algo", "dcn_forward_plan", "dcnv4_fused_forward",
                 "dcnv4_fused_forward_algo", "msda_forward", "msda_forward_points",
                 "msda_mask_value", "dcn_output_size", "dcn_status_string", "dcn_last_cuda_error",
                 "dcn_launch_count", "dcn_device_flags", "dcn_debug_checks", "dcn_version")
DCN_ALGO_AUTO = 0
DCN_ALGO_GATHER = 1
DCN_ALGO_SIMT = 1
DCN_ALGO_BAND = 2
DCN_ALGO_TENSOR = 3
ALGO_CODES = {"auto": DCN_ALGO_AUTO, "gather": DCN_ALGO_GATHER, "band": DCN_ALGO_BAND}
# dynconv_forward_algo's kernels
DYNCONV_ALGO_CODES = {"auto": DCN_ALGO_AUTO, "simt": DCN_ALGO_SIMT, "tensor": DCN_ALGO_TENSOR}

# every symbol include/dcn.h declares, with its ctypes signature
_VP = ctypes.c_void_p
_I = ctypes.c_int
_LL = ctypes.c_longlong
SIGNATURES = {
    "dcn_forward": (_I, [_VP, _VP, _VP, _VP] + [_I] * 12 + [_VP]),
    "dcn_forward_algo": (_I, [_VP, _VP, _VP, _VP] + [_I] * 13 + [_VP]),
    "dcn_forward_plan": (_I, [_I] * 13 + [ctypes.POINTER(ctypes.c_int)]),
    "dcn_device_flags": (_I, [_I]),
    "dcn_debug_checks": (_I, []),
    "msda_forward": (_I, [_VP] * 6 + [_I] * 7 + [_VP]),
    "msda_forward_points": (_I, [_VP] * 4 + [_I] + [_VP] * 4 + [_I] * 7 + [_VP]),
    "msda_mask_value": (_I, [_VP] * 3 + [_I] * 5 + [_VP]),
    "dcn_backward_workspace_size": (_LL, [_I] * 5),
    "dcn_backward": (_I, [_VP] * 8 + [_LL] + [_I] * 12 + [_VP]),
    "dcn_backward_static_scratch": (_I, [_VP] * 7 + [_I] * 12 + [_VP]),
    "msda_backward_workspace_size": (_LL, [_I] * 5),
    "msda_backward": (_I, [_VP] * 10 + [_LL] + [_I] * 8 + [_VP]),
    "dynconv_forward": (_I, [_VP] * 3 + [_I] * 8 + [_VP]),
    "dynconv_forward_algo": (_I, [_VP] * 3 + [_I] * 9 + [_VP]),
    "dcnv4_fused_forward": (_I, [_VP] * 4 + [_I] * 10 + [_VP]),
    "dcnv4_fused_forward_algo": (_I, [_VP] * 4 + [_I] * 11 + [_VP]),
    "dcn_output_size": (_I, [_I] * 5),
    "dcn_status_string": (ctypes.c_char_p, [_I]),
    "dcn_last_cuda_error": (_I, []),
    "dcn_launch_count": (ctypes.c_uint64, []),
    "dcn_version": (_I, []),
}

_lib = None


class DcnError(RuntimeError):
    """A dcn_status_t other than DCN_OK."""

    def __init__(self, status, where):
        self.status = status
        text = _load().dcn_status_string(status).decode()
        detail = ""
        if status == DCN_ERR_CUDA:
            detail = f" (cudaError {_load().dcn_last_cuda_error()})"
        super().__init__(f"{where}: {text}{detail} [status {status}]")


def _load():
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(
                f"{LIB_PATH} is missing: build it with "
                "`python -m deformable_attention_sampling_b200.build`")
        lib = ctypes.CDLL(LIB_PATH)
        for name, (res, args) in SIGNATURES.items():
            fn = getattr(lib, name)
            fn.restype = res
            fn.argtypes = args
        _lib = lib
    return _lib


def library():
    """The loaded ctypes library (loads it on first use)."""
    return _load()


_debug_lib = None


def debug_library():
    """The debug library (libdcn_b200_debug.so: the forward and status calls
    with device-side address and level-table checks), loaded on first use."""
    global _debug_lib
    if _debug_lib is None:
        if not os.path.exists(DEBUG_LIB_PATH):
            raise RuntimeError(
                f"{DEBUG_LIB_PATH} is missing: build it with "
                "`python -m deformable_attention_sampling_b200.build`")
        lib = ctypes.CDLL(DEBUG_LIB_PATH)
        for name in DEBUG_SYMBOLS:
            res, args = SIGNATURES[name]
            fn = getattr(lib, name)
            fn.restype = res
            fn.argtypes = args
        _debug_lib = lib
    return _debug_lib


def _ptr(p):
    if p is None:
        return None
    if isinstance(p, int):
        return p
    return int(p.data_ptr())


def _stream(s):
    if s is None:
        import torch
        return int(torch.cuda.current_stream().cuda_stream)
    if isinstance(s, int):
        return s
    return int(s.cuda_stream)


def _check(status, where):
    if status != DCN_OK:
        raise DcnError(status, where)


def dcn_forward(x, offset, mask, out, N, H, W, C, G, kh, kw, stride, pad, dil,
                softmax_flag, dtype, stream=None):
    """C dcn_forward; raises DcnError on a non-OK status."""
    _check(_load().dcn_forward(_ptr(x), _ptr(offset), _ptr(mask), _ptr(out), N, H, W, C, G,
                               kh, kw, stride, pad, dil, softmax_flag, dtype, _stream(stream)),
           "dcn_forward")


def dcn_forward_algo(x, offset, mask, out, N, H, W, C, G, kh, kw, stride, pad, dil,
                     softmax_flag, dtype, algo, stream=None):
    """C dcn_forward_algo (algo: DCN_ALGO_AUTO / _GATHER / _BAND); raises
    DcnError on a non-OK status."""
    _check(_load().dcn_forward_algo(_ptr(x), _ptr(offset), _ptr(mask), _ptr(out), N, H, W, C,
                                    G, kh, kw, stride, pad, dil, softmax_flag, dtype, algo,
                                    _stream(stream)),
           "dcn_forward_algo")


PLAN_FIELDS = ("algo", "rows_per_step", "margin", "ring_rows", "sampler_warps",
               "steps_in_flight", "runs_per_row", "smem_bytes")


def dcn_forward_plan(N, H, W, C, G, kh, kw, stride, pad, dil, softmax_flag, dtype,
                     algo=DCN_ALGO_AUTO, lib=None):
    """C dcn_forward_plan: the kernel dcn_forward_algo runs for this shape and
    the band kernel's launch shape, as a dict over PLAN_FIELDS (host only, no
    GPU needed); raises DcnError on a non-OK status."""
    plan = (ctypes.c_int * 8)()
    _check((lib or _load()).dcn_forward_plan(N, H, W, C, G, kh, kw, stride, pad, dil,
                                             softmax_flag, dtype, algo, plan),
           "dcn_forward_plan")
    return dict(zip(PLAN_FIELDS, list(plan)))


def dcn_device_flags(reset=False, lib=None):
    """C dcn_device_flags: the status word of the current device (DCN_FLAG_*
    bits), cleared when reset; synchronous.  `lib`: the debug library handle
    instead of the release library."""
    r = (lib or _load()).dcn_device_flags(1 if reset else 0)
    if r < 0:
        raise DcnError(r, "dcn_device_flags")
    return r


def dcn_debug_checks(lib=None):
    """1 for the debug library (device-side checks), 0 for the release one."""
    return int((lib or _load()).dcn_debug_checks())


def msda_forward(value, spatial_shapes, level_start, sampling_loc, attn_w, out, N, Lq, M, D,
                 L, K, dtype, stream=None):
    """C msda_forward; raises DcnError on a non-OK status."""
    _check(_load().msda_forward(_ptr(value), _ptr(spatial_shapes), _ptr(level_start),
                                _ptr(sampling_loc), _ptr(attn_w), _ptr(out), N, Lq, M, D, L,
                                K, dtype, _stream(stream)),
           "msda_forward")


def dcn_backward_workspace_size(N, H, W, C, dtype):
    return int(_load().dcn_backward_workspace_size(N, H, W, C, dtype))


def dcn_backward(x, offset, mask, grad_out, grad_x, grad_offset, grad_mask, workspace,
                 workspace_bytes, N, H, W, C, G, kh, kw, stride, pad, dil, softmax_flag, dtype,
                 stream=None):
    """C dcn_backward; raises DcnError on a non-OK status."""
    _check(_load().dcn_backward(_ptr(x), _ptr(offset), _ptr(mask), _ptr(grad_out), _ptr(grad_x),
                                _ptr(grad_offset), _ptr(grad_mask), _ptr(workspace),
                                workspace_bytes, N, H, W, C, G, kh, kw, stride, pad, dil,
                                softmax_flag, dtype, _stream(stream)),
           "dcn_backward")


# bytes of the library's static grad_x accumulator (DCN_STATIC_SCRATCH_BYTES)
STATIC_SCRATCH_BYTES = 16 << 20


def dcn_backward_static_scratch(x, offset, mask, grad_out, grad_x, grad_offset, grad_mask, N, H,
                                W, C, G, kh, kw, stride, pad, dil, softmax_flag, dtype,
                                stream=None):
    """C dcn_backward_static_scratch (no workspace argument; the library's own
    per-device accumulator); raises DcnError on a non-OK status."""
    _check(_load().dcn_backward_static_scratch(
        _ptr(x), _ptr(offset), _ptr(mask), _ptr(grad_out), _ptr(grad_x), _ptr(grad_offset),
        _ptr(grad_mask), N, H, W, C, G, kh, kw, stride, pad, dil, softmax_flag, dtype,
        _stream(stream)), "dcn_backward_static_scratch")


def msda_backward_workspace_size(N, S, M, D, dtype):
    return int(_load().msda_backward_workspace_size(N, S, M, D, dtype))


def msda_backward(value, spatial_shapes, level_start, sampling_loc, attn_w, grad_out,
                  grad_value, grad_loc, grad_attn, workspace, workspace_bytes, N, S, Lq, M, D,
                  L, K, dtype, stream=None):
    """C msda_backward; raises DcnError on a non-OK status."""
    _check(_load().msda_backward(_ptr(value), _ptr(spatial_shapes), _ptr(level_start),
                                 _ptr(sampling_loc), _ptr(attn_w), _ptr(grad_out),
                                 _ptr(grad_value), _ptr(grad_loc), _ptr(grad_attn),
                                 _ptr(workspace), workspace_bytes, N, S, Lq, M, D, L, K, dtype,
                                 _stream(stream)),
           "msda_backward")


def dynconv_forward(x, weights, out, N, H, W, C, G, K, softmax_flag, dtype, stream=None):
    """C dynconv_forward; raises DcnError on a non-OK status."""
    _check(_load().dynconv_forward(_ptr(x), _ptr(weights), _ptr(out), N, H, W, C, G, K,
                                   softmax_flag, dtype, _stream(stream)),
           "dynconv_forward")


def dynconv_forward_algo(x, weights, out, N, H, W, C, G, K, softmax_flag, dtype, algo,
                         stream=None):
    """C dynconv_forward_algo; raises DcnError on a non-OK status."""
    _check(_load().dynconv_forward_algo(_ptr(x), _ptr(weights), _ptr(out), N, H, W, C, G, K,
                                        softmax_flag, dtype, algo, _stream(stream)),
           "dynconv_forward_algo")


def msda_forward_points(value, spatial_shapes, level_start, reference, ref_dim, valid_ratios,
                        offsets, attn_w, out, N, Lq, M, D, L, K, dtype, stream=None):
    """C msda_forward_points; raises DcnError on a non-OK status."""
    _check(_load().msda_forward_points(_ptr(value), _ptr(spatial_shapes), _ptr(level_start),
                                       _ptr(reference), ref_dim, _ptr(valid_ratios),
                                       _ptr(offsets), _ptr(attn_w), _ptr(out), N, Lq, M, D, L,
                                       K, dtype, _stream(stream)),
           "msda_forward_points")


def msda_mask_value(value, mask, out, N, S, M, D, dtype, stream=None):
    """C msda_mask_value; raises DcnError on a non-OK status."""
    _check(_load().msda_mask_value(_ptr(value), _ptr(mask), _ptr(out), N, S, M, D, dtype,
                                   _stream(stream)),
           "msda_mask_value")


def dcnv4_fused_forward(x, w_om, b_om, out, N, H, W, C, G, kh, kw, pad, dil, dtype,
                        stream=None):
    """C dcnv4_fused_forward; raises DcnError on a non-OK status."""
    _check(_load().dcnv4_fused_forward(_ptr(x), _ptr(w_om), _ptr(b_om), _ptr(out), N, H, W, C,
                                       G, kh, kw, pad, dil, dtype, _stream(stream)),
           "dcnv4_fused_forward")


def dcnv4_fused_forward_algo(x, w_om, b_om, out, N, H, W, C, G, kh, kw, pad, dil, dtype, algo,
                             stream=None):
    """C dcnv4_fused_forward_algo; raises DcnError on a non-OK status."""
    _check(_load().dcnv4_fused_forward_algo(_ptr(x), _ptr(w_om), _ptr(b_om), _ptr(out), N, H, W,
                                            C, G, kh, kw, pad, dil, dtype, algo,
                                            _stream(stream)),
           "dcnv4_fused_forward_algo")


def dcn_output_size(n_in, k, stride, pad, dil):
    return int(_load().dcn_output_size(n_in, k, stride, pad, dil))


def dcn_status_string(status):
    return _load().dcn_status_string(status).decode()


def dcn_last_cuda_error():
    return int(_load().dcn_last_cuda_error())


def dcn_launch_count():
    return int(_load().dcn_launch_count())


def dcn_version():
    return int(_load().dcn_version())


# ------------------------------------------------------------ tensor helpers

def dtype_code(t):
    """dcn_dtype_t of a torch tensor."""
    import torch
    codes = {torch.float32: 0, torch.float16: 1, torch.bfloat16: 2}
    if t.dtype not in codes:
        raise TypeError(f"unsupported dtype {t.dtype}")
    return codes[t.dtype]


def _require(cond, msg):
    if not cond:
        raise ValueError(msg)


def dcn(x, offset, mask, kh=3, kw=3, stride=1, pad=1, dil=1, softmax_flag=0, out=None,
        stream=None, algo="auto"):
    """dcn_forward_algo on torch CUDA tensors; allocates `out` when not given.

    x [N, H, W, C], offset [N, Ho, Wo, G, K, 2], mask [N, Ho, Wo, G, K], all of
    one dtype (float32 / float16 / bfloat16), contiguous, on one CUDA device.
    algo: "auto" (dcn_forward), "gather" or "band".
    """
    import torch
    _require(x.dim() == 4 and mask.dim() == 5 and offset.dim() == 6,
             "expected x [N,H,W,C], offset [N,Ho,Wo,G,K,2], mask [N,Ho,Wo,G,K]")
    N, H, W, C = x.shape
    G = mask.shape[3]
    Ho = dcn_output_size(H, kh, stride, pad, dil)
    Wo = dcn_output_size(W, kw, stride, pad, dil)
    K = kh * kw
    _require(tuple(offset.shape) == (N, Ho, Wo, G, K, 2), "offset has the wrong shape")
    _require(tuple(mask.shape) == (N, Ho, Wo, G, K), "mask has the wrong shape")
    _require(offset.dtype == x.dtype and mask.dtype == x.dtype, "mixed dtypes")
    _require(x.is_cuda and offset.is_cuda and mask.is_cuda, "tensors must be on a CUDA device")
    _require(x.is_contiguous() and offset.is_contiguous() and mask.is_contiguous(),
             "tensors must be contiguous")
    if out is None:
        out = torch.empty((N, Ho, Wo, C), dtype=x.dtype, device=x.device)
    _require(tuple(out.shape) == (N, Ho, Wo, C) and out.dtype == x.dtype and out.is_contiguous(),
             "out has the wrong shape, dtype or layout")
    _require(algo in ALGO_CODES, f"algo must be one of {sorted(ALGO_CODES)}")
    dcn_forward_algo(x, offset, mask, out, N, H, W, C, G, kh, kw, stride, pad, dil,
                     softmax_flag, dtype_code(x), ALGO_CODES[algo], stream)
    return out


def msda(value, spatial_shapes, level_start, sampling_loc, attn_w, out=None, stream=None):
    """msda_forward on torch CUDA tensors; allocates `out` when not given.

    value [N, S, M, D], spatial_shapes [L, 2] int64 (H, W), level_start [L] int64,
    sampling_loc [N, Lq, M, L, K, 2], attn_w [N, Lq, M, L, K].
    """
    import torch
    _require(value.dim() == 4 and attn_w.dim() == 5 and sampling_loc.dim() == 6,
             "expected value [N,S,M,D], loc [N,Lq,M,L,K,2], attn [N,Lq,M,L,K]")
    N, S, M, D = value.shape
    _, Lq, _, L, K = attn_w.shape
    _require(tuple(sampling_loc.shape) == (N, Lq, M, L, K, 2), "sampling_loc has the wrong shape")
    _require(tuple(attn_w.shape[:3]) == (N, Lq, M), "attn_w has the wrong shape")
    _require(tuple(spatial_shapes.shape) == (L, 2) and tuple(level_start.shape) == (L,),
             "spatial_shapes / level_start have the wrong shape")
    _require(spatial_shapes.dtype == torch.int64 and level_start.dtype == torch.int64,
             "spatial_shapes / level_start must be int64")
    _require(sampling_loc.dtype == value.dtype and attn_w.dtype == value.dtype, "mixed dtypes")
    for t in (value, spatial_shapes, level_start, sampling_loc, attn_w):
        _require(t.is_cuda and t.is_contiguous(), "tensors must be contiguous CUDA tensors")
    if out is None:
        out = torch.empty((N, Lq, M * D), dtype=value.dtype, device=value.device)
    _require(tuple(out.shape) == (N, Lq, M * D) and out.dtype == value.dtype and out.is_contiguous(),
             "out has the wrong shape, dtype or layout")
    msda_forward(value, spatial_shapes, level_start, sampling_loc, attn_w, out, N, Lq, M, D, L,
                 K, dtype_code(value), stream)
    return out


def _workspace(nbytes, device, workspace):
    """A caller-given workspace tensor, or a new one of nbytes (16-byte aligned)."""
    import torch
    if nbytes <= 0:
        return None, 0
    if workspace is None:
        workspace = torch.empty(nbytes // 4, dtype=torch.float32, device=device)
    _require(workspace.is_cuda and workspace.is_contiguous(), "workspace must be a CUDA tensor")
    have = workspace.numel() * workspace.element_size()
    _require(have >= nbytes, f"workspace holds {have} bytes, {nbytes} needed")
    return workspace, have


def dcn_grad(x, offset, mask, grad_out, kh=3, kw=3, stride=1, pad=1, dil=1, softmax_flag=0,
             workspace=None, stream=None):
    """dcn_backward on torch CUDA tensors: returns (grad_x, grad_offset, grad_mask).

    The float32 accumulator for grad_x of 16-bit data comes from `workspace`
    when given (a CUDA tensor of at least dcn_backward_workspace_size bytes),
    else a new tensor.
    """
    import torch
    _require(x.dim() == 4 and mask.dim() == 5 and offset.dim() == 6,
             "expected x [N,H,W,C], offset [N,Ho,Wo,G,K,2], mask [N,Ho,Wo,G,K]")
    N, H, W, C = x.shape
    G = mask.shape[3]
    Ho = dcn_output_size(H, kh, stride, pad, dil)
    Wo = dcn_output_size(W, kw, stride, pad, dil)
    K = kh * kw
    _require(tuple(offset.shape) == (N, Ho, Wo, G, K, 2), "offset has the wrong shape")
    _require(tuple(mask.shape) == (N, Ho, Wo, G, K), "mask has the wrong shape")
    _require(tuple(grad_out.shape) == (N, Ho, Wo, C), "grad_out has the wrong shape")
    for t in (offset, mask, grad_out):
        _require(t.dtype == x.dtype, "mixed dtypes")
    for t in (x, offset, mask, grad_out):
        _require(t.is_cuda and t.is_contiguous(), "tensors must be contiguous CUDA tensors")
    code = dtype_code(x)
    ws, ws_bytes = _workspace(dcn_backward_workspace_size(N, H, W, C, code), x.device, workspace)
    gx = torch.empty_like(x)
    goff = torch.empty_like(offset)
    gmask = torch.empty_like(mask)
    dcn_backward(x, offset, mask, grad_out, gx, goff, gmask, ws, ws_bytes, N, H, W, C, G, kh,
                 kw, stride, pad, dil, softmax_flag, code, stream)
    return gx, goff, gmask


def msda_grad(value, spatial_shapes, level_start, sampling_loc, attn_w, grad_out,
              workspace=None, stream=None):
    """msda_backward on torch CUDA tensors: returns (grad_value, grad_loc, grad_attn)."""
    import torch
    N, S, M, D = value.shape
    _, Lq, _, L, K = attn_w.shape
    _require(tuple(sampling_loc.shape) == (N, Lq, M, L, K, 2), "sampling_loc has the wrong shape")
    _require(tuple(grad_out.shape) == (N, Lq, M * D), "grad_out has the wrong shape")
    _require(spatial_shapes.dtype == torch.int64 and level_start.dtype == torch.int64,
             "spatial_shapes / level_start must be int64")
    for t in (sampling_loc, attn_w, grad_out):
        _require(t.dtype == value.dtype, "mixed dtypes")
    for t in (value, spatial_shapes, level_start, sampling_loc, attn_w, grad_out):
        _require(t.is_cuda and t.is_contiguous(), "tensors must be contiguous CUDA tensors")
    code = dtype_code(value)
    ws, ws_bytes = _workspace(msda_backward_workspace_size(N, S, M, D, code), value.device,
                              workspace)
    gv = torch.empty_like(value)
    gl = torch.empty_like(sampling_loc)
    ga = torch.empty_like(attn_w)
    msda_backward(value, spatial_shapes, level_start, sampling_loc, attn_w, grad_out, gv, gl, ga,
                  ws, ws_bytes, N, S, Lq, M, D, L, K, code, stream)
    return gv, gl, ga


def dynconv(x, weights, K, softmax_flag=1, out=None, stream=None, algo="auto"):
    """dynconv_forward_algo (the ContMix core) on torch CUDA tensors.

    x [N, H, W, C], weights [N, H, W, G, K*K] (tap ky * K + kx), one dtype.
    algo: "auto" (the tensor-core kernel where it applies), "tensor" or "simt".
    """
    import torch
    _require(x.dim() == 4 and weights.dim() == 5, "expected x [N,H,W,C], weights [N,H,W,G,K*K]")
    N, H, W, C = x.shape
    G = weights.shape[3]
    _require(tuple(weights.shape) == (N, H, W, G, K * K), "weights has the wrong shape")
    _require(weights.dtype == x.dtype, "mixed dtypes")
    for t in (x, weights):
        _require(t.is_cuda and t.is_contiguous(), "tensors must be contiguous CUDA tensors")
    if out is None:
        out = torch.empty_like(x)
    _require(tuple(out.shape) == (N, H, W, C) and out.dtype == x.dtype and out.is_contiguous(),
             "out has the wrong shape, dtype or layout")
    _require(algo in DYNCONV_ALGO_CODES, f"algo must be one of {sorted(DYNCONV_ALGO_CODES)}")
    dynconv_forward_algo(x, weights, out, N, H, W, C, G, K, softmax_flag, dtype_code(x),
                         DYNCONV_ALGO_CODES[algo], stream)
    return out


def msda_points(value, spatial_shapes, level_start, reference, offsets, attn_w,
                valid_ratios=None, out=None, stream=None):
    """msda_forward_points on torch CUDA tensors: reference [N, Lq, 2 or 4],
    offsets [N, Lq, M, L, K, 2], valid_ratios [N, L, 2] or None."""
    import torch
    N, S, M, D = value.shape
    _, Lq, _, L, K = attn_w.shape
    ref_dim = reference.shape[-1]
    _require(tuple(reference.shape) == (N, Lq, ref_dim) and ref_dim in (2, 4),
             "reference must be [N, Lq, 2] or [N, Lq, 4]")
    _require(tuple(offsets.shape) == (N, Lq, M, L, K, 2), "offsets has the wrong shape")
    _require(valid_ratios is None or tuple(valid_ratios.shape) == (N, L, 2),
             "valid_ratios must be [N, L, 2]")
    for t in (value, reference, offsets, attn_w) + ((valid_ratios,) if valid_ratios is not None else ()):
        _require(t.is_cuda and t.is_contiguous() and t.dtype == value.dtype,
                 "tensors must be contiguous CUDA tensors of one dtype")
    if out is None:
        out = torch.empty((N, Lq, M * D), dtype=value.dtype, device=value.device)
    msda_forward_points(value, spatial_shapes, level_start, reference, ref_dim, valid_ratios,
                        offsets, attn_w, out, N, Lq, M, D, L, K, dtype_code(value), stream)
    return out


def mask_value(value, mask, out=None, stream=None):
    """msda_mask_value on torch CUDA tensors (mask [N, S] bool or uint8);
    out=value masks in place."""
    import torch
    N, S, M, D = value.shape
    _require(tuple(mask.shape) == (N, S), "mask must be [N, S]")
    m = mask.to(torch.uint8) if mask.dtype != torch.uint8 else mask
    _require(m.is_cuda and m.is_contiguous() and value.is_contiguous(), "contiguous CUDA tensors")
    if out is None:
        out = torch.empty_like(value)
    msda_mask_value(value, m, out, N, S, M, D, dtype_code(value), stream)
    return out


def dcnv4_fused(x, w_om, b_om=None, groups=4, kh=3, kw=3, pad=1, dil=1, out=None, stream=None,
                algo="auto"):
    """dcnv4_fused_forward_algo on torch CUDA tensors: x [N, H, W, C], w_om
    [G*kh*kw*3, C], b_om [G*kh*kw*3] or None; algo "auto", "gather" or "band"."""
    import torch
    N, H, W, C = x.shape
    J = groups * kh * kw * 3
    _require(tuple(w_om.shape) == (J, C), "w_om must be [G*K*3, C]")
    _require(b_om is None or tuple(b_om.shape) == (J,), "b_om must be [G*K*3]")
    for t in (x, w_om) + ((b_om,) if b_om is not None else ()):
        _require(t.is_cuda and t.is_contiguous() and t.dtype == x.dtype,
                 "tensors must be contiguous CUDA tensors of one dtype")
    if out is None:
        out = torch.empty_like(x)
    _require(algo in ALGO_CODES, f"algo must be one of {sorted(ALGO_CODES)}")
    dcnv4_fused_forward_algo(x, w_om, b_om, out, N, H, W, C, groups, kh, kw, pad, dil,
                             dtype_code(x), ALGO_CODES[algo], stream)
    return out
