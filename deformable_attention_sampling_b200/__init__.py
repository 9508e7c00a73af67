"""Deformable sampling-aggregation on NVIDIA B200 (sm_100a).

DCNv3 / DCNv4 deformable convolution core and the multi-scale deformable
attention (MSDeformAttn) core, forward and backward, as hand-written CUDA kernels behind a
C interface (include/dcn.h, libdcn_b200.so).  This package is the thin Python
binding: it marshals pointers, sizes and streams and runs nothing itself.

    import deformable_attention_sampling_b200 as dcnb
    out = dcnb.dcn(x, offset, mask)          # torch CUDA tensors, NHWC
    out = dcnb.msda(value, shapes, starts, loc, attn)
    gx, goff, gmask = dcnb.dcn_grad(x, offset, mask, grad_out)
    gv, gloc, gattn = dcnb.msda_grad(value, shapes, starts, loc, attn, grad_out)
    out = dcnb.dynconv(x, weights, K)        # ContMix core: per-pixel K x K kernels
"""
from ._binding import (  # noqa: F401
    ALGO_CODES,
    DCN_ALGO_AUTO,
    DCN_ALGO_BAND,
    DCN_ALGO_GATHER,
    DCN_ALGO_SIMT,
    DCN_ALGO_TENSOR,
    DYNCONV_ALGO_CODES,
    DCN_ERR_CUDA,
    DCN_ERR_INVALID_ARG,
    DCN_ERR_MISALIGNED,
    DCN_ERR_UNSUPPORTED,
    DCN_OK,
    DTYPE_CODES,
    LIB_PATH,
    SIGNATURES,
    DcnError,
    dcn,
    STATIC_SCRATCH_BYTES,
    dcn_backward,
    dcn_backward_static_scratch,
    dcn_backward_workspace_size,
    dcn_forward,
    dcn_forward_algo,
    dcn_forward_plan,
    PLAN_FIELDS,
    DCN_FLAG_BAD_LEVELS,
    DCN_FLAG_OUT_OF_BOUNDS,
    DCN_FLAG_WAIT_TIMEOUT,
    DEBUG_LIB_PATH,
    dcn_debug_checks,
    dcn_device_flags,
    debug_library,
    dcn_grad,
    dcn_last_cuda_error,
    dcn_launch_count,
    dcn_output_size,
    dcnv4_fused,
    dcnv4_fused_forward,
    dcnv4_fused_forward_algo,
    dcn_status_string,
    dcn_version,
    dtype_code,
    dynconv,
    dynconv_forward,
    dynconv_forward_algo,
    library,
    msda,
    msda_backward,
    msda_backward_workspace_size,
    msda_forward,
    msda_forward_points,
    msda_mask_value,
    msda_points,
    mask_value,
    msda_grad,
)
