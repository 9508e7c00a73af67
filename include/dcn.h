/*
 * dcn.h - C interface of libdcn_b200.so: deformable sampling-aggregation
 * (DCNv3 / DCNv4 core) and multi-scale deformable attention (MSDeformAttn core)
 * forward and backward on NVIDIA B200 (sm_100a).
 *
 * Conventions shared by every entry point
 *   - All tensor pointers are DEVICE pointers owned by the caller.  The library
 *     allocates nothing, never synchronises, and launches its kernels
 *     asynchronously on `stream` (a cudaStream_t; NULL is the legacy default
 *     stream).  The caller keeps the buffers alive until the stream has run.
 *   - Tensors are contiguous, row-major, in the layouts stated per call.
 *   - `dtype` (dcn_dtype_t) applies to every floating tensor of the call
 *     (inputs and output).  Arithmetic is float32 throughout: 16-bit inputs are
 *     widened exactly, products and sums are float32, and the output is rounded
 *     once, to nearest even.
 *   - `out` must not overlap any input (DCN_ERR_INVALID_ARG).
 *   - No C++ exception crosses this interface; every entry point returns a
 *     dcn_status_t.  On an error nothing is launched and `out` is untouched,
 *     except DCN_ERR_CUDA, which reports a failed launch.
 *   - Thread safety: calls are independent and may come from several host
 *     threads; each runs on the stream it is given.
 */
#ifndef DCN_B200_H
#define DCN_B200_H

#include <stdint.h>

/* symbols of the shared library (it is built with hidden default visibility) */
#if defined(__GNUC__)
#define DCN_API __attribute__((visibility("default")))
#else
#define DCN_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef enum { DCN_F32 = 0, DCN_F16 = 1, DCN_BF16 = 2 } dcn_dtype_t;

typedef enum {
    DCN_OK = 0,
    DCN_ERR_INVALID_ARG = -1,  /* bad dimension, null pointer, unknown dtype, aliasing */
    DCN_ERR_UNSUPPORTED = -2,  /* valid request beyond the library's stated limits */
    DCN_ERR_MISALIGNED = -3,   /* a pointer not aligned to its element size */
    DCN_ERR_CUDA = -4          /* the kernel launch failed (see dcn_last_cuda_error) */
} dcn_status_t;

/*
 * dcn_forward - DCNv3 / DCNv4 deformable sampling-aggregation, forward.
 *
 * Defined by "InternImage: Deformable Convolutions at Scale" ch.1-4 (learned
 * offsets, bilinear read with zero padding, groups) and the "DCNv4" note,
 * "Why Is Sampling Just 9 Points Still Slow?" (y_g(p0) = sum_k m_gk x_g(p0 +
 * p_k + dp_gk)) and "1. Remove Softmax".  For every output pixel (oy, ox),
 * group g < G and channel c < D = C / G:
 *
 *   out[n][oy][ox][g*D + c] = sum_{ix < kw, iy < kh} m[k] * B(x[n][.][.][g*D + c], px, py)
 *     k  = ix * kh + iy
 *     px = ox*stride - pad + ix*dil + offset[n][oy][ox][g][k][0]
 *     py = oy*stride - pad + iy*dil + offset[n][oy][ox][g][k][1]
 *     m[k] = mask[n][oy][ox][g][k]                       (softmax_flag = 0, DCNv4)
 *     m[k] = softmax over k of mask[n][oy][ox][g][.]     (softmax_flag = 1, DCNv3)
 *   B(f, px, py): bilinear read, corners floor(p) and floor(p) + 1 with weights
 *   (1-a)(1-b), a(1-b), (1-a)b, ab (a, b the fractional parts); corners outside
 *   the map read 0 (no clamping, no renormalisation).
 *
 * Layouts (channels-last):
 *   x      [N][H][W][C]
 *   offset [N][Ho][Wo][G][K][2]   (dx, dy) in pixels, x along W, K = kh * kw
 *   mask   [N][Ho][Wo][G][K]      modulation m, or logits when softmax_flag = 1
 *   out    [N][Ho][Wo][C]
 *   Ho = (H + 2*pad - dil*(kh - 1) - 1) / stride + 1, Wo likewise with W, kw.
 *
 * Limits: H, W, pad, stride, dil <= 65536; kh * kw <= 1024; one group's
 * channels D * element size <= 1024 bytes (at most 32 threads per (pixel,
 * group)); one image of x and of out below 2^31 bytes; N * Ho * Wo * G below
 * 2^31 (DCN_ERR_UNSUPPORTED otherwise).  N = 0 launches nothing and
 * returns DCN_OK.  Offsets may be any value: a tap whose corners all fall
 * outside the map, however far, contributes 0; a NaN offset makes its tap
 * contribute 0.  Non-finite x or mask values give unspecified (but never
 * trapping) results.
 * Errors: DCN_ERR_INVALID_ARG for N < 0, any other dimension <= 0 (pad < 0),
 * C % G != 0, Ho or Wo <= 0, softmax_flag not 0/1, an unknown dtype, a null
 * pointer (N > 0) or out overlapping an input; DCN_ERR_MISALIGNED when a
 * pointer is not aligned to the element size.
 */
DCN_API int dcn_forward(const void* x, const void* offset, const void* mask, void* out,
                int N, int H, int W, int C, int G, int kh, int kw,
                int stride, int pad, int dil, int softmax_flag, int dtype,
                void* stream);

/*
 * dcn_forward_algo - dcn_forward with a choice of kernel.
 *
 * The same operator, arguments, layouts, limits and errors as dcn_forward
 * (which is dcn_forward_algo with DCN_ALGO_AUTO); `algo` picks the kernel:
 *   DCN_ALGO_GATHER  corners read through the L1 cache; every shape;
 *   DCN_ALGO_BAND    the input rows a CTA's output rows can reach (window plus
 *                    a margin of up to 6 rows for the offsets) staged in shared
 *                    memory by bulk copies, corners read from there (taps whose
 *                    offsets leave the band read global memory); only for
 *                    16-bit data with 16 channels per group, C * 2 a multiple
 *                    of 128 bytes, all four tensors 16-byte aligned, offset and
 *                    mask rows of a multiple of 16 bytes and a band that fits in
 *                    shared memory (W * C * 2 bytes per row): DCN_ERR_UNSUPPORTED
 *                    otherwise;
 *   DCN_ALGO_AUTO    the band kernel where it applies, else the gather kernel.
 * The two kernels round the same float32 sums; their outputs may differ in the
 * last bit where the order of the float32 additions differs.
 * Errors: as dcn_forward, plus DCN_ERR_INVALID_ARG for an unknown `algo`.
 */
typedef enum {
    DCN_ALGO_AUTO = 0,
    DCN_ALGO_GATHER = 1,
    DCN_ALGO_SIMT = 1,      /* dynconv_forward_algo: the CUDA-core (FFMA) kernel */
    DCN_ALGO_BAND = 2,
    DCN_ALGO_TENSOR = 3     /* dynconv_forward_algo: the tensor-core kernel */
} dcn_algo_t;

DCN_API int dcn_forward_algo(const void* x, const void* offset, const void* mask, void* out,
                     int N, int H, int W, int C, int G, int kh, int kw,
                     int stride, int pad, int dil, int softmax_flag, int dtype,
                     int algo, void* stream);

/*
 * dcn_forward_plan - which kernel dcn_forward_algo runs for a shape, and the
 * band kernel's launch shape.  Host only: no CUDA call, no device memory.
 *
 * Arguments as dcn_forward_algo without the tensors and the stream; the
 * tensors are taken to be 16-byte aligned.  `plan` (caller-owned, 8 ints) is
 * written on DCN_OK only:
 *   plan[0]  DCN_ALGO_BAND or DCN_ALGO_GATHER, the kernel that runs; 0 when
 *            N = 0 (nothing is launched; plan[1..7] still describe the shape)
 *   plan[1]  band kernel: output rows per step            (0 for the gather kernel)
 *   plan[2]  band kernel: offset margin, input rows staged above and below
 *            the window rows
 *   plan[3]  band kernel: input rows in the shared-memory ring
 *   plan[4]  band kernel: sampler warps per CTA (one more warp issues the copies)
 *   plan[5]  band kernel: steps in flight
 *   plan[6]  band kernel: warp runs (32 items) per output row
 *   plan[7]  band kernel: dynamic shared memory per CTA, bytes
 * A CTA of the band kernel owns a contiguous range of output rows (numbered
 * n * Ho + oy over the batch), one CTA per SM.
 * Errors: those of dcn_forward_algo that the shape decides (DCN_ERR_INVALID_ARG,
 * DCN_ERR_UNSUPPORTED, including DCN_ALGO_BAND on a shape the band kernel
 * does not take), and DCN_ERR_INVALID_ARG for a null `plan`.
 */
DCN_API int dcn_forward_plan(int N, int H, int W, int C, int G, int kh, int kw,
                     int stride, int pad, int dil, int softmax_flag, int dtype,
                     int algo, int* plan);

/*
 * dcn_device_flags - the per-device status word of the library's kernels.
 *
 * Bits (sticky until reset):
 *   DCN_FLAG_WAIT_TIMEOUT   a bounded wait of a band kernel's pipeline gave up
 *                           after about two seconds; its CTA stopped, so the
 *                           output of that call is incomplete;
 *   DCN_FLAG_OUT_OF_BOUNDS  (debug library only) a kernel computed a gather,
 *                           shared-memory or store address outside its buffer;
 *                           the access was skipped (a load read zeros);
 *   DCN_FLAG_BAD_LEVELS     (debug library only) an MSDA level table that is not
 *                           a gap-free, in-order list of positive shapes; the
 *                           call then reads no value rows.
 * Returns the word of the current device and clears it when reset != 0. The
 * read is a synchronous copy: it waits for the device's preceding work.
 * No counterpart on the pages: a guard of this library's own kernels.
 * Returns DCN_ERR_CUDA if the read fails.
 */
#define DCN_FLAG_WAIT_TIMEOUT 1
#define DCN_FLAG_OUT_OF_BOUNDS 2
#define DCN_FLAG_BAD_LEVELS 4

DCN_API int dcn_device_flags(int reset);

/*
 * dcn_debug_checks - 1 when this library was built with the device-side
 * checks (the debug library, libdcn_b200_debug.so: every DCN and MSDA forward
 * gather and store address is checked against its buffer, and the MSDA level
 * table on the device), else 0. The debug library has the same interface and
 * the same results; it is slower.
 */
DCN_API int dcn_debug_checks(void);

/*
 * msda_forward - multi-scale deformable attention core, forward.
 *
 * Defined by "Deformable DETR: Learn Where to Read", "A learned location can
 * fall between cells" (x = u W_l - 1/2, y = v H_l - 1/2, bilinear tent weights
 * over the four floor/ceil neighbours, zero outside, no clamping, no
 * renormalisation) and "Mix samples with a per-head budget" (h_m = sum over
 * levels l and points k of A_mlk times the sample, heads concatenated before
 * the output projection, which is not part of this call):
 *
 *   out[n][q][h*D + c] = sum_{l < L, k < K} attn_w[n][q][h][l][k] *
 *                        S_l(value[n][start_l + .][h][c], sampling_loc[n][q][h][l][k])
 *
 * Layouts:
 *   value          [N][S][M][D]       levels concatenated row-major, level l at
 *                                     rows [start_l, start_l + H_l W_l)
 *   spatial_shapes [L][2] int64       (H_l, W_l), DEVICE memory
 *   level_start    [L]    int64       start_l, DEVICE memory
 *   sampling_loc   [N][Lq][M][L][K][2] normalised (u, v) = (x, y), any real value
 *   attn_w         [N][Lq][M][L][K]   already normalised weights (used as given)
 *   out            [N][Lq][M*D]
 *   S is taken as level_start[L-1] + H_{L-1} * W_{L-1} (levels stored in order,
 *   without gaps).
 *
 * The device contents of spatial_shapes and level_start are a precondition
 * (positive shapes, starts inside value); they are not validated, because that
 * would need a synchronisation.
 * Limits: L <= 16, K <= 64, one head's channels D * element size <= 1024
 * bytes, N * Lq * M below 2^31 (DCN_ERR_UNSUPPORTED otherwise); S below 2^31
 * rows (a precondition, like the level table).  N = 0 or Lq = 0 launches
 * nothing and returns DCN_OK.
 * Errors: DCN_ERR_INVALID_ARG for N < 0, Lq < 0, M, D, L or K <= 0, an unknown
 * dtype, a null pointer (N * Lq > 0) or out overlapping an input;
 * DCN_ERR_MISALIGNED when a pointer is not aligned to its element size.
 */
DCN_API int msda_forward(const void* value, const int64_t* spatial_shapes,
                 const int64_t* level_start, const void* sampling_loc,
                 const void* attn_w, void* out, int N, int Lq, int M, int D,
                 int L, int K, int dtype, void* stream);

/*
 * dcnv4_fused_forward - DCNv4 core fed by its merged offset / mask linear.
 *
 * Defined by the "DCNv4" note, "1. Remove Softmax" (one linear layer gives
 * each location its G*K offset pairs and G*K modulation scalars, used without
 * a softmax) and the passages of dcn_forward.  For every pixel p:
 *   om[p][j] = sum_c w_om[j][c] * x[p][c] + b_om[j],  j < J = G * K * 3
 *   offset[p][g][k][c2] = om[p][(g*K + k)*2 + c2],  mask[p][g][k] = om[p][2GK + g*K + k]
 *   out = dcn_forward(x, offset, mask) with stride 1 and softmax_flag 0.
 * The offsets and masks are computed per warp on the tensor cores (16-bit
 * inputs, float32 accumulation), kept in float32 in shared memory and never
 * written to global memory.
 *
 * Layouts: x [N][H][W][C], w_om [J][C], b_om [J] (or NULL for no bias),
 * out [N][H][W][C]; all 16-bit (f16 or bf16).
 * Limits: dtype f16 / bf16 (f32: DCN_ERR_UNSUPPORTED); odd kh, kw with
 * pad * 2 == dil * (kh - 1) == dil * (kw - 1) (the output keeps the input
 * size); C a multiple of 16, at most 128; a warp's run of (pixel, group) items must hold
 * whole pixels (32 / TPI a multiple of G); the limits of dcn_forward.
 * Errors: as dcn_forward; DCN_ERR_MISALIGNED unless x and out are 4-byte
 * aligned and w_om, b_om aligned to the element size.
 */
DCN_API int dcnv4_fused_forward(const void* x, const void* w_om, const void* b_om, void* out,
                 int N, int H, int W, int C, int G, int kh, int kw, int pad, int dil,
                 int dtype, void* stream);

/*
 * dcnv4_fused_forward_algo - dcnv4_fused_forward with a choice of kernel.
 *
 * The same operator, arguments, layouts and errors as dcnv4_fused_forward
 * (which is this call with DCN_ALGO_AUTO); `algo` picks the kernel:
 *   DCN_ALGO_GATHER  corners read through L1, the linear per warp run on the
 *                    warp-level tensor-core path (mma.sync);
 *   DCN_ALGO_BAND    input rows staged in shared memory (as dcn_forward_algo's
 *                    band kernel) and the linear of each step's pixels (up to
 *                    128) as one tcgen05 product (M = 128, N = 3GK rounded up to
 *                    16, K = C) with float32 accumulators in tensor memory, fed
 *                    by tensor-map loads; only for 16 channels per group, C a
 *                    multiple of 64 up to 256, 3 G K <= 256, W <= 128 and
 *                    16-byte aligned x, w_om and out: DCN_ERR_UNSUPPORTED
 *                    otherwise;
 *   DCN_ALGO_AUTO    the band kernel where it applies, else the gather kernel.
 * Both keep the offsets and masks in float32 on chip; the two products add in
 * different orders, so outputs may differ in the last bits.
 * Errors: as dcnv4_fused_forward, plus DCN_ERR_INVALID_ARG for an unknown
 * `algo`.
 */
DCN_API int dcnv4_fused_forward_algo(const void* x, const void* w_om, const void* b_om,
                 void* out, int N, int H, int W, int C, int G, int kh, int kw, int pad,
                 int dil, int dtype, int algo, void* stream);

/*
 * msda_forward_points - msda_forward fed from reference points or boxes.
 *
 * Defined by "Deformable DETR: Learn Where to Read", "A reference links
 * resolutions without equating their pixels" and helper 1: a query's
 * reference is in valid-image coordinates; level l's valid ratio r =
 * (W_valid / W_l, H_valid / H_l) scales it into the level's padded frame, and
 *   point reference (cx, cy):        s = (cx, cy) * r + offset / (W_l, H_l)
 *   box reference (cx, cy, w, h):    s = (cx, cy) * r + offset / K * (w, h) * r / 2
 * (componentwise, no clamping); then exactly msda_forward with location s.
 * The locations are formed in the kernel and never stored.
 *
 * Arguments: as msda_forward, with
 *   reference     [N][Lq][ref_dim]   ref_dim = 2 (point) or 4 (box), dtype
 *   valid_ratios  [N][L][2]          (x, y) ratios in dtype, or NULL for all 1
 *   offsets       [N][Lq][M][L][K][2] in place of sampling_loc
 * Padding masks are not applied here: zero the masked value rows first
 * (msda_mask_value), as the module does before the sampling core.
 * Errors: as msda_forward; DCN_ERR_INVALID_ARG also for ref_dim not 2 / 4 or
 * a NULL reference; DCN_ERR_MISALIGNED for a reference or ratio pointer not
 * aligned to the element size.
 */
DCN_API int msda_forward_points(const void* value, const int64_t* spatial_shapes,
                 const int64_t* level_start, const void* reference, int ref_dim,
                 const void* valid_ratios, const void* offsets, const void* attn_w, void* out,
                 int N, int Lq, int M, int D, int L, int K, int dtype, void* stream);

/*
 * msda_mask_value - zero the value rows of padded positions.
 *
 * "Deformable DETR", "A reference links resolutions ...": the attention module
 * zeroes projected values at masked positions, so that a read near a
 * valid-image edge mixes valid features with zeros.  For every n < N, s < S:
 *   out[n][s][.][.] = mask[n][s] ? 0 : value[n][s][.][.]
 * value / out [N][S][M][D] in dtype, mask [N][S] bytes (non-zero = masked).
 * out may be value itself (in place); otherwise it must not overlap it.
 * Errors: DCN_ERR_INVALID_ARG for a bad dimension, dtype, NULL pointer (N > 0)
 * or overlap; DCN_ERR_MISALIGNED for value / out not aligned to the element size.
 */
DCN_API int msda_mask_value(const void* value, const unsigned char* mask, void* out, int N,
                 int S, int M, int D, int dtype, void* stream);

/*
 * dcn_backward_workspace_size - bytes of scratch that dcn_backward needs.
 *
 * grad_x is a scatter (every tap adds to four pixels), accumulated in float32:
 * for 16-bit data in a float32 copy of x's shape that the caller provides,
 * N * H * W * C * 4 bytes; for float32 data in grad_x itself (0 bytes).
 * Returns the byte count, or DCN_ERR_INVALID_ARG (< 0) for a negative or
 * zero dimension (N < 0) or an unknown dtype.
 */
DCN_API long long dcn_backward_workspace_size(int N, int H, int W, int C, int dtype);

/*
 * dcn_backward - gradients of dcn_forward with respect to x, offset and mask.
 *
 * Defined by the same passages as dcn_forward, differentiated: "InternImage"
 * ch.2 (the bilinear read is differentiable in the sampling position, which is
 * how the offsets learn) and ch.3 / "DCNv4" "1. Remove Softmax" (the
 * modulation with and without the softmax).  With go = grad_out:
 *
 *   grad_x[n][y][x][g*D+c]  = sum over taps (oy, ox, k) whose corner (y, x) is
 *                             inside the map of m[k] * w_corner * go[n][oy][ox][g*D+c]
 *   grad_offset[..][k][0]   = m[k] * sum_c go * dB/dpx,  [1]: dB/dpy, where
 *                             dB/dpx = (1-b)(v01 - v00) + b(v11 - v10) and
 *                             dB/dpy = (1-a)(v10 - v00) + a(v11 - v01), corners
 *                             outside the map read 0; at an integer position the
 *                             derivative is the one of the cell to the right/below
 *   dL/dm[k]                = sum_c go * B(x, px, py)
 *   grad_mask[..][k]        = dL/dm[k]                              (softmax_flag = 0)
 *                           = m[k] * (dL/dm[k] - sum_j m[j] dL/dm[j])  (softmax_flag = 1:
 *                             the gradient with respect to the logits)
 *
 * Arguments: x, offset, mask, softmax_flag, the sizes and dtype exactly as
 * given to dcn_forward; grad_out [N][Ho][Wo][C]; outputs grad_x [N][H][W][C],
 * grad_offset [N][Ho][Wo][G][K][2] and grad_mask [N][Ho][Wo][G][K], all in
 * `dtype` and all overwritten.  `workspace` is caller-owned device scratch of
 * at least dcn_backward_workspace_size() bytes, 16-byte aligned (ignored and
 * may be NULL for float32); its contents on entry do not matter.
 * Launches, in stream order: a zero fill of the float32 accumulator, the
 * gradient kernel, and for 16-bit data the rounding of the accumulator into
 * grad_x.  grad_x is a float32 sum whose order of additions is not fixed
 * (hardware reductions), so its last bits may differ from run to run;
 * grad_offset and grad_mask are deterministic.
 * Limits: those of dcn_forward, plus: the shared-memory slice of one warp
 * (the run's offsets, masks and their gradients: 6 * K * es * 32 / TPI bytes,
 * and 4 * K * 32 / TPI more for softmax_flag = 1) at most 200 KiB
 * (DCN_ERR_UNSUPPORTED otherwise; K <= 169 always fits).
 * Errors: as dcn_forward, for every pointer; DCN_ERR_INVALID_ARG also when an
 * output overlaps an input, another output or the workspace, or when
 * workspace_bytes is too small; DCN_ERR_MISALIGNED for a workspace not
 * aligned to 16 bytes.
 */
DCN_API int dcn_backward(const void* x, const void* offset, const void* mask,
                 const void* grad_out, void* grad_x, void* grad_offset, void* grad_mask,
                 void* workspace, long long workspace_bytes, int N, int H, int W, int C,
                 int G, int kh, int kw, int stride, int pad, int dil, int softmax_flag,
                 int dtype, void* stream);

/* Size of the library's own static grad_x accumulator (one per device). */
#define DCN_STATIC_SCRATCH_BYTES (16LL << 20)

/*
 * dcn_backward_static_scratch - dcn_backward with the library's own scratch.
 *
 * The pages describe no counterpart: this is an interface convenience, not a
 * step of the method.  It is for callers that cannot hand dcn_backward a
 * workspace: a C host program with no device allocator of its own at call
 * time, or code that must not allocate once it has started (a fixed memory
 * budget).  Arguments, results, launches and errors are those of
 * dcn_backward, without `workspace` / `workspace_bytes`: for 16-bit data the
 * float32 grad_x accumulator is a statically sized array in the library's
 * device code (DCN_STATIC_SCRATCH_BYTES per device, reserved when the
 * library's device code is loaded on that device).  No call allocates.
 *   - Limit: N * H * W * C * 4 <= DCN_STATIC_SCRATCH_BYTES for f16 / bf16
 *     (N * H * W * C <= 4194304); beyond it DCN_ERR_UNSUPPORTED, nothing
 *     launched.  float32 data needs no scratch and has no such limit.
 *   - The first call on a device (with 16-bit data) looks up the array's
 *     device address with cudaGetSymbolAddress, with that device current,
 *     and caches it; a failure returns DCN_ERR_CUDA.  Make that first call
 *     before any stream capture on the device.
 *   - The accumulator is zero-filled by every call (it needs no clearing
 *     between calls), but there is one per device: calls whose work overlaps
 *     in time on one device (other streams, other host threads) race on it
 *     and give wrong grad_x.  Calls issued in order on one stream are safe.
 */
DCN_API int dcn_backward_static_scratch(const void* x, const void* offset, const void* mask,
                 const void* grad_out, void* grad_x, void* grad_offset, void* grad_mask,
                 int N, int H, int W, int C, int G, int kh, int kw, int stride, int pad,
                 int dil, int softmax_flag, int dtype, void* stream);

/*
 * msda_backward_workspace_size - bytes of scratch that msda_backward needs:
 * a float32 accumulator for grad_value, N * S * M * D * 4 bytes for 16-bit
 * data, 0 for float32 (accumulated in grad_value itself); DCN_ERR_INVALID_ARG
 * (< 0) for a bad dimension or dtype.
 */
DCN_API long long msda_backward_workspace_size(int N, int S, int M, int D, int dtype);

/*
 * msda_backward - gradients of msda_forward with respect to value,
 * sampling_loc and attn_w.
 *
 * Defined by the passages of msda_forward, differentiated ("A learned
 * location can fall between cells": the read is differentiable in the
 * location).  With go = grad_out[n][q][h*D + c], x = u W_l - 1/2,
 * y = v H_l - 1/2, a, b their fractional parts and A = attn_w[n][q][h][l][k]:
 *
 *   grad_value[n][start_l + r][h][c] += A * w_corner * go   for each corner r in the level
 *   grad_loc[..][0] = A * W_l * sum_c go * ((1-b)(v01 - v00) + b(v11 - v10))
 *   grad_loc[..][1] = A * H_l * sum_c go * ((1-a)(v10 - v00) + a(v11 - v01))
 *   grad_attn[..]   = sum_c go * S_l(value, loc)
 *
 * Arguments: as msda_forward, plus S (value rows per batch item, equal to
 * level_start[L-1] + H_{L-1} W_{L-1}), grad_out [N][Lq][M*D] and the outputs
 * grad_value [N][S][M][D], grad_loc [N][Lq][M][L][K][2] and grad_attn
 * [N][Lq][M][L][K], all in `dtype` and all overwritten.  `workspace` as for
 * dcn_backward, of msda_backward_workspace_size() bytes.  grad_value's last
 * bits depend on the order of hardware reductions; the others are
 * deterministic.  Same launch sequence, limits and errors as msda_forward and
 * dcn_backward (a warp's shared slice, 6 * L * K * es * 32 / TPI bytes, at
 * most 200 KiB).
 */
DCN_API int msda_backward(const void* value, const int64_t* spatial_shapes,
                  const int64_t* level_start, const void* sampling_loc, const void* attn_w,
                  const void* grad_out, void* grad_value, void* grad_loc, void* grad_attn,
                  void* workspace, long long workspace_bytes, int N, int S, int Lq, int M,
                  int D, int L, int K, int dtype, void* stream);

/*
 * dynconv_forward - dynamic local aggregation (the ContMix core), forward.
 *
 * Defined by the "OverLoCK" note, "ContMix: Put the Whole Image into the
 * Kernel", steps 4-5: a softmax turns each location's K*K numbers into its own
 * K x K kernel per channel group, which is applied to the zero-padded K x K
 * neighbourhood of that group's channels (taps row-major, as the note's unfold
 * with padding K / 2 orders them).  For every pixel (y, x), group g < G and
 * channel c < D = C / G:
 *
 *   out[n][y][x][g*D + c] = sum_{ky, kx < K} A[ky*K + kx] * x[n][y + ky - K/2][x + kx - K/2][g*D + c]
 *     A = softmax over t of weights[n][y][x][g][t]   (softmax_flag = 1)
 *     A = weights[n][y][x][g][.] as given             (softmax_flag = 0)
 *   with x = 0 outside the map.  It is dcn_forward with every offset zero,
 *   stride 1, pad K / 2, and the tap order ky * K + kx.
 *
 * Layouts: x [N][H][W][C], weights [N][H][W][G][K*K], out [N][H][W][C].
 * Limits: K odd, K <= 31; one group's channels a multiple of 32 bytes
 * (D * element size % 32 == 0: 16 f16 / bf16 or 8 f32 channels per 32 bytes);
 * H, W <= 65536; one image of x below 2^31 bytes (DCN_ERR_UNSUPPORTED
 * otherwise).  N = 0 launches nothing.
 * Errors: DCN_ERR_INVALID_ARG for a bad dimension, an even K, C % G != 0,
 * softmax_flag not 0/1, an unknown dtype, a null pointer (N > 0) or out
 * overlapping an input; DCN_ERR_MISALIGNED unless x and weights are 16-byte
 * aligned and out is 32-byte aligned.
 */
DCN_API int dynconv_forward(const void* x, const void* weights, void* out, int N, int H,
                 int W, int C, int G, int K, int softmax_flag, int dtype, void* stream);

/*
 * dynconv_forward_algo - dynconv_forward with the kernel chosen by `algo`.
 *
 *   DCN_ALGO_TENSOR  each kernel row of 16 consecutive outputs as a banded
 *                    16 x 32 matrix (the locations' K numbers) times the
 *                    window row (32 columns x 16 channels) on the tensor cores
 *                    (mma.sync m16n8k16, float32 accumulation); the softmaxed
 *                    numbers enter as a 16-bit high part plus the 16-bit
 *                    rounding of the remainder.  Only for f16 / bf16 data and
 *                    K = 7 or 13: DCN_ERR_UNSUPPORTED otherwise.  A non-finite
 *                    x value inside the 32-column window of a 16-output block
 *                    makes all of that block's outputs of the row non-finite
 *                    (the band's zeros multiply it), where the definition
 *                    leaves outputs that do not reach it unaffected.
 *   DCN_ALGO_SIMT    (= DCN_ALGO_GATHER) the CUDA-core kernel: float32 FMAs
 *                    over the staged window, any dtype and odd K <= 31.
 *   DCN_ALGO_AUTO    the tensor-core kernel where it applies, else the CUDA-core one.
 * The two kernels add the same products in different orders; their outputs
 * may differ in the last bit.
 * Errors: as dynconv_forward, plus DCN_ERR_INVALID_ARG for an unknown `algo`.
 */
DCN_API int dynconv_forward_algo(const void* x, const void* weights, void* out, int N, int H,
                 int W, int C, int G, int K, int softmax_flag, int dtype, int algo,
                 void* stream);

/* Output size of the deformable window: (in + 2 pad - dil (k - 1) - 1) / stride + 1,
 * or a value <= 0 when the window does not fit. */
DCN_API int dcn_output_size(int in, int k, int stride, int pad, int dil);

/* Static English text for a dcn_status_t value (never NULL). */
DCN_API const char* dcn_status_string(int status);

/* The cudaError_t of the most recent DCN_ERR_CUDA in the calling thread (0 if none). */
DCN_API int dcn_last_cuda_error(void);

/* Number of kernels this library has launched in this process (all threads). */
DCN_API uint64_t dcn_launch_count(void);

/* Library version as MAJOR * 10000 + MINOR * 100 + PATCH. */
DCN_API int dcn_version(void);

#ifdef __cplusplus
}
#endif

#endif /* DCN_B200_H */
