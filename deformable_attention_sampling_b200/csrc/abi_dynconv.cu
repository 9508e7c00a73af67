// C interface of libdcn_b200.so: dynconv_forward (the ContMix core).
#include "abi_common.cuh"
#include "dynconv_fwd.cuh"
#include "dynconv_mma.cuh"

using namespace dcnb_abi;

namespace {

template <typename T, int KT>
const void* dynconv_kernel_k(int softmax) {
    return softmax ? (const void*)dcnb::dynconv_fwd_kernel<T, true, KT>
                   : (const void*)dcnb::dynconv_fwd_kernel<T, false, KT>;
}

template <typename T>
const void* dynconv_kernel_for(int softmax, int K) {
    switch (K) {
        case 7: return dynconv_kernel_k<T, 7>(softmax);
        case 13: return dynconv_kernel_k<T, 13>(softmax);
        default: return dynconv_kernel_k<T, 0>(softmax);
    }
}

template <typename T, int KT>
const void* dynconv_mma_kernel_k(int softmax) {
    return softmax ? (const void*)dcnb::dynconv_mma_kernel<T, true, KT>
                   : (const void*)dcnb::dynconv_mma_kernel<T, false, KT>;
}

// The tensor-core kernel for this dtype and K, or null.
template <typename T>
const void* dynconv_mma_kernel_for(int softmax, int K) {
    switch (K) {
        case 7: return dynconv_mma_kernel_k<T, 7>(softmax);
        case 13: return dynconv_mma_kernel_k<T, 13>(softmax);
        default: return nullptr;
    }
}

}  // namespace

extern "C" {

int dynconv_forward(const void* x, const void* weights, void* out, int N, int H, int W, int C,
                    int G, int K, int softmax_flag, int dtype, void* stream) {
    return dynconv_forward_algo(x, weights, out, N, H, W, C, G, K, softmax_flag, dtype,
                                DCN_ALGO_AUTO, stream);
}

int dynconv_forward_algo(const void* x, const void* weights, void* out, int N, int H, int W,
                         int C, int G, int K, int softmax_flag, int dtype, int algo,
                         void* stream) {
    if (algo != DCN_ALGO_AUTO && algo != DCN_ALGO_SIMT && algo != DCN_ALGO_TENSOR)
        return DCN_ERR_INVALID_ARG;
    const int es = elem_bytes(dtype);
    if (es == 0 || N < 0 || H <= 0 || W <= 0 || C <= 0 || G <= 0 || C % G != 0 || K <= 0 ||
        K % 2 != 1 || (softmax_flag != 0 && softmax_flag != 1))
        return DCN_ERR_INVALID_ARG;
    const int D = C / G;
    if (K > dcnb::kDynMaxK || H > kMaxDim || W > kMaxDim || (D * es) % 32 != 0)
        return DCN_ERR_UNSUPPORTED;
    const long long pixels = (long long)N * H * W;
    if ((long long)H * W * C * es > kInt31 || pixels * G > kInt31 ||
        (long long)H * W * G * K * K > kInt31)
        return DCN_ERR_UNSUPPORTED;
    if (N == 0) return DCN_OK;
    if (!x || !weights || !out) return DCN_ERR_INVALID_ARG;
    if ((uintptr_t)x % 16 != 0 || (uintptr_t)out % 32 != 0 || (uintptr_t)weights % 16 != 0)
        return DCN_ERR_MISALIGNED;
    const long long xb = pixels * C * es;
    if (overlaps(out, xb, x, xb) || overlaps(out, xb, weights, pixels * G * K * K * es))
        return DCN_ERR_INVALID_ARG;

    dcnb::DynArgs a;
    if (algo != DCN_ALGO_SIMT) {
        // the tensor-core kernel: 16-bit data, a compiled K, 8 x 32 output tiles
        const void* fn = nullptr;
        if (dtype == DCN_F16) fn = dynconv_mma_kernel_for<__half>(softmax_flag, K);
        if (dtype == DCN_BF16) fn = dynconv_mma_kernel_for<__nv_bfloat16>(softmax_flag, K);
        if (fn) {
            a.x = x;
            a.w = weights;
            a.out = out;
            a.H = H;
            a.W = W;
            a.C = C;
            a.G = G;
            a.D = D;
            a.K = K;
            a.th = dcnb::kMmaRows;
            a.tiles_x = (W + dcnb::kMmaCols - 1) / dcnb::kMmaCols;
            a.tiles_y = (H + dcnb::kMmaRows - 1) / dcnb::kMmaRows;
            a.chunks = D * es / 32;
            a.win_rows = dcnb::kMmaRows + K - 1;
            a.row_bytes = dcnb::dyn_row_bytes(dcnb::kMmaWinCols);
            a.xs_bytes = a.win_rows * a.row_bytes;
            a.ws_bytes = 0;
            const int smem = dcnb::dyn_mma_smem(K);
            const long long ctas = (long long)N * a.tiles_y * a.tiles_x * G * a.chunks;
            if (ctas > kInt31 || smem > kMaxBwdSmemBytes) return DCN_ERR_UNSUPPORTED;
            return launch_grid(fn, a, (int)ctas, dcnb::kMmaThreads, smem, stream);
        }
        if (algo == DCN_ALGO_TENSOR) return DCN_ERR_UNSUPPORTED;
    }

    // tile rows: 8 on maps up to 64 rows (more CTAs), else 16
    const int th = H <= 64 ? 8 : 16;
    a.x = x;
    a.w = weights;
    a.out = out;
    a.H = H;
    a.W = W;
    a.C = C;
    a.G = G;
    a.D = D;
    a.K = K;
    a.th = th;
    a.tiles_x = (W + dcnb::kDynTileW - 1) / dcnb::kDynTileW;
    a.tiles_y = (H + th - 1) / th;
    a.chunks = D * es / 32;
    a.win_rows = th + K - 1;
    a.row_bytes = dcnb::dyn_row_bytes(dcnb::kDynTileW + K - 1);
    a.xs_bytes = a.win_rows * a.row_bytes;
    // the compiled kernel sizes keep their weights in registers: no slots
    const bool fixed_k = K == 7 || K == 13;
    a.ws_bytes = fixed_k ? 0 : ((K * dcnb::dyn_wstride(th) * 4) + 15) & ~15;
    const int raw_bytes = 2 * th * dcnb::kDynTileW * dcnb::dyn_slot_bytes(K, es);   // two buffers
    const int smem = a.xs_bytes + a.ws_bytes + raw_bytes;
    if (smem > kMaxBwdSmemBytes) return DCN_ERR_UNSUPPORTED;
    const long long ctas = (long long)N * a.tiles_y * a.tiles_x * G * a.chunks;
    if (ctas > kInt31) return DCN_ERR_UNSUPPORTED;

    const void* fn = nullptr;
    switch (dtype) {
        case DCN_F32: fn = dynconv_kernel_for<float>(softmax_flag, K); break;
        case DCN_F16: fn = dynconv_kernel_for<__half>(softmax_flag, K); break;
        case DCN_BF16: fn = dynconv_kernel_for<__nv_bfloat16>(softmax_flag, K); break;
        default: break;
    }
    if (!fn) return DCN_ERR_UNSUPPORTED;
    return launch_grid(fn, a, (int)ctas, th * dcnb::kDynSegs, smem, stream);
}

}  // extern "C"
