// C interface of libdcn_b200.so: dcn_forward (argument checks, launch
// shape, dispatch to the sm_100a DCN forward kernels).
#include "abi_common.cuh"
#include "dcn_fwd.cuh"

using namespace dcnb_abi;

namespace {

template <typename T, int VB>
const void* dcn_kernel_for(int softmax, int kh, int kw) {
    using namespace dcnb;
    if (kh == 3 && kw == 3)   // the common window: taps fully unrolled
        return softmax ? (const void*)dcn_fwd_kernel<T, VB, true, 3>
                       : (const void*)dcn_fwd_kernel<T, VB, false, 3>;
    return softmax ? (const void*)dcn_fwd_kernel<T, VB, true>
                   : (const void*)dcn_fwd_kernel<T, VB, false>;
}

template <typename T>
const void* dcn_kernel_vb(int vb, int kh, int kw, int softmax) {
    switch (vb) {
        case 32: return dcn_kernel_for<T, 32>(softmax, kh, kw);
        case 16: return dcn_kernel_for<T, 16>(softmax, kh, kw);
        case 8: return dcn_kernel_for<T, 8>(softmax, kh, kw);
        case 4: return dcn_kernel_for<T, 4>(softmax, kh, kw);
        default: break;
    }
    if constexpr (sizeof(T) == 2) {
        if (vb == 2) return dcn_kernel_for<T, 2>(softmax, kh, kw);
    }
    return nullptr;
}

}  // namespace

extern "C" {

int dcn_forward(const void* x, const void* offset, const void* mask, void* out, int N, int H,
                int W, int C, int G, int kh, int kw, int stride, int pad, int dil,
                int softmax_flag, int dtype, void* stream) {
    const int es = elem_bytes(dtype);
    if (es == 0 || N < 0 || H <= 0 || W <= 0 || C <= 0 || G <= 0 || C % G != 0 || kh <= 0 ||
        kw <= 0 || stride <= 0 || pad < 0 || dil <= 0 || (softmax_flag != 0 && softmax_flag != 1))
        return DCN_ERR_INVALID_ARG;
    if (H > kMaxDim || W > kMaxDim || pad > kMaxDim || stride > kMaxDim || dil > kMaxDim ||
        kh > kMaxDim || kw > kMaxDim || (long long)kh * kw > kMaxTaps)
        return DCN_ERR_UNSUPPORTED;
    const int Ho = dcn_output_size(H, kh, stride, pad, dil);
    const int Wo = dcn_output_size(W, kw, stride, pad, dil);
    if (Ho <= 0 || Wo <= 0) return DCN_ERR_INVALID_ARG;
    const int D = C / G;
    const int K = kh * kw;
    const long long img_bytes = (long long)H * W * C * es;
    const long long out_img_bytes = (long long)Ho * Wo * C * es;
    const long long items = (long long)N * Ho * Wo * G;
    if (img_bytes > kInt31 || out_img_bytes > kInt31 || items > kInt31 ||
        (long long)N * Ho * Wo > kInt31)
        return DCN_ERR_UNSUPPORTED;
    if (N == 0) return DCN_OK;
    if (!x || !offset || !mask || !out) return DCN_ERR_INVALID_ARG;
    if ((((uintptr_t)x | (uintptr_t)offset | (uintptr_t)mask | (uintptr_t)out) % es) != 0)
        return DCN_ERR_MISALIGNED;
    const long long x_bytes = img_bytes * N;
    const long long o_bytes = out_img_bytes * N;
    const long long off_bytes = items * K * 2 * es;
    const long long m_bytes = items * K * es;
    if (overlaps(out, o_bytes, x, x_bytes) || overlaps(out, o_bytes, offset, off_bytes) ||
        overlaps(out, o_bytes, mask, m_bytes))
        return DCN_ERR_INVALID_ARG;

    const int vb = pick_vector_bytes(es, D, (uintptr_t)x | (uintptr_t)out);
    if (vb == 0) return DCN_ERR_MISALIGNED;
    const int cpt = vb / es;
    const int tpi = D / cpt;
    if (tpi > 32) return DCN_ERR_UNSUPPORTED;   // one item must fit in a warp
    const int run_items = 32 / tpi;
    const int row_items = Wo * G;
    const int runs_per_row = (row_items + run_items - 1) / run_items;
    int sms = 148;
    {
        int device = 0;
        if (cudaGetDevice(&device) == cudaSuccess)
            (void)cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, device);
        (void)cudaGetLastError();
    }
    const TileShape ts =
        choose_tile(N, Ho, runs_per_row, kh * dil, sms, dcnb::kDcnMaxWarps, 25);
    const int warps = ts.h * ts.w;
    const int tiles_x = (runs_per_row + ts.w - 1) / ts.w;
    const long long tiles_per_image = (long long)((Ho + ts.h - 1) / ts.h) * tiles_x;
    const long long num_tiles = tiles_per_image * N;
    if (num_tiles > kInt31) return DCN_ERR_UNSUPPORTED;
    // per-warp shared slice for the run's offsets and masks; unstaged when the
    // CTA's slices would not fit in the default shared-memory window
    int stage_elems = run_items * K;
    const int slice = ((2 * stage_elems * es + 15) & ~15) + ((stage_elems * es + 15) & ~15);
    int smem = slice * warps;
    if (smem > kMaxStageBytes) {
        stage_elems = 0;
        smem = 0;
    }

    dcnb::DcnArgs a;
    a.x = x;
    a.offset = offset;
    a.mask = mask;
    a.out = out;
    a.H = H;
    a.W = W;
    a.C = C;
    a.G = G;
    a.D = D;
    a.kh = kh;
    a.kw = kw;
    a.K = K;
    a.stride = stride;
    a.pad = pad;
    a.dil = dil;
    a.Ho = Ho;
    a.Wo = Wo;
    a.tpi = tpi;
    a.run_items = run_items;
    a.runs_per_row = runs_per_row;
    a.tile_h = ts.h;
    a.tile_w = ts.w;
    a.tiles_x = tiles_x;
    a.tiles_per_image = (int)tiles_per_image;
    a.num_tiles = (int)num_tiles;
    a.stage_elems = stage_elems;
    a.prefetch = (((uintptr_t)x | (uintptr_t)(C * es)) % 16) == 0 ? 1 : 0;
    a.div_G = make_div((uint32_t)G);
    a.div_tpi = make_div((uint32_t)tpi);
    a.div_tile_w = make_div((uint32_t)ts.w);
    a.div_tiles_x = make_div((uint32_t)tiles_x);
    a.div_tiles_per_image = make_div((uint32_t)tiles_per_image);
    a.pix_bytes = (uint32_t)(C * es);
    a.row_bytes = (uint32_t)((long long)W * C * es);
    a.img_bytes = img_bytes;
    a.w_om = nullptr;
    a.b_om = nullptr;
    a.J = 0;

    const void* fn = nullptr;
    switch (dtype) {
        case DCN_F32: fn = dcn_kernel_vb<float>(vb, kh, kw, softmax_flag); break;
        case DCN_F16: fn = dcn_kernel_vb<__half>(vb, kh, kw, softmax_flag); break;
        case DCN_BF16: fn = dcn_kernel_vb<__nv_bfloat16>(vb, kh, kw, softmax_flag); break;
        default: break;
    }
    if (!fn) return DCN_ERR_UNSUPPORTED;
    return launch(fn, a, a.num_tiles, 32 * warps, smem, stream);
}

// msda_forward and its reference-point variants: `sampling_loc` holds the
// locations (ref_dim = 0) or the offsets (ref_dim = 2 / 4, with `ref` and

}  // extern "C"
