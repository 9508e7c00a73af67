// C interface of libdcn_b200.so: dcnv4_fused_forward (the DCNv4 core fed by
// its merged offset / mask linear).
#include "abi_common.cuh"
#include "dcn_fwd.cuh"

using namespace dcnb_abi;

namespace {

template <typename T, int VB>
const void* dcn_fused_kernel_for(int kh, int kw) {
    using namespace dcnb;
    if (kh == 3 && kw == 3) return (const void*)dcn_fwd_kernel<T, VB, false, 3, true>;
    return (const void*)dcn_fwd_kernel<T, VB, false, 0, true>;
}

template <typename T>
const void* dcn_fused_kernel_vb(int vb, int kh, int kw) {
    switch (vb) {
        case 32: return dcn_fused_kernel_for<T, 32>(kh, kw);
        case 16: return dcn_fused_kernel_for<T, 16>(kh, kw);
        case 8: return dcn_fused_kernel_for<T, 8>(kh, kw);
        case 4: return dcn_fused_kernel_for<T, 4>(kh, kw);
        case 2: return dcn_fused_kernel_for<T, 2>(kh, kw);
        default: return nullptr;
    }
}

}  // namespace

extern "C" {

int dcnv4_fused_forward(const void* x, const void* w_om, const void* b_om, void* out, int N,
                        int H, int W, int C, int G, int kh, int kw, int pad, int dil, int dtype,
                        void* stream) {
    const int es = elem_bytes(dtype);
    if (es == 0 || N < 0 || H <= 0 || W <= 0 || C <= 0 || G <= 0 || C % G != 0 || kh <= 0 ||
        kw <= 0 || pad < 0 || dil <= 0)
        return DCN_ERR_INVALID_ARG;
    if (dtype == DCN_F32) return DCN_ERR_UNSUPPORTED;   // the linear runs on 16-bit tensor cores
    // stride 1 and a same-size window: the linear is applied at each output pixel
    if (kh % 2 != 1 || kw % 2 != 1 || pad * 2 != dil * (kh - 1) || pad * 2 != dil * (kw - 1))
        return DCN_ERR_UNSUPPORTED;
    if (H > kMaxDim || W > kMaxDim || dil > kMaxDim || (long long)kh * kw > kMaxTaps ||
        C % 16 != 0)
        return DCN_ERR_UNSUPPORTED;
    const int D = C / G;
    const int K = kh * kw;
    const int J = G * K * 3;
    const long long img_bytes = (long long)H * W * C * es;
    const long long items = (long long)N * H * W * G;
    if (img_bytes > kInt31 || items > kInt31 || (long long)J * C > kInt31)
        return DCN_ERR_UNSUPPORTED;
    if (N == 0) return DCN_OK;
    if (!x || !w_om || !out) return DCN_ERR_INVALID_ARG;
    if ((((uintptr_t)x | (uintptr_t)out) % 4) != 0 || ((uintptr_t)w_om % es) != 0 ||
        ((uintptr_t)b_om % es) != 0)
        return DCN_ERR_MISALIGNED;
    const long long xb = img_bytes * N;
    if (overlaps(out, xb, x, xb) || overlaps(out, xb, w_om, (long long)J * C * es) ||
        (b_om && overlaps(out, xb, b_om, (long long)J * es)))
        return DCN_ERR_INVALID_ARG;

    const int vb = pick_vector_bytes(es, D, (uintptr_t)x | (uintptr_t)out);
    if (vb == 0) return DCN_ERR_MISALIGNED;
    const int cpt = vb / es;
    const int tpi = D / cpt;
    if (tpi > 32) return DCN_ERR_UNSUPPORTED;
    const int run_items = 32 / tpi;
    if (run_items % G != 0) return DCN_ERR_UNSUPPORTED;   // runs must hold whole pixels
    const int row_items = W * G;
    const int runs_per_row = (row_items + run_items - 1) / run_items;
    int sms = 148;
    {
        int device = 0;
        if (cudaGetDevice(&device) == cudaSuccess)
            (void)cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, device);
        (void)cudaGetLastError();
    }
    if (C > 16 * dcnb::kFusedMaxKSteps) return DCN_ERR_UNSUPPORTED;
    const int stage_elems = run_items * K;
    const int slice = ((2 * stage_elems * 4 + 15) & ~15) + ((stage_elems * 4 + 15) & ~15);
    const int rows = (J + 15) & ~15;
    const int front = ((rows * dcnb::fused_w_stride(C) * es + 15) & ~15) + ((J * 4 + 15) & ~15);
    int cap = (kMaxBwdSmemBytes - front) / slice;
    if (cap < 1) return DCN_ERR_UNSUPPORTED;
    if (cap > dcnb::kDcnMaxWarps) cap = dcnb::kDcnMaxWarps;
    const TileShape ts = choose_tile(N, H, runs_per_row, kh * dil, sms, cap, 25);
    const int warps = ts.h * ts.w;
    const int tiles_x = (runs_per_row + ts.w - 1) / ts.w;
    const long long tiles_per_image = (long long)((H + ts.h - 1) / ts.h) * tiles_x;
    const long long num_tiles = tiles_per_image * N;
    if (num_tiles > kInt31) return DCN_ERR_UNSUPPORTED;
    const int smem = front + slice * warps;

    dcnb::DcnArgs a;
    a.x = x;
    a.offset = nullptr;
    a.mask = nullptr;
    a.out = out;
    a.H = H;
    a.W = W;
    a.C = C;
    a.G = G;
    a.D = D;
    a.kh = kh;
    a.kw = kw;
    a.K = K;
    a.stride = 1;
    a.pad = pad;
    a.dil = dil;
    a.Ho = H;
    a.Wo = W;
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
    a.w_om = w_om;
    a.b_om = b_om;
    a.J = J;

    const void* fn = nullptr;
    switch (dtype) {
        case DCN_F16: fn = dcn_fused_kernel_vb<__half>(vb, kh, kw); break;
        case DCN_BF16: fn = dcn_fused_kernel_vb<__nv_bfloat16>(vb, kh, kw); break;
        default: break;
    }
    if (!fn) return DCN_ERR_UNSUPPORTED;
    return launch(fn, a, a.num_tiles, 32 * warps, smem, stream);
}

}  // extern "C"
