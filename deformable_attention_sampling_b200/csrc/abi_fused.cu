// C interface of libdcn_b200.so: dcnv4_fused_forward and
// dcnv4_fused_forward_algo (the DCNv4 core fed by its merged offset / mask
// linear).  Two kernels:
//   - the band kernel with the linear on tcgen05 (dcn_band_fused.cuh): 16-bit
//     data, 16 channels per group, C a multiple of 64 up to 256, 3 G K <= 256
//     outputs, W <= 128, 16-byte aligned tensors and a band that fits in
//     shared memory;
//   - the gather kernel with the linear on warp-level mma.sync (dcn_fwd.cuh,
//     FUSED): every other shape.
#include "abi_common.cuh"
#include "dcn_band_fused.cuh"
#include "dcn_fwd.cuh"

using namespace dcnb_abi;

namespace {

constexpr int kFusedSmemLimit = 227 * 1024;
constexpr int kFusedMaxStages = 3;

// The fused kernel runs its taps in a loop for every window size: with the
// four roles' code in one kernel, the 3 x 3 sampler unrolled over its taps
// stalled on instruction fetch (2.8 "no instruction" stalls per issue) and
// took 133.8 us per 64 x 56 x 56 x 64 fp16 launch against 114.0 us looped.
template <typename T>
const void* band_fused_kernel_for(int /*kh*/, int /*kw*/) {
    return (const void*)dcnb::dcn_band_fused_kernel<T, 0>;
}

// Launch configuration of the tcgen05 band kernel, or false when the shape or
// the pointers do not qualify (or a tensor map cannot be made).
bool band_fused_config(const void* x, const void* w_om, const void* b_om, void* out, int N,
                       int H, int W, int C, int G, int kh, int kw, int pad, int dil, bool bf16,
                       dcnb::BandFusedArgs* f, int* smem, int* threads) {
    const int es = 2;
    const int D = C / G;
    const int K = kh * kw;
    const int J = 3 * G * K;
    if (D != 16 || C % 64 != 0 || C > 256 || J > 256 || W > 128) return false;
    if ((((uintptr_t)x | (uintptr_t)w_om | (uintptr_t)out) % 16) != 0 ||
        ((uintptr_t)b_om % es) != 0)
        return false;
    const int NJ = (J + 15) / 16 * 16;
    const int kchunks = C / 64;
    const long long row_bytes = (long long)W * C * es;
    const int row_items = W * G;
    const int run_items = 32 / dcnb::kBandLanesPerItem;
    const int runs_per_row = (row_items + run_items - 1) / run_items;
    const int consumer_warps = dcnb::kFusedMaxThreads / 32 - 2 - dcnb::kFusedEpilogueWarps;
    const uint32_t w_bytes = (uint32_t)kchunks * (uint32_t)NJ * 128u;
    const uint32_t om_stride = (uint32_t)((J + 3) / 4 * 4);
    // candidates in order of preference: offset margin (taps that leave the
    // band are slow) and steps in flight (the product's result must be ready
    // before the samplers reach its step), then the most output rows per step
    static const int kPlans[][2] = {{6, 3}, {5, 3}, {6, 2}, {5, 2}, {4, 3}, {4, 2},
                                    {3, 3}, {3, 2}, {2, 3}, {2, 2}};
    for (const auto& plan : kPlans) {
        const int margin = plan[0], ns = plan[1];
        if (pad > margin + (kh - 1) * dil) continue;
        {
            if (ns > kFusedMaxStages || (uint32_t)ns * (uint32_t)NJ > 512u) continue;
            for (int th = std::min(4, std::min(128 / W, H)); th >= 1; --th) {
            // A stage: the step's th * W pixel rows, rounded to 64 or 128 (the
            // product reads 128 rows; rows past the tile only reach accumulator
            // lanes that are never read)
            const int a_rows_alloc = th * W <= 64 ? 64 : 128;
            const uint32_t a_bytes = (uint32_t)kchunks * (uint32_t)a_rows_alloc * 128u;
            const uint32_t om_bytes = (uint32_t)((th * W * om_stride * 4 + 15) / 16 * 16);
            const int band = dcnb::band_rows(th, 1, kh, dil, margin);
            const int band_in_map = std::min(band, H);
            long long ring = band + (long long)(ns - 1) * th;
            ring = std::min(ring, 2LL * H);
            ring = std::max<long long>(ring, band_in_map);
            // 1 KB of alignment slack, tiles, ring, om buffers, barriers
            // (2 per step in flight for the ring and 4 for the product, plus
            // the weight tile's), descriptors, the TMEM address and the bias
            const long long bytes = 1024 + w_bytes + (long long)ns * a_bytes + ring * row_bytes +
                                    (long long)ns * om_bytes + (6LL * ns + 1) * 8 +
                                    (long long)ns * dcnb::kBandDescInts * 4 + 16 + NJ * 4;
            const long long tx = band_in_map * row_bytes + (long long)kchunks * th * W * 128;
            if (bytes > kFusedSmemLimit || tx >= (1 << 20)) continue;
            uint32_t tmem_cols = 32;
            while (tmem_cols < (uint32_t)(ns * NJ)) tmem_cols <<= 1;
            dcnb::BandArgs& a = f->b;
            a.x = x;
            a.offset = nullptr;
            a.mask = nullptr;
            a.out = out;
            a.H = H;
            a.W = W;
            a.C = C;
            a.G = G;
            a.kh = kh;
            a.kw = kw;
            a.K = K;
            a.stride = 1;
            a.pad = pad;
            a.dil = dil;
            a.Ho = H;
            a.Wo = W;
            a.rows_total = N * H;
            a.th = th;
            a.margin = margin;
            a.ring_rows = (int)ring;
            a.consumer_warps = consumer_warps;
            a.stages = ns;
            a.runs_per_row = runs_per_row;
            a.row_bytes = (uint32_t)row_bytes;
            a.pix_bytes = (uint32_t)(C * es);
            a.off_row_bytes = 0;
            a.mask_row_bytes = 0;
            a.ring_bytes = (uint32_t)(ring * row_bytes);
            a.stage_bytes = 0;
            a.div_G = make_div((uint32_t)G);
            a.div_Ho = make_div((uint32_t)H);
            a.div_runs = make_div((uint32_t)runs_per_row);
            a.flags = nullptr;
            a.x_bytes = (long long)N * H * row_bytes;
            a.out_bytes = (long long)N * H * row_bytes;
            f->b_om = b_om;
            f->J = J;
            f->NJ = NJ;
            f->kchunks = kchunks;
            f->a_rows = th * W;
            f->consumer_warps = consumer_warps;
            f->tmem_cols = tmem_cols;
            f->a_bytes = a_bytes;
            f->a_box_bytes = (uint32_t)kchunks * (uint32_t)(th * W) * 128u;
            f->w_bytes = w_bytes;
            f->om_stride = om_stride;
            f->om_bytes = om_bytes;
            if (!encode_tmap_2d(&f->tmap_x, x, bf16, (uint64_t)C, (uint64_t)N * H * W,
                                (uint64_t)C * es, 64, (uint32_t)(th * W)) ||
                !encode_tmap_2d(&f->tmap_w, w_om, bf16, (uint64_t)C, (uint64_t)J,
                                (uint64_t)C * es, 64, (uint32_t)NJ))
                return false;
            *smem = (int)bytes;
            *threads = 32 * (consumer_warps + 2 + dcnb::kFusedEpilogueWarps);
            return true;
            }
        }
    }
    return false;
}

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

int dcnv4_fused_forward_algo(const void* x, const void* w_om, const void* b_om, void* out,
                             int N, int H, int W, int C, int G, int kh, int kw, int pad, int dil,
                             int dtype, int algo, void* stream) {
    const int es = elem_bytes(dtype);
    if (algo != DCN_ALGO_AUTO && algo != DCN_ALGO_GATHER && algo != DCN_ALGO_BAND)
        return DCN_ERR_INVALID_ARG;
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

    if (algo != DCN_ALGO_GATHER) {
        dcnb::BandFusedArgs f;
        int smem = 0, threads = 0;
        if (band_fused_config(x, w_om, b_om, out, N, H, W, C, G, kh, kw, pad, dil,
                              dtype == DCN_BF16, &f, &smem, &threads)) {
            f.b.flags = device_flags_word();
            const void* fn = dtype == DCN_F16 ? band_fused_kernel_for<__half>(kh, kw)
                                              : band_fused_kernel_for<__nv_bfloat16>(kh, kw);
            // one CTA per SM (the shared-memory footprint allows no more)
            return launch(fn, f, f.b.rows_total, threads, smem, stream);
        }
        if (algo == DCN_ALGO_BAND) return DCN_ERR_UNSUPPORTED;
    }

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
    a.flags = device_flags_word();
    a.x_bytes = img_bytes * N;
    a.out_bytes = img_bytes * N;

    const void* fn = nullptr;
    switch (dtype) {
        case DCN_F16: fn = dcn_fused_kernel_vb<__half>(vb, kh, kw); break;
        case DCN_BF16: fn = dcn_fused_kernel_vb<__nv_bfloat16>(vb, kh, kw); break;
        default: break;
    }
    if (!fn) return DCN_ERR_UNSUPPORTED;
    return launch(fn, a, a.num_tiles, 32 * warps, smem, stream);
}

int dcnv4_fused_forward(const void* x, const void* w_om, const void* b_om, void* out, int N,
                        int H, int W, int C, int G, int kh, int kw, int pad, int dil, int dtype,
                        void* stream) {
    return dcnv4_fused_forward_algo(x, w_om, b_om, out, N, H, W, C, G, kh, kw, pad, dil, dtype,
                                    DCN_ALGO_AUTO, stream);
}

}  // extern "C"
