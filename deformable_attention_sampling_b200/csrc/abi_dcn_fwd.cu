// C interface of libdcn_b200.so: dcn_forward and dcn_forward_algo (argument
// checks, choice between the two forward kernels, launch shape, dispatch), and
// dcn_forward_plan (the same choice and launch shape, on the host only).
//
// Two kernels compute the same operator:
//   - the band kernel (dcn_band.cuh): input rows staged in shared memory by
//     bulk copies, conflict-free corner reads; 16-bit data, 16 channels per
//     group, pixels of a multiple of 128 bytes, 16-byte aligned tensors and
//     rows, and a band of rows that fits in shared memory;
//   - the gather kernel (dcn_fwd.cuh): corners read through L1; every shape.
// DCN_ALGO_AUTO takes the band kernel where it applies.
#include "abi_common.cuh"
#include "dcn_band.cuh"
#include "dcn_fwd.cuh"

using namespace dcnb_abi;

namespace {

constexpr int kBandMarginRows = 6;     // offset margin of the band, at most
constexpr int kBandMinMarginRows = 2;
constexpr int kBandSmemLimit = 227 * 1024;
constexpr int kBandTargetItems = 14 * 32;   // items per step
#ifndef DCN_BAND_STAGES
#define DCN_BAND_STAGES 2
#endif
constexpr int kBandStepsInFlight = DCN_BAND_STAGES;   // 2 .. dcnb::kBandMaxStages
static_assert(kBandStepsInFlight >= 2 && kBandStepsInFlight <= dcnb::kBandMaxStages, "stages");

template <typename T>
const void* band_kernel_for(int softmax, int kh, int kw) {
    using namespace dcnb;
    if (kh == 3 && kw == 3)
        return softmax ? (const void*)dcn_band_kernel<T, true, 3>
                       : (const void*)dcn_band_kernel<T, false, 3>;
    return softmax ? (const void*)dcn_band_kernel<T, true, 0>
                   : (const void*)dcn_band_kernel<T, false, 0>;
}

// Launch shape of the band kernel for a problem shape (tensors taken to be
// 16-byte aligned), or false when the shape does not qualify.  Host only.
struct BandPlan {
    int th;              // output rows per step
    int margin;          // offset margin of the band, rows above and below
    int ring;            // input rows in the shared-memory ring
    int warps;           // sampler warps (one more warp produces)
    int runs_per_row;    // warp runs per output row
    long long row_bytes, off_row, mask_row, stage, smem;
};

bool band_plan(int H, int W, int C, int G, int kh, int kw, int stride, int pad, int dil,
               int Ho, int Wo, int es, BandPlan* p) {
    const int D = C / G;
    const int K = kh * kw;
    if (es != 2 || D != 16 || (C * es) % 128 != 0) return false;
    const long long row_bytes = (long long)W * C * es;
    const long long off_row = (long long)Wo * G * K * 2 * es;
    const long long mask_row = (long long)Wo * G * K * es;
    if (off_row % 16 != 0 || mask_row % 16 != 0) return false;
    const long long row_items = (long long)Wo * G;
    const int run_items = 32 / dcnb::kBandLanesPerItem;
    const int runs_per_row = (int)((row_items + run_items - 1) / run_items);
    int th = (int)((kBandTargetItems + row_items - 1) / row_items);
    th = std::max(1, std::min(th, std::min(4, Ho)));
    // runs are dealt to the sampler warps round-robin over the CTA's whole
    // range, so two warps more than a step's runs start on the next step while
    // the others finish this one (measured at N = 64, 56 x 56, C = 64, G = 4:
    // 71.0 us with 16 warps, 71.9 with 15, 73.9 with 14; 17 and 18 spill)
    const int warps = std::min(dcnb::kBandMaxConsumerWarps, th * runs_per_row + 2);
    const long long stage = (th * (off_row + mask_row) + 127) / 128 * 128;
    for (int margin = kBandMarginRows; margin >= kBandMinMarginRows; --margin) {
        if (pad > margin + (kh - 1) * dil) break;   // every band must meet the map
        const int band = dcnb::band_rows(th, stride, kh, dil, margin);
        const int band_in_map = std::min(band, H);
        long long ring = band + (long long)(kBandStepsInFlight - 1) * th * stride;
        ring = std::min(ring, 2LL * H);
        ring = std::max<long long>(ring, band_in_map);
        const long long bytes = ring * row_bytes + kBandStepsInFlight * stage +
                                kBandStepsInFlight * 16 +
                                kBandStepsInFlight * dcnb::kBandDescInts * 4;
        // one step's copies must fit in an mbarrier transaction count
        if (bytes > kBandSmemLimit || band_in_map * row_bytes + stage >= (1 << 20)) continue;
        p->th = th;
        p->margin = margin;
        p->ring = (int)ring;
        p->warps = warps;
        p->runs_per_row = runs_per_row;
        p->row_bytes = row_bytes;
        p->off_row = off_row;
        p->mask_row = mask_row;
        p->stage = stage;
        p->smem = bytes;
        return true;
    }
    return false;
}

// Launch configuration of the band kernel for this call, or false when the
// shape or the pointers do not qualify.
bool band_config(const void* x, const void* offset, const void* mask, void* out, int N, int H,
                 int W, int C, int G, int kh, int kw, int stride, int pad, int dil, int Ho,
                 int Wo, int es, dcnb::BandArgs* a, int* smem, int* threads) {
    if ((((uintptr_t)x | (uintptr_t)offset | (uintptr_t)mask | (uintptr_t)out) % 16) != 0)
        return false;
    BandPlan p;
    if (!band_plan(H, W, C, G, kh, kw, stride, pad, dil, Ho, Wo, es, &p)) return false;
    a->x = x;
    a->offset = offset;
    a->mask = mask;
    a->out = out;
    a->H = H;
    a->W = W;
    a->C = C;
    a->G = G;
    a->kh = kh;
    a->kw = kw;
    a->K = kh * kw;
    a->stride = stride;
    a->pad = pad;
    a->dil = dil;
    a->Ho = Ho;
    a->Wo = Wo;
    a->rows_total = N * Ho;
    a->th = p.th;
    a->margin = p.margin;
    a->ring_rows = p.ring;
    a->consumer_warps = p.warps;
    a->stages = kBandStepsInFlight;
    a->runs_per_row = p.runs_per_row;
    a->row_bytes = (uint32_t)p.row_bytes;
    a->pix_bytes = (uint32_t)(C * es);
    a->off_row_bytes = (uint32_t)p.off_row;
    a->mask_row_bytes = (uint32_t)p.mask_row;
    a->ring_bytes = (uint32_t)(p.ring * p.row_bytes);
    a->stage_bytes = (uint32_t)p.stage;
    a->div_G = make_div((uint32_t)G);
    a->div_Ho = make_div((uint32_t)Ho);
    a->div_runs = make_div((uint32_t)p.runs_per_row);
    a->flags = device_flags_word();
    a->x_bytes = (long long)N * H * p.row_bytes;
    a->out_bytes = (long long)N * Ho * Wo * C * es;
    *smem = (int)p.smem;
    *threads = 32 * (p.warps + 1);
    return true;
}

// Argument checks shared by dcn_forward_algo and dcn_forward_plan (shapes,
// flags, dtype, algo, size limits); the output size on DCN_OK.
int check_dcn_shape(int N, int H, int W, int C, int G, int kh, int kw, int stride, int pad,
                    int dil, int softmax_flag, int dtype, int algo, int* Ho_out, int* Wo_out) {
    const int es = elem_bytes(dtype);
    if (algo != DCN_ALGO_AUTO && algo != DCN_ALGO_GATHER && algo != DCN_ALGO_BAND)
        return DCN_ERR_INVALID_ARG;
    if (es == 0 || N < 0 || H <= 0 || W <= 0 || C <= 0 || G <= 0 || C % G != 0 || kh <= 0 ||
        kw <= 0 || stride <= 0 || pad < 0 || dil <= 0 || (softmax_flag != 0 && softmax_flag != 1))
        return DCN_ERR_INVALID_ARG;
    if (H > kMaxDim || W > kMaxDim || pad > kMaxDim || stride > kMaxDim || dil > kMaxDim ||
        kh > kMaxDim || kw > kMaxDim || (long long)kh * kw > kMaxTaps)
        return DCN_ERR_UNSUPPORTED;
    const int Ho = dcn_output_size(H, kh, stride, pad, dil);
    const int Wo = dcn_output_size(W, kw, stride, pad, dil);
    if (Ho <= 0 || Wo <= 0) return DCN_ERR_INVALID_ARG;
    const long long img_bytes = (long long)H * W * C * es;
    const long long out_img_bytes = (long long)Ho * Wo * C * es;
    const long long items = (long long)N * Ho * Wo * G;
    if (img_bytes > kInt31 || out_img_bytes > kInt31 || items > kInt31 ||
        (long long)N * Ho * Wo > kInt31)
        return DCN_ERR_UNSUPPORTED;
    *Ho_out = Ho;
    *Wo_out = Wo;
    return DCN_OK;
}

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

int dcn_forward_algo(const void* x, const void* offset, const void* mask, void* out, int N,
                     int H, int W, int C, int G, int kh, int kw, int stride, int pad, int dil,
                     int softmax_flag, int dtype, int algo, void* stream) {
    int Ho = 0, Wo = 0;
    const int rc = check_dcn_shape(N, H, W, C, G, kh, kw, stride, pad, dil, softmax_flag, dtype,
                                   algo, &Ho, &Wo);
    if (rc != DCN_OK) return rc;
    const int es = elem_bytes(dtype);
    const int D = C / G;
    const int K = kh * kw;
    const long long img_bytes = (long long)H * W * C * es;
    const long long out_img_bytes = (long long)Ho * Wo * C * es;
    const long long items = (long long)N * Ho * Wo * G;
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

    if (algo != DCN_ALGO_GATHER) {
        dcnb::BandArgs b;
        int smem = 0, threads = 0;
        if (band_config(x, offset, mask, out, N, H, W, C, G, kh, kw, stride, pad, dil, Ho, Wo,
                        es, &b, &smem, &threads)) {
            const void* fn = dtype == DCN_F16 ? band_kernel_for<__half>(softmax_flag, kh, kw)
                                              : band_kernel_for<__nv_bfloat16>(softmax_flag, kh, kw);
            // one CTA per SM, each a contiguous range of output rows
            return launch(fn, b, b.rows_total, threads, smem, stream);
        }
        if (algo == DCN_ALGO_BAND) return DCN_ERR_UNSUPPORTED;
    }

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
    a.flags = device_flags_word();
    a.x_bytes = img_bytes * N;
    a.out_bytes = out_img_bytes * N;

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

int dcn_forward_plan(int N, int H, int W, int C, int G, int kh, int kw, int stride, int pad,
                     int dil, int softmax_flag, int dtype, int algo, int* plan) {
    if (!plan) return DCN_ERR_INVALID_ARG;
    int Ho = 0, Wo = 0;
    const int rc = check_dcn_shape(N, H, W, C, G, kh, kw, stride, pad, dil, softmax_flag, dtype,
                                   algo, &Ho, &Wo);
    if (rc != DCN_OK) return rc;
    const int es = elem_bytes(dtype);
    int out[8] = {0, 0, 0, 0, 0, 0, 0, 0};
    BandPlan p;
    if (algo != DCN_ALGO_GATHER &&
        band_plan(H, W, C, G, kh, kw, stride, pad, dil, Ho, Wo, es, &p)) {
        out[0] = DCN_ALGO_BAND;
        out[1] = p.th;
        out[2] = p.margin;
        out[3] = p.ring;
        out[4] = p.warps;
        out[5] = kBandStepsInFlight;
        out[6] = p.runs_per_row;
        out[7] = (int)p.smem;
    } else {
        if (algo == DCN_ALGO_BAND) return DCN_ERR_UNSUPPORTED;
        const int D = C / G;
        const int vb = pick_vector_bytes(es, D, 0);
        if (vb == 0 || D / (vb / es) > 32) return DCN_ERR_UNSUPPORTED;
        out[0] = DCN_ALGO_GATHER;
    }
    if (N == 0) out[0] = DCN_ALGO_AUTO;   // nothing is launched
    for (int i = 0; i < 8; ++i) plan[i] = out[i];
    return DCN_OK;
}

int dcn_forward(const void* x, const void* offset, const void* mask, void* out, int N, int H,
                int W, int C, int G, int kh, int kw, int stride, int pad, int dil,
                int softmax_flag, int dtype, void* stream) {
    return dcn_forward_algo(x, offset, mask, out, N, H, W, C, G, kh, kw, stride, pad, dil,
                            softmax_flag, dtype, DCN_ALGO_AUTO, stream);
}


}  // extern "C"
