// C interface of libdcn_b200.so: msda_forward, its reference-point variants
// (msda_forward_points) and msda_mask_value.
#include "abi_common.cuh"
#include "msda_fwd.cuh"

using namespace dcnb_abi;

namespace {

template <typename T, int REF>
const void* msda_kernel_ref(int vb) {
    using namespace dcnb;
    switch (vb) {
        case 32: return (const void*)msda_fwd_kernel<T, 32, REF>;
        case 16: return (const void*)msda_fwd_kernel<T, 16, REF>;
        case 8: return (const void*)msda_fwd_kernel<T, 8, REF>;
        case 4: return (const void*)msda_fwd_kernel<T, 4, REF>;
        default: break;
    }
    if constexpr (sizeof(T) == 2) {
        if (vb == 2) return (const void*)msda_fwd_kernel<T, 2, REF>;
    }
    return nullptr;
}

template <typename T>
const void* msda_kernel_vb(int vb, int ref_dim) {
    switch (ref_dim) {
        case 0: return msda_kernel_ref<T, 0>(vb);
        case 2: return msda_kernel_ref<T, 2>(vb);
        case 4: return msda_kernel_ref<T, 4>(vb);
        default: return nullptr;
    }
}

}  // namespace

extern "C" {

static int msda_launch(const void* value, const int64_t* spatial_shapes,
                       const int64_t* level_start, const void* sampling_loc, const void* attn_w,
                       void* out, int N, int Lq, int M, int D, int L, int K, int dtype,
                       void* stream, const void* ref, int ref_dim, const void* vr) {
    const int es = elem_bytes(dtype);
    if (es == 0 || N < 0 || Lq < 0 || M <= 0 || D <= 0 || L <= 0 || K <= 0)
        return DCN_ERR_INVALID_ARG;
    if (L > dcnb::kMsdaMaxLevels || K > 64) return DCN_ERR_UNSUPPORTED;
    const long long items = (long long)N * Lq * M;
    if (items > kInt31 || (long long)M * D * es > kInt31) return DCN_ERR_UNSUPPORTED;
    if (items == 0) return DCN_OK;
    if (!value || !spatial_shapes || !level_start || !sampling_loc || !attn_w || !out)
        return DCN_ERR_INVALID_ARG;
    if ((((uintptr_t)value | (uintptr_t)sampling_loc | (uintptr_t)attn_w | (uintptr_t)out) %
         es) != 0 ||
        (((uintptr_t)spatial_shapes | (uintptr_t)level_start) % 8) != 0)
        return DCN_ERR_MISALIGNED;
    const int LK = L * K;
    const long long o_bytes = items * D * es;
    if (overlaps(out, o_bytes, sampling_loc, items * LK * 2 * es) ||
        overlaps(out, o_bytes, attn_w, items * LK * es) ||
        overlaps(out, o_bytes, spatial_shapes, (long long)L * 16) ||
        overlaps(out, o_bytes, level_start, (long long)L * 8) ||
        (uintptr_t)out == (uintptr_t)value)
        return DCN_ERR_INVALID_ARG;
    if (ref_dim != 0) {
        if (!ref) return DCN_ERR_INVALID_ARG;
        if ((((uintptr_t)ref | (uintptr_t)vr) % es) != 0) return DCN_ERR_MISALIGNED;
        if (overlaps(out, o_bytes, ref, (long long)N * Lq * ref_dim * es) ||
            (vr && overlaps(out, o_bytes, vr, (long long)N * L * 2 * es)))
            return DCN_ERR_INVALID_ARG;
    }

    const int vb = pick_vector_bytes(es, D, (uintptr_t)value | (uintptr_t)out);
    if (vb == 0) return DCN_ERR_MISALIGNED;
    const int cpt = vb / es;
    const int tpi = D / cpt;
    if (tpi > 32) return DCN_ERR_UNSUPPORTED;   // one item must fit in a warp
    const int run_items = 32 / tpi;
    // per-warp shared slice for the run's locations and weights; unstaged when
    // the CTA's slices would not fit in the default shared-memory window
    int stage_elems = run_items * LK;
    const int loc_stride = staged_row_stride(run_items, LK * 2, 2, es);
    const int w_stride = staged_row_stride(run_items, LK, 1, es);
    const int slice = run_items * (loc_stride + w_stride) * es;
    int smem = slice * dcnb::kMsdaWarps;
    if (smem > kMaxStageBytes) {
        stage_elems = 0;
        smem = 0;
    }

    dcnb::MsdaArgs a;
    a.value = value;
    a.shapes = spatial_shapes;
    a.level_start = level_start;
    a.loc = sampling_loc;
    a.attn = attn_w;
    a.out = out;
    a.Lq = Lq;
    a.M = M;
    a.D = D;
    a.L = L;
    a.K = K;
    a.tpi = tpi;
    a.run_items = run_items;
    a.total_items = (int)items;
    a.num_runs = (int)((items + run_items - 1) / run_items);
    a.stage_elems = stage_elems;
    a.loc_stride = loc_stride;
    a.w_stride = w_stride;
    a.div_M = make_div((uint32_t)M);
    a.div_Lq = make_div((uint32_t)Lq);
    a.div_tpi = make_div((uint32_t)tpi);
    a.ref = ref;
    a.vr = vr;
    a.flags = device_flags_word();

    const void* fn = nullptr;
    switch (dtype) {
        case DCN_F32: fn = msda_kernel_vb<float>(vb, ref_dim); break;
        case DCN_F16: fn = msda_kernel_vb<__half>(vb, ref_dim); break;
        case DCN_BF16: fn = msda_kernel_vb<__nv_bfloat16>(vb, ref_dim); break;
        default: break;
    }
    if (!fn) return DCN_ERR_UNSUPPORTED;
    // one unit of work per warp: a CTA's warps share its range of runs
    const int num_ctas = (a.num_runs + dcnb::kMsdaWarps - 1) / dcnb::kMsdaWarps;
    return launch(fn, a, num_ctas, dcnb::kMsdaThreads, smem, stream);
}

int msda_forward(const void* value, const int64_t* spatial_shapes, const int64_t* level_start,
                 const void* sampling_loc, const void* attn_w, void* out, int N, int Lq, int M,
                 int D, int L, int K, int dtype, void* stream) {
    return msda_launch(value, spatial_shapes, level_start, sampling_loc, attn_w, out, N, Lq, M,
                       D, L, K, dtype, stream, nullptr, 0, nullptr);
}

int msda_forward_points(const void* value, const int64_t* spatial_shapes,
                        const int64_t* level_start, const void* reference, int ref_dim,
                        const void* valid_ratios, const void* offsets, const void* attn_w,
                        void* out, int N, int Lq, int M, int D, int L, int K, int dtype,
                        void* stream) {
    if (ref_dim != 2 && ref_dim != 4) return DCN_ERR_INVALID_ARG;
    return msda_launch(value, spatial_shapes, level_start, offsets, attn_w, out, N, Lq, M, D, L,
                       K, dtype, stream, reference, ref_dim, valid_ratios);
}

int msda_mask_value(const void* value, const unsigned char* mask, void* out, int N, int S,
                    int M, int D, int dtype, void* stream) {
    const int es = elem_bytes(dtype);
    if (es == 0 || N < 0 || S <= 0 || M <= 0 || D <= 0) return DCN_ERR_INVALID_ARG;
    const long long row_bytes = (long long)M * D * es;
    if (row_bytes > kInt31 || (long long)N * S > kInt31) return DCN_ERR_UNSUPPORTED;
    if (N == 0) return DCN_OK;
    if (!value || !mask || !out) return DCN_ERR_INVALID_ARG;
    if ((((uintptr_t)value | (uintptr_t)out) % es) != 0) return DCN_ERR_MISALIGNED;
    const long long bytes = row_bytes * N * S;
    if ((out != value && overlaps(out, bytes, value, bytes)) ||
        overlaps(out, bytes, mask, (long long)N * S))
        return DCN_ERR_INVALID_ARG;
    dcnb::MaskArgs m;
    m.value = value;
    m.mask = mask;
    m.out = out;
    m.rows = (long long)N * S;
    m.row_bytes = (int)row_bytes;
    m.vec16 = ((((uintptr_t)value | (uintptr_t)out) % 16) == 0 && row_bytes % 16 == 0) ? 1 : 0;
    const long long units = m.vec16 ? bytes / 16 : bytes;
    const long long blocks = (units + 255) / 256;
    return launch((const void*)dcnb::msda_mask_value_kernel, m,
                  (int)std::min(blocks, 1LL << 20), 256, 0, stream);
}

}  // extern "C"
