// C interface of libdcn_b200.so (declared in include/dcn.h): argument
// validation, launch-shape choice and dispatch to the sm_100a kernels.
//
// Nothing here allocates or synchronises; every launch goes to the caller's
// stream.  Errors are reported as dcn_status_t values and never as exceptions.
#include <cuda_runtime.h>

#include <atomic>
#include <mutex>

#include "dcn.h"
#include "dcn_fwd.cuh"
#include "msda_fwd.cuh"

namespace {

using dcnb::FastDiv;

std::atomic<unsigned long long> g_launches{0};
thread_local int g_last_cuda_error = 0;

constexpr int kMaxDim = 65536;        // H, W, pad, stride, dil
constexpr int kMaxTaps = 1024;        // kh * kw
constexpr int kMaxStageBytes = 48 * 1024;
constexpr long long kInt31 = 2147483647LL;

FastDiv make_div(uint32_t d) {
    uint32_t shift = 0;
    while ((1ull << shift) < d) ++shift;
    const unsigned long long mul = ((1ull << 32) * ((1ull << shift) - d)) / d + 1;
    return FastDiv{d, (uint32_t)mul, shift};
}

int elem_bytes(int dtype) {
    switch (dtype) {
        case DCN_F32: return 4;
        case DCN_F16: return 2;
        case DCN_BF16: return 2;
        default: return 0;
    }
}

// Widest per-thread vector (bytes) that divides one group's channel span and
// keeps every thread's address aligned for the given base pointers.
int pick_vector_bytes(int es, int D, uintptr_t bases) {
    const int span = D * es;
    for (int vb = 32; vb >= es; vb >>= 1) {
        if (span % vb == 0 && (bases % (uintptr_t)vb) == 0) return vb;
    }
    return 0;
}

bool overlaps(const void* a, long long abytes, const void* b, long long bbytes) {
    const uintptr_t a0 = (uintptr_t)a, b0 = (uintptr_t)b;
    return a0 < b0 + (uintptr_t)bbytes && b0 < a0 + (uintptr_t)abytes;
}

// Grid size: one resident wave of CTAs (SM count x CTAs per SM), or fewer
// when there are fewer blocks; each CTA then strides over the blocks.
struct GridCacheEntry {
    const void* fn;
    int device;
    int smem;
    int ctas_per_sm;
    int sms;
};
std::mutex g_grid_mutex;
GridCacheEntry g_grid_cache[64];
int g_grid_cache_n = 0;

int wave_size(const void* fn, int threads, int smem) {
    int device = 0;
    if (cudaGetDevice(&device) != cudaSuccess) return 0;
    {
        std::lock_guard<std::mutex> lock(g_grid_mutex);
        for (int i = 0; i < g_grid_cache_n; ++i) {
            const GridCacheEntry& e = g_grid_cache[i];
            if (e.fn == fn && e.device == device && e.smem == smem) return e.ctas_per_sm * e.sms;
        }
    }
    int sms = 0, per_sm = 0;
    if (cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, device) != cudaSuccess)
        return 0;
    if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, fn, threads, smem) != cudaSuccess)
        return 0;
    if (per_sm < 1) per_sm = 1;
    std::lock_guard<std::mutex> lock(g_grid_mutex);
    if (g_grid_cache_n < 64) g_grid_cache[g_grid_cache_n++] = {fn, device, smem, per_sm, sms};
    return per_sm * sms;
}

template <typename Args>
int launch(const void* fn, const Args& args, int num_blocks, int threads, int smem,
           void* stream) {
    const int wave = wave_size(fn, threads, smem);
    if (wave <= 0) {
        g_last_cuda_error = (int)cudaGetLastError();
        return DCN_ERR_CUDA;
    }
    const int grid = num_blocks < wave ? num_blocks : wave;
    void* params[] = {const_cast<Args*>(&args)};
    const cudaError_t err = cudaLaunchKernel(fn, dim3(grid), dim3(threads), params,
                                             (size_t)smem, (cudaStream_t)stream);
    if (err != cudaSuccess) {
        g_last_cuda_error = (int)err;
        (void)cudaGetLastError();   // clear the launch error we just reported
        return DCN_ERR_CUDA;
    }
    g_launches.fetch_add(1, std::memory_order_relaxed);
    return DCN_OK;
}

// ---------------------------------------------------------------- DCN ------

template <typename T, int VB>
const void* dcn_kernel_for(int kh, int kw, int softmax) {
    using namespace dcnb;
    if (kh == 3 && kw == 3) {
        return softmax ? (const void*)dcn_fwd_kernel<T, VB, 3, 3, true>
                       : (const void*)dcn_fwd_kernel<T, VB, 3, 3, false>;
    }
    return softmax ? (const void*)dcn_fwd_kernel<T, VB, 0, 0, true>
                   : (const void*)dcn_fwd_kernel<T, VB, 0, 0, false>;
}

template <typename T>
const void* dcn_kernel_vb(int vb, int kh, int kw, int softmax) {
    switch (vb) {
        case 32: return dcn_kernel_for<T, 32>(kh, kw, softmax);
        case 16: return dcn_kernel_for<T, 16>(kh, kw, softmax);
        case 8: return dcn_kernel_for<T, 8>(kh, kw, softmax);
        case 4: return dcn_kernel_for<T, 4>(kh, kw, softmax);
        default: break;
    }
    if constexpr (sizeof(T) == 2) {
        if (vb == 2) return dcn_kernel_for<T, 2>(kh, kw, softmax);
    }
    return nullptr;
}

// ---------------------------------------------------------------- MSDA -----

template <typename T>
const void* msda_kernel_vb(int vb) {
    using namespace dcnb;
    switch (vb) {
        case 32: return (const void*)msda_fwd_kernel<T, 32>;
        case 16: return (const void*)msda_fwd_kernel<T, 16>;
        case 8: return (const void*)msda_fwd_kernel<T, 8>;
        case 4: return (const void*)msda_fwd_kernel<T, 4>;
        default: break;
    }
    if constexpr (sizeof(T) == 2) {
        if (vb == 2) return (const void*)msda_fwd_kernel<T, 2>;
    }
    return nullptr;
}

}  // namespace

extern "C" {

int dcn_output_size(int in, int k, int stride, int pad, int dil) {
    if (in <= 0 || k <= 0 || stride <= 0 || pad < 0 || dil <= 0) return 0;
    const long long span = (long long)in + 2LL * pad - (long long)dil * (k - 1) - 1;
    if (span < 0) return 0;
    return (int)(span / stride + 1);
}

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
    if (tpi > dcnb::kDcnThreads) return DCN_ERR_UNSUPPORTED;
    int items_per_cta = dcnb::kDcnThreads / tpi;
    const int per_item_stage = K * 3 * es;
    if (items_per_cta * per_item_stage + 32 > kMaxStageBytes)
        items_per_cta = (kMaxStageBytes - 32) / per_item_stage;
    if (items_per_cta < 1) return DCN_ERR_UNSUPPORTED;
    const int smem = ((items_per_cta * K * 2 * es + 15) & ~15) + items_per_cta * K * es;

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
    a.items_per_cta = items_per_cta;
    a.total_items = (int)items;
    a.num_blocks = (int)((items + items_per_cta - 1) / items_per_cta);
    a.div_G = make_div((uint32_t)G);
    a.div_Wo = make_div((uint32_t)Wo);
    a.div_Ho = make_div((uint32_t)Ho);
    a.div_tpi = make_div((uint32_t)tpi);
    a.pix_bytes = (uint32_t)(C * es);
    a.row_bytes = (uint32_t)((long long)W * C * es);
    a.img_bytes = img_bytes;

    const void* fn = nullptr;
    switch (dtype) {
        case DCN_F32: fn = dcn_kernel_vb<float>(vb, kh, kw, softmax_flag); break;
        case DCN_F16: fn = dcn_kernel_vb<__half>(vb, kh, kw, softmax_flag); break;
        case DCN_BF16: fn = dcn_kernel_vb<__nv_bfloat16>(vb, kh, kw, softmax_flag); break;
        default: break;
    }
    if (!fn) return DCN_ERR_UNSUPPORTED;
    return launch(fn, a, a.num_blocks, dcnb::kDcnThreads, smem, stream);
}

int msda_forward(const void* value, const int64_t* spatial_shapes, const int64_t* level_start,
                 const void* sampling_loc, const void* attn_w, void* out, int N, int Lq, int M,
                 int D, int L, int K, int dtype, void* stream) {
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

    const int vb = pick_vector_bytes(es, D, (uintptr_t)value | (uintptr_t)out);
    if (vb == 0) return DCN_ERR_MISALIGNED;
    const int cpt = vb / es;
    const int tpi = D / cpt;
    if (tpi > dcnb::kMsdaThreads) return DCN_ERR_UNSUPPORTED;
    int items_per_cta = dcnb::kMsdaThreads / tpi;
    const int per_item_stage = LK * 3 * es;
    if (items_per_cta * per_item_stage + 32 > kMaxStageBytes)
        items_per_cta = (kMaxStageBytes - 32) / per_item_stage;
    if (items_per_cta < 1) return DCN_ERR_UNSUPPORTED;
    const int smem = ((items_per_cta * LK * 2 * es + 15) & ~15) + items_per_cta * LK * es;

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
    a.items_per_cta = items_per_cta;
    a.total_items = (int)items;
    a.num_blocks = (int)((items + items_per_cta - 1) / items_per_cta);
    a.div_M = make_div((uint32_t)M);
    a.div_Lq = make_div((uint32_t)Lq);
    a.div_tpi = make_div((uint32_t)tpi);

    const void* fn = nullptr;
    switch (dtype) {
        case DCN_F32: fn = msda_kernel_vb<float>(vb); break;
        case DCN_F16: fn = msda_kernel_vb<__half>(vb); break;
        case DCN_BF16: fn = msda_kernel_vb<__nv_bfloat16>(vb); break;
        default: break;
    }
    if (!fn) return DCN_ERR_UNSUPPORTED;
    return launch(fn, a, a.num_blocks, dcnb::kMsdaThreads, smem, stream);
}

const char* dcn_status_string(int status) {
    switch (status) {
        case DCN_OK: return "ok";
        case DCN_ERR_INVALID_ARG: return "invalid argument";
        case DCN_ERR_UNSUPPORTED: return "unsupported shape or size";
        case DCN_ERR_MISALIGNED: return "misaligned pointer";
        case DCN_ERR_CUDA: return "CUDA launch failed";
        default: return "unknown status";
    }
}

int dcn_last_cuda_error(void) { return g_last_cuda_error; }

uint64_t dcn_launch_count(void) { return g_launches.load(std::memory_order_relaxed); }

int dcn_version(void) { return 10000; }

}  // extern "C"
