// C interface of libdcn_b200.so (declared in include/dcn.h): argument
// validation, launch-shape choice and dispatch to the sm_100a kernels.
//
// Nothing here allocates or synchronises; every launch goes to the caller's
// stream.  Errors are reported as dcn_status_t values and never as exceptions.
#include <cuda_runtime.h>

#include <algorithm>
#include <atomic>
#include <cmath>
#include <mutex>

#include "dcn.h"
#include "dcn_bwd.cuh"
#include "dcn_fwd.cuh"
#include "dynconv_fwd.cuh"
#include "msda_bwd.cuh"
#include "msda_fwd.cuh"

namespace {

using dcnb::FastDiv;

std::atomic<unsigned long long> g_launches{0};
thread_local int g_last_cuda_error = 0;

constexpr int kMaxDim = 65536;        // H, W, pad, stride, dil
constexpr int kMaxTaps = 1024;        // kh * kw
constexpr int kMaxStageBytes = 48 * 1024;
constexpr int kMaxBwdSliceBytes = 200 * 1024;   // shared slice of one backward warp
constexpr int kMaxBwdSmemBytes = 220 * 1024;    // of one backward CTA (opt-in size)
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
// when there are fewer work units; each CTA then takes a contiguous share.
//
// The first time a kernel runs on a device with a given shared-memory size,
// its preferred shared-memory carveout is set to what its resident CTAs need
// (the rest of the SM's 256 KB array stays L1, which the gathers live in);
// the carveout of a kernel only ever grows, so no earlier configuration loses
// occupancy.
struct GridCacheEntry {
    const void* fn;
    int device;
    int threads;
    int smem;
    int ctas_per_sm;
    int sms;
    int carveout;
};
std::mutex g_grid_mutex;
GridCacheEntry g_grid_cache[64];
int g_grid_cache_n = 0;

int wave_size(const void* fn, int threads, int smem) {
    int device = 0;
    if (cudaGetDevice(&device) != cudaSuccess) return 0;
    std::lock_guard<std::mutex> lock(g_grid_mutex);
    int carve_set = -1;
    for (int i = 0; i < g_grid_cache_n; ++i) {
        const GridCacheEntry& e = g_grid_cache[i];
        if (e.fn == fn && e.device == device) {
            if (e.smem == smem && e.threads == threads) return e.ctas_per_sm * e.sms;
            if (e.carveout > carve_set) carve_set = e.carveout;
        }
    }
    int sms = 0, smem_sm = 0, per_sm = 0;
    if (cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, device) != cudaSuccess ||
        cudaDeviceGetAttribute(&smem_sm, cudaDevAttrMaxSharedMemoryPerMultiprocessor, device) !=
            cudaSuccess)
        return 0;
    if (smem > 48 * 1024) {
        // beyond the default window: opt in (the limit of a function only grows)
        cudaFuncAttributes attr;
        if (cudaFuncGetAttributes(&attr, fn) != cudaSuccess) return 0;
        if (attr.maxDynamicSharedSizeBytes < smem &&
            cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize, smem) !=
                cudaSuccess)
            return 0;
    }
    if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, fn, threads, smem) != cudaSuccess)
        return 0;
    if (per_sm < 1) per_sm = 1;
    // shared memory the resident CTAs need (1 KB per CTA is reserved by the system)
    const long long need = (long long)per_sm * (smem + 1024);
    int carve = smem_sm > 0 ? (int)((need * 100 + smem_sm - 1) / smem_sm) : -1;
    if (carve > 100) carve = 100;
    if (carve < carve_set) carve = carve_set;
    if (carve >= 0 &&
        cudaFuncSetAttribute(fn, cudaFuncAttributePreferredSharedMemoryCarveout, carve) ==
            cudaSuccess) {
        int per_sm2 = 0;
        if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm2, fn, threads, smem) !=
                cudaSuccess || per_sm2 < per_sm) {
            (void)cudaGetLastError();
            (void)cudaFuncSetAttribute(fn, cudaFuncAttributePreferredSharedMemoryCarveout,
                                       cudaSharedmemCarveoutDefault);
            carve = -1;
        }
    } else {
        (void)cudaGetLastError();
        carve = -1;
    }
    if (g_grid_cache_n < 64)
        g_grid_cache[g_grid_cache_n++] = {fn, device, threads, smem, per_sm, sms, carve};
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

// One CTA per work unit (no persistent loop): the grid is the unit count.
template <typename Args>
int launch_grid(const void* fn, const Args& args, int num_blocks, int threads, int smem,
                void* stream) {
    if (wave_size(fn, threads, smem) <= 0) {   // sets the shared-memory attributes
        g_last_cuda_error = (int)cudaGetLastError();
        return DCN_ERR_CUDA;
    }
    void* params[] = {const_cast<Args*>(&args)};
    const cudaError_t err = cudaLaunchKernel(fn, dim3(num_blocks), dim3(threads), params,
                                             (size_t)smem, (cudaStream_t)stream);
    if (err != cudaSuccess) {
        g_last_cuda_error = (int)err;
        (void)cudaGetLastError();
        return DCN_ERR_CUDA;
    }
    g_launches.fetch_add(1, std::memory_order_relaxed);
    return DCN_OK;
}

// ---------------------------------------------------------------- DCN ------

// Tile shape of the DCN kernel: tile_h output rows x tile_w warp runs, one
// warp per run, at most kDcnMaxWarps warps per CTA.  A CTA sweeps its tiles
// along the row, so its L1 footprint is its band's input rows (tile rows plus
// the window and offset halo) times a sliding column window; the SM's L1 only
// holds the footprint of about one such band.  The choice minimises the
// product of
//   - padded work      (rows and runs beyond the map in the last tiles),
//   - vertical overfetch ((tile_h + halo) / tile_h input rows per output row),
//   - the tail         (the last wave of tiles only partly fills the SMs),
//   - latency exposure (fewer resident warps cover less gather latency).
// On small maps (at most kSmallMapRows output rows) a band of the image fits
// in L1 whatever the tile, and measured time is set by resident warps: there
// tiles are capped at 8 warps so that three CTAs share an SM.  On larger maps
// L1 reuse dominates and tiles grow up to kDcnMaxWarps rows (one CTA per SM).
struct TileShape {
    int h, w;
};

constexpr int kSmallMapRows = 64;

// `cap` is the kernel's warp limit per CTA and `warps_by_regs` the warps one
// SM holds at the kernel's register count.
TileShape choose_tile(int N, int Ho, int runs, int kernel_extent, int sms,
                      int cap = dcnb::kDcnMaxWarps, int warps_by_regs = 25) {
    const int kWarpsPerSmByRegs = warps_by_regs;   // forward: 80 registers per thread
    const int max_warps = Ho <= kSmallMapRows ? (cap < 8 ? cap : 8) : cap;
    const double halo = kernel_extent + 2.0 * dcnb::kPrefetchMargin;
    TileShape best{1, 1};
    double best_cost = 1e300;
    for (int h = 1; h <= max_warps && h <= Ho; ++h) {
        for (int w = 1; h * w <= max_warps && w <= runs; ++w) {
            const int warps = h * w;
            if (warps < 8 && warps < Ho * runs && warps < max_warps) continue;
            const long long bands = (Ho + h - 1) / h, tx = (runs + w - 1) / w;
            const double pad_work = (double)(bands * h * tx * w) / ((double)Ho * runs);
            const double overfetch = (h + halo) / h;
            int ctas = kWarpsPerSmByRegs / warps;
            if (ctas < 1) ctas = 1;
            const double per_slot = (double)N * bands * tx / ((double)sms * ctas);
            const double tail = (per_slot < 1.0 ? 1.0 : std::ceil(per_slot)) / per_slot;
            const int resident = warps * ctas < 24 ? warps * ctas : 24;
            const double latency = 1.0 + 8.0 / resident;
            const double cost = pad_work * overfetch * tail * latency;
            if (cost < best_cost) {
                best_cost = cost;
                best = TileShape{h, w};
            }
        }
    }
    return best;
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

// ---------------------------------------------------------------- MSDA -----

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

// ------------------------------------------------------------ backward ---

template <typename T, int VB, bool PAIR = false>
const void* dcn_bwd_kernel_for(int softmax, int kh, int kw) {
    using namespace dcnb;
    if (kh == 3 && kw == 3)
        return softmax ? (const void*)dcn_bwd_kernel<T, VB, true, 3, PAIR>
                       : (const void*)dcn_bwd_kernel<T, VB, false, 3, PAIR>;
    return softmax ? (const void*)dcn_bwd_kernel<T, VB, true, 0, PAIR>
                   : (const void*)dcn_bwd_kernel<T, VB, false, 0, PAIR>;
}

template <typename T>
const void* dcn_bwd_kernel_vb(int vb, int kh, int kw, int softmax, int pair) {
    if (pair) {   // 8 channels per lane
        if (vb == 8 * (int)sizeof(T))
            return dcn_bwd_kernel_for<T, 8 * sizeof(T), true>(softmax, kh, kw);
        return nullptr;
    }
    switch (vb) {
        case 32: return dcn_bwd_kernel_for<T, 32>(softmax, kh, kw);
        case 16: return dcn_bwd_kernel_for<T, 16>(softmax, kh, kw);
        case 8: return dcn_bwd_kernel_for<T, 8>(softmax, kh, kw);
        case 4: return dcn_bwd_kernel_for<T, 4>(softmax, kh, kw);
        default: break;
    }
    if constexpr (sizeof(T) == 2) {
        if (vb == 2) return dcn_bwd_kernel_for<T, 2>(softmax, kh, kw);
    }
    return nullptr;
}

template <typename T>
const void* msda_bwd_kernel_vb(int vb, int pair) {
    using namespace dcnb;
    if (pair) {   // 8 channels per lane
        if (vb == 8 * (int)sizeof(T)) return (const void*)msda_bwd_kernel<T, 8 * sizeof(T), true>;
        return nullptr;
    }
    switch (vb) {
        case 32: return (const void*)msda_bwd_kernel<T, 32>;
        case 16: return (const void*)msda_bwd_kernel<T, 16>;
        case 8: return (const void*)msda_bwd_kernel<T, 8>;
        case 4: return (const void*)msda_bwd_kernel<T, 4>;
        default: break;
    }
    if constexpr (sizeof(T) == 2) {
        if (vb == 2) return (const void*)msda_bwd_kernel<T, 2>;
    }
    return nullptr;
}

// Widest float32 reduction (4, 2 or 1 floats) whose every address is aligned:
// the accumulator base, the pixel stride (floats) and the lane's channel
// chunk (cpt floats) must all be multiples of it.
int pick_red_vec(const void* acc, long long pix_floats, int cpt) {
    for (int rv = 4; rv > 1; rv >>= 1) {
        if ((uintptr_t)acc % (uintptr_t)(4 * rv) == 0 && pix_floats % rv == 0 && cpt % rv == 0)
            return rv;
    }
    return 1;
}

// Per-lane vector width of a backward kernel.  Where a group's (head's)
// channels split into an even number of 8-channel lanes and the accumulator's
// 32-byte sectors line up with them, 8 channels per lane (one float32 sector)
// so that lane pairs reduce whole sectors (*pair = 1); otherwise the forward's
// widest vector.
int pick_bwd_vector_bytes(int es, int D, uintptr_t bases, const void* acc,
                          long long pix_floats, int* pair) {
    *pair = 0;
    const int vb8 = 8 * es;
    if (D % 16 == 0 && bases % (uintptr_t)vb8 == 0 && (uintptr_t)acc % 32 == 0 &&
        pix_floats % 8 == 0) {
        *pair = 1;
        return vb8;
    }
    return pick_vector_bytes(es, D, bases);
}

// The accumulator set-up and wrap-up launches around a backward kernel.
int launch_zero(float* p, long long n, void* stream) {
    if (n <= 0) return DCN_OK;
    const long long blocks = (n / 4 + dcnb::kUtilThreads - 1) / dcnb::kUtilThreads + 1;
    return launch((const void*)dcnb::zero_f32_kernel, dcnb::ZeroArgs{p, n},
                  (int)std::min(blocks, 1LL << 20), dcnb::kUtilThreads, 0, stream);
}

template <typename T>
int launch_round(const float* src, void* dst, long long n, void* stream) {
    if (n <= 0) return DCN_OK;
    const int vec4 = ((uintptr_t)dst % (4 * sizeof(T))) == 0 ? 1 : 0;
    const long long blocks = (n / 4 + dcnb::kUtilThreads - 1) / dcnb::kUtilThreads + 1;
    return launch((const void*)dcnb::round_f32_kernel<T>,
                  dcnb::RoundArgs<T>{src, static_cast<T*>(dst), n, vec4},
                  (int)std::min(blocks, 1LL << 20), dcnb::kUtilThreads, 0, stream);
}

int launch_round_dtype(int dtype, const float* src, void* dst, long long n, void* stream) {
    switch (dtype) {
        case DCN_F16: return launch_round<__half>(src, dst, n, stream);
        case DCN_BF16: return launch_round<__nv_bfloat16>(src, dst, n, stream);
        default: return DCN_OK;   // float32 accumulates in place
    }
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
    const TileShape ts = choose_tile(N, Ho, runs_per_row, kh * dil, sms);
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
// the optional valid ratios `vr`).
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
    const int slice = ((2 * stage_elems * es + 15) & ~15) + ((stage_elems * es + 15) & ~15);
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
    a.div_M = make_div((uint32_t)M);
    a.div_Lq = make_div((uint32_t)Lq);
    a.div_tpi = make_div((uint32_t)tpi);
    a.ref = ref;
    a.vr = vr;

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

long long dcn_backward_workspace_size(int N, int H, int W, int C, int dtype) {
    const int es = elem_bytes(dtype);
    if (es == 0 || N < 0 || H <= 0 || W <= 0 || C <= 0) return DCN_ERR_INVALID_ARG;
    if (dtype == DCN_F32) return 0;
    return (long long)N * H * W * C * 4;
}

int dcn_backward(const void* x, const void* offset, const void* mask, const void* grad_out,
                 void* grad_x, void* grad_offset, void* grad_mask, void* workspace,
                 long long workspace_bytes, int N, int H, int W, int C, int G, int kh, int kw,
                 int stride, int pad, int dil, int softmax_flag, int dtype, void* stream) {
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
    if (!x || !offset || !mask || !grad_out || !grad_x || !grad_offset || !grad_mask)
        return DCN_ERR_INVALID_ARG;
    if ((((uintptr_t)x | (uintptr_t)offset | (uintptr_t)mask | (uintptr_t)grad_out |
          (uintptr_t)grad_x | (uintptr_t)grad_offset | (uintptr_t)grad_mask) % es) != 0)
        return DCN_ERR_MISALIGNED;
    const long long need_ws = dcn_backward_workspace_size(N, H, W, C, dtype);
    if (need_ws > 0) {
        if (!workspace || workspace_bytes < need_ws) return DCN_ERR_INVALID_ARG;
        if ((uintptr_t)workspace % 16 != 0) return DCN_ERR_MISALIGNED;
    }
    const long long x_bytes = img_bytes * N;
    const long long go_bytes = out_img_bytes * N;
    const long long off_bytes = items * K * 2 * es;
    const long long m_bytes = items * K * es;
    {
        const void* in_p[4] = {x, offset, mask, grad_out};
        const long long in_b[4] = {x_bytes, off_bytes, m_bytes, go_bytes};
        const void* out_p[4] = {grad_x, grad_offset, grad_mask, workspace};
        const long long out_b[4] = {x_bytes, off_bytes, m_bytes, need_ws > 0 ? need_ws : 0};
        for (int i = 0; i < 4; ++i) {
            if (out_b[i] == 0) continue;
            for (int j = 0; j < 4; ++j)
                if (overlaps(out_p[i], out_b[i], in_p[j], in_b[j])) return DCN_ERR_INVALID_ARG;
            for (int j = 0; j < i; ++j)
                if (out_b[j] > 0 && overlaps(out_p[i], out_b[i], out_p[j], out_b[j]))
                    return DCN_ERR_INVALID_ARG;
        }
    }

    float* acc = dtype == DCN_F32 ? static_cast<float*>(grad_x) : static_cast<float*>(workspace);
    int pair = 0;
    const int vb = pick_bwd_vector_bytes(es, D, (uintptr_t)x | (uintptr_t)grad_out, acc, C,
                                         &pair);
    if (vb == 0) return DCN_ERR_MISALIGNED;
    const int cpt = vb / es;
    const int tpi = D / cpt;
    if (tpi > 32) return DCN_ERR_UNSUPPORTED;
    const int run_items = 32 / tpi;
    const int slice = dcnb::bwd_slice(run_items, K, es, softmax_flag != 0).total();
    if (slice > kMaxBwdSliceBytes) return DCN_ERR_UNSUPPORTED;
    int cap = kMaxBwdSmemBytes / slice;
    if (cap > dcnb::kDcnBwdMaxWarps) cap = dcnb::kDcnBwdMaxWarps;
    const int row_items = Wo * G;
    const int runs_per_row = (row_items + run_items - 1) / run_items;
    int sms = 148;
    {
        int device = 0;
        if (cudaGetDevice(&device) == cudaSuccess)
            (void)cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, device);
        (void)cudaGetLastError();
    }
    // 128 registers per thread: 16 warps per SM
    const TileShape ts = choose_tile(N, Ho, runs_per_row, kh * dil, sms, cap, 16);
    const int warps = ts.h * ts.w;
    const int tiles_x = (runs_per_row + ts.w - 1) / ts.w;
    const long long tiles_per_image = (long long)((Ho + ts.h - 1) / ts.h) * tiles_x;
    const long long num_tiles = tiles_per_image * N;
    if (num_tiles > kInt31) return DCN_ERR_UNSUPPORTED;

    dcnb::DcnBwdArgs b;
    dcnb::DcnArgs& a = b.f;
    a.x = x;
    a.offset = offset;
    a.mask = mask;
    a.out = nullptr;
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
    a.stage_elems = run_items * K;
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
    b.grad_out = grad_out;
    b.grad_offset = grad_offset;
    b.grad_mask = grad_mask;
    b.gx_acc = acc;
    b.red_vec = pick_red_vec(acc, C, cpt);

    const void* fn = nullptr;
    switch (dtype) {
        case DCN_F32: fn = dcn_bwd_kernel_vb<float>(vb, kh, kw, softmax_flag, pair); break;
        case DCN_F16: fn = dcn_bwd_kernel_vb<__half>(vb, kh, kw, softmax_flag, pair); break;
        case DCN_BF16:
            fn = dcn_bwd_kernel_vb<__nv_bfloat16>(vb, kh, kw, softmax_flag, pair);
            break;
        default: break;
    }
    if (!fn) return DCN_ERR_UNSUPPORTED;
    const long long acc_elems = (long long)N * H * W * C;
    int rc = launch_zero(acc, acc_elems, stream);
    if (rc != DCN_OK) return rc;
    rc = launch(fn, b, a.num_tiles, 32 * warps, slice * warps, stream);
    if (rc != DCN_OK) return rc;
    return launch_round_dtype(dtype, acc, grad_x, acc_elems, stream);
}

int dynconv_forward(const void* x, const void* weights, void* out, int N, int H, int W, int C,
                    int G, int K, int softmax_flag, int dtype, void* stream) {
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

    // tile rows: 8 on maps up to 64 rows (more CTAs), else 16
    const int th = H <= 64 ? 8 : 16;
    dcnb::DynArgs a;
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

long long msda_backward_workspace_size(int N, int S, int M, int D, int dtype) {
    const int es = elem_bytes(dtype);
    if (es == 0 || N < 0 || S <= 0 || M <= 0 || D <= 0) return DCN_ERR_INVALID_ARG;
    if (dtype == DCN_F32) return 0;
    return (long long)N * S * M * D * 4;
}

int msda_backward(const void* value, const int64_t* spatial_shapes, const int64_t* level_start,
                  const void* sampling_loc, const void* attn_w, const void* grad_out,
                  void* grad_value, void* grad_loc, void* grad_attn, void* workspace,
                  long long workspace_bytes, int N, int S, int Lq, int M, int D, int L, int K,
                  int dtype, void* stream) {
    const int es = elem_bytes(dtype);
    if (es == 0 || N < 0 || S <= 0 || Lq < 0 || M <= 0 || D <= 0 || L <= 0 || K <= 0)
        return DCN_ERR_INVALID_ARG;
    if (L > dcnb::kMsdaMaxLevels || K > 64) return DCN_ERR_UNSUPPORTED;
    const long long items = (long long)N * Lq * M;
    if (items > kInt31 || (long long)M * D * es > kInt31) return DCN_ERR_UNSUPPORTED;
    if (N == 0) return DCN_OK;
    if (!value || !spatial_shapes || !level_start || !grad_value) return DCN_ERR_INVALID_ARG;
    if (items > 0 && (!sampling_loc || !attn_w || !grad_out || !grad_loc || !grad_attn))
        return DCN_ERR_INVALID_ARG;
    if ((((uintptr_t)value | (uintptr_t)sampling_loc | (uintptr_t)attn_w | (uintptr_t)grad_out |
          (uintptr_t)grad_value | (uintptr_t)grad_loc | (uintptr_t)grad_attn) % es) != 0 ||
        (((uintptr_t)spatial_shapes | (uintptr_t)level_start) % 8) != 0)
        return DCN_ERR_MISALIGNED;
    const long long need_ws = msda_backward_workspace_size(N, S, M, D, dtype);
    if (need_ws > 0) {
        if (!workspace || workspace_bytes < need_ws) return DCN_ERR_INVALID_ARG;
        if ((uintptr_t)workspace % 16 != 0) return DCN_ERR_MISALIGNED;
    }
    const int LK = L * K;
    const long long v_bytes = (long long)N * S * M * D * es;
    {
        const void* in_p[6] = {value, spatial_shapes, level_start, sampling_loc, attn_w, grad_out};
        const long long in_b[6] = {v_bytes, (long long)L * 16, (long long)L * 8,
                                   items * LK * 2 * es, items * LK * es, items * D * es};
        const void* out_p[4] = {grad_value, grad_loc, grad_attn, workspace};
        const long long out_b[4] = {v_bytes, items * LK * 2 * es, items * LK * es,
                                    need_ws > 0 ? need_ws : 0};
        for (int i = 0; i < 4; ++i) {
            if (out_b[i] == 0) continue;
            for (int j = 0; j < 6; ++j)
                if (in_b[j] > 0 && overlaps(out_p[i], out_b[i], in_p[j], in_b[j]))
                    return DCN_ERR_INVALID_ARG;
            for (int j = 0; j < i; ++j)
                if (out_b[j] > 0 && overlaps(out_p[i], out_b[i], out_p[j], out_b[j]))
                    return DCN_ERR_INVALID_ARG;
        }
    }

    float* acc =
        dtype == DCN_F32 ? static_cast<float*>(grad_value) : static_cast<float*>(workspace);
    int pair = 0;
    const int vb = pick_bwd_vector_bytes(es, D, (uintptr_t)value | (uintptr_t)grad_out, acc,
                                         (long long)M * D, &pair);
    if (vb == 0) return DCN_ERR_MISALIGNED;
    const int cpt = vb / es;
    const int tpi = D / cpt;
    if (tpi > 32) return DCN_ERR_UNSUPPORTED;
    const int run_items = 32 / tpi;
    const int slice = dcnb::msda_bwd_slice(run_items, LK, es).total();
    if (slice > kMaxBwdSliceBytes || slice * dcnb::kMsdaWarps > kMaxBwdSmemBytes)
        return DCN_ERR_UNSUPPORTED;

    const long long acc_elems = (long long)N * S * M * D;
    dcnb::MsdaBwdArgs b;
    dcnb::MsdaArgs& a = b.f;
    a.value = value;
    a.shapes = spatial_shapes;
    a.level_start = level_start;
    a.loc = sampling_loc;
    a.attn = attn_w;
    a.out = nullptr;
    a.Lq = Lq;
    a.M = M;
    a.D = D;
    a.L = L;
    a.K = K;
    a.tpi = tpi;
    a.run_items = run_items;
    a.total_items = (int)items;
    a.num_runs = (int)((items + run_items - 1) / run_items);
    a.stage_elems = run_items * LK;
    a.div_M = make_div((uint32_t)M);
    a.div_Lq = make_div((uint32_t)(Lq > 0 ? Lq : 1));
    a.div_tpi = make_div((uint32_t)tpi);
    a.ref = nullptr;
    a.vr = nullptr;
    b.grad_out = grad_out;
    b.grad_loc = grad_loc;
    b.grad_attn = grad_attn;
    b.gv_acc = acc;
    b.S = S;
    b.red_vec = pick_red_vec(acc, (long long)M * D, cpt);

    const void* fn = nullptr;
    switch (dtype) {
        case DCN_F32: fn = msda_bwd_kernel_vb<float>(vb, pair); break;
        case DCN_F16: fn = msda_bwd_kernel_vb<__half>(vb, pair); break;
        case DCN_BF16: fn = msda_bwd_kernel_vb<__nv_bfloat16>(vb, pair); break;
        default: break;
    }
    if (!fn) return DCN_ERR_UNSUPPORTED;
    int rc = launch_zero(acc, acc_elems, stream);
    if (rc != DCN_OK) return rc;
    if (items > 0) {
        const int num_ctas = (a.num_runs + dcnb::kMsdaWarps - 1) / dcnb::kMsdaWarps;
        rc = launch(fn, b, num_ctas, dcnb::kMsdaThreads, slice * dcnb::kMsdaWarps, stream);
        if (rc != DCN_OK) return rc;
    }
    return launch_round_dtype(dtype, acc, grad_value, acc_elems, stream);
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

// ------------------------------------------- backward without caller scratch
//
// dcn_backward needs a float32 accumulator for grad_x of 16-bit data, and it
// takes it from the caller.  Some callers have no device memory to hand over
// at call time: a plain C host program that has no allocator of its own, or
// code that must not allocate once it has started (a fixed device-memory
// budget set at initialisation).  For them this file keeps one statically
// sized accumulator per device, placed in the module's global memory when the
// library's device code is loaded, and dcn_backward_static_scratch runs the
// unchanged dcn_backward path with it.  Nothing is allocated per call.

namespace {

constexpr long long kStaticScratchBytes = DCN_STATIC_SCRATCH_BYTES;   // 16 MiB
constexpr int kMaxScratchDevices = 64;

__device__ __align__(256) float g_static_scratch[kStaticScratchBytes / 4];

std::mutex g_scratch_mutex;
void* g_scratch_ptr[kMaxScratchDevices] = {};

// Device address of the static accumulator on the current device, looked up
// (cudaGetSymbolAddress) the first time a device asks and cached after that.
int static_scratch(void** out) {
    int device = 0;
    cudaError_t err = cudaGetDevice(&device);
    if (err != cudaSuccess) {
        g_last_cuda_error = (int)err;
        (void)cudaGetLastError();
        return DCN_ERR_CUDA;
    }
    if (device < 0 || device >= kMaxScratchDevices) return DCN_ERR_UNSUPPORTED;
    std::lock_guard<std::mutex> lock(g_scratch_mutex);
    if (g_scratch_ptr[device] == nullptr) {
        void* p = nullptr;
        err = cudaGetSymbolAddress(&p, g_static_scratch);
        if (err != cudaSuccess || p == nullptr) {
            g_last_cuda_error = (int)(err != cudaSuccess ? err : cudaErrorInvalidSymbol);
            (void)cudaGetLastError();
            return DCN_ERR_CUDA;
        }
        g_scratch_ptr[device] = p;
    }
    *out = g_scratch_ptr[device];
    return DCN_OK;
}

}  // namespace

extern "C" {

int dcn_backward_static_scratch(const void* x, const void* offset, const void* mask,
                                const void* grad_out, void* grad_x, void* grad_offset,
                                void* grad_mask, int N, int H, int W, int C, int G, int kh,
                                int kw, int stride, int pad, int dil, int softmax_flag,
                                int dtype, void* stream) {
    const long long need = dcn_backward_workspace_size(N, H, W, C, dtype);
    if (need < 0) return DCN_ERR_INVALID_ARG;
    if (need > kStaticScratchBytes) return DCN_ERR_UNSUPPORTED;
    void* ws = nullptr;
    if (need > 0) {
        const int rc = static_scratch(&ws);
        if (rc != DCN_OK) return rc;
    }
    return dcn_backward(x, offset, mask, grad_out, grad_x, grad_offset, grad_mask, ws,
                        need > 0 ? kStaticScratchBytes : 0, N, H, W, C, G, kh, kw, stride, pad,
                        dil, softmax_flag, dtype, stream);
}

}  // extern "C"
