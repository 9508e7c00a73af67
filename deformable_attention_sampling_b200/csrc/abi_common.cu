// C interface of libdcn_b200.so, shared part: the launch helpers of
// abi_common.cuh, the tile choice of the L1-path DCN kernels, and the status,
// version and size queries declared in include/dcn.h.
#include <mutex>

#include "abi_common.cuh"
#include "dcn_fwd.cuh"

namespace dcnb_abi {

std::atomic<unsigned long long> g_launches{0};
thread_local int g_last_cuda_error = 0;

int sm_count() {
    int sms = 148, device = 0;
    if (cudaGetDevice(&device) == cudaSuccess)
        (void)cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, device);
    (void)cudaGetLastError();
    return sms > 0 ? sms : 148;
}

namespace {

using EncodeTiledFn = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                   const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                   const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                   CUtensorMapL2promotion, CUtensorMapFloatOOBfill);
std::once_flag g_encode_once;
EncodeTiledFn g_encode = nullptr;

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

}  // namespace

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
constexpr int kSmallMapRows = 64;

// Status word of the kernels (DCN_FLAG_* bits), one per device; its device
// address is looked up once per device.
__device__ unsigned int g_device_flags;

constexpr int kMaxScratchDevices = 64;
std::mutex g_timeout_mutex;
unsigned int* g_timeout_ptr[kMaxScratchDevices] = {};

unsigned int* device_flags_word() {
    int device = 0;
    if (cudaGetDevice(&device) != cudaSuccess || device < 0 || device >= kMaxScratchDevices) {
        (void)cudaGetLastError();
        return nullptr;
    }
    std::lock_guard<std::mutex> lock(g_timeout_mutex);
    if (g_timeout_ptr[device] == nullptr) {
        void* p = nullptr;
        if (cudaGetSymbolAddress(&p, g_device_flags) != cudaSuccess) {
            (void)cudaGetLastError();
            return nullptr;
        }
        g_timeout_ptr[device] = static_cast<unsigned int*>(p);
    }
    return g_timeout_ptr[device];
}

bool encode_tmap_2d(CUtensorMap* map, const void* base, bool bf16, uint64_t inner,
                    uint64_t outer, uint64_t row_bytes, uint32_t box_inner, uint32_t box_outer) {
    std::call_once(g_encode_once, [] {
        void* fn = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &fn, cudaEnableDefault, &q) ==
                cudaSuccess && q == cudaDriverEntryPointSuccess)
            g_encode = reinterpret_cast<EncodeTiledFn>(fn);
        (void)cudaGetLastError();
    });
    if (!g_encode) return false;
    const cuuint64_t dims[2] = {inner, outer};
    const cuuint64_t strides[1] = {row_bytes};
    const cuuint32_t box[2] = {box_inner, box_outer};
    const cuuint32_t elem_strides[2] = {1, 1};
    return g_encode(map, bf16 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16 : CU_TENSOR_MAP_DATA_TYPE_FLOAT16,
                    2, const_cast<void*>(base), dims, strides, box, elem_strides,
                    CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                    CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                    CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

TileShape choose_tile(int N, int Ho, int runs, int kernel_extent, int sms, int cap,
                      int warps_by_regs) {
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

int staged_row_stride(int items, int row_elems, int read_elems, int es) {
    const int row_bytes = (row_elems * es + 15) & ~15;
    const int read_bytes = read_elems * es;
    int best_stride = row_bytes, best_worst = 1 << 30;
    for (int pad = 0; pad < 128; pad += 16) {
        const int stride = row_bytes + pad;
        int worst = 0;
        for (int off = 0; off + read_bytes <= row_elems * es && worst < best_worst;
             off += read_bytes) {
            // distinct 4-byte words per bank among the items' reads at `off`
            int words[32][32];
            int count[32] = {0};
            for (int i = 0; i < items && i < 32; ++i) {
                const int first = (i * stride + off) >> 2;
                const int last = (i * stride + off + read_bytes - 1) >> 2;
                for (int wd = first; wd <= last; ++wd) {
                    const int bank = wd & 31;
                    bool seen = false;
                    for (int j = 0; j < count[bank]; ++j) seen = seen || words[bank][j] == wd;
                    if (!seen && count[bank] < 32) words[bank][count[bank]++] = wd;
                }
            }
            for (int b = 0; b < 32; ++b) worst = std::max(worst, count[b]);
        }
        if (worst < best_worst) {
            best_worst = worst;
            best_stride = stride;
        }
        if (best_worst <= 1) break;
    }
    return best_stride / es;
}

}  // namespace dcnb_abi

using namespace dcnb_abi;

extern "C" {

int dcn_output_size(int in, int k, int stride, int pad, int dil) {
    if (in <= 0 || k <= 0 || stride <= 0 || pad < 0 || dil <= 0) return 0;
    const long long span = (long long)in + 2LL * pad - (long long)dil * (k - 1) - 1;
    if (span < 0) return 0;
    return (int)(span / stride + 1);
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

int dcn_device_flags(int reset) {
    unsigned int v = 0;
    if (cudaMemcpyFromSymbol(&v, g_device_flags, sizeof(v)) != cudaSuccess) {
        g_last_cuda_error = (int)cudaGetLastError();
        return DCN_ERR_CUDA;
    }
    if (reset) {
        const unsigned int zero = 0;
        if (cudaMemcpyToSymbol(g_device_flags, &zero, sizeof(zero)) != cudaSuccess) {
            g_last_cuda_error = (int)cudaGetLastError();
            return DCN_ERR_CUDA;
        }
    }
    return (int)(v & 0x7fffffffu);
}

int dcn_debug_checks(void) {
#ifdef DCN_DEBUG
    return 1;
#else
    return 0;
#endif
}

int dcn_last_cuda_error(void) { return g_last_cuda_error; }

uint64_t dcn_launch_count(void) { return g_launches.load(std::memory_order_relaxed); }

int dcn_version(void) { return 10000; }

}  // extern "C"
