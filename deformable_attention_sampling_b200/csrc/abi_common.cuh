// Host-side helpers shared by the translation units of the C interface:
// argument checks, launch-shape choice and launching.  Nothing here allocates
// or synchronises; every launch goes to the caller's stream.
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>

#include <algorithm>
#include <atomic>
#include <cmath>
#include <cstdint>

#include "common.cuh"
#include "dcn.h"

namespace dcnb_abi {

using dcnb::FastDiv;

// launches issued by the library, and the last CUDA error seen by this thread
extern std::atomic<unsigned long long> g_launches;
extern thread_local int g_last_cuda_error;

constexpr int kMaxDim = 65536;        // H, W, pad, stride, dil
constexpr int kMaxTaps = 1024;        // kh * kw
constexpr int kMaxStageBytes = 48 * 1024;
constexpr int kMaxBwdSliceBytes = 200 * 1024;   // shared slice of one backward warp
constexpr int kMaxBwdSmemBytes = 220 * 1024;    // of one backward CTA (opt-in size)
constexpr long long kInt31 = 2147483647LL;

inline FastDiv make_div(uint32_t d) {
    uint32_t shift = 0;
    while ((1ull << shift) < d) ++shift;
    const unsigned long long mul = ((1ull << 32) * ((1ull << shift) - d)) / d + 1;
    return FastDiv{d, (uint32_t)mul, shift};
}

inline int elem_bytes(int dtype) {
    switch (dtype) {
        case DCN_F32: return 4;
        case DCN_F16: return 2;
        case DCN_BF16: return 2;
        default: return 0;
    }
}

// Widest per-thread vector (bytes) that divides one group's channel span and
// keeps every thread's address aligned for the given base pointers.
inline int pick_vector_bytes(int es, int D, uintptr_t bases) {
    const int span = D * es;
    for (int vb = 32; vb >= es; vb >>= 1) {
        if (span % vb == 0 && (bases % (uintptr_t)vb) == 0) return vb;
    }
    return 0;
}

inline bool overlaps(const void* a, long long abytes, const void* b, long long bbytes) {
    const uintptr_t a0 = (uintptr_t)a, b0 = (uintptr_t)b;
    return a0 < b0 + (uintptr_t)bbytes && b0 < a0 + (uintptr_t)abytes;
}

// Multiprocessor count of the current device (148 when it cannot be read).
int sm_count();

// Grid size: one resident wave of CTAs (SM count x CTAs per SM) of kernel fn
// at this block size and dynamic shared memory, 0 on a CUDA error.
//
// The first time a kernel runs on a device with a given shared-memory size,
// its preferred shared-memory carveout is set to what its resident CTAs need
// (the rest of the SM's 256 KB array stays L1, which the gathers live in);
// the carveout of a kernel only ever grows, so no earlier configuration loses
// occupancy.  Kernels above 48 KB of dynamic shared memory are opted in.
int wave_size(const void* fn, int threads, int smem);

// Persistent launch: at most one resident wave of CTAs, or fewer when there
// are fewer work units; each CTA then takes a contiguous share.
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
        (void)cudaGetLastError();   // clear the launch error just reported
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

// Tile shape of the L1-path DCN kernels: tile_h output rows x tile_w warp
// runs, one warp per run (see choose_tile in abi_common.cu).
struct TileShape {
    int h, w;
};

// `cap` is the kernel's warp limit per CTA and `warps_by_regs` the warps one
// SM holds at the kernel's register count.
TileShape choose_tile(int N, int Ho, int runs, int kernel_extent, int sms, int cap,
                      int warps_by_regs);

// Item stride, in elements, of a warp's staged slice in shared memory: the
// run's `items` rows of `row_elems` elements (`es` bytes each) are copied
// from consecutive global rows, and at every step each item reads
// `read_elems` elements at the same offset of its row.  The stride is the row
// rounded up to 16 bytes plus the multiple of 16 bytes that leaves the
// fewest of those reads in one of the 32 four-byte banks (rows of a power of
// two bytes would put every item in the same bank).
int staged_row_stride(int items, int row_elems, int read_elems, int es);

// Device address of the kernels' status word (DCN_FLAG_* bits) on the current
// device (looked up once per device), or null.
unsigned int* device_flags_word();

// A 2-D tensor map over a row-major matrix of 16-bit elements (`inner`
// elements per row, `outer` rows, rows `row_bytes` apart) for tile loads of
// box_inner x box_outer elements with the 128-byte swizzle; out-of-range box
// elements read as zero.  The encoder comes from the driver through the
// runtime's entry-point query (no link-time dependency on libcuda).  False on
// any error.
bool encode_tmap_2d(CUtensorMap* map, const void* base, bool bf16, uint64_t inner,
                    uint64_t outer, uint64_t row_bytes, uint32_t box_inner, uint32_t box_outer);

}  // namespace dcnb_abi
