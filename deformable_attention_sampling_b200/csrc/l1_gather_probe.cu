// Gather-rate probe: the bytes per SM clock that random 32-byte vector loads
// (one ld.global.nc.v8.b32 per lane, the corner load of the sampling kernels)
// sustain on this GPU, as the per-SM footprint grows from L1-resident to
// L2-resident, plus shared-memory 16-byte gathers for comparison.  It
// calibrates the on-chip roofline that bench.py reports beside the HBM one.
//
//   python -m deformable_attention_sampling_b200.build --probe
//   deformable_attention_sampling_b200/_lib/l1_gather_probe
//
// Every index is reduced modulo its buffer, so every access stays in bounds.
#include <cuda_runtime.h>

#include <cstdint>
#include <cstdio>

namespace {

constexpr int kIters = 2048;
constexpr int kThreads = 256;
constexpr int kSmemBytes = 32 * 1024;

__device__ __forceinline__ uint32_t next(uint32_t& s) {
    s = s * 1664525u + 1013904223u;   // 32-bit LCG (Numerical Recipes constants)
    return s >> 8;
}

// Each CTA gathers 32-byte sectors from a window of `win` sectors starting at
// `blockIdx.x * stride` (stride 0: every CTA shares one window).
__global__ void gather_global(const uint8_t* __restrict__ buf, uint32_t sectors, uint32_t win,
                              uint32_t stride, uint32_t* sink) {
    uint32_t s = threadIdx.x * 7919u + blockIdx.x * 104729u;
    const uint32_t base = (blockIdx.x * stride) % sectors;
    uint32_t acc = 0;
    for (int i = 0; i < kIters; ++i) {
        const uint32_t sec = (base + next(s) % win) % sectors;
        uint32_t a0, a1, a2, a3, a4, a5, a6, a7;
        asm volatile("ld.global.nc.v8.b32 {%0,%1,%2,%3,%4,%5,%6,%7}, [%8];"
                     : "=r"(a0), "=r"(a1), "=r"(a2), "=r"(a3), "=r"(a4), "=r"(a5), "=r"(a6),
                       "=r"(a7)
                     : "l"(buf + (size_t)sec * 32));
        acc += a0 ^ a1 ^ a2 ^ a3 ^ a4 ^ a5 ^ a6 ^ a7;
    }
    if (acc == 0x12345678u) sink[0] = acc;
}

// 16-byte shared-memory gathers: random chunks, or conflict-free (lane i of a
// warp reads chunk base + i).
template <bool CONFLICT_FREE>
__global__ void gather_shared(const uint8_t* __restrict__ buf, uint32_t* sink) {
    __shared__ __align__(16) uint8_t sm[kSmemBytes];
    for (int i = threadIdx.x; i < kSmemBytes / 16; i += blockDim.x)
        reinterpret_cast<uint4*>(sm)[i] = reinterpret_cast<const uint4*>(buf)[i];
    __syncthreads();
    uint32_t s = threadIdx.x * 7919u + blockIdx.x * 104729u;
    const uint32_t lane = threadIdx.x & 31;
    uint32_t acc = 0;
    for (int i = 0; i < kIters; ++i) {
        const uint32_t r = next(s);
        const uint32_t chunk = CONFLICT_FREE ? (((r & ~31u) + lane) % (kSmemBytes / 16))
                                             : (r % (kSmemBytes / 16));
        const uint32_t addr = (uint32_t)__cvta_generic_to_shared(sm + chunk * 16);
        uint32_t a0, a1, a2, a3;
        asm volatile("ld.shared.v4.b32 {%0,%1,%2,%3}, [%4];"
                     : "=r"(a0), "=r"(a1), "=r"(a2), "=r"(a3) : "r"(addr));
        acc += a0 ^ a1 ^ a2 ^ a3;
    }
    if (acc == 0x12345678u) sink[0] = acc;
}

double bytes_per_clk_per_sm(float ms, double bytes, int sms, int mhz) {
    return bytes / (ms * 1e-3 * mhz * 1e6) / sms;
}

}  // namespace

int main() {
    const size_t bytes = 256u << 20;
    uint8_t* buf = nullptr;
    uint32_t* sink = nullptr;
    if (cudaMalloc(&buf, bytes) != cudaSuccess || cudaMalloc(&sink, 64) != cudaSuccess) {
        std::printf("allocation failed\n");
        return 1;
    }
    cudaMemset(buf, 1, bytes);
    int sms = 0, khz = 0;
    cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, 0);
    cudaDeviceGetAttribute(&khz, cudaDevAttrClockRate, 0);
    const int mhz = khz / 1000;
    const int ctas_per_sm = 4, grid = sms * ctas_per_sm;
    const uint32_t sectors = (uint32_t)(bytes / 32);
    cudaEvent_t a, b;
    cudaEventCreate(&a);
    cudaEventCreate(&b);
    std::printf("SMs %d, clock %d MHz (rates below assume this clock)\n", sms, mhz);
    std::printf("%-46s %10s %14s\n", "random 32 B global gathers", "ms", "B/clk/SM");
    for (uint32_t kb : {8u, 24u, 40u, 56u, 80u, 128u, 256u, 1024u}) {
        for (int shared : {1, 0}) {
            const uint32_t win = kb * 1024 / 32, stride = shared ? 0 : win;
            gather_global<<<grid, kThreads>>>(buf, sectors, win, stride, sink);
            cudaEventRecord(a);
            gather_global<<<grid, kThreads>>>(buf, sectors, win, stride, sink);
            cudaEventRecord(b);
            cudaEventSynchronize(b);
            float ms = 0.f;
            cudaEventElapsedTime(&ms, a, b);
            char label[96];
            std::snprintf(label, sizeof label, "  %4u KB window, %s", kb,
                          shared ? "shared by all CTAs" : "one per CTA (4 per SM)");
            std::printf("%-46s %10.3f %14.1f\n", label, ms,
                        bytes_per_clk_per_sm(ms, (double)grid * kThreads * kIters * 32, sms, mhz));
        }
    }
    for (int cf : {0, 1}) {
        auto k = cf ? gather_shared<true> : gather_shared<false>;
        k<<<grid, kThreads>>>(buf, sink);
        cudaEventRecord(a);
        k<<<grid, kThreads>>>(buf, sink);
        cudaEventRecord(b);
        cudaEventSynchronize(b);
        float ms = 0.f;
        cudaEventElapsedTime(&ms, a, b);
        std::printf("%-46s %10.3f %14.1f\n",
                    cf ? "16 B shared gathers, conflict-free" : "16 B shared gathers, random",
                    ms, bytes_per_clk_per_sm(ms, (double)grid * kThreads * kIters * 16, sms, mhz));
    }
    const cudaError_t err = cudaDeviceSynchronize();
    std::printf("status: %s\n", cudaGetErrorString(err));
    return err == cudaSuccess ? 0 : 1;
}
