// Dynamic local aggregation (the ContMix core), sm_100a SIMT kernel.
//
// Operator ("OverLoCK" note, "ContMix: Put the Whole Image into the Kernel",
// steps 4-5): every location has, per channel group, its own K x K kernel (a
// softmax over its K*K numbers), applied to the zero-padded K x K
// neighbourhood of that group's channels:
//   out[n,y,x,g*D+c] = sum_{ky,kx} A[n,y,x,g,ky*K+kx] * x[n, y+ky-K/2, x+kx-K/2, g*D+c]
// It is a DCN with every offset zero, so nothing is gathered: a CTA stages the
// input window of an output tile once in shared memory and every staged pixel
// feeds up to K*K outputs.
//
// Work decomposition (one CTA = one tile of TH rows x 32 columns, one group,
// one 32-byte channel chunk):
//   thread  = 4 consecutive output columns (P = 4) of one row, CPT channels
//             (32 bytes: 16 fp16 / bf16 or 8 fp32); 8 threads span the tile's
//             32 columns, so a warp covers 4 rows.
//   window  = rows [y0 - K/2, y0 + TH - 1 + K/2], columns likewise, copied with
//             cp.async (zero-filled outside the map, all copies in flight at
//             once); pixel c of a window row sits at byte c*32 + (c/4)*16, so
//             the 32-byte loads of a warp (threads 4 columns apart) spread over
//             all banks.
//   weights = one kernel row (ky) at a time: the K numbers of every location
//             are copied by lane groups with coalesced loads into a
//             double-buffered raw shared buffer (the next row is fetched while
//             the current one is used), then the thread that owns a location
//             turns them into float32 weights in its own slots [kx][row][col]
//             (row stride 33: conflict-free).  With the softmax the maximum of
//             each location's K*K numbers comes from a pre-pass, each weight is
//             exp2((z - max) log2 e), computed once, the owner sums them in
//             registers and divides its outputs by the sum at the end.
// Per kernel row the thread slides along x: each window pixel it loads (two
// 16-byte shared loads, widened once) is multiplied into the up to four
// outputs whose taps cover it, with packed FFMA2 into float32 accumulators.
#pragma once

#include "common.cuh"

namespace dcnb {

constexpr int kDynP = 4;            // output columns per thread
constexpr int kDynTileW = 32;       // output columns per tile
constexpr int kDynSegs = kDynTileW / kDynP;
constexpr int kDynMaxK = 31;

struct DynArgs {
    const void* x;           // [N][H][W][C]
    const void* w;           // [N][H][W][G][K*K]
    void* out;               // [N][H][W][C]
    int H, W, C, G, D, K;
    int th;                  // tile rows
    int tiles_x, tiles_y, chunks;
    int win_rows, row_bytes; // staged window: rows, bytes per row (padded)
    int xs_bytes, ws_bytes;  // shared-memory parts
};

__host__ __device__ inline int dyn_pixel_byte(int c) { return c * 32 + (c >> 2) * 16; }

__host__ __device__ inline int dyn_row_bytes(int cols) { return ((cols + 3) >> 2) * 144; }

// floats per kx slice of a staged kernel row: TH rows of 33, plus one so that
// the slices of consecutive kx start in different banks
__host__ __device__ inline int dyn_wstride(int th) { return th * (kDynTileW + 1) + 1; }

// 16-byte asynchronous global -> shared copy; src_bytes = 0 writes zeros.
__device__ __forceinline__ void cp_async16(void* dst, const void* src, uint32_t src_bytes) {
    const uint32_t d = (uint32_t)__cvta_generic_to_shared(dst);
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" :: "r"(d), "l"(src),
                 "r"(src_bytes) : "memory");
}

constexpr int kDynStageUnroll = 8;   // loads in flight per lane while staging weights

// Words per location in the raw weight buffer: the K numbers of one kernel row
// (16-bit or 32-bit), rounded up to an odd count so that the locations a warp
// reads at once fall in different banks.
__host__ __device__ inline int dyn_raw_words(int K, int es) {
    const int w = (K * es + 3) / 4;
    return w | 1;
}

template <typename T, bool SOFTMAX>
__global__ void __launch_bounds__(256) dynconv_fwd_kernel(const DynArgs a) {
    constexpr int CPT = 32 / (int)sizeof(T);
    constexpr int es = (int)sizeof(T);
    constexpr int U = kDynStageUnroll;
    constexpr float kLog2e = 1.4426950408889634f;
    extern __shared__ __align__(16) unsigned char smem[];
    const int TH = a.th;
    const int NP = TH * kDynTileW;                  // locations of the tile
    const int K = a.K, KK = K * K, r = K >> 1;
    const int RW = dyn_raw_words(K, es);            // raw words per location
    const int RP = kDynTileW + 1;                   // locations per raw / ws row (padded)
    unsigned char* xs = smem;
    float* ws = reinterpret_cast<float*>(smem + a.xs_bytes);
    uint32_t* raw = reinterpret_cast<uint32_t*>(smem + a.xs_bytes + a.ws_bytes);
    const int raw_words = TH * RP * RW;             // one buffer
    float* s_max = reinterpret_cast<float*>(raw + 2 * raw_words);

    const int tid = threadIdx.x;
    const int nthreads = blockDim.x;
    const int lane = tid & 31;
    const int warp = tid >> 5;
    const int nwarps = nthreads >> 5;

    // tile coordinates: blockIdx.x = (((n * tiles_y + ty) * tiles_x + tx) * G + g) * chunks + q
    int b = blockIdx.x;
    const int q = b % a.chunks;
    b /= a.chunks;
    const int g = b % a.G;
    b /= a.G;
    const int tx = b % a.tiles_x;
    b /= a.tiles_x;
    const int ty = b % a.tiles_y;
    const int n = b / a.tiles_y;
    const int y0 = ty * TH, x0 = tx * kDynTileW;
    const long long ch0 = (long long)g * a.D + (long long)q * CPT;   // first channel

    // ---- stage the input window: asynchronous 16-byte copies, zeros outside ----
    const int win_cols = kDynTileW + K - 1;
    const long long pix_bytes = (long long)a.C * es;
    const char* xin = static_cast<const char*>(a.x) + (long long)n * a.H * a.W * pix_bytes +
                      ch0 * es;
    for (int e = tid; e < a.win_rows * win_cols * 2; e += nthreads) {
        const int half = e & 1;
        const int pix = e >> 1;
        const int wr = pix / win_cols, wc = pix - wr * win_cols;
        const int gy = y0 - r + wr, gx = x0 - r + wc;
        const bool inside = (unsigned)gy < (unsigned)a.H && (unsigned)gx < (unsigned)a.W;
        const char* src = inside ? xin + ((long long)gy * a.W + gx) * pix_bytes + half * 16 : xin;
        cp_async16(xs + wr * a.row_bytes + dyn_pixel_byte(wc) + half * 16, src, inside ? 16u : 0u);
    }
    asm volatile("cp.async.commit_group;" ::: "memory");

    // weights of the tile: location (row, col) starts at wt + row * w_row + col * w_col
    const T* wt = static_cast<const T*>(a.w) +
                  ((((long long)n * a.H + y0) * a.W + x0) * a.G + g) * KK;
    const int w_col = a.G * KK;
    const int w_row = a.W * w_col;
    auto in_map = [&](int row, int col) { return y0 + row < a.H && x0 + col < a.W; };

    // ---- softmax: maximum of each location's K*K numbers (a warp per location) ----
    if constexpr (SOFTMAX) {
        for (int pix0 = warp * 4; pix0 < NP; pix0 += nwarps * 4) {
            float m[4];
#pragma unroll
            for (int u = 0; u < 4; ++u) {
                const int pix = pix0 + u;
                const int row = pix / kDynTileW, col = pix - row * kDynTileW;
                m[u] = -INFINITY;
                if (pix < NP && in_map(row, col)) {
                    const T* wp = wt + row * w_row + col * w_col;
                    for (int t = lane; t < KK; t += 32) m[u] = fmaxf(m[u], Elem<T>::one(wp + t));
                }
            }
#pragma unroll
            for (int u = 0; u < 4; ++u) {
#pragma unroll
                for (int o = 16; o > 0; o >>= 1)
                    m[u] = fmaxf(m[u], __shfl_xor_sync(0xffffffffu, m[u], o));
                if (lane == 0 && pix0 + u < NP) s_max[pix0 + u] = m[u];
            }
        }
    }

    // Copy kernel row ky of every location into raw buffer `buf` (lanes over
    // the K numbers of a location, 16 or 32 lanes per location, U locations in
    // flight per lane).  Locations outside the map copy nothing.
    const int lpp = K <= 16 ? 16 : 32;
    const int ppw = 32 / lpp;
    const int sub = lane / lpp, kx_l = lane - sub * lpp;
    auto copy_row = [&](int ky, int buf) {
        T* dst = reinterpret_cast<T*>(raw + buf * raw_words);
        for (int base = warp * ppw * U; base < NP; base += nwarps * ppw * U) {
            T v[U];
#pragma unroll
            for (int u = 0; u < U; ++u) {
                const int pix = base + u * ppw + sub;
                const int row = pix / kDynTileW, col = pix - row * kDynTileW;
                if (pix < NP && kx_l < K && in_map(row, col))
                    v[u] = wt[row * w_row + col * w_col + ky * K + kx_l];
            }
#pragma unroll
            for (int u = 0; u < U; ++u) {
                const int pix = base + u * ppw + sub;
                const int row = pix / kDynTileW, col = pix - row * kDynTileW;
                if (pix < NP && kx_l < K && in_map(row, col))
                    dst[(row * RP + col) * RW * (4 / es) + kx_l] = v[u];
            }
        }
    };

    // ---- this thread's outputs: 4 columns of one row ----
    const int seg = tid % kDynSegs;
    const int row = tid / kDynSegs;
    const int col0 = seg * kDynP;
    float acc[kDynP][CPT];
#pragma unroll
    for (int p = 0; p < kDynP; ++p)
#pragma unroll
        for (int i = 0; i < CPT; ++i) acc[p][i] = 0.f;
    float mloc[kDynP], ssum[kDynP];
    bool mine[kDynP];

    const int wstride = dyn_wstride(TH);
    copy_row(0, 0);
    asm volatile("cp.async.wait_all;" ::: "memory");
    __syncthreads();
#pragma unroll
    for (int p = 0; p < kDynP; ++p) {
        mine[p] = in_map(row, col0 + p);
        mloc[p] = SOFTMAX && mine[p] ? s_max[row * kDynTileW + col0 + p] * kLog2e : 0.f;
        ssum[p] = 0.f;
    }

    for (int ky = 0; ky < K; ++ky) {
        if (ky > 0) __syncthreads();   // raw row ky complete; raw row ky - 1 consumed
        // this thread's weights of kernel row ky: exp (softmax) once per tap,
        // into its own slots of ws (read back only by this thread)
        {
            const T* src = reinterpret_cast<const T*>(raw + (ky & 1) * raw_words);
            float* wk = ws + row * RP + col0;
#pragma unroll
            for (int p = 0; p < kDynP; ++p) {
                const T* rp = src + (row * RP + col0 + p) * RW * (4 / es);
                for (int kx = 0; kx < K; ++kx) {
                    float e = 0.f;
                    if (mine[p]) {
                        const float z = Elem<T>::one(rp + kx);
                        if constexpr (SOFTMAX) {
                            e = exp2f(fmaf(z, kLog2e, -mloc[p]));
                            ssum[p] += e;
                        } else {
                            e = z;
                        }
                    }
                    wk[kx * wstride + p] = e;
                }
            }
        }
        // prefetch kernel row ky + 1 into the other buffer while computing
        if (ky + 1 < K) copy_row(ky + 1, (ky + 1) & 1);

        // slide along the window row (row + ky) over columns col0 .. col0 + K + P - 2
        const unsigned char* xrow = xs + (row + ky) * a.row_bytes;
        const float* wk = ws + row * RP + col0;
        for (int j = 0; j < K + kDynP - 1; ++j) {
            const unsigned char* px = xrow + dyn_pixel_byte(col0 + j);
            uint32_t wv[8];
            const uint4 lo = *reinterpret_cast<const uint4*>(px);
            const uint4 hi = *reinterpret_cast<const uint4*>(px + 16);
            wv[0] = lo.x; wv[1] = lo.y; wv[2] = lo.z; wv[3] = lo.w;
            wv[4] = hi.x; wv[5] = hi.y; wv[6] = hi.z; wv[7] = hi.w;
            float f[CPT];
            widen<T, CPT>(wv, f);
#pragma unroll
            for (int p = 0; p < kDynP; ++p) {
                const int kx = j - p;
                if (kx >= 0 && kx < K) axpy<CPT>(acc[p], wk[kx * wstride + p], f);
            }
        }
    }

    // ---- normalise (softmax) and store ----
    char* obase = static_cast<char*>(a.out) + (long long)n * a.H * a.W * pix_bytes + ch0 * es;
#pragma unroll
    for (int p = 0; p < kDynP; ++p) {
        if (mine[p]) {
            if constexpr (SOFTMAX) {
                const float inv = 1.f / ssum[p];
#pragma unroll
                for (int i = 0; i < CPT; ++i) acc[p][i] *= inv;
            }
            uint32_t o[8];
            narrow<T, CPT>(acc[p], o);
            store_vec<32>(obase + ((long long)(y0 + row) * a.W + (x0 + col0 + p)) * pix_bytes, o);
        }
    }
}

}  // namespace dcnb
