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
//   thread  = P = 2 consecutive output columns of one row, CPT channels
//             (32 bytes: 16 fp16 / bf16 or 8 fp32); 16 threads span the tile's
//             32 columns, so a warp covers 2 rows.
//   window  = rows [y0 - K/2, y0 + TH - 1 + K/2], columns likewise, copied with
//             cp.async (zero-filled outside the map, all copies in flight at
//             once); pixel c of a window row sits at byte c*32 + (c/4)*16, so
//             the 32-byte loads of a warp (threads 2 columns apart) spread over
//             the banks.
//   weights = one kernel row (ky) at a time: the K numbers of every location
//             are copied with 16-byte cp.async blocks (from the block that holds
//             the first number, the last copy clipped to the row's end) into a
//             double-buffered raw shared buffer, the next row in flight while
//             the current one is used; the thread that owns a location reads
//             them at any alignment and writes float32 weights into its own
//             slots [kx][row][col] (row stride 33: conflict-free).  The softmax
//             runs online per location: a running maximum keeps exp finite,
//             each weight is exp2((z - max) log2 e), computed once, and the
//             running sum and the owner's accumulators are rescaled when the
//             maximum grows; the output is divided by the sum at the end.
// Per kernel row the thread slides along x: each window pixel it loads (two
// 16-byte shared loads, widened once) is multiplied into the up to P outputs
// whose taps cover it, with packed FFMA2 into float32 accumulators.
#pragma once

#include "common.cuh"

namespace dcnb {

constexpr int kDynP = 2;            // output columns per thread (2: measured faster than 4, more warps)
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

// Bytes of one location's slot in the raw weight buffer: the K numbers of a
// kernel row start anywhere within their first 16-byte block, so the slot
// holds ceil((K * es + 15) / 16) whole blocks.
__host__ __device__ inline int dyn_slot_bytes(int K, int es) { return ((K * es + 15 + 15) / 16) * 16; }

// KT > 0: the kernel size fixed at compile time (the workloads' 7 and 13).
// Each thread then keeps its locations' weights of the current kernel row in
// registers (no float32 weight slots in shared memory, so more CTAs fit on an
// SM) and the sliding loop unrolls.  KT = 0: any odd K up to kDynMaxK.
template <typename T, bool SOFTMAX, int KT = 0>
__global__ void __launch_bounds__(256) dynconv_fwd_kernel(const DynArgs a) {
    constexpr int CPT = 32 / (int)sizeof(T);
    constexpr int es = (int)sizeof(T);
    constexpr float kLog2e = 1.4426950408889634f;
    extern __shared__ __align__(16) unsigned char smem[];
    const int TH = a.th;
    const int NP = TH * kDynTileW;                  // locations of the tile
    const int K = KT ? KT : a.K, KK = K * K, r = K >> 1;
    const int SB = dyn_slot_bytes(K, es);
    unsigned char* xs = smem;
    float* ws = reinterpret_cast<float*>(smem + a.xs_bytes);
    unsigned char* raw = smem + a.xs_bytes + a.ws_bytes;   // two buffers of NP slots

    const int tid = threadIdx.x;
    const int nthreads = blockDim.x;

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
    // slot of location (row, col): ordered [col % P][row][col / P], so that the
    // owners of one column offset read consecutive slots
    auto slot = [&](int row, int col) {
        return ((col % kDynP) * TH + row) * kDynSegs + col / kDynP;
    };

    // Copy kernel row ky of every location of the tile into raw buffer `buf`:
    // whole 16-byte blocks from the block holding the row's first number,
    // each copy clipped to the row's last byte (nothing past it is read).
    auto copy_row = [&](int ky, int buf) {
        unsigned char* dst0 = raw + buf * NP * SB;
        for (int loc = tid; loc < NP; loc += nthreads) {
            const int row = loc / kDynTileW, col = loc - row * kDynTileW;
            if (!in_map(row, col)) continue;
            const char* first = reinterpret_cast<const char*>(wt + row * w_row + col * w_col + ky * K);
            const char* last = first + K * es;
            const char* blk = reinterpret_cast<const char*>((uintptr_t)first & ~(uintptr_t)15);
            unsigned char* dst = dst0 + slot(row, col) * SB;
            for (; blk < last; blk += 16, dst += 16) {
                const long long left = last - blk;
                cp_async16(dst, blk, left >= 16 ? 16u : (uint32_t)left);
            }
        }
        asm volatile("cp.async.commit_group;" ::: "memory");
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
    float mrun[kDynP], ssum[kDynP];
    bool mine[kDynP];
    int skew[kDynP];    // byte offset of the row's first number within its block
#pragma unroll
    for (int p = 0; p < kDynP; ++p) {
        mine[p] = in_map(row, col0 + p);
        mrun[p] = -INFINITY;
        ssum[p] = 0.f;
        skew[p] = (int)((uintptr_t)(wt + row * w_row + (col0 + p) * w_col) & 15);
    }
    const int wstride = dyn_wstride(TH);
    float* wk = ws + row * (kDynTileW + 1) + col0;
    float wreg[kDynP][KT ? KT : 1];   // KT > 0: this row's weights of the thread's locations
    (void)wreg;
    auto put_w = [&](int p, int kx, float v) {
        if constexpr (KT > 0) wreg[p][kx] = v;
        else wk[kx * wstride + p] = v;
    };

    copy_row(0, 0);
    for (int ky = 0; ky < K; ++ky) {
        if (ky + 1 < K) {
            if (ky > 0) __syncthreads();      // raw buffer (ky + 1) & 1 is no longer read
            copy_row(ky + 1, (ky + 1) & 1);
            asm volatile("cp.async.wait_group 1;" ::: "memory");   // window and row ky landed
        } else {
            asm volatile("cp.async.wait_all;" ::: "memory");
        }
        __syncthreads();

        // this thread's weights of kernel row ky, into its own slots of ws
#pragma unroll
        for (int p = 0; p < kDynP; ++p) {
            if (!mine[p]) {
#pragma unroll
                for (int kx = 0; kx < K; ++kx) put_w(p, kx, 0.f);
                continue;
            }
            const int sk = (skew[p] + ky * K * es) & 15;
            const T* zr = reinterpret_cast<const T*>(raw + (ky & 1) * NP * SB +
                                                     slot(row, col0 + p) * SB + sk);
            if constexpr (SOFTMAX) {
                float m = mrun[p];
                for (int kx = 0; kx < K; ++kx) m = fmaxf(m, Elem<T>::one(zr + kx));
                const float sc = exp2f((mrun[p] - m) * kLog2e);   // 0 on the first row
                mrun[p] = m;
                const float ml = m * kLog2e;
                float srow = 0.f;
#pragma unroll
                for (int kx = 0; kx < K; ++kx) {
                    const float e = exp2f(fmaf(Elem<T>::one(zr + kx), kLog2e, -ml));
                    srow += e;
                    put_w(p, kx, e);
                }
                ssum[p] = fmaf(ssum[p], sc, srow);
#pragma unroll
                for (int i = 0; i < CPT; ++i) acc[p][i] *= sc;
            } else {
#pragma unroll
                for (int kx = 0; kx < K; ++kx) put_w(p, kx, Elem<T>::one(zr + kx));
            }
        }

        // slide along the window row (row + ky) over columns col0 .. col0 + K + P - 2
        const unsigned char* xrow = xs + (row + ky) * a.row_bytes;
#pragma unroll
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
                if (kx >= 0 && kx < K) {
                    if constexpr (KT > 0) axpy<CPT>(acc[p], wreg[p][kx], f);
                    else axpy<CPT>(acc[p], wk[kx * wstride + p], f);
                }
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
