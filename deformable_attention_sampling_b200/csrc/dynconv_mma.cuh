// Dynamic local aggregation (the ContMix core) on the tensor cores.
//
// Same operator as dynconv_fwd_kernel ("OverLoCK" note, "ContMix: Put the
// Whole Image into the Kernel", steps 4-5), for 16-bit data and the compiled
// kernel sizes.  One kernel row ky of 16 consecutive outputs of an image row
// is a matrix product:
//   out[i][c] += sum_j A_ky[i][j] * X_ky[j][c]      i < 16 outputs, c < 16 channels
//   A_ky[i][j] = weight(i, ky, kx = j - i)  for 0 <= j - i < K, else 0
//   X_ky[j][c] = x[y + ky - K/2][x0 + j - K/2][c]   (the window row)
// A is banded: row i holds its location's K numbers starting at column i, so
// j < 16 + K - 1 <= 32 and two k-steps of mma.m16n8k16 cover it.  Each
// location's weights are split into a 16-bit high part and the 16-bit
// rounding of the remainder; the two products are accumulated in float32, so
// the weights enter the sum to about 2^-22 (f16) / 2^-17 (bf16) of their
// value, and x enters exactly.
//
// A is built in shared memory (its zeros are written once: the band of every
// row sits at the same columns for every ky) and read with ldmatrix; the
// window rows are staged as in the SIMT kernel and read with ldmatrix.trans
// as the column-major B operand.  These operands are assembled per warp in
// registers and shared memory, which is why this path uses the warp-level
// mma.sync: a tcgen05 product would read A from shared memory or TMEM at
// 128 rows x 32 columns per k-range, six tenths of it zeros, and for N = 16
// channels those operand reads, not the arithmetic, would set its time.
//
// Work decomposition (one CTA = 8 output rows x 32 columns of one group and
// one 16-channel chunk; 8 warps):
//   warp  = one output row, as two blocks of 16 columns;
//   lane  = one location (column) of the row for the softmax: the numbers of
//           kernel row ky + 1 of the warp's 32 locations are copied into
//           their slots (8-byte cp.async; at K = 13 four lanes per location,
//           at K = 7 each lane its own; warp barriers only) while each lane
//           reads its location's row ky, updates its running maximum and sum
//           (online softmax, as the SIMT kernel), and writes its band of A
//           (high and low parts) for both k-steps;
//   mma   = per block and k-step: A (ldmatrix.x4, high and low), B
//           (ldmatrix.x4.trans: 16 window columns x 16 channels), four
//           m16n8k16 products into float32 accumulators (16 per lane).
// The accumulators of a location are scaled when its running maximum grows
// and divided by its sum at the end.
#pragma once

#include <cuda_bf16.h>
#include <cuda_fp16.h>

#include "dynconv_fwd.cuh"

namespace dcnb {

constexpr int kMmaRows = 8;          // output rows per CTA (one warp each)
constexpr int kMmaCols = 32;         // output columns per CTA (two blocks of 16)
constexpr int kMmaWinCols = 48;      // window columns staged: both blocks' two k-steps
constexpr int kMmaThreads = 32 * kMmaRows;
constexpr int kMmaTileBytes = 16 * 32;                 // one 16 x 16 16-bit tile
constexpr int kMmaWarpTiles = 2 * 2 * 2;               // block x k-step x (high, low)
// the second block's four tiles sit 64 bytes further: with that shift the
// 32 lanes' band stores of every word fall in 32 distinct banks
constexpr int kMmaBlockPad = 64;
constexpr int kMmaWarpBytes = kMmaWarpTiles * kMmaTileBytes + kMmaBlockPad;

// Shared-memory offset of tile (block bb, k-step s, part: 0 high, 1 low).
__host__ __device__ inline int mma_tile_offset(int bb, int s, int part) {
    return ((bb * 2 + s) * 2 + part) * kMmaTileBytes + bb * kMmaBlockPad;
}

// 8-byte units of a location's slot for one kernel row in the raw buffer:
// its K numbers from the 8-byte unit holding the first, rounded up to an odd
// count, so that the 8-byte loads of 16 lanes (one wavefront) hit distinct
// bank pairs.
__host__ __device__ inline int dyn_mma_slot_units(int K) {
    const int u = (2 * K + 6 + 7) / 8;
    return u | 1;
}
__host__ __device__ inline int dyn_mma_slot_words(int K) { return 2 * dyn_mma_slot_units(K); }

// Byte offset of element (row i, column jj) of a 16 x 16 tile of 16-bit
// values: rows of 32 bytes, the two 16-byte halves of rows 4-7 and 12-15
// swapped, so that the 8 row addresses of an ldmatrix fall in distinct banks.
__host__ __device__ inline int mma_tile_byte(int i, int jj) {
    return i * 32 + ((((jj >> 3) ^ (i >> 2)) & 1) << 4) + (jj & 7) * 2;
}

template <typename T>
struct MmaOps;

template <>
struct MmaOps<__half> {
    // (lo, hi) -> one word, lo in the low 16 bits
    static __device__ __forceinline__ uint32_t pack(float lo, float hi) {
        __half2 h = __floats2half2_rn(lo, hi);
        return *reinterpret_cast<uint32_t*>(&h);
    }
    static __device__ __forceinline__ float2 unpack(uint32_t w) {
        __half2 h = *reinterpret_cast<__half2*>(&w);
        return __half22float2(h);
    }
    static __device__ __forceinline__ void mma(float* d, const uint32_t* a, uint32_t b0,
                                               uint32_t b1) {
        asm volatile(
            "mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 "
            "{%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, {%0,%1,%2,%3};"
            : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
            : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
    }
};

template <>
struct MmaOps<__nv_bfloat16> {
    static __device__ __forceinline__ uint32_t pack(float lo, float hi) {
        __nv_bfloat162 h = __floats2bfloat162_rn(lo, hi);
        return *reinterpret_cast<uint32_t*>(&h);
    }
    static __device__ __forceinline__ float2 unpack(uint32_t w) {
        // bf16 is the upper half of a float32
        return make_float2(__uint_as_float(w << 16), __uint_as_float(w & 0xffff0000u));
    }
    static __device__ __forceinline__ void mma(float* d, const uint32_t* a, uint32_t b0,
                                               uint32_t b1) {
        asm volatile(
            "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 "
            "{%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, {%0,%1,%2,%3};"
            : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
            : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
    }
};

__device__ __forceinline__ void ldsm_x4(uint32_t addr, uint32_t* r) {
    asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0,%1,%2,%3}, [%4];"
                 : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]) : "r"(addr) : "memory");
}

__device__ __forceinline__ void ldsm_x4_trans(uint32_t addr, uint32_t* r) {
    asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0,%1,%2,%3}, [%4];"
                 : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]) : "r"(addr) : "memory");
}

// 2^x by the hardware approximation (relative error about 2^-22; 2^-inf = 0)
__device__ __forceinline__ float ex2_approx(float x) {
    float y;
    asm("ex2.approx.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}

__device__ __forceinline__ void sts32(uint32_t addr, uint32_t v) {
    asm volatile("st.shared.b32 [%0], %1;" :: "r"(addr), "r"(v) : "memory");
}

// Shared-memory bytes of the tensor-core kernel for kernel size K: the window
// (rows of dyn_row_bytes(kMmaWinCols)), two raw buffers of kernel-row numbers
// and each warp's A tiles.
__host__ __device__ inline int dyn_mma_raw_bytes(int K) {
    return ((2 * kMmaRows * kMmaCols * dyn_mma_slot_words(K) + 1) * 4 + 15) & ~15;
}

__host__ __device__ inline int dyn_mma_smem(int K) {
    return (kMmaRows + K - 1) * dyn_row_bytes(kMmaWinCols) + dyn_mma_raw_bytes(K) +
           kMmaRows * kMmaWarpBytes;
}

// 8-byte asynchronous global -> shared copy of src_bytes (0..8) bytes, zero-filled.
__device__ __forceinline__ void cp_async8(uint32_t dst, const void* src, uint32_t src_bytes) {
    asm volatile("cp.async.ca.shared.global [%0], [%1], 8, %2;" :: "r"(dst), "l"(src),
                 "r"(src_bytes) : "memory");
}

__device__ __forceinline__ uint2 lds64(uint32_t addr) {
    uint2 v;
    asm volatile("ld.shared.v2.u32 {%0,%1}, [%2];" : "=r"(v.x), "=r"(v.y) : "r"(addr) : "memory");
    return v;
}

template <typename T, bool SOFTMAX, int K>
__global__ void __launch_bounds__(kMmaThreads, 2) dynconv_mma_kernel(const DynArgs a) {
    static_assert(sizeof(T) == 2, "16-bit data");
    static_assert(K % 2 == 1 && K <= 17, "two k-steps of 16 columns cover the band");
    constexpr int es = 2;
    constexpr int R = K / 2;
    constexpr int NWORD = (K + 1) / 2;   // words of a row's band
    constexpr float kLog2e = 1.4426950408889634f;
    using Ops = MmaOps<T>;
    extern __shared__ __align__(16) unsigned char smem[];
    constexpr int NP = kMmaRows * kMmaCols;   // locations of the tile
    const int SW = dyn_mma_slot_words(K);
    unsigned char* xs = smem;
    uint32_t* raw = reinterpret_cast<uint32_t*>(smem + a.xs_bytes);   // two buffers of NP slots
    unsigned char* at = smem + a.xs_bytes + dyn_mma_raw_bytes(K);

    const int tid = threadIdx.x;
    const int warp = tid >> 5, lane = tid & 31;

    // tile: blockIdx.x = (((n * tiles_y + ty) * tiles_x + tx) * G + g) * chunks + q
    int blk = blockIdx.x;
    const int q = blk % a.chunks;
    blk /= a.chunks;
    const int g = blk % a.G;
    blk /= a.G;
    const int tx = blk % a.tiles_x;
    blk /= a.tiles_x;
    const int ty = blk % a.tiles_y;
    const int n = blk / a.tiles_y;
    const int y0 = ty * kMmaRows, x0 = tx * kMmaCols;
    const long long ch0 = (long long)g * a.D + (long long)q * 16;   // first channel
    const long long pix_bytes = (long long)a.C * es;

    // ---- the input window: rows y0 - R .. y0 + 7 + R, columns x0 - R .. x0 - R + 47 ----
    const char* xin = static_cast<const char*>(a.x) + (long long)n * a.H * a.W * pix_bytes +
                      ch0 * es;
    for (int e = tid; e < a.win_rows * kMmaWinCols * 2; e += kMmaThreads) {
        const int half = e & 1;
        const int pix = e >> 1;
        const int wr = pix / kMmaWinCols, wc = pix - wr * kMmaWinCols;
        const int gy = y0 - R + wr, gx = x0 - R + wc;
        const bool inside = (unsigned)gy < (unsigned)a.H && (unsigned)gx < (unsigned)a.W;
        const char* src = inside ? xin + ((long long)gy * a.W + gx) * pix_bytes + half * 16 : xin;
        cp_async16(xs + wr * a.row_bytes + dyn_pixel_byte(wc) + half * 16, src, inside ? 16u : 0u);
    }
    asm volatile("cp.async.commit_group;" ::: "memory");

    // this warp's A tiles (mma_tile_offset); zero once: only the bands are rewritten
    unsigned char* aw = at + warp * kMmaWarpBytes;
    for (int i = lane; i < kMmaWarpBytes / 16; i += 32)
        reinterpret_cast<uint4*>(aw)[i] = make_uint4(0u, 0u, 0u, 0u);
    const uint32_t aw_s = (uint32_t)__cvta_generic_to_shared(aw);
    const uint32_t xs_s = (uint32_t)__cvta_generic_to_shared(xs);

    // raw weights of the tile: location (row, col) starts at wt + row * w_row + col * w_col
    const T* wt = static_cast<const T*>(a.w) +
                  ((((long long)n * a.H + y0) * a.W + x0) * a.G + g) * (K * K);
    const int w_col = a.G * K * K;
    const int w_row = a.W * w_col;
    auto in_map = [&](int row, int col) { return y0 + row < a.H && x0 + col < a.W; };
    // A warp stages the numbers of its own row's 32 locations; each thread then
    // reads those of its own location (warp, lane).  Kernel row ky goes to
    // buffer ky & 1 as 8-byte units from the one holding the row's first
    // number, the last clipped to the row's end.  The 32 locations' rows sit
    // w_col numbers apart in global memory, so a copy instruction whose lanes
    // take one location each touches 32 lines.
    const bool mine = in_map(warp, lane);
    const char* row_w = reinterpret_cast<const char*>(wt + warp * w_row);
    const char* my_w = row_w + (long long)lane * w_col * es;
    const uint32_t row_slot = (uint32_t)__cvta_generic_to_shared(raw) +
                              (uint32_t)(warp * kMmaCols * SW * 4);
    const uint32_t my_slot = row_slot + (uint32_t)(lane * SW * 4);
    // units a kernel row can span (from the 8-byte unit of its first number)
    constexpr int NUC = (2 * K + 6 + 7) / 8;
    // Four units (K = 13): four lanes per location, one unit each, so a copy
    // instruction touches eight locations' lines (247.8 -> 238.4 us per
    // 64 x 56 x 56 x 64 launch).  Three units (K = 7): a lane per location
    // (the packed mapping of 32 x 3 units measured 127.0 against 123.0 us).
    constexpr bool kWarpCopy = NUC >= 4;
    auto copy_row = [&](int ky) {
        if constexpr (!kWarpCopy) {
            // each thread its own location's units
            if (mine) {
                const char* first = my_w + ky * K * es;
                const char* last = first + K * es;
                const char* u8 = reinterpret_cast<const char*>((uintptr_t)first & ~(uintptr_t)7);
                uint32_t dst = my_slot + (uint32_t)((ky & 1) * NP * SW * 4);
                for (; u8 < last; u8 += 8, dst += 8) {
                    const long long left = last - u8;
                    cp_async8(dst, u8, left >= 8 ? 8u : (uint32_t)left);
                }
            }
        } else {
            // UPL lanes per location: copy f of the row's 32 x UPL (location,
            // unit) pairs is location f / UPL, unit f % UPL
            constexpr int UPL = NUC <= 4 ? 4 : 8;
#pragma unroll
            for (int pass = 0; pass < UPL; ++pass) {
                const int f = pass * 32 + lane;
                const int col = f / UPL, unit = f - col * UPL;
                if (in_map(warp, col)) {
                    const char* first = row_w + ((long long)col * w_col + ky * K) * es;
                    const char* last = first + K * es;
                    const char* u8 = reinterpret_cast<const char*>((uintptr_t)first &
                                                                   ~(uintptr_t)7) + 8 * unit;
                    if (u8 < last) {
                        const long long left = last - u8;
                        const uint32_t dst = row_slot + (uint32_t)(col * SW * 4) +
                                             (uint32_t)((ky & 1) * NP * SW * 4) + 8u * unit;
                        cp_async8(dst, u8, left >= 8 ? 8u : (uint32_t)left);
                    }
                }
            }
        }
        asm volatile("cp.async.commit_group;" ::: "memory");
    };

    // ---- softmax role: this lane's location (warp, lane) = block bb, row i ----
    const int skew = (int)((uintptr_t)my_w & 7);
    const int bb_own = lane >> 4, i_own = lane & 15;
    uint32_t waddr[NWORD];   // shared address of band word k in the high tile
#pragma unroll
    for (int k = 0; k < NWORD; ++k) {
        const int j0 = 2 * (i_own >> 1) + 2 * k;   // first column of word k
        waddr[k] = aw_s + (uint32_t)(mma_tile_offset(bb_own, j0 >> 4, 0) +
                                     mma_tile_byte(i_own, j0 & 15));
    }
    // odd rows start their band in the upper half of a word: word k is the
    // upper half of pair k - 1 and the lower half of pair k
    const uint32_t sel = (i_own & 1) ? 0x5432u : 0x7654u;
    float mrun = -INFINITY, ssum = 0.f;

    // ---- product role ----
    const int gq = lane >> 2, tq = lane & 3;
    const uint32_t a_off = (uint32_t)mma_tile_byte(lane & 15, (lane >> 4) * 8);
    const int kb = (lane & 7) + ((lane >> 3) & 1) * 8;   // window column of this lane's B row
    const int nh = lane >> 4;                            // channel half of its B row
    float acc[2][2][4];
#pragma unroll
    for (int bb = 0; bb < 2; ++bb)
#pragma unroll
        for (int nt = 0; nt < 2; ++nt)
#pragma unroll
            for (int i = 0; i < 4; ++i) acc[bb][nt][i] = 0.f;

    // B rows of this lane for (block, k-step): window columns 16 bb + 16 s + kb
    uint32_t boff[2][2];
#pragma unroll
    for (int bb = 0; bb < 2; ++bb)
#pragma unroll
        for (int s = 0; s < 2; ++s)
            boff[bb][s] = (uint32_t)(dyn_pixel_byte(bb * 16 + s * 16 + kb) + nh * 16);

    copy_row(0);
    asm volatile("cp.async.wait_group 0;" ::: "memory");
    __syncthreads();   // the window (every warp's copies) and the zeroed A tiles
#pragma unroll 1
    for (int ky = 0; ky < K; ++ky) {
        // the warp's row ky + 1 in flight while row ky is used; buffer
        // (ky + 1) & 1 was last read at row ky - 1, by every lane of the warp
        // before this barrier
        __syncwarp();
        if (ky + 1 < K) {
            copy_row(ky + 1);
            asm volatile("cp.async.wait_group 1;" ::: "memory");
        } else {
            asm volatile("cp.async.wait_group 0;" ::: "memory");
        }
        __syncwarp();   // every lane's copies of row ky have landed

        // this location's numbers of kernel row ky (0 outside the map)
        float e[2 * NWORD];
        e[2 * NWORD - 1] = 0.f;
        float sc = 1.f;
        if (mine) {
            // the row's numbers start at byte o = (skew + ky K es) & 7 of the slot:
            // load the slot, drop o / 4 words, realign the half-word pairs, widen
            constexpr int NU = (2 * K + 6 + 7) / 8 | 1;   // = dyn_mma_slot_units(K)
            const int o = (skew + ky * K * es) & 7;
            const uint32_t zs = my_slot + (uint32_t)((ky & 1) * NP * SW * 4);
            uint32_t wv[2 * NU];
#pragma unroll
            for (int u = 0; u < NU; ++u) {
                const uint2 v = lds64(zs + 8 * u);
                wv[2 * u] = v.x;
                wv[2 * u + 1] = v.y;
            }
            const bool wshift = o >= 4;
            const uint32_t al = (o & 2) ? 0x5432u : 0x3210u;
            uint32_t wa[NWORD + 1];
#pragma unroll
            for (int k = 0; k <= NWORD; ++k) wa[k] = wshift ? wv[k + 1] : wv[k];
            float z[2 * NWORD];
#pragma unroll
            for (int k = 0; k < NWORD; ++k) {
                const float2 f = Ops::unpack(__byte_perm(wa[k], wa[k + 1], al));
                z[2 * k] = f.x;
                z[2 * k + 1] = f.y;
            }
            if constexpr (SOFTMAX) {
                // maximum as a tree (independent pairs), exponentials with ex2.approx
                float t[K];
#pragma unroll
                for (int kx = 0; kx < K; ++kx) t[kx] = z[kx];
#pragma unroll
                for (int step = 1; step < K; step *= 2)
#pragma unroll
                    for (int kx = 0; kx + step < K; kx += 2 * step)
                        t[kx] = fmaxf(t[kx], t[kx + step]);
                const float m = fmaxf(mrun, t[0]);
                sc = ex2_approx((mrun - m) * kLog2e);   // 0 on the first row
                mrun = m;
                const float ml = m * kLog2e;
                float s0 = 0.f, s1 = 0.f;
#pragma unroll
                for (int kx = 0; kx < K; ++kx) {
                    e[kx] = ex2_approx(fmaf(z[kx], kLog2e, -ml));
                    if (kx & 1) s1 += e[kx];
                    else s0 += e[kx];
                }
                const float srow = s0 + s1;
                ssum = fmaf(ssum, sc, srow);
            } else {
#pragma unroll
                for (int kx = 0; kx < K; ++kx) e[kx] = z[kx];
            }
        } else {
#pragma unroll
            for (int kx = 0; kx < K; ++kx) e[kx] = 0.f;
        }

        // the band of row i_own: high parts, and (softmax) the rounded remainders
        uint32_t prev_h = 0u, prev_l = 0u;
#pragma unroll
        for (int k = 0; k < NWORD; ++k) {
            const uint32_t ph = Ops::pack(e[2 * k], e[2 * k + 1]);
            sts32(waddr[k], __byte_perm(prev_h, ph, sel));
            prev_h = ph;
            if constexpr (SOFTMAX) {
                const float2 hv = Ops::unpack(ph);
                const uint32_t pl = Ops::pack(e[2 * k] - hv.x, e[2 * k + 1] - hv.y);
                sts32(waddr[k] + kMmaTileBytes, __byte_perm(prev_l, pl, sel));
                prev_l = pl;
            }
        }
        __syncwarp();

        // the accumulators of a location follow its running maximum
        if constexpr (SOFTMAX) {
#pragma unroll
            for (int bb = 0; bb < 2; ++bb) {
                const float s_lo = __shfl_sync(0xffffffffu, sc, bb * 16 + gq);
                const float s_hi = __shfl_sync(0xffffffffu, sc, bb * 16 + gq + 8);
#pragma unroll
                for (int nt = 0; nt < 2; ++nt) {
                    acc[bb][nt][0] *= s_lo;
                    acc[bb][nt][1] *= s_lo;
                    acc[bb][nt][2] *= s_hi;
                    acc[bb][nt][3] *= s_hi;
                }
            }
        }

        // products of window row warp + ky
        const uint32_t xrow = xs_s + (uint32_t)((warp + ky) * a.row_bytes);
#pragma unroll
        for (int bb = 0; bb < 2; ++bb) {
#pragma unroll
            for (int s = 0; s < 2; ++s) {
                const uint32_t tile = aw_s + (uint32_t)mma_tile_offset(bb, s, 0);
                uint32_t ah[4], bf[4];
                ldsm_x4(tile + a_off, ah);
                ldsm_x4_trans(xrow + boff[bb][s], bf);
                Ops::mma(acc[bb][0], ah, bf[0], bf[1]);
                Ops::mma(acc[bb][1], ah, bf[2], bf[3]);
                if constexpr (SOFTMAX) {
                    uint32_t al[4];
                    ldsm_x4(tile + kMmaTileBytes + a_off, al);
                    Ops::mma(acc[bb][0], al, bf[0], bf[1]);
                    Ops::mma(acc[bb][1], al, bf[2], bf[3]);
                }
            }
        }
        __syncwarp();   // the A tiles are rewritten for the next kernel row
    }

    // ---- normalise and store: lane (gq, tq) holds rows gq, gq + 8 of each block,
    // channels nt * 8 + 2 tq, +1 ----
    const int oy = y0 + warp;
    char* obase = static_cast<char*>(a.out) + ((long long)n * a.H + oy) * a.W * pix_bytes +
                  (ch0 + 2 * tq) * es;
#pragma unroll
    for (int bb = 0; bb < 2; ++bb) {
        float inv_lo = 1.f, inv_hi = 1.f;
        if constexpr (SOFTMAX) {
            inv_lo = 1.f / __shfl_sync(0xffffffffu, ssum, bb * 16 + gq);
            inv_hi = 1.f / __shfl_sync(0xffffffffu, ssum, bb * 16 + gq + 8);
        }
        const int c_lo = x0 + bb * 16 + gq, c_hi = c_lo + 8;
#pragma unroll
        for (int nt = 0; nt < 2; ++nt) {
            if (oy < a.H && c_lo < a.W)
                *reinterpret_cast<uint32_t*>(obase + (long long)c_lo * pix_bytes + nt * 16) =
                    Ops::pack(acc[bb][nt][0] * inv_lo, acc[bb][nt][1] * inv_lo);
            if (oy < a.H && c_hi < a.W)
                *reinterpret_cast<uint32_t*>(obase + (long long)c_hi * pix_bytes + nt * 16) =
                    Ops::pack(acc[bb][nt][2] * inv_hi, acc[bb][nt][3] * inv_hi);
        }
    }
}

}  // namespace dcnb
