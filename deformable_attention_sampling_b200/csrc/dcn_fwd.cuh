// DCNv3 / DCNv4 deformable sampling-aggregation forward, sm_100a SIMT kernel.
//
// Operator ("InternImage: Deformable Convolutions at Scale" ch.1-4; "DCNv4",
// "Why Is Sampling Just 9 Points Still Slow?" and "1. Remove Softmax"):
//   out[n,oy,ox,g*D+c] = sum_k m[g,k] * bilinear(x[n,:,:,g*D+c], p0 + p_k + dp[g,k])
// with zero padding outside the map and m either used as given (DCNv4) or
// soft-maxed over the K taps of the group (DCNv3).
//
// Work decomposition
//   item  = one (output pixel, group) pair; items are numbered pixel-major,
//           group-minor: the memory order of offset, mask and out.  TPI = D/CPT
//           threads serve an item, each owning CPT consecutive channels (CPT *
//           sizeof(T) = VB <= 32 bytes: one 256-bit load per corner).
//   run   = 32/TPI consecutive items of one output row, served by one warp.  A
//           run is contiguous in offset, mask and out.
//   tile  = kDcnWarps runs at the same position in consecutive output rows.  A
//           CTA sweeps a contiguous range of tiles, ordered along the row, so
//           its gathers reuse the L1 lines its neighbours brought in.
//
// Per run the warp copies the run's offsets and masks (two contiguous spans)
// into its own slice of shared memory with coalesced 16-byte loads and then
// syncs only itself; there is no CTA-wide barrier.  Per tap a thread splits
// the offset into floor and fraction (exact for 16-bit inputs), forms per-axis
// weights that are zero for corners outside the map, and issues four
// unconditional vector loads whose coordinates are clamped into the map (a
// clamped corner has weight 0, so its data never contributes).  One warp of
// each CTA bulk-prefetches into L2 the x rows of the CTA's next tiles, so that
// the gathers' L1 misses find their data in L2 instead of HBM.
// Channels accumulate in float32 with packed FFMA2; the result is rounded once
// and stored with one streaming vector store.
//
// The sampler uses no tensor cores: the work is a gather and a weighted sum,
// not a contraction.  The binding limit is the SM's L1 data path for
// scattered 32-byte gathers.  Only the FUSED variant's front end (the merged
// offset / mask linear) is a contraction, and it runs on the tensor cores.
#pragma once

#include <type_traits>

#include "common.cuh"

namespace dcnb {

constexpr int kDcnMaxWarps = 24;             // warps per CTA = runs per tile, at most
constexpr int kDcnMaxThreads = 32 * kDcnMaxWarps;
// Offset floors are clamped to +-kBigCoord before the integer conversion; a
// tap that far out has all four corners outside every supported map
// (H, W <= 2^16), and fminf / fmaxf map a NaN offset to the bound.
constexpr float kBigCoord = 4194304.0f;      // 2^22

struct DcnArgs {
    const void* x;
    const void* offset;
    const void* mask;
    void* out;
    int H, W, C, G, D;
    int kh, kw, K;
    int stride, pad, dil;
    int Ho, Wo;
    int tpi;                  // threads per item
    int run_items;            // items per warp run (32 / tpi)
    int runs_per_row;         // ceil(Wo * G / run_items)
    int tile_h;               // output rows per tile
    int tile_w;               // runs per tile row; the CTA has tile_h * tile_w warps
    int tiles_x;              // ceil(runs_per_row / tile_w)
    int tiles_per_image;      // ceil(Ho / tile_h) * tiles_x
    int num_tiles;            // N * tiles_per_image
    int stage_elems;          // staged mask elements per warp (run_items * K); 0 = unstaged
    int prefetch;             // 1: bulk-prefetch upcoming tiles' x rows into L2
    FastDiv div_G, div_tpi, div_tile_w, div_tiles_x, div_tiles_per_image;
    uint32_t pix_bytes;       // C * sizeof(T): byte stride between neighbouring pixels
    uint32_t row_bytes;       // W * C * sizeof(T)
    long long img_bytes;      // H * W * C * sizeof(T)
    // fused front end only: the merged offset / mask linear
    const void* w_om;         // [J][C], J = G * K * 3 (offsets in [G][K][2] order, then masks)
    const void* b_om;         // [J] or null
    int J;
    unsigned int* flags;      // status word (device), or null
    long long x_bytes;        // bytes of x and of out (bounds of the debug library's checks)
    long long out_bytes;
};

// ---------------------------------------------- fused DCNv4 front end ----
//
// "DCNv4" note, "1. Remove Softmax": one linear layer gives every location its
// G*K offset pairs and G*K modulation scalars.  In the fused kernel each warp
// computes them for its run's pixels on the tensor cores (mma.sync m16n8k16,
// 16-bit inputs, float32 accumulation: a 16-pixel x 8-output tile per
// instruction) straight into its shared slice, in float32, so the offsets and
// masks never travel through HBM and are never rounded to 16 bits.

template <typename T>
__device__ __forceinline__ void mma_16816(float* c, const uint32_t* a, uint32_t b0, uint32_t b1);

template <>
__device__ __forceinline__ void mma_16816<__half>(float* c, const uint32_t* a, uint32_t b0,
                                                  uint32_t b1) {
    asm volatile("mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 "
                 "{%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, {%0,%1,%2,%3};"
                 : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
                 : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

template <>
__device__ __forceinline__ void mma_16816<__nv_bfloat16>(float* c, const uint32_t* a, uint32_t b0,
                                                         uint32_t b1) {
    asm volatile("mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 "
                 "{%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, {%0,%1,%2,%3};"
                 : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
                 : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

template <>
__device__ __forceinline__ void mma_16816<float>(float*, const uint32_t*, uint32_t, uint32_t) {}

// Row stride (elements) of the staged weight matrix: C plus 8, so that the
// eight rows a B fragment reads start in different banks.
__host__ __device__ inline int fused_w_stride(int C) { return C + 8; }

// om[pixel][j] = sum_c W[j][c] x[pixel][c] + b[j] for the npix pixels of one
// run (row `xrow`, first pixel pix0), written to s_off[pixel * 2GK + j]
// (j < 2GK) and s_mask[pixel * GK + j - 2GK].  Ws: staged W (rows padded to
// a multiple of 16 with zeros), bs: bias.  All 32 lanes take part.
constexpr int kFusedMaxKSteps = 8;   // C <= 128: the A fragments of a run stay in registers

template <typename T>
__device__ __forceinline__ void fused_front_end(const T* xrow, int pix0, int npix, int C, int J,
                                                int GK, const T* Ws, const float* bs,
                                                float* s_off, float* s_mask, int lane) {
    const int gid = lane >> 2, tig = lane & 3;
    const int WS = fused_w_stride(C);
    const int G2K = 2 * GK;
    const int KS = C >> 4;
    for (int m0 = 0; m0 < npix; m0 += 16) {
        const int r0 = m0 + gid, r1 = m0 + gid + 8;           // this lane's two pixel rows
        // the run's A fragments for every k-step, loaded once
        uint32_t afr[kFusedMaxKSteps][4];
        {
            const T* x0 = xrow + (long long)(pix0 + r0) * C + 2 * tig;
            const T* x1 = xrow + (long long)(pix0 + r1) * C + 2 * tig;
#pragma unroll
            for (int ks = 0; ks < kFusedMaxKSteps; ++ks) {
                afr[ks][0] = afr[ks][1] = afr[ks][2] = afr[ks][3] = 0u;
                if (ks < KS) {
                    if (r0 < npix) {
                        afr[ks][0] = *reinterpret_cast<const uint32_t*>(x0 + ks * 16);
                        afr[ks][2] = *reinterpret_cast<const uint32_t*>(x0 + ks * 16 + 8);
                    }
                    if (r1 < npix) {
                        afr[ks][1] = *reinterpret_cast<const uint32_t*>(x1 + ks * 16);
                        afr[ks][3] = *reinterpret_cast<const uint32_t*>(x1 + ks * 16 + 8);
                    }
                }
            }
        }
        // two 8-output tiles per step: independent accumulator chains
        for (int n0 = 0; n0 < J; n0 += 16) {
            float c[2][4] = {{0.f, 0.f, 0.f, 0.f}, {0.f, 0.f, 0.f, 0.f}};
            const T* w0 = Ws + (n0 + gid) * WS + 2 * tig;
            const T* w1 = w0 + 8 * WS;
#pragma unroll
            for (int ks = 0; ks < kFusedMaxKSteps; ++ks) {
                if (ks < KS) {
                    mma_16816<T>(c[0], afr[ks], *reinterpret_cast<const uint32_t*>(w0 + ks * 16),
                                 *reinterpret_cast<const uint32_t*>(w0 + ks * 16 + 8));
                    mma_16816<T>(c[1], afr[ks], *reinterpret_cast<const uint32_t*>(w1 + ks * 16),
                                 *reinterpret_cast<const uint32_t*>(w1 + ks * 16 + 8));
                }
            }
            // epilogue: c[t][0..1] row r0, c[t][2..3] row r1, outputs j and j + 1
#pragma unroll
            for (int t = 0; t < 2; ++t) {
                const int j = n0 + 8 * t + 2 * tig;
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    const int r = e < 2 ? r0 : r1;
                    const int jj = j + (e & 1);
                    if (r < npix && jj < J) {
                        const float v = c[t][e] + bs[jj];
                        if (jj < G2K) s_off[r * G2K + jj] = v;
                        else s_mask[r * GK + (jj - G2K)] = v;
                    }
                }
            }
        }
    }
}

// Copy `elems` elements of T from global `src` to shared `dst` with the lanes
// of one warp (widest access the addresses and size allow; streaming loads).
template <typename T>
__device__ __forceinline__ void warp_stage(T* dst, const T* src, int elems, int lane) {
    const int nbytes = elems * (int)sizeof(T);
    const uintptr_t a = (uintptr_t)src | (uintptr_t)dst | (uintptr_t)nbytes;
    if ((a & 15) == 0) {
        const uint4* s = reinterpret_cast<const uint4*>(src);
        uint4* d = reinterpret_cast<uint4*>(dst);
        for (int i = lane; i < (nbytes >> 4); i += 32) {
            uint4 v;
            asm("ld.global.nc.L1::no_allocate.v4.u32 {%0,%1,%2,%3}, [%4];"
                : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w) : "l"(s + i));
            d[i] = v;
        }
    } else if ((a & 7) == 0) {
        const uint2* s = reinterpret_cast<const uint2*>(src);
        uint2* d = reinterpret_cast<uint2*>(dst);
        for (int i = lane; i < (nbytes >> 3); i += 32) {
            uint2 v;
            asm("ld.global.nc.L1::no_allocate.v2.u32 {%0,%1}, [%2];"
                : "=r"(v.x), "=r"(v.y) : "l"(s + i));
            d[i] = v;
        }
    } else if ((a & 3) == 0) {
        const uint32_t* s = reinterpret_cast<const uint32_t*>(src);
        uint32_t* d = reinterpret_cast<uint32_t*>(dst);
        for (int i = lane; i < (nbytes >> 2); i += 32) d[i] = __ldg(s + i);
    } else {
        const unsigned short* s = reinterpret_cast<const unsigned short*>(src);
        unsigned short* d = reinterpret_cast<unsigned short*>(dst);
        for (int i = lane; i < (nbytes >> 1); i += 32) d[i] = __ldg(s + i);
    }
}

// Tiles ahead of the current one whose x rows are prefetched into L2, and the
// margin (pixels) added around a tile's undeformed window for the offsets.
constexpr int kPrefetchAhead = 2;
constexpr int kPrefetchMargin = 4;

// A tile's batch item, first output row and first run (tiles are numbered
// image-major, then band of tile_h rows, then tile_w runs along the row).
struct TileCoord {
    int n, oy0, run0;
};

__device__ __forceinline__ TileCoord decode_tile(const DcnArgs& a, int tile) {
    const int n = (int)a.div_tiles_per_image.div((uint32_t)tile);
    const int rem = tile - n * a.tiles_per_image;
    const int band = (int)a.div_tiles_x.div((uint32_t)rem);
    const int tx = rem - band * a.tiles_x;
    return TileCoord{n, band * a.tile_h, tx * a.tile_w};
}

// Bulk-prefetch into L2 the rows of x that `tile` gathers from (its output
// rows' window plus a margin for the offsets), one contiguous span per input
// row, issued by the lanes of one warp.  A prefetch is only a hint: it moves
// no data into the kernel and changes no result.  Requires 16-byte aligned
// x rows and pixels (checked on the host).
__device__ __forceinline__ void prefetch_tile_x(const DcnArgs& a, int tile, int lane) {
    if (tile >= a.num_tiles) return;
    const TileCoord tc = decode_tile(a, tile);
    const int n = tc.n;
    const int oy0 = tc.oy0;
    const int oy1 = min(oy0 + a.tile_h, a.Ho) - 1;
    const int i0 = tc.run0 * a.run_items;
    const int i1 = min(i0 + a.tile_w * a.run_items, a.Wo * a.G) - 1;
    const int ox0 = (int)a.div_G.div((uint32_t)i0), ox1 = (int)a.div_G.div((uint32_t)i1);
    const int y_lo = max(oy0 * a.stride - a.pad - kPrefetchMargin, 0);
    const int y_hi = min(oy1 * a.stride - a.pad + (a.kh - 1) * a.dil + kPrefetchMargin, a.H - 1);
    const int x_lo = max(ox0 * a.stride - a.pad - kPrefetchMargin, 0);
    const int x_hi = min(ox1 * a.stride - a.pad + (a.kw - 1) * a.dil + kPrefetchMargin, a.W - 1);
    if (y_lo > y_hi || x_lo > x_hi) return;
    const uint32_t span = (uint32_t)(x_hi - x_lo + 1) * a.pix_bytes;
    const char* base = static_cast<const char*>(a.x) + (long long)n * a.img_bytes +
                       (long long)x_lo * a.pix_bytes;
    for (int y = y_lo + lane; y <= y_hi; y += 32) {
        const char* p = base + (long long)y * a.row_bytes;
        asm volatile("cp.async.bulk.prefetch.L2.global [%0], %1;" :: "l"(p), "r"(span)
                     : "memory");
    }
}

// One tap of one item: the four corner weights (zero for a corner outside the
// map) and the byte offsets, within the image, of the four corners to load
// (coordinates clamped into the map, so every load is in bounds).
struct TapGeom {
    uint32_t off[4];
    float w[4];
};

__device__ __forceinline__ TapGeom tap_geometry(const DcnArgs& a, int bxk, int byk, float dx,
                                                float dy, float m) {
    TapGeom t;
    float fx = floorf(dx), fy = floorf(dy);
    const float ax = dx - fx, ay = dy - fy;
    fx = fminf(fmaxf(fx, -kBigCoord), kBigCoord);
    fy = fminf(fmaxf(fy, -kBigCoord), kBigCoord);
    const int x0 = bxk + (int)fx, y0 = byk + (int)fy;
    const int x1 = x0 + 1, y1 = y0 + 1;
    const bool vx0 = (unsigned)x0 < (unsigned)a.W, vx1 = (unsigned)x1 < (unsigned)a.W;
    const bool vy0 = (unsigned)y0 < (unsigned)a.H, vy1 = (unsigned)y1 < (unsigned)a.H;
    // per-axis weights, zero for a corner outside the map
    const float wx0 = vx0 ? 1.f - ax : 0.f, wx1 = vx1 ? ax : 0.f;
    const float wy0 = vy0 ? (1.f - ay) * m : 0.f, wy1 = vy1 ? ay * m : 0.f;
    t.w[0] = wx0 * wy0;
    t.w[1] = wx1 * wy0;
    t.w[2] = wx0 * wy1;
    t.w[3] = wx1 * wy1;
    // coordinates clamped into the map: every load is in bounds
    const uint32_t cx0 = vx0 ? (uint32_t)x0 : 0u, cx1 = vx1 ? (uint32_t)x1 : 0u;
    const uint32_t cy0 = vy0 ? (uint32_t)y0 : 0u, cy1 = vy1 ? (uint32_t)y1 : 0u;
    const uint32_t r0 = cy0 * a.row_bytes, r1 = cy1 * a.row_bytes;
    const uint32_t c0 = cx0 * a.pix_bytes, c1 = cx1 * a.pix_bytes;
    t.off[0] = r0 + c0;
    t.off[1] = r0 + c1;
    t.off[2] = r1 + c0;
    t.off[3] = r1 + c1;
    return t;
}

// KF > 0: a fixed KF x KF window, whose taps are fully unrolled (tap indices,
// kernel offsets and shared-memory addresses fold into constants; measured
// 10% faster for 3 x 3).  KF = 0: any window, taps in a rolled loop.
// FUSED: offsets and masks come from the merged linear of the DCNv4 front end
// (fused_front_end, float32 in shared memory) instead of global tensors;
// stride 1, runs aligned to whole pixels (checked on the host).
template <typename T, int VB, bool SOFTMAX, int KF = 0, bool FUSED = false>
__global__ void __launch_bounds__(kDcnMaxThreads, 1) dcn_fwd_kernel(const DcnArgs a) {
    constexpr int UNROLL = KF ? KF * KF : 1;
    constexpr int CPT = VB / (int)sizeof(T);
    constexpr int NW = VB >= 4 ? VB / 4 : 1;
    using OT = typename std::conditional<FUSED, float, T>::type;   // staged offset / mask type
    extern __shared__ __align__(16) unsigned char smem[];

    const int kh = KF ? KF : a.kh;
    const int kw = KF ? KF : a.kw;
    const int K = kh * kw;
    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    const bool staged = FUSED || a.stage_elems > 0;
    // fused: the staged weight matrix and bias come first
    unsigned char* wsm = smem;
    int front = 0;
    if constexpr (FUSED) {
        const int rows = (a.J + 15) & ~15;
        front = ((rows * fused_w_stride(a.C) * (int)sizeof(T) + 15) & ~15) + ((a.J * 4 + 15) & ~15);
    }
    // this warp's slice of shared memory: offsets, then masks
    const int off_slice = ((2 * a.stage_elems * (int)sizeof(OT)) + 15) & ~15;
    const int slice = off_slice + ((a.stage_elems * (int)sizeof(OT) + 15) & ~15);
    OT* s_off = reinterpret_cast<OT*>(smem + front + warp * slice);
    OT* s_mask = reinterpret_cast<OT*>(smem + front + warp * slice + off_slice);
    if constexpr (FUSED) {
        // stage W (rows padded to a multiple of 16 with zeros) and the bias
        const int rows = (a.J + 15) & ~15;
        const int WS = fused_w_stride(a.C);
        T* Ws = reinterpret_cast<T*>(wsm);
        const T* wg = static_cast<const T*>(a.w_om);
        for (int e = threadIdx.x; e < rows * a.C; e += blockDim.x) {
            const int j = e / a.C, c = e - j * a.C;
            Ws[j * WS + c] = j < a.J ? wg[e] : Elem<T>::from(0.f);
        }
        float* bs = reinterpret_cast<float*>(wsm + ((rows * WS * (int)sizeof(T) + 15) & ~15));
        for (int j = threadIdx.x; j < a.J; j += blockDim.x)
            bs[j] = a.b_om ? Elem<T>::one(static_cast<const T*>(a.b_om) + j) : 0.f;
        __syncthreads();
    }

    const int li = (int)a.div_tpi.div((uint32_t)lane);     // item within the run
    const int chunk = lane - li * a.tpi;                    // channel chunk of the item
    const int row_items = a.Wo * a.G;
    const int warp_row = (int)a.div_tile_w.div((uint32_t)warp);   // this warp's row in a tile
    const int warp_col = warp - warp_row * a.tile_w;               // and its run

    // contiguous, balanced range of tiles for this CTA
    const int t_begin = (int)(((long long)a.num_tiles * blockIdx.x) / gridDim.x);
    const int t_end = (int)(((long long)a.num_tiles * (blockIdx.x + 1)) / gridDim.x);

    if (a.prefetch && warp == 0) {
        for (int t = t_begin; t < min(t_begin + kPrefetchAhead, t_end); ++t)
            prefetch_tile_x(a, t, lane);
    }

    for (int tile = t_begin; tile < t_end; ++tile) {
        if (a.prefetch && warp == 0 && tile + kPrefetchAhead < t_end)
            prefetch_tile_x(a, tile + kPrefetchAhead, lane);
        const TileCoord tc = decode_tile(a, tile);
        const int n = tc.n;
        const int oy = tc.oy0 + warp_row;
        const int run = tc.run0 + warp_col;
        if (oy >= a.Ho || run >= a.runs_per_row) continue;   // warp-uniform
        const int i0 = run * a.run_items;                    // first item of the run in its row
        const int nitems = min(a.run_items, row_items - i0);
        const long long item_base = ((long long)n * a.Ho + oy) * row_items + i0;

        const OT* offp;
        const OT* maskp;
        if (staged) {
            __syncwarp();                                    // previous run's reads are done
            if constexpr (FUSED) {
                const int rows = (a.J + 15) & ~15;
                const T* Ws = reinterpret_cast<const T*>(wsm);
                const float* bs = reinterpret_cast<const float*>(
                    wsm + ((rows * fused_w_stride(a.C) * (int)sizeof(T) + 15) & ~15));
                const T* xrow = static_cast<const T*>(a.x) + ((long long)n * a.H + oy) * a.W * a.C;
                fused_front_end<T>(xrow, i0 / a.G, (nitems + a.G - 1) / a.G, a.C, a.J, a.G * K,
                                   Ws, bs, s_off, s_mask, lane);
            } else {
                warp_stage(s_off, static_cast<const T*>(a.offset) + item_base * K * 2,
                           nitems * K * 2, lane);
                warp_stage(s_mask, static_cast<const T*>(a.mask) + item_base * K, nitems * K,
                           lane);
            }
            __syncwarp();
            offp = s_off + li * K * 2;
            maskp = s_mask + li * K;
        } else {
            offp = reinterpret_cast<const OT*>(static_cast<const T*>(a.offset) +
                                               (item_base + li) * K * 2);
            maskp = reinterpret_cast<const OT*>(static_cast<const T*>(a.mask) +
                                                (item_base + li) * K);
        }
        if (li >= nitems) continue;

        const int item_in_row = i0 + li;
        const int ox = (int)a.div_G.div((uint32_t)item_in_row);
        const int g = item_in_row - ox * a.G;
        const char* xb = static_cast<const char*>(a.x) + (long long)n * a.img_bytes +
                         (long long)(g * a.D + chunk * CPT) * (int)sizeof(T);
        const int bx = ox * a.stride - a.pad;
        const int by = oy * a.stride - a.pad;

        // DCNv3: stable softmax of the group's K logits
        float zmax = 0.f, inv_sum = 1.f;
        if constexpr (SOFTMAX) {
            zmax = Elem<OT>::one(maskp);
            for (int k = 1; k < K; ++k) zmax = fmaxf(zmax, Elem<OT>::one(maskp + k));
            float s = 0.f;
            for (int k = 0; k < K; ++k) s += expf(Elem<OT>::one(maskp + k) - zmax);
            inv_sum = 1.f / s;
        }
        auto modulation = [&](int k) {
            const float z = Elem<OT>::one(maskp + k);
            if constexpr (SOFTMAX) return expf(z - zmax) * inv_sum;
            return z;
        };

        float acc[CPT];
#pragma unroll
        for (int i = 0; i < CPT; ++i) acc[i] = 0.f;

        // Rolling corner pipeline over the taps (k = ix * kh + iy, walked with
        // iy fastest): the geometry of tap k+1 is computed while tap k's four
        // loads are in flight, and each corner's registers are refilled with
        // tap k+1's corner right after they are consumed.  Four loads stay in
        // flight with the registers of one tap.
        uint32_t v[4][NW];
        float w[4];
        int nix = 0, niy = 0;            // the next tap to prepare
        auto geometry = [&]() {
            const int k = nix * kh + niy;
            float dx, dy;
            load_pair<OT>(offp + 2 * k, dx, dy);
            const TapGeom t = tap_geometry(a, bx + nix * a.dil, by + niy * a.dil, dx, dy,
                                           modulation(k));
            if (++niy == kh) {
                niy = 0;
                ++nix;
            }
            return t;
        };
        // a corner load (clamped into the map, so always inside x; the debug
        // library checks it and reads zeros instead when it is not)
        const char* x_lo = static_cast<const char*>(a.x);
        auto corner = [&](uint32_t off, uint32_t* dst) {
            const char* src = xb + off;
            if (DCN_IN_BOUNDS(src >= x_lo && src + VB <= x_lo + a.x_bytes, a.flags)) {
                load_vec<VB>(src, dst);
            } else {
#pragma unroll
                for (int i = 0; i < NW; ++i) dst[i] = 0u;
            }
        };
        {
            const TapGeom t0 = geometry();
#pragma unroll
            for (int c = 0; c < 4; ++c) {
                corner(t0.off[c], v[c]);
                w[c] = t0.w[c];
            }
        }
#pragma unroll UNROLL
        for (int k = 0; k < K; ++k) {
            const bool more = k + 1 < K;
            TapGeom tn;
            if (more) tn = geometry();
            float f[CPT];
#pragma unroll
            for (int c = 0; c < 4; ++c) {
                widen<T, CPT>(v[c], f);
                axpy<CPT>(acc, w[c], f);
                if (more) corner(tn.off[c], v[c]);
            }
            if (more) {
#pragma unroll
                for (int c = 0; c < 4; ++c) w[c] = tn.w[c];
            }
        }

        uint32_t o[NW];
        narrow<T, CPT>(acc, o);
        char* ob = static_cast<char*>(a.out) +
                   ((item_base + li) * a.D + chunk * CPT) * (int)sizeof(T);
        const char* o_lo = static_cast<const char*>(a.out);
        if (DCN_IN_BOUNDS(ob >= o_lo && ob + VB <= o_lo + a.out_bytes, a.flags))
            store_vec<VB>(ob, o);
    }
}

}  // namespace dcnb
