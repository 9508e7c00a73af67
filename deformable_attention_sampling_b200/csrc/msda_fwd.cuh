// Multi-scale deformable attention (MSDeformAttn core) forward, sm_100a SIMT.
//
// Operator ("Deformable DETR: Learn Where to Read", "A learned location can
// fall between cells" and "Mix samples with a per-head budget"):
//   out[n,q,h*D+c] = sum_{l,k} A[n,q,h,l,k] * S_l(value[n, start_l + ., h, c], loc[n,q,h,l,k])
//   S_l(f, u, v): x = u W_l - 1/2, y = v H_l - 1/2; bilinear over the four
//   floor/ceil neighbours, zero outside, no clamping, no renormalisation.
//
// Work decomposition mirrors the DCN kernel:
//   item = one (batch, query, head) triple, numbered in the memory order of
//          loc, attn and out; TPI = D / CPT threads share it, each owning CPT
//          consecutive channels (CPT * sizeof(T) <= 32 bytes: one vector load
//          per corner).
//   run  = 32 / TPI consecutive items served by one warp (at D = 32 fp32: the
//          8 heads of one query).  A run is contiguous in loc, attn and out;
//          the warp stages its run's locations and weights into its own slice
//          of shared memory and syncs only itself.
// Each CTA takes a contiguous range of runs.  Per item the L*K taps run as a
// rolling corner pipeline: the next tap's geometry is computed while the
// current tap's four loads are in flight, and each corner's registers are
// refilled with the next tap's corner as soon as they are consumed.  Corners
// outside the level are loaded from a clamped in-level address with zero
// weight.
//
// Location arithmetic: x = u W - 1/2 is formed as hi = u*W, lo = fma(u, W, -hi)
// (the exact rounding error of the product), x0 = floor(hi - 1/2) and
// a = (hi - 1/2 - x0) + lo, renormalised into [0, 1).  This keeps the
// fractional part accurate to ~1e-7 px where a plain float32 product would be
// off by up to half an ulp of u*W (~4e-6 px at W = 150).
#pragma once

#include "common.cuh"

namespace dcnb {

constexpr int kMsdaWarps = 4;
constexpr int kMsdaThreads = 32 * kMsdaWarps;
constexpr int kMsdaMaxLevels = 16;

struct MsdaArgs {
    const void* value;
    const int64_t* shapes;       // [L][2] (H_l, W_l), device
    const int64_t* level_start;  // [L], device
    const void* loc;             // locations, or offsets for the reference variants
    const void* attn;
    void* out;
    int Lq, M, D, L, K;
    int tpi;                     // threads per item
    int run_items;               // items per warp run (32 / tpi)
    int total_items;             // N * Lq * M
    int num_runs;                // ceil(total_items / run_items)
    int stage_elems;             // staged weights per warp (run_items * L * K); 0 = unstaged
    int loc_stride, w_stride;    // item strides (elements) of the staged slices
    FastDiv div_M, div_Lq, div_tpi;
    const void* ref;             // reference variants: [N][Lq][2 or 4] in valid-image units
    const void* vr;              // [N][L][2] valid ratios (W_valid / W, H_valid / H) or null
    unsigned int* flags;         // status word (device), or null
};

// Integer cell and fraction of the normalised coordinate u on a level of
// `size` pixels: returns a in [0, 1) and writes the clamped floor to *cell.
__device__ __forceinline__ float level_coord(float u, float size, int* cell) {
    const float hi = u * size;
    const float lo = fmaf(u, size, -hi);   // exact residual of the product
    const float xs = hi - 0.5f;
    float fx = floorf(xs);
    float a = (xs - fx) + lo;
    if (a >= 1.f) {
        a -= 1.f;
        fx += 1.f;
    } else if (a < 0.f) {
        a += 1.f;
        fx -= 1.f;
    }
    fx = fminf(fmaxf(fx, -4194304.f), 4194304.f);   // +-2^22; NaN -> far outside
    *cell = (int)fx;
    return a;
}

// One tap: byte offsets (from the item's value base) of the four corners to
// load, clamped into the level, and their weights (zero outside the level).
struct MsdaTap {
    long long off[4];
    float w[4];
};

// Cell and fraction of a pixel-space coordinate x (already u W - 1/2),
// formed in double precision by the caller: a few float32 roundings of a
// position near 150 px would already move samples by ~1e-5 px.
__device__ __forceinline__ float pixel_coord(double x, int* cell) {
    double fx = floor(x);
    const float a = fminf(fmaxf((float)(x - fx), 0.f), 1.f);   // NaN: far outside, a = 0
    fx = fmin(fmax(fx, -4194304.0), 4194304.0);                // +-2^22
    *cell = (int)fx;
    return a;
}

__device__ __forceinline__ MsdaTap msda_corners(const int (*lvl)[3], long long pix_bytes, int l,
                                                int x0, float ax, int y0, float ay, float A);

__device__ __forceinline__ MsdaTap msda_tap(const int (*lvl)[3], long long pix_bytes, int l,
                                            float u, float v, float A) {
    const int Hl = lvl[l][0], Wl = lvl[l][1];
    int x0, y0;
    const float ax = level_coord(u, (float)Wl, &x0);
    const float ay = level_coord(v, (float)Hl, &y0);
    return msda_corners(lvl, pix_bytes, l, x0, ax, y0, ay, A);
}

// The four corners of cell (x0, y0) with fractions (ax, ay) on level l.
__device__ __forceinline__ MsdaTap msda_corners(const int (*lvl)[3], long long pix_bytes, int l,
                                                int x0, float ax, int y0, float ay, float A) {
    MsdaTap t;
    const int Hl = lvl[l][0], Wl = lvl[l][1];
    const int x1 = x0 + 1, y1 = y0 + 1;
    const bool vx0 = (unsigned)x0 < (unsigned)Wl, vx1 = (unsigned)x1 < (unsigned)Wl;
    const bool vy0 = (unsigned)y0 < (unsigned)Hl, vy1 = (unsigned)y1 < (unsigned)Hl;
    const float wx0 = vx0 ? 1.f - ax : 0.f, wx1 = vx1 ? ax : 0.f;
    const float wy0 = vy0 ? (1.f - ay) * A : 0.f, wy1 = vy1 ? ay * A : 0.f;
    t.w[0] = wx0 * wy0;
    t.w[1] = wx1 * wy0;
    t.w[2] = wx0 * wy1;
    t.w[3] = wx1 * wy1;
    const int cx0 = vx0 ? x0 : 0, cx1 = vx1 ? x1 : 0;
    const int cy0 = vy0 ? y0 : 0, cy1 = vy1 ? y1 : 0;
    // an empty level (non-positive shape) loads row 0 with zero weights
    const long long start = (Hl > 0 && Wl > 0) ? (long long)lvl[l][2] : 0;
    const long long row0 = start + (long long)cy0 * Wl;
    const long long row1 = start + (long long)cy1 * Wl;
    t.off[0] = (row0 + cx0) * pix_bytes;
    t.off[1] = (row0 + cx1) * pix_bytes;
    t.off[2] = (row1 + cx0) * pix_bytes;
    t.off[3] = (row1 + cx1) * pix_bytes;
    return t;
}

// Element of `es` bytes, moved as an integer.
template <int ES>
struct Word;
template <>
struct Word<4> {
    using type = uint32_t;
};
template <>
struct Word<2> {
    using type = unsigned short;
};

// Copy `rows` rows of `row_elems` elements of T between consecutive rows in
// global memory and shared rows `stride` elements apart, with the lanes of
// one warp; 16-byte vectors when the addresses and sizes allow, else single
// elements.  IN: global -> shared; otherwise shared -> global.
template <typename T, bool IN>
__device__ __forceinline__ void msda_stage_rows(T* shared, int stride, T* global, int row_elems,
                                                int rows, int lane) {
    constexpr int es = (int)sizeof(T);
    const int row_bytes = row_elems * es;
    const uintptr_t al = (uintptr_t)global | (uintptr_t)shared | (uintptr_t)row_bytes |
                         (uintptr_t)(stride * es);
    if ((al & 15) == 0) {
        const int vpr = row_bytes >> 4;
        const int svs = (stride * es) >> 4;
        uint4* g = reinterpret_cast<uint4*>(global);
        uint4* sh = reinterpret_cast<uint4*>(shared);
        for (int i = lane; i < rows * vpr; i += 32) {
            const int r = i / vpr;
            const int si = r * svs + (i - r * vpr);
            if constexpr (IN) {
                uint4 x;
                asm("ld.global.nc.L1::no_allocate.v4.u32 {%0,%1,%2,%3}, [%4];"
                    : "=r"(x.x), "=r"(x.y), "=r"(x.z), "=r"(x.w) : "l"(g + i));
                sh[si] = x;
            } else {
                g[i] = sh[si];
            }
        }
    } else {
        using W = typename Word<es>::type;
        W* g = reinterpret_cast<W*>(global);
        W* sh = reinterpret_cast<W*>(shared);
        for (int i = lane; i < rows * row_elems; i += 32) {
            const int r = i / row_elems;
            const int si = r * stride + (i - r * row_elems);
            if constexpr (IN)
                sh[si] = __ldg(g + i);
            else
                g[i] = sh[si];
        }
    }
}

// REF = 0: sampling_loc holds the normalised locations.  REF = 2 / 4: it holds
// the offsets of the reference-point variants ("Deformable DETR", "A reference
// links resolutions without equating their pixels" and helper 1), and the
// pixel position is formed here from the point (cx, cy) or box (cx, cy, w, h)
// reference of the query and the level's valid ratio r:
//   point: x = (cx r) W + dx - 1/2                  (s = cx r + dx / W)
//   box:   x = ((cx + dx w / (2K)) r) W - 1/2       (s = cx r + dx / K * w * r / 2)
// Five CTAs (20 warps) per SM for the plain path, four for the reference
// variants, whose double-precision location arithmetic needs the registers.
template <typename T, int VB, int REF = 0>
__global__ void __launch_bounds__(kMsdaThreads, REF == 0 ? 5 : 4)
    msda_fwd_kernel(const MsdaArgs a) {
    constexpr int CPT = VB / (int)sizeof(T);
    constexpr int NW = VB >= 4 ? VB / 4 : 1;
    extern __shared__ __align__(16) unsigned char smem[];
    __shared__ int s_lvl[kMsdaMaxLevels][3];   // H_l, W_l, start_l
    __shared__ long long s_S;

    const int L = a.L, K = a.K;
    const int LK = L * K;
    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    const bool staged = a.stage_elems > 0;
    // item rows a.loc_stride / a.w_stride elements apart (multiples of 16 bytes)
    const int loc_slice = a.run_items * a.loc_stride * (int)sizeof(T);
    const int slice = loc_slice + a.run_items * a.w_stride * (int)sizeof(T);
    T* s_loc = reinterpret_cast<T*>(smem + warp * slice);
    T* s_w = reinterpret_cast<T*>(smem + warp * slice + loc_slice);

    if (threadIdx.x < L) {
        // a non-positive shape (a broken precondition) makes the level empty
        // instead of turning the unsigned bounds tests into no-ops
        s_lvl[threadIdx.x][0] = (int)max(a.shapes[2 * threadIdx.x], (int64_t)0);
        s_lvl[threadIdx.x][1] = (int)max(a.shapes[2 * threadIdx.x + 1], (int64_t)0);
        s_lvl[threadIdx.x][2] = (int)a.level_start[threadIdx.x];
    }
    if (threadIdx.x == 0)
        s_S = a.level_start[L - 1] + a.shapes[2 * (L - 1)] * a.shapes[2 * (L - 1) + 1];
#ifdef DCN_DEBUG
    // the debug library checks the level table on the device: positive shapes,
    // levels in order without gaps from row 0; otherwise the call reads no
    // value rows (and writes no output)
    __shared__ int s_bad;
    if (threadIdx.x == 0) {
        int bad = 0;
        long long expect = 0;
        for (int l = 0; l < L; ++l) {
            if (a.shapes[2 * l] <= 0 || a.shapes[2 * l + 1] <= 0 || a.level_start[l] != expect)
                bad = 1;
            expect = a.level_start[l] + a.shapes[2 * l] * a.shapes[2 * l + 1];
        }
        s_bad = bad;
        if (bad) set_flag(a.flags, kFlagBadLevels);
    }
    __syncthreads();
    if (s_bad) return;
#endif
    __syncthreads();

    const int li = (int)a.div_tpi.div((uint32_t)lane);   // item within the run
    const int chunk = lane - li * a.tpi;
    const long long pix_bytes = (long long)a.M * a.D * (int)sizeof(T);   // one value row

    // contiguous, balanced range of runs for this CTA, split into one
    // contiguous sub-range per warp: consecutive queries of one warp reuse
    // each other's value rows through L1, while the CTA's warps, working far
    // apart, do not queue on the same lines' misses at the same time
    const int r_begin = (int)(((long long)a.num_runs * blockIdx.x) / gridDim.x);
    const int r_end = (int)(((long long)a.num_runs * (blockIdx.x + 1)) / gridDim.x);
    const int w_begin = r_begin + (int)(((long long)(r_end - r_begin) * warp) / kMsdaWarps);
    const int w_end = r_begin + (int)(((long long)(r_end - r_begin) * (warp + 1)) / kMsdaWarps);

    for (int run = w_begin; run < w_end; ++run) {
        const int item0 = run * a.run_items;
        const int nitems = min(a.run_items, a.total_items - item0);
        const T* locp;
        const T* wp;
        if (staged) {
            __syncwarp();
            msda_stage_rows<T, true>(
                s_loc, a.loc_stride,
                const_cast<T*>(static_cast<const T*>(a.loc)) + (long long)item0 * LK * 2, LK * 2,
                nitems, lane);
            msda_stage_rows<T, true>(
                s_w, a.w_stride,
                const_cast<T*>(static_cast<const T*>(a.attn)) + (long long)item0 * LK, LK,
                nitems, lane);
            __syncwarp();
            locp = s_loc + li * a.loc_stride;
            wp = s_w + li * a.w_stride;
        } else {
            locp = static_cast<const T*>(a.loc) + (long long)(item0 + li) * LK * 2;
            wp = static_cast<const T*>(a.attn) + (long long)(item0 + li) * LK;
        }
        if (li >= nitems) continue;

        const int item = item0 + li;                  // (n * Lq + q) * M + h
        const int nq = (int)a.div_M.div((uint32_t)item);
        const int h = item - nq * a.M;
        const int n = (int)a.div_Lq.div((uint32_t)nq);
        const char* vb = static_cast<const char*>(a.value) +
                         ((long long)n * s_S * a.M + h) * a.D * (int)sizeof(T) +
                         (long long)chunk * CPT * (int)sizeof(T);
        // reference variants: the query's reference, the batch item's ratios
        float rcx = 0.f, rcy = 0.f, rw = 0.f, rh = 0.f;
        const T* vrp = nullptr;
        if constexpr (REF != 0) {
            const T* rp = static_cast<const T*>(a.ref) + (long long)nq * REF;
            rcx = Elem<T>::one(rp);
            rcy = Elem<T>::one(rp + 1);
            if constexpr (REF == 4) {   // box size (w, h)
                rw = Elem<T>::one(rp + 2);
                rh = Elem<T>::one(rp + 3);
            }
            if (a.vr) vrp = static_cast<const T*>(a.vr) + (long long)n * L * 2;
        }
        float rx = 1.f, ry = 1.f;   // valid ratios of the current level

        float acc[CPT];
#pragma unroll
        for (int i = 0; i < CPT; ++i) acc[i] = 0.f;

        // rolling corner pipeline over the L*K taps (level-major)
        uint32_t v[4][NW];
        float w[4];
        int nl = 0, nt = 0;                  // level and index of the next tap
        auto geometry = [&]() {
            float u, vv;
            load_pair<T>(locp + 2 * nt, u, vv);
            MsdaTap t;
            if constexpr (REF == 0) {
                t = msda_tap(s_lvl, pix_bytes, nl, u, vv, Elem<T>::one(wp + nt));
            } else {
                if (vrp && nt == nl * K) {    // first tap of a level
                    rx = Elem<T>::one(vrp + 2 * nl);
                    ry = Elem<T>::one(vrp + 2 * nl + 1);
                }
                const double Wl = (double)s_lvl[nl][1], Hl = (double)s_lvl[nl][0];
                double x, y;
                if constexpr (REF == 2) {
                    x = fma((double)rcx * rx, Wl, (double)u) - 0.5;
                    y = fma((double)rcy * ry, Hl, (double)vv) - 0.5;
                } else {
                    const double half_k = 0.5 / (double)K;
                    x = fma((double)u * half_k, (double)rw, (double)rcx) * rx * Wl - 0.5;
                    y = fma((double)vv * half_k, (double)rh, (double)rcy) * ry * Hl - 0.5;
                }
                int x0, y0;
                const float ax = pixel_coord(x, &x0);
                const float ay = pixel_coord(y, &y0);
                t = msda_corners(s_lvl, pix_bytes, nl, x0, ax, y0, ay, Elem<T>::one(wp + nt));
            }
            ++nt;
            if (nt == (nl + 1) * K) ++nl;
            return t;
        };
        // a corner load (clamped into its level, so always inside value; the
        // debug library checks it against the image's rows and reads zeros
        // instead when it is not)
        const long long img_bytes_v = s_S * pix_bytes;
        const long long lane_off = (long long)h * a.D * (int)sizeof(T) +
                                   (long long)chunk * CPT * (int)sizeof(T);
        auto corner = [&](long long off, uint32_t* dst) {
            if (DCN_IN_BOUNDS(off >= 0 && off + lane_off + VB <= img_bytes_v, a.flags)) {
                load_vec<VB>(vb + off, dst);
            } else {
#pragma unroll
                for (int i = 0; i < NW; ++i) dst[i] = 0u;
            }
        };
        (void)img_bytes_v;
        (void)lane_off;
        {
            const MsdaTap t0 = geometry();
#pragma unroll
            for (int c = 0; c < 4; ++c) {
                corner(t0.off[c], v[c]);
                w[c] = t0.w[c];
            }
        }
#pragma unroll 1
        for (int t = 0; t < LK; ++t) {
            const bool more = t + 1 < LK;
            MsdaTap tn;
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
                   ((long long)nq * a.M * a.D + h * a.D + chunk * CPT) * (int)sizeof(T);
        store_vec<VB>(ob, o);
    }
}

}  // namespace dcnb

namespace dcnb {

// value rows whose mask byte is set become 0 ("Deformable DETR": the attention
// module zeroes projected values at masked positions); out may be value.
struct MaskArgs {
    const void* value;
    const unsigned char* mask;   // [N][S]
    void* out;
    long long rows;              // N * S
    int row_bytes;               // M * D * element size
    int vec16;                   // 1: rows, value and out are 16-byte aligned
};

static __global__ void __launch_bounds__(256) msda_mask_value_kernel(const MaskArgs m) {
    const long long tid = (long long)blockIdx.x * blockDim.x + threadIdx.x;
    const long long nthreads = (long long)gridDim.x * blockDim.x;
    const char* src = static_cast<const char*>(m.value);
    char* dst = static_cast<char*>(m.out);
    if (m.vec16) {
        const int per_row = m.row_bytes >> 4;
        const long long total = m.rows * per_row;
        for (long long i = tid; i < total; i += nthreads) {
            const long long row = i / per_row;
            uint4 v = make_uint4(0u, 0u, 0u, 0u);
            if (!m.mask[row]) v = reinterpret_cast<const uint4*>(src)[i];
            reinterpret_cast<uint4*>(dst)[i] = v;
        }
    } else {
        const long long total = m.rows * m.row_bytes;
        for (long long i = tid; i < total; i += nthreads) {
            const long long row = i / m.row_bytes;
            dst[i] = m.mask[row] ? 0 : src[i];
        }
    }
}

}  // namespace dcnb
