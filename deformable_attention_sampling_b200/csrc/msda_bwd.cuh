// Multi-scale deformable attention (MSDeformAttn core) backward, sm_100a SIMT.
//
// Gradients of out[n,q,h*D+c] = sum_{l,k} A * S_l(value, loc) ("Deformable
// DETR: Learn Where to Read", "A learned location can fall between cells":
// the read is differentiable in the location, which is how the offsets learn):
//   grad_value  scatter: each corner receives A * w_corner * go
//   grad_loc    A * W_l * dS/da, A * H_l * dS/db  (x = u W_l - 1/2, so
//               dx/du = W_l; one-sided at integer positions)
//   grad_attn   <go, S_l(value, loc)>
// The work decomposition is the forward's (item = (batch, query, head), TPI
// threads of CPT channels, warp runs of 32/TPI items, per-warp staging).  Per
// tap each thread forms the corner dot products P_c = sum over its channels
// of go * value_corner and combines them as the DCN backward does; the three
// per-tap sums are reduced over the item's threads with shuffles.  grad_value
// goes to a float32 accumulator through vector reductions in L2, whole
// 32-byte sectors per lane pair where the channel split allows (as in the
// DCN backward).
#pragma once

#include "dcn_bwd.cuh"
#include "msda_fwd.cuh"

namespace dcnb {

struct MsdaBwdArgs {
    MsdaArgs f;              // forward geometry; f.out is unused
    const void* grad_out;    // [N][Lq][M*D]
    void* grad_loc;          // [N][Lq][M][L][K][2]
    void* grad_attn;         // [N][Lq][M][L][K]
    float* gv_acc;           // float32 [N][S][M][D], zero on entry
    long long S;             // value rows per batch item
    int red_vec;             // floats per reduction instruction: 4, 2 or 1
};

// One tap: element offsets (from the item's value base) of the four corners,
// clamped into the level; the fractions; a bit per corner inside the level.
struct MsdaBwdTap {
    long long off[4];
    float ax, ay;
    uint32_t valid;
    float Wl, Hl;
};

__device__ __forceinline__ MsdaBwdTap msda_bwd_tap(const int (*lvl)[3], long long pix_elems,
                                                   int l, float u, float v) {
    MsdaBwdTap t;
    const int Hl = lvl[l][0], Wl = lvl[l][1];
    int x0, y0;
    const float ax = level_coord(u, (float)Wl, &x0);
    const float ay = level_coord(v, (float)Hl, &y0);
    // a NaN location lands far outside with a finite fraction
    t.ax = fminf(fmaxf(ax, 0.f), 1.f);
    t.ay = fminf(fmaxf(ay, 0.f), 1.f);
    t.Wl = (float)Wl;
    t.Hl = (float)Hl;
    const int x1 = x0 + 1, y1 = y0 + 1;
    const bool vx0 = (unsigned)x0 < (unsigned)Wl, vx1 = (unsigned)x1 < (unsigned)Wl;
    const bool vy0 = (unsigned)y0 < (unsigned)Hl, vy1 = (unsigned)y1 < (unsigned)Hl;
    t.valid = (uint32_t)(vx0 && vy0) | ((uint32_t)(vx1 && vy0) << 1) |
              ((uint32_t)(vx0 && vy1) << 2) | ((uint32_t)(vx1 && vy1) << 3);
    const int cx0 = vx0 ? x0 : 0, cx1 = vx1 ? x1 : 0;
    const int cy0 = vy0 ? y0 : 0, cy1 = vy1 ? y1 : 0;
    const long long start = (Hl > 0 && Wl > 0) ? (long long)lvl[l][2] : 0;
    const long long row0 = start + (long long)cy0 * Wl;
    const long long row1 = start + (long long)cy1 * Wl;
    t.off[0] = (row0 + cx0) * pix_elems;
    t.off[1] = (row0 + cx1) * pix_elems;
    t.off[2] = (row1 + cx0) * pix_elems;
    t.off[3] = (row1 + cx1) * pix_elems;
    return t;
}

// Byte sizes of one warp's shared slice: staged locations and weights, then
// grad_loc and grad_attn of the run, item rows loc_stride / w_stride elements
// apart (each a multiple of 16 bytes).
struct MsdaBwdSlice {
    int loc, attn;
    __host__ __device__ int total() const { return 2 * (loc + attn); }
};

__host__ __device__ inline MsdaBwdSlice msda_bwd_slice(int run_items, int loc_stride,
                                                       int w_stride, int es) {
    MsdaBwdSlice s;
    s.loc = run_items * loc_stride * es;
    s.attn = run_items * w_stride * es;
    return s;
}

// PAIR: the sector-paired scatter (CPT = 8, an even number of lanes per item).
// 128 registers: four 4-warp CTAs per SM (measured faster than a register cap
// that fits six, which spills).
template <typename T, int VB, bool PAIR = false>
__global__ void __launch_bounds__(kMsdaThreads, 4) msda_bwd_kernel(const MsdaBwdArgs b) {
    constexpr int CPT = VB / (int)sizeof(T);
    constexpr int NW = VB >= 4 ? VB / 4 : 1;
    constexpr int es = (int)sizeof(T);
    extern __shared__ __align__(16) unsigned char smem[];
    __shared__ int s_lvl[kMsdaMaxLevels][3];
    const MsdaArgs& a = b.f;

    const int L = a.L, K = a.K;
    const int LK = L * K;
    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    const MsdaBwdSlice sl = msda_bwd_slice(a.run_items, a.loc_stride, a.w_stride, es);
    unsigned char* my = smem + warp * sl.total();
    T* s_loc = reinterpret_cast<T*>(my);
    T* s_w = reinterpret_cast<T*>(my + sl.loc);
    T* s_gloc = reinterpret_cast<T*>(my + sl.loc + sl.attn);
    T* s_gw = reinterpret_cast<T*>(my + 2 * sl.loc + sl.attn);

    if (threadIdx.x < L) {
        s_lvl[threadIdx.x][0] = (int)max(a.shapes[2 * threadIdx.x], (int64_t)0);
        s_lvl[threadIdx.x][1] = (int)max(a.shapes[2 * threadIdx.x + 1], (int64_t)0);
        s_lvl[threadIdx.x][2] = (int)a.level_start[threadIdx.x];
    }
    __syncthreads();

    const int li_raw = (int)a.div_tpi.div((uint32_t)lane);
    const int chunk = lane - li_raw * a.tpi;
    const long long pix_elems = (long long)a.M * a.D;   // one value row

    const int r_begin = (int)(((long long)a.num_runs * blockIdx.x) / gridDim.x);
    const int r_end = (int)(((long long)a.num_runs * (blockIdx.x + 1)) / gridDim.x);

    // one contiguous sub-range of runs per warp (as in the forward)
    const int w_begin = r_begin + (int)(((long long)(r_end - r_begin) * warp) / kMsdaWarps);
    const int w_end = r_begin + (int)(((long long)(r_end - r_begin) * (warp + 1)) / kMsdaWarps);
    for (int run = w_begin; run < w_end; ++run) {
        const int item0 = run * a.run_items;
        const int nitems = min(a.run_items, a.total_items - item0);
        __syncwarp();
        msda_stage_rows<T, true>(
            s_loc, a.loc_stride,
            const_cast<T*>(static_cast<const T*>(a.loc)) + (long long)item0 * LK * 2, LK * 2,
            nitems, lane);
        msda_stage_rows<T, true>(
            s_w, a.w_stride,
            const_cast<T*>(static_cast<const T*>(a.attn)) + (long long)item0 * LK, LK, nitems,
            lane);
        __syncwarp();

        // lanes without an item shadow item 0 with a zero upstream gradient
        const bool active = li_raw < nitems;
        const int li = active ? li_raw : 0;
        const T* locp = s_loc + li * a.loc_stride;
        const T* wp = s_w + li * a.w_stride;
        const int item = item0 + li;                  // (n * Lq + q) * M + h
        const int nq = (int)a.div_M.div((uint32_t)item);
        const int h = item - nq * a.M;
        const int n = (int)a.div_Lq.div((uint32_t)nq);
        const long long base = ((long long)n * b.S * a.M + h) * a.D + (long long)chunk * CPT;
        const char* vb = static_cast<const char*>(a.value) + base * es;
        float* gvb = b.gv_acc + base;

        float go[CPT];
        {
            uint32_t w[NW];
            load_vec<VB>(static_cast<const char*>(b.grad_out) +
                             ((long long)nq * a.M * a.D + h * a.D + chunk * CPT) * es,
                         w);
            widen<T, CPT>(w, go);
            if (!active) {
#pragma unroll
                for (int i = 0; i < CPT; ++i) go[i] = 0.f;
            }
        }
        static_assert(!PAIR || CPT == 8, "the paired scatter needs 8 channels per lane");
        PairScatter ps;
        if constexpr (PAIR) ps = pair_setup(go, chunk);

        uint32_t v[4][NW];
        int nl = 0, nt = 0;
        auto geometry = [&]() {
            float u, vv;
            load_pair<T>(locp + 2 * nt, u, vv);
            const MsdaBwdTap t = msda_bwd_tap(s_lvl, pix_elems, nl, u, vv);
            ++nt;
            if (nt == (nl + 1) * K) ++nl;
            return t;
        };
        MsdaBwdTap cur = geometry();
#pragma unroll
        for (int c = 0; c < 4; ++c) load_vec<VB>(vb + cur.off[c] * es, v[c]);

#pragma unroll 1
        for (int t = 0; t < LK; ++t) {
            const bool more = t + 1 < LK;
            MsdaBwdTap nxt;
            if (more) nxt = geometry();
            float P[4];
#pragma unroll
            for (int c = 0; c < 4; ++c) {
                float f[CPT];
                widen<T, CPT>(v[c], f);
                P[c] = (cur.valid >> c) & 1u ? dot<CPT>(go, f) : 0.f;
                if (more) load_vec<VB>(vb + nxt.off[c] * es, v[c]);
            }
            const float A = Elem<T>::one(wp + t);
            const float wx0 = 1.f - cur.ax, wx1 = cur.ax;
            const float wy0 = 1.f - cur.ay, wy1 = cur.ay;
#pragma unroll
            for (int c = 0; c < 4; ++c) {
                const float wc = (c & 1 ? wx1 : wx0) * (c & 2 ? wy1 : wy0);
                if (active && ((cur.valid >> c) & 1u)) {
                    if constexpr (PAIR)
                        scatter_pair(gvb + cur.off[c], A * wc, ps);
                    else
                        scatter_scaled<CPT>(gvb + cur.off[c], A * wc, go, b.red_vec);
                }
            }
            float gs = wy0 * (wx0 * P[0] + wx1 * P[1]) + wy1 * (wx0 * P[2] + wx1 * P[3]);
            float da = wy0 * (P[1] - P[0]) + wy1 * (P[3] - P[2]);
            float db = wx0 * (P[2] - P[0]) + wx1 * (P[3] - P[1]);
            gs = item_sum(gs, a.tpi, li_raw * a.tpi, chunk);
            da = item_sum(da, a.tpi, li_raw * a.tpi, chunk);
            db = item_sum(db, a.tpi, li_raw * a.tpi, chunk);
            if (active && chunk == 0) {
                s_gloc[li * a.loc_stride + 2 * t] = Elem<T>::from(A * cur.Wl * da);
                s_gloc[li * a.loc_stride + 2 * t + 1] = Elem<T>::from(A * cur.Hl * db);
                s_gw[li * a.w_stride + t] = Elem<T>::from(gs);
            }
            if (more) cur = nxt;
        }
        __syncwarp();
        msda_stage_rows<T, false>(s_gloc, a.loc_stride,
                                  static_cast<T*>(b.grad_loc) + (long long)item0 * LK * 2,
                                  LK * 2, nitems, lane);
        msda_stage_rows<T, false>(s_gw, a.w_stride,
                                  static_cast<T*>(b.grad_attn) + (long long)item0 * LK, LK,
                                  nitems, lane);
    }
}

}  // namespace dcnb
