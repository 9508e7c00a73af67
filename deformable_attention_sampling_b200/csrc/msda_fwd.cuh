// Multi-scale deformable attention (MSDeformAttn core) forward, sm_100a SIMT.
//
// Operator ("Deformable DETR: Learn Where to Read", "A learned location can
// fall between cells" and "Mix samples with a per-head budget"):
//   out[n,q,h*D+c] = sum_{l,k} A[n,q,h,l,k] * S_l(value[n, start_l + ., h, c], loc[n,q,h,l,k])
//   S_l(f, u, v): x = u W_l - 1/2, y = v H_l - 1/2; bilinear over the four
//   floor/ceil neighbours, zero outside, no clamping, no renormalisation.
//
// Work decomposition mirrors the DCN kernel: a work item is one (batch,
// query, head) triple, numbered in the memory order of loc / attn / out, and
// TPI = D / CPT threads share it, each owning CPT consecutive channels
// (CPT * sizeof(T) <= 32 bytes: one vector load per corner).  The CTA stages
// its block's locations and weights (contiguous spans) into shared memory.
//
// Location arithmetic: x = u W - 1/2 is formed as hi = u*W, lo = fma(u, W, -hi)
// (the exact rounding error of the product), x0 = floor(hi - 1/2) and
// a = (hi - 1/2 - x0) + lo, renormalised into [0, 1).  This keeps the
// fractional part accurate to ~1e-7 px where a plain float32 product would be
// off by up to half an ulp of u*W (~4e-6 px at W = 150).
#pragma once

#include "common.cuh"

namespace dcnb {

constexpr int kMsdaThreads = 128;
constexpr int kMsdaMaxLevels = 16;

struct MsdaArgs {
    const void* value;
    const int64_t* shapes;       // [L][2] (H_l, W_l), device
    const int64_t* level_start;  // [L], device
    const void* loc;
    const void* attn;
    void* out;
    int Lq, M, D, L, K;
    int tpi;
    int items_per_cta;
    int total_items;             // N * Lq * M
    int num_blocks;
    FastDiv div_M, div_Lq, div_tpi;
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

template <typename T, int VB>
__global__ void __launch_bounds__(kMsdaThreads, 4) msda_fwd_kernel(const MsdaArgs a) {
    constexpr int CPT = VB / (int)sizeof(T);
    constexpr int NW = VB >= 4 ? VB / 4 : 1;
    extern __shared__ __align__(16) unsigned char smem[];
    __shared__ int s_lvl[kMsdaMaxLevels][3];   // H_l, W_l, start_l
    __shared__ long long s_S;

    const int L = a.L, K = a.K;
    const int LK = L * K;
    T* s_loc = reinterpret_cast<T*>(smem);
    const int loc_span = ((a.items_per_cta * LK * 2 * (int)sizeof(T)) + 15) & ~15;
    T* s_w = reinterpret_cast<T*>(smem + loc_span);

    if (threadIdx.x < L) {
        // a non-positive shape (a broken precondition) makes the level empty
        // instead of turning the unsigned bounds tests below into no-ops
        s_lvl[threadIdx.x][0] = (int)max(a.shapes[2 * threadIdx.x], (int64_t)0);
        s_lvl[threadIdx.x][1] = (int)max(a.shapes[2 * threadIdx.x + 1], (int64_t)0);
        s_lvl[threadIdx.x][2] = (int)a.level_start[threadIdx.x];
    }
    if (threadIdx.x == 0)
        s_S = a.level_start[L - 1] + a.shapes[2 * (L - 1)] * a.shapes[2 * (L - 1) + 1];

    const int li = (int)a.div_tpi.div(threadIdx.x);
    const int chunk = (int)threadIdx.x - li * a.tpi;
    const long long pix_bytes = (long long)a.M * a.D * (int)sizeof(T);   // one value row

    for (int blk = blockIdx.x; blk < a.num_blocks; blk += gridDim.x) {
        const int item0 = blk * a.items_per_cta;
        const int nitems = min(a.items_per_cta, a.total_items - item0);
        __syncthreads();
        stage_span(s_loc, static_cast<const T*>(a.loc) + (long long)item0 * LK * 2,
                   nitems * LK * 2 * (int)sizeof(T));
        stage_span(s_w, static_cast<const T*>(a.attn) + (long long)item0 * LK,
                   nitems * LK * (int)sizeof(T));
        __syncthreads();
        if (li >= nitems) continue;

        const int item = item0 + li;                  // (n * Lq + q) * M + h
        const int nq = (int)a.div_M.div((uint32_t)item);
        const int h = item - nq * a.M;
        const int n = (int)a.div_Lq.div((uint32_t)nq);

        const char* vb = static_cast<const char*>(a.value) +
                         ((long long)n * s_S * a.M + h) * a.D * (int)sizeof(T) +
                         (long long)chunk * CPT * (int)sizeof(T);
        const T* locp = s_loc + li * LK * 2;
        const T* wp = s_w + li * LK;

        float acc[CPT];
#pragma unroll
        for (int i = 0; i < CPT; ++i) acc[i] = 0.f;
        uint32_t r00[NW], r01[NW], r10[NW], r11[NW];
#pragma unroll
        for (int i = 0; i < NW; ++i) r00[i] = r01[i] = r10[i] = r11[i] = 0u;

        for (int l = 0; l < L; ++l) {
            const int Hl = s_lvl[l][0], Wl = s_lvl[l][1];
            const char* lb = vb + (long long)s_lvl[l][2] * pix_bytes;
            const float Wf = (float)Wl, Hf = (float)Hl;
#pragma unroll 2
            for (int k = 0; k < K; ++k) {
                const int t = l * K + k;
                float u, v;
                load_pair<T>(locp + 2 * t, u, v);
                const float A = Elem<T>::one(wp + t);
                int x0, y0;
                const float ax = level_coord(u, Wf, &x0);
                const float ay = level_coord(v, Hf, &y0);
                const bool vx0 = (unsigned)x0 < (unsigned)Wl;
                const bool vx1 = (unsigned)(x0 + 1) < (unsigned)Wl;
                const bool vy0 = (unsigned)y0 < (unsigned)Hl;
                const bool vy1 = (unsigned)(y0 + 1) < (unsigned)Hl;
                const float mb1 = A * ay;
                const float mb0 = A - mb1;
                const float w00 = (vx0 && vy0) ? (1.f - ax) * mb0 : 0.f;
                const float w01 = (vx1 && vy0) ? ax * mb0 : 0.f;
                const float w10 = (vx0 && vy1) ? (1.f - ax) * mb1 : 0.f;
                const float w11 = (vx1 && vy1) ? ax * mb1 : 0.f;
                // value rows of the four corners; in-bounds rows lie in [0, S)
                const int q00 = (int)((uint32_t)y0 * (uint32_t)Wl + (uint32_t)x0);
                const int q10 = q00 + Wl;
                if (vx0 && vy0) load_vec<VB>(lb + (long long)q00 * pix_bytes, r00);
                if (vx1 && vy0) load_vec<VB>(lb + (long long)(q00 + 1) * pix_bytes, r01);
                if (vx0 && vy1) load_vec<VB>(lb + (long long)q10 * pix_bytes, r10);
                if (vx1 && vy1) load_vec<VB>(lb + (long long)(q10 + 1) * pix_bytes, r11);
                float f[CPT];
                widen<T, CPT>(r00, f);
                axpy<CPT>(acc, w00, f);
                widen<T, CPT>(r01, f);
                axpy<CPT>(acc, w01, f);
                widen<T, CPT>(r10, f);
                axpy<CPT>(acc, w10, f);
                widen<T, CPT>(r11, f);
                axpy<CPT>(acc, w11, f);
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
