// DCNv3 / DCNv4 deformable sampling-aggregation forward, sm_100a SIMT kernel.
//
// Operator ("InternImage: Deformable Convolutions at Scale" ch.1-4; "DCNv4",
// "Why Is Sampling Just 9 Points Still Slow?" and "1. Remove Softmax"):
//   out[n,oy,ox,g*D+c] = sum_k m[g,k] * bilinear(x[n,:,:,g*D+c], p0 + p_k + dp[g,k])
// with zero padding outside the map and m either used as given (DCNv4) or
// soft-maxed over the K taps of the group (DCNv3).
//
// Work decomposition.  A work item is one (output pixel, group) pair; items
// are numbered pixel-major, group-minor, which is exactly the memory order of
// the offset and mask tensors ([N,Ho,Wo,G,K,...]).  Each item is handled by
// TPI = D / CPT threads, each owning CPT consecutive channels of the group
// (CPT * sizeof(T) = VB bytes, at most 32: one 256-bit load per corner).
// A block of items is therefore contiguous in offset, mask and out.
//
//   1. The CTA copies its block's offsets and masks (one contiguous span each)
//      into shared memory with coalesced 16-byte loads: every value is read
//      from HBM once and each thread then reads its own item's K triples.
//   2. Per tap, the thread splits the offset into integer and fractional parts
//      (floor(d), d - floor(d): exact for 16-bit inputs), forms the four
//      corner weights (1-a)(1-b)m, a(1-b)m, (1-a)b m, ab m once for its CPT
//      channels, zeroes the weight of every corner outside the map and issues
//      one predicated vector load per in-bounds corner.  A corner outside the
//      map is never loaded: its registers keep the previous (finite) data and
//      its weight is zero.
//   3. The CPT channels accumulate in float32 with packed FFMA2; the result is
//      rounded once to T and written with one streaming vector store.
// No tensor cores: the work is a gather and a weighted sum, not a contraction.
#pragma once

#include "common.cuh"

namespace dcnb {

constexpr int kDcnThreads = 128;
// Offsets are clamped to +-kBigCoord before the integer conversion; any tap
// that far out has all four corners outside every supported map (H, W <= 2^16),
// and a NaN offset maps to -kBigCoord (fminf/fmaxf return the non-NaN operand).
constexpr float kBigCoord = 4194304.0f;   // 2^22

struct DcnArgs {
    const void* x;
    const void* offset;
    const void* mask;
    void* out;
    int H, W, C, G, D;
    int kh, kw, K;
    int stride, pad, dil;
    int Ho, Wo;
    int tpi;              // threads per item
    int items_per_cta;    // items staged and computed per block
    int total_items;      // N * Ho * Wo * G   (< 2^31)
    int num_blocks;       // ceil(total_items / items_per_cta)
    FastDiv div_G, div_Wo, div_Ho, div_tpi;
    uint32_t pix_bytes;   // C * sizeof(T): byte stride between neighbouring pixels
    uint32_t row_bytes;   // W * C * sizeof(T)
    long long img_bytes;  // H * W * C * sizeof(T)
};

// KH, KW: compile-time window (0 = runtime a.kh / a.kw).
template <typename T, int VB, int KH, int KW, bool SOFTMAX>
__global__ void __launch_bounds__(kDcnThreads, 4) dcn_fwd_kernel(const DcnArgs a) {
    constexpr int CPT = VB / (int)sizeof(T);
    constexpr int NW = VB >= 4 ? VB / 4 : 1;
    extern __shared__ __align__(16) unsigned char smem[];

    const int kh = KH ? KH : a.kh;
    const int kw = KW ? KW : a.kw;
    const int K = kh * kw;
    T* s_off = reinterpret_cast<T*>(smem);
    const int off_span = ((a.items_per_cta * K * 2 * (int)sizeof(T)) + 15) & ~15;
    T* s_mask = reinterpret_cast<T*>(smem + off_span);

    const int li = (int)a.div_tpi.div(threadIdx.x);          // item within the block
    const int chunk = (int)threadIdx.x - li * a.tpi;          // channel chunk of the item

    for (int blk = blockIdx.x; blk < a.num_blocks; blk += gridDim.x) {
        const int item0 = blk * a.items_per_cta;
        const int nitems = min(a.items_per_cta, a.total_items - item0);
        __syncthreads();   // the previous block's shared reads are complete
        stage_span(s_off, static_cast<const T*>(a.offset) + (long long)item0 * K * 2,
                   nitems * K * 2 * (int)sizeof(T));
        stage_span(s_mask, static_cast<const T*>(a.mask) + (long long)item0 * K,
                   nitems * K * (int)sizeof(T));
        __syncthreads();
        if (li >= nitems) continue;

        const int item = item0 + li;
        const int pix = (int)a.div_G.div((uint32_t)item);     // n*Ho*Wo + oy*Wo + ox
        const int g = item - pix * a.G;
        const int t = (int)a.div_Wo.div((uint32_t)pix);
        const int ox = pix - t * a.Wo;
        const int n = (int)a.div_Ho.div((uint32_t)t);
        const int oy = t - n * a.Ho;

        const char* xb = static_cast<const char*>(a.x) + (long long)n * a.img_bytes +
                         (long long)(g * a.D + chunk * CPT) * (int)sizeof(T);
        const T* offp = s_off + li * K * 2;
        const T* maskp = s_mask + li * K;
        const int bx = ox * a.stride - a.pad;
        const int by = oy * a.stride - a.pad;

        // DCNv3: stable softmax of the group's K logits
        float zmax = 0.f, inv_sum = 1.f;
        if constexpr (SOFTMAX) {
            zmax = Elem<T>::one(maskp);
            for (int k = 1; k < K; ++k) zmax = fmaxf(zmax, Elem<T>::one(maskp + k));
            float s = 0.f;
            for (int k = 0; k < K; ++k) s += expf(Elem<T>::one(maskp + k) - zmax);
            inv_sum = 1.f / s;
        }

        float acc[CPT];
#pragma unroll
        for (int i = 0; i < CPT; ++i) acc[i] = 0.f;
        uint32_t r00[NW], r01[NW], r10[NW], r11[NW];   // stale data stays finite
#pragma unroll
        for (int i = 0; i < NW; ++i) r00[i] = r01[i] = r10[i] = r11[i] = 0u;

#pragma unroll 1
        for (int ix = 0; ix < kw; ++ix) {
#pragma unroll
            for (int iy = 0; iy < kh; ++iy) {
                const int k = ix * kh + iy;
                float dx, dy;
                load_pair<T>(offp + 2 * k, dx, dy);
                float m = Elem<T>::one(maskp + k);
                if constexpr (SOFTMAX) m = expf(m - zmax) * inv_sum;

                // integer and fractional parts of the offset
                float fx = floorf(dx), fy = floorf(dy);
                const float ax = dx - fx, ay = dy - fy;
                fx = fminf(fmaxf(fx, -kBigCoord), kBigCoord);
                fy = fminf(fmaxf(fy, -kBigCoord), kBigCoord);
                const int x0 = bx + ix * a.dil + (int)fx;
                const int y0 = by + iy * a.dil + (int)fy;
                const bool vx0 = (unsigned)x0 < (unsigned)a.W;
                const bool vx1 = (unsigned)(x0 + 1) < (unsigned)a.W;
                const bool vy0 = (unsigned)y0 < (unsigned)a.H;
                const bool vy1 = (unsigned)(y0 + 1) < (unsigned)a.H;

                const float mb1 = m * ay;
                const float mb0 = m - mb1;
                const float w00 = (vx0 && vy0) ? (1.f - ax) * mb0 : 0.f;
                const float w01 = (vx1 && vy0) ? ax * mb0 : 0.f;
                const float w10 = (vx0 && vy1) ? (1.f - ax) * mb1 : 0.f;
                const float w11 = (vx1 && vy1) ? ax * mb1 : 0.f;

                // byte offsets within the image; only in-bounds corners are used,
                // and those lie in [0, 2^31), so 32-bit wrap-around is harmless
                const uint32_t o00 = (uint32_t)y0 * a.row_bytes + (uint32_t)x0 * a.pix_bytes;
                const uint32_t o01 = o00 + a.pix_bytes;
                const uint32_t o10 = o00 + a.row_bytes;
                const uint32_t o11 = o10 + a.pix_bytes;
                if (vx0 && vy0) load_vec<VB>(xb + (int)o00, r00);
                if (vx1 && vy0) load_vec<VB>(xb + (int)o01, r01);
                if (vx0 && vy1) load_vec<VB>(xb + (int)o10, r10);
                if (vx1 && vy1) load_vec<VB>(xb + (int)o11, r11);

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
                   ((long long)pix * a.C + g * a.D + chunk * CPT) * (int)sizeof(T);
        store_vec<VB>(ob, o);
    }
}

}  // namespace dcnb
