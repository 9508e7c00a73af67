// DCNv3 / DCNv4 deformable sampling-aggregation backward, sm_100a SIMT kernel.
//
// Gradients of out[n,oy,ox,g*D+c] = sum_k m_k * B(x_g, p_k) ("InternImage"
// ch.2-3 and "DCNv4" "1. Remove Softmax": the op is differentiable in x, in
// the offsets through the bilinear weights, and in the modulation):
//   grad_x     scatter: each corner of each tap receives m_k * w_corner * go
//   grad_off   m_k * dB/dpx, m_k * dB/dpy  (one-sided at integer positions,
//              where floor() jumps: the derivative of the right-hand cell)
//   grad_mask  <go, B(x_g, p_k)>, and for DCNv3 the softmax Jacobian on top:
//              dL/dz_k = m_k * (dL/dm_k - sum_j m_j dL/dm_j).
//
// Work decomposition, tiles and shared-memory staging are the forward's: an
// item is an (output pixel, group) pair served by TPI threads that own CPT
// channels each; a warp serves a run of 32/TPI items of one output row.  Per
// tap a thread forms, for each of the four corners, the dot product
// P_c = sum over its channels of go * x_corner, then
//   dL/dm_k = wy0 (wx0 P00 + wx1 P01) + wy1 (wx0 P10 + wx1 P11)
//   dB/da   = wy0 (P01 - P00) + wy1 (P11 - P10)
//   dB/db   = wx0 (P10 - P00) + wx1 (P11 - P01)
// with P = 0 for corners outside the map, and reduces the three over the
// item's threads with warp shuffles.  The grad_x scatter goes to a float32
// accumulator with vector reductions (red.global.add.v4.f32: 16 bytes per
// instruction, resolved in L2), issued so that each instruction of a lane
// pair fills whole 32-byte sectors when an item has an even number of 8-channel
// lanes (the reduction throughput of L2 is per sector); the caller's launch
// sequence zeroes the accumulator first and, for 16-bit data, rounds it into
// grad_x afterwards.
// grad_offset and grad_mask of a run are collected in the warp's shared slice
// and written with coalesced stores.
#pragma once

#include "dcn_fwd.cuh"

namespace dcnb {

constexpr int kDcnBwdMaxWarps = 16;   // 128 registers: 16 warps per SM
constexpr int kDcnBwdMaxThreads = 32 * kDcnBwdMaxWarps;

struct DcnBwdArgs {
    DcnArgs f;                 // forward geometry; f.out is unused
    const void* grad_out;      // [N][Ho][Wo][C]
    void* grad_offset;         // [N][Ho][Wo][G][K][2]
    void* grad_mask;           // [N][Ho][Wo][G][K]
    float* gx_acc;             // float32 [N][H][W][C], zero on entry
    int red_vec;               // floats per reduction instruction: 4, 2 or 1
};

// ------------------------------------------------------------ reductions --

__device__ __forceinline__ void red_add4(float* p, float a, float b, float c, float d) {
    asm volatile("red.global.add.v4.f32 [%0], {%1,%2,%3,%4};"
                 :: "l"(p), "f"(a), "f"(b), "f"(c), "f"(d) : "memory");
}
__device__ __forceinline__ void red_add2(float* p, float a, float b) {
    asm volatile("red.global.add.v2.f32 [%0], {%1,%2};" :: "l"(p), "f"(a), "f"(b) : "memory");
}
__device__ __forceinline__ void red_add1(float* p, float a) {
    asm volatile("red.global.add.f32 [%0], %1;" :: "l"(p), "f"(a) : "memory");
}

// p[i] += coef * g[i] for i < CPT, with the widest reduction `rv` allows
// (rv divides CPT and p is aligned to rv floats; checked on the host).
template <int CPT>
__device__ __forceinline__ void scatter_scaled(float* p, float coef, const float* g, int rv) {
    if constexpr (CPT % 4 == 0) {
        if (rv == 4) {
#pragma unroll
            for (int i = 0; i < CPT; i += 4)
                red_add4(p + i, coef * g[i], coef * g[i + 1], coef * g[i + 2], coef * g[i + 3]);
            return;
        }
    }
    if constexpr (CPT % 2 == 0) {
        if (rv == 2) {
#pragma unroll
            for (int i = 0; i < CPT; i += 2) red_add2(p + i, coef * g[i], coef * g[i + 1]);
            return;
        }
    }
#pragma unroll
    for (int i = 0; i < CPT; ++i) red_add1(p + i, coef * g[i]);
}

// Copy `elems` elements of T from shared `src` (16-byte aligned) to global
// `dst` with the lanes of one warp, using the widest store that the
// destination address and the size allow.
template <typename T>
__device__ __forceinline__ void warp_stage_out(T* dst, const T* src, int elems, int lane) {
    const int nbytes = elems * (int)sizeof(T);
    const uintptr_t al = (uintptr_t)dst | (uintptr_t)nbytes;
    if ((al & 15) == 0) {
        const uint4* s = reinterpret_cast<const uint4*>(src);
        uint4* d = reinterpret_cast<uint4*>(dst);
        for (int i = lane; i < (nbytes >> 4); i += 32) d[i] = s[i];
    } else if ((al & 7) == 0) {
        const uint2* s = reinterpret_cast<const uint2*>(src);
        uint2* d = reinterpret_cast<uint2*>(dst);
        for (int i = lane; i < (nbytes >> 3); i += 32) d[i] = s[i];
    } else if ((al & 3) == 0) {
        const uint32_t* s = reinterpret_cast<const uint32_t*>(src);
        uint32_t* d = reinterpret_cast<uint32_t*>(dst);
        for (int i = lane; i < (nbytes >> 2); i += 32) d[i] = s[i];
    } else {
        const unsigned short* s = reinterpret_cast<const unsigned short*>(src);
        unsigned short* d = reinterpret_cast<unsigned short*>(dst);
        for (int i = lane; i < (nbytes >> 1); i += 32) d[i] = s[i];
    }
}

// Sector-paired scatter (CPT = 8, an even number of lanes per item).  L2
// resolves reductions per 32-byte sector, so two 16-byte reductions to one
// sector cost as much as two full ones.  The two lanes 2j, 2j+1 of an item own
// 8 channels each (one float32 sector each); in the first instruction both
// add to lane 2j's sector (lane 2j its channels 0-3, lane 2j+1 lane 2j's
// channels 4-7), in the second both add to lane 2j+1's sector.  The values a
// lane adds are fixed per item: v1 / v2 and the float offsets d1 / d2 come
// from pair_setup, so the scatter itself is branch-free.
struct PairScatter {
    float v1[4], v2[4];
    int d1, d2;
};

// Every lane of the warp must call it (one shuffle exchange per item).
__device__ __forceinline__ PairScatter pair_setup(const float* go, int chunk) {
    PairScatter ps;
    const bool odd = chunk & 1;
    float recv[4];
#pragma unroll
    for (int i = 0; i < 4; ++i)   // the partner's half that this lane adds
        recv[i] = __shfl_xor_sync(0xffffffffu, odd ? go[i] : go[4 + i], 1);
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        ps.v1[i] = odd ? recv[i] : go[i];        // lane 2j's sector
        ps.v2[i] = odd ? go[4 + i] : recv[i];    // lane 2j+1's sector
    }
    ps.d1 = odd ? -4 : 0;
    ps.d2 = odd ? 4 : 8;
    return ps;
}

// p = this lane's first channel in the accumulator
__device__ __forceinline__ void scatter_pair(float* p, float coef, const PairScatter& ps) {
    red_add4(p + ps.d1, coef * ps.v1[0], coef * ps.v1[1], coef * ps.v1[2], coef * ps.v1[3]);
    red_add4(p + ps.d2, coef * ps.v2[0], coef * ps.v2[1], coef * ps.v2[2], coef * ps.v2[3]);
}

// sum_i a[i] * b[i] for i < CPT (two lanes per FFMA2)
template <int CPT>
__device__ __forceinline__ float dot(const float* a, const float* b) {
    float2 s = make_float2(0.f, 0.f);
#pragma unroll
    for (int i = 0; i + 1 < CPT; i += 2)
        s = __ffma2_rn(make_float2(a[i], a[i + 1]), make_float2(b[i], b[i + 1]), s);
    float r = s.x + s.y;
    if constexpr (CPT % 2 == 1) r = fmaf(a[CPT - 1], b[CPT - 1], r);
    return r;
}

// Sum of v over the `tpi` consecutive lanes that serve one item (lanes
// [base, base + tpi)); every lane of the warp must call it.  Power-of-two
// groups use a butterfly, other group sizes a rotation.
__device__ __forceinline__ float item_sum(float v, int tpi, int base, int chunk) {
    if (tpi == 1) return v;
    if ((tpi & (tpi - 1)) == 0) {
        for (int s = 1; s < tpi; s <<= 1) v += __shfl_xor_sync(0xffffffffu, v, s);
        return v;
    }
    float total = v;
    for (int s = 1; s < tpi; ++s) {
        int src = chunk + s;
        if (src >= tpi) src -= tpi;
        total += __shfl_sync(0xffffffffu, v, base + src);
    }
    return total;
}

// One tap of one item for the backward: byte offsets (within the image) of the
// four corners, clamped into the map; the fractions; a bit per corner that
// lies inside the map (bit c for corner c = 00, 01, 10, 11 as (y, x)).
struct BwdTap {
    uint32_t off[4];
    float ax, ay;
    uint32_t valid;
};

__device__ __forceinline__ BwdTap bwd_tap(const DcnArgs& a, int bxk, int byk, float dx,
                                          float dy) {
    BwdTap t;
    float fx = floorf(dx), fy = floorf(dy);
    fx = fminf(fmaxf(fx, -kBigCoord), kBigCoord);
    fy = fminf(fmaxf(fy, -kBigCoord), kBigCoord);
    // exact for finite offsets within the clamp; NaN or far taps (all corners
    // outside) get a finite fraction so that their zero products stay zero
    t.ax = fminf(fmaxf(dx - fx, 0.f), 1.f);
    t.ay = fminf(fmaxf(dy - fy, 0.f), 1.f);
    const int x0 = bxk + (int)fx, y0 = byk + (int)fy;
    const int x1 = x0 + 1, y1 = y0 + 1;
    const bool vx0 = (unsigned)x0 < (unsigned)a.W, vx1 = (unsigned)x1 < (unsigned)a.W;
    const bool vy0 = (unsigned)y0 < (unsigned)a.H, vy1 = (unsigned)y1 < (unsigned)a.H;
    t.valid = (uint32_t)(vx0 && vy0) | ((uint32_t)(vx1 && vy0) << 1) |
              ((uint32_t)(vx0 && vy1) << 2) | ((uint32_t)(vx1 && vy1) << 3);
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

// Byte sizes of the parts of one warp's shared slice (each a multiple of 16):
// staged offsets and masks (inputs), then grad_offset and grad_mask (outputs),
// then, for DCNv3, the float32 dL/dm of every tap of the run.
struct BwdSlice {
    int off_in, mask_in, off_out, mask_out, gm;
    __host__ __device__ int total() const { return off_in + mask_in + off_out + mask_out + gm; }
};

__host__ __device__ inline BwdSlice bwd_slice(int run_items, int K, int es, bool softmax) {
    BwdSlice s;
    s.off_in = (2 * run_items * K * es + 15) & ~15;
    s.mask_in = (run_items * K * es + 15) & ~15;
    s.off_out = s.off_in;
    s.mask_out = s.mask_in;
    s.gm = softmax ? ((run_items * K * 4 + 15) & ~15) : 0;
    return s;
}

// PAIR: the sector-paired scatter (CPT = 8, an even number of lanes per item),
// chosen on the host; otherwise plain vector reductions of width b.red_vec.
template <typename T, int VB, bool SOFTMAX, int KF = 0, bool PAIR = false>
__global__ void __launch_bounds__(kDcnBwdMaxThreads, 1) dcn_bwd_kernel(const DcnBwdArgs b) {
    constexpr int UNROLL = KF ? KF * KF : 1;
    constexpr int CPT = VB / (int)sizeof(T);
    constexpr int NW = VB >= 4 ? VB / 4 : 1;
    constexpr int es = (int)sizeof(T);
    extern __shared__ __align__(16) unsigned char smem[];
    const DcnArgs& a = b.f;

    const int kh = KF ? KF : a.kh;
    const int kw = KF ? KF : a.kw;
    const int K = kh * kw;
    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    const BwdSlice sl = bwd_slice(a.run_items, K, es, SOFTMAX);
    unsigned char* my = smem + warp * sl.total();
    T* s_off = reinterpret_cast<T*>(my);
    T* s_mask = reinterpret_cast<T*>(my + sl.off_in);
    T* s_goff = reinterpret_cast<T*>(my + sl.off_in + sl.mask_in);
    T* s_gmask = reinterpret_cast<T*>(my + sl.off_in + sl.mask_in + sl.off_out);
    float* s_gm = reinterpret_cast<float*>(my + sl.off_in + sl.mask_in + sl.off_out +
                                           sl.mask_out);

    const int li_raw = (int)a.div_tpi.div((uint32_t)lane);   // item within the run
    const int chunk = lane - li_raw * a.tpi;
    const int row_items = a.Wo * a.G;
    const int warp_row = (int)a.div_tile_w.div((uint32_t)warp);
    const int warp_col = warp - warp_row * a.tile_w;

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
        const int i0 = run * a.run_items;
        const int nitems = min(a.run_items, row_items - i0);
        const long long item_base = ((long long)n * a.Ho + oy) * row_items + i0;

        __syncwarp();   // the previous run's shared reads and writes are done
        warp_stage(s_off, static_cast<const T*>(a.offset) + item_base * K * 2, nitems * K * 2,
                   lane);
        warp_stage(s_mask, static_cast<const T*>(a.mask) + item_base * K, nitems * K, lane);
        __syncwarp();

        // Lanes past the run's last item (or past the last whole item of the
        // warp) shadow item 0 with a zero upstream gradient: they take part in
        // the shuffles and write nothing.
        const bool active = li_raw < nitems;
        const int li = active ? li_raw : 0;
        const T* offp = s_off + li * K * 2;
        const T* maskp = s_mask + li * K;
        const int item_in_row = i0 + li;
        const int ox = (int)a.div_G.div((uint32_t)item_in_row);
        const int g = item_in_row - ox * a.G;
        const long long ch = (long long)g * a.D + chunk * CPT;   // first channel of the lane
        const char* xb = static_cast<const char*>(a.x) + (long long)n * a.img_bytes + ch * es;
        float* gxb = b.gx_acc + (long long)n * a.H * a.W * a.C + ch;
        const int bx = ox * a.stride - a.pad;
        const int by = oy * a.stride - a.pad;

        float go[CPT];
        {
            uint32_t w[NW];
            load_vec<VB>(static_cast<const char*>(b.grad_out) +
                             ((item_base + li) * a.D + chunk * CPT) * es,
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

        float zmax = 0.f, inv_sum = 1.f;
        if constexpr (SOFTMAX) {
            zmax = Elem<T>::one(maskp);
            for (int k = 1; k < K; ++k) zmax = fmaxf(zmax, Elem<T>::one(maskp + k));
            float s = 0.f;
            for (int k = 0; k < K; ++k) s += expf(Elem<T>::one(maskp + k) - zmax);
            inv_sum = 1.f / s;
        }
        auto modulation = [&](int k) {
            const float z = Elem<T>::one(maskp + k);
            if constexpr (SOFTMAX) return expf(z - zmax) * inv_sum;
            return z;
        };

        // rolling corner pipeline over the taps, as in the forward
        uint32_t v[4][NW];
        int nix = 0, niy = 0;
        auto geometry = [&]() {
            const int k = nix * kh + niy;
            float dx, dy;
            load_pair<T>(offp + 2 * k, dx, dy);
            const BwdTap t = bwd_tap(a, bx + nix * a.dil, by + niy * a.dil, dx, dy);
            if (++niy == kh) {
                niy = 0;
                ++nix;
            }
            return t;
        };
        BwdTap cur = geometry();
#pragma unroll
        for (int c = 0; c < 4; ++c) load_vec<VB>(xb + cur.off[c], v[c]);
        float dot_mg = 0.f;   // sum_k m_k dL/dm_k (DCNv3)

#pragma unroll UNROLL
        for (int k = 0; k < K; ++k) {
            const bool more = k + 1 < K;
            BwdTap nxt;
            if (more) nxt = geometry();
            float P[4];
#pragma unroll
            for (int c = 0; c < 4; ++c) {
                float f[CPT];
                widen<T, CPT>(v[c], f);
                P[c] = (cur.valid >> c) & 1u ? dot<CPT>(go, f) : 0.f;
                if (more) load_vec<VB>(xb + nxt.off[c], v[c]);
            }
            const float m = modulation(k);
            const float wx0 = 1.f - cur.ax, wx1 = cur.ax;
            const float wy0 = 1.f - cur.ay, wy1 = cur.ay;
            // grad_x scatter of this tap's four corners
#pragma unroll
            for (int c = 0; c < 4; ++c) {
                const float wc = (c & 1 ? wx1 : wx0) * (c & 2 ? wy1 : wy0);
                if (active && ((cur.valid >> c) & 1u)) {
                    if constexpr (PAIR)
                        scatter_pair(gxb + cur.off[c] / es, m * wc, ps);
                    else
                        scatter_scaled<CPT>(gxb + cur.off[c] / es, m * wc, go, b.red_vec);
                }
            }
            float gm = wy0 * (wx0 * P[0] + wx1 * P[1]) + wy1 * (wx0 * P[2] + wx1 * P[3]);
            float da = wy0 * (P[1] - P[0]) + wy1 * (P[3] - P[2]);
            float db = wx0 * (P[2] - P[0]) + wx1 * (P[3] - P[1]);
            gm = item_sum(gm, a.tpi, li_raw * a.tpi, chunk);
            da = item_sum(da, a.tpi, li_raw * a.tpi, chunk);
            db = item_sum(db, a.tpi, li_raw * a.tpi, chunk);
            if (active && chunk == 0) {
                const int idx = li * K + k;
                s_goff[2 * idx] = Elem<T>::from(m * da);
                s_goff[2 * idx + 1] = Elem<T>::from(m * db);
                if constexpr (SOFTMAX) {
                    s_gm[idx] = gm;
                    dot_mg = fmaf(m, gm, dot_mg);
                } else {
                    s_gmask[idx] = Elem<T>::from(gm);
                }
            }
            if (more) cur = nxt;
        }

        if constexpr (SOFTMAX) {
            if (active && chunk == 0) {
                for (int k = 0; k < K; ++k) {
                    const int idx = li * K + k;
                    s_gmask[idx] = Elem<T>::from(modulation(k) * (s_gm[idx] - dot_mg));
                }
            }
        }
        __syncwarp();
        warp_stage_out(static_cast<T*>(b.grad_offset) + item_base * K * 2, s_goff,
                       nitems * K * 2, lane);
        warp_stage_out(static_cast<T*>(b.grad_mask) + item_base * K, s_gmask, nitems * K, lane);
    }
}

}  // namespace dcnb

namespace dcnb {

// ------------------------------------------------ accumulator set-up / wrap-up

constexpr int kUtilThreads = 256;

struct ZeroArgs {
    float* p;
    long long n;
};

template <typename T>
struct RoundArgs {
    const float* src;
    T* dst;
    long long n;
    int vec4;
};

// p[0, n) = 0, with 16-byte stores on the aligned body.
static __global__ void __launch_bounds__(kUtilThreads) zero_f32_kernel(const ZeroArgs z) {
    float* p = z.p;
    const long long n = z.n;
    const long long tid = (long long)blockIdx.x * blockDim.x + threadIdx.x;
    const long long nthreads = (long long)gridDim.x * blockDim.x;
    long long head = (long long)(((16u - ((uintptr_t)p & 15u)) & 15u) >> 2);
    if (head > n) head = n;
    const long long nv = (n - head) >> 2;
    if (tid < head) p[tid] = 0.f;
    float4* body = reinterpret_cast<float4*>(p + head);
    for (long long i = tid; i < nv; i += nthreads) body[i] = make_float4(0.f, 0.f, 0.f, 0.f);
    const long long tail = head + nv * 4;
    if (tid < n - tail) p[tail + tid] = 0.f;
}

// dst[i] = round(src[i]) for i < n.  src is 16-byte aligned; vec4 = 1 when dst
// is aligned to four elements, so that each thread converts a float4 at once.
template <typename T>
__global__ void __launch_bounds__(kUtilThreads) round_f32_kernel(const RoundArgs<T> r) {
    const float* src = r.src;
    T* dst = r.dst;
    const long long n = r.n;
    const int vec4 = r.vec4;
    const long long tid = (long long)blockIdx.x * blockDim.x + threadIdx.x;
    const long long nthreads = (long long)gridDim.x * blockDim.x;
    long long done = 0;
    if (vec4) {
        const long long nv = n >> 2;
        const float4* s = reinterpret_cast<const float4*>(src);
        for (long long i = tid; i < nv; i += nthreads) {
            float4 f;
            asm("ld.global.nc.L1::no_allocate.v4.f32 {%0,%1,%2,%3}, [%4];"
                : "=f"(f.x), "=f"(f.y), "=f"(f.z), "=f"(f.w) : "l"(s + i));
            const float fs[4] = {f.x, f.y, f.z, f.w};
            uint32_t w[4];
            narrow<T, 4>(fs, w);
            if constexpr (sizeof(T) == 4) {
                store_vec<16>(dst + 4 * i, w);
            } else {
                store_vec<8>(dst + 4 * i, w);
            }
        }
        done = nv * 4;
    }
    for (long long i = done + tid; i < n; i += nthreads) dst[i] = Elem<T>::from(src[i]);
}

}  // namespace dcnb
