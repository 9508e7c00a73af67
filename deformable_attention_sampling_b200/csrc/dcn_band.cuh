// DCNv3 / DCNv4 forward with the input neighbourhood staged in shared memory
// (sm_100a): the "band" kernel for 16-bit data with 16 channels per group.
//
// Operator: as dcn_fwd.cuh ("InternImage: Deformable Convolutions at Scale"
// ch.1-4; "DCNv4", "Why Is Sampling Just 9 Points Still Slow?" and "1. Remove
// Softmax"):
//   out[n,oy,ox,g*16+c] = sum_k m[g,k] * bilinear(x[n,:,:,g*16+c], p0 + p_k + dp[g,k])
// zero outside the map; m as given (DCNv4) or soft-maxed over K (DCNv3).
//
// Why a band.  The DCNv4 note ("Why Is Sampling Just 9 Points Still Slow?",
// "2. Move Less Data") puts the compulsory traffic near 3.7 HWC against 36
// corner reads per (pixel, group): the time goes into moving corners, not
// arithmetic.  Corner reads gathered straight through L1 cost one cache tag
// lookup per 32-byte sector, at random positions.  Here every CTA copies the
// full-width input rows its output rows can reach (the undeformed window plus
// a margin of `margin` rows above and below for the offsets) into a ring of
// rows in shared memory, in the map's own NHWC byte order, with bulk copies
// (cp.async.bulk, completion on an mbarrier), and gathers corners from there.
//
// Conflict-free gathers.  With a pixel of C * 2 bytes, a multiple of 128, the
// 32-byte span of group g in any pixel of any staged row lies in banks
// 8 (g mod 4) .. 8 (g mod 4) + 7: the bank of a corner read depends on its
// group and 16-byte half only, never on the (data-dependent) sampling
// position.  Each lane owns one (pixel, group) item, and lanes 4-7 of every
// group of eight read the halves in the opposite order to lanes 0-3, so each
// quarter warp's eight 16-byte reads fall in eight different bank quads: every
// ld.shared.v4 of a warp completes in the minimum four wavefronts.
//
// Pipeline.  A CTA owns a contiguous range of output rows (all images, flat
// n * Ho + oy) and walks it in steps of up to `th` rows of one image.  One
// producer thread issues, per step, the bulk copies of the input rows the step
// adds to the ring and of the step's offset and mask rows (one contiguous span
// each) into one of kBandStages stage buffers, with the byte count on that
// stage's `full` barrier; the consumer warps wait on it, sample the step's
// items, and arrive on the stage's `empty` barrier.  Ring rows are addressed
// by a running "virtual" row number (slot = virtual mod ring_rows); before
// overwriting slots the producer waits until every step that reads them is
// done, so a new image's band can start at any point of the ring.
//
// Taps whose offsets leave the band (|dy| >= margin, about 0.3% at
// dy ~ N(0, 2 px) and a margin of 6 rows) read their four corners from global
// memory instead, under a warp-uniform branch.
//
// Every wait is bounded (about two seconds of %globaltimer); a wait that
// runs out records a timeout in the status word and the thread leaves.
#pragma once

#include <type_traits>

#include "common.cuh"

namespace dcnb {

// Steps in flight (stage buffers of offsets and masks, descriptors, barrier
// pairs): a launch parameter between 2 and kBandMaxStages.
constexpr int kBandMaxStages = 4;
// Lanes per (pixel, group) item of the band samplers: 1 (each lane reads both
// 16-byte halves of the group, 16 channels) or 2 (one half each).  Sampler
// warps per CTA, with the producer warp: 17 warps of up to 120 registers at
// one lane per item, 25 warps of up to 72 registers at two.
#ifndef DCN_BAND_LPI
#define DCN_BAND_LPI 1
#endif
constexpr int kBandLanesPerItem = DCN_BAND_LPI;
static_assert(kBandLanesPerItem == 1 || kBandLanesPerItem == 2, "1 or 2 lanes per item");
// Tap geometry computed one (1) or two (2) taps ahead of the accumulation.
#ifndef DCN_BAND_AHEAD
#define DCN_BAND_AHEAD 1
#endif
#ifndef DCN_BAND_WARPS
#define DCN_BAND_WARPS (DCN_BAND_LPI == 1 ? 16 : 24)
#endif
constexpr int kBandMaxConsumerWarps = DCN_BAND_WARPS;
constexpr int kBandMaxThreads = 32 * (kBandMaxConsumerWarps + 1);
constexpr int kBandDescInts = 8;
constexpr unsigned long long kBandWaitNs = 2000000000ull;   // bound of every wait
// Offset floors are clamped to +-2^22 before the integer conversion; a tap
// that far out has all four corners outside every supported map (H, W <=
// 2^16), and fminf / fmaxf map a NaN offset to the bound.
constexpr float kBandBigCoord = 4194304.0f;

struct BandArgs {
    const void* x;
    const void* offset;
    const void* mask;
    void* out;
    int H, W, C, G;
    int kh, kw, K;
    int stride, pad, dil;
    int Ho, Wo;
    int rows_total;           // N * Ho output rows, numbered n * Ho + oy
    int th;                   // output rows per step (at most)
    int margin;               // offset margin of the band, rows above and below
    int ring_rows;            // rows in the ring
    int consumer_warps;       // warps that sample; one more warp produces
    int stages;               // steps in flight: stage buffers, descriptors, barrier pairs
    int runs_per_row;         // ceil(Wo * G / items per warp run)
    uint32_t row_bytes;       // W * C * 2: one input row
    uint32_t pix_bytes;       // C * 2
    uint32_t off_row_bytes;   // Wo * G * K * 2 * 2: offsets of one output row
    uint32_t mask_row_bytes;  // Wo * G * K * 2
    uint32_t ring_bytes;      // ring_rows * row_bytes (128-byte multiple)
    uint32_t stage_bytes;     // th * (off_row_bytes + mask_row_bytes), 128-byte multiple
    FastDiv div_G, div_Ho, div_runs;
    unsigned int* flags;      // status word (device), or null
    long long x_bytes;        // bytes of x and of out (bounds of the debug library's checks)
    long long out_bytes;
};

__host__ __device__ inline int band_rows(int th, int stride, int kh, int dil, int margin) {
    return (th - 1) * stride + (kh - 1) * dil + 2 * margin + 1;
}

// ------------------------------------------------ barriers, bulk copies ----

__device__ __forceinline__ uint32_t smem_u32(const void* p) {
    return (uint32_t)__cvta_generic_to_shared(p);
}

__device__ __forceinline__ unsigned long long global_ns() {
    unsigned long long t;
    asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
    return t;
}

__device__ __forceinline__ void mbar_init(uint64_t* bar, uint32_t count) {
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" :: "r"(smem_u32(bar)), "r"(count)
                 : "memory");
}

__device__ __forceinline__ void mbar_fence_init() {
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}

__device__ __forceinline__ void mbar_arrive(uint64_t* bar) {
    asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" :: "r"(smem_u32(bar)) : "memory");
}

__device__ __forceinline__ void mbar_arrive_expect_tx(uint64_t* bar, uint32_t bytes) {
    asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;"
                 :: "r"(smem_u32(bar)), "r"(bytes) : "memory");
}

__device__ __forceinline__ bool mbar_try_wait(uint64_t* bar, uint32_t parity) {
    uint32_t done;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(done) : "r"(smem_u32(bar)), "r"(parity) : "memory");
    return done != 0;
}

// Wait for the phase of `bar` with the given parity to complete, for at most
// kBandWaitNs; false (and a timeout recorded in *err) if it did not.
__device__ __forceinline__ bool mbar_wait(uint64_t* bar, uint32_t parity, unsigned int* err) {
    if (mbar_try_wait(bar, parity)) return true;
    const unsigned long long t0 = global_ns();
    for (;;) {
        for (int i = 0; i < 64; ++i)
            if (mbar_try_wait(bar, parity)) return true;
        if (global_ns() - t0 > kBandWaitNs) {
            set_flag(err, kFlagWaitTimeout);
            return false;
        }
    }
}

// Bulk copy of `bytes` (a multiple of 16; both addresses 16-byte aligned) from
// global memory into this CTA's shared memory, completing on `bar`.
__device__ __forceinline__ void bulk_g2s(void* dst, const void* src, uint32_t bytes,
                                         uint64_t* bar) {
    asm volatile(
        "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];"
        :: "r"(smem_u32(dst)), "l"(src), "r"(bytes), "r"(smem_u32(bar)) : "memory");
}

// 16 bytes from shared memory (32-bit shared address).  Volatile, so that it
// is never merged with a read of the same address in an earlier step, and
// never moved above the barrier wait that makes the data valid.
__device__ __forceinline__ void lds128(uint32_t addr, uint32_t* w) {
    asm volatile("ld.shared.v4.b32 {%0,%1,%2,%3}, [%4];"
                 : "=r"(w[0]), "=r"(w[1]), "=r"(w[2]), "=r"(w[3]) : "r"(addr));
}

// An (x, y) offset pair and one modulation of type OT from shared memory
// (32-bit shared addresses), widened to float32.  Volatile for the same reason
// as lds128.
template <typename OT>
__device__ __forceinline__ void lds_pair(uint32_t addr, float& x, float& y) {
    if constexpr (sizeof(OT) == 4) {
        asm volatile("ld.shared.v2.f32 {%0,%1}, [%2];" : "=f"(x), "=f"(y) : "r"(addr));
    } else {
        uint32_t w;
        asm volatile("ld.shared.b32 %0, [%1];" : "=r"(w) : "r"(addr));
        x = Elem<OT>::lo(w);
        y = Elem<OT>::hi(w);
    }
}

template <typename OT>
__device__ __forceinline__ float lds_one(uint32_t addr) {
    if constexpr (sizeof(OT) == 4) {
        float v;
        asm volatile("ld.shared.f32 %0, [%1];" : "=f"(v) : "r"(addr));
        return v;
    } else {
        unsigned short h;
        asm volatile("ld.shared.b16 %0, [%1];" : "=h"(h) : "r"(addr));
        return Elem<OT>::lo((uint32_t)h);
    }
}

// ------------------------------------------------------------- steps -------

// The step that starts at flat output row `cur` (< end): image n, first row o,
// rows nrows (at most th, never past the image or the CTA's range).
struct BandStep {
    int n, o, nrows;
};

__device__ __forceinline__ BandStep band_step(const BandArgs& a, int cur, int end) {
    BandStep s;
    s.n = (int)a.div_Ho.div((uint32_t)cur);
    s.o = cur - s.n * a.Ho;
    s.nrows = min(min(a.th, a.Ho - s.o), end - cur);
    return s;
}

// Descriptor of a step, written by the producer before the step's copies:
// band rows [y_lo, y_hi] of image n (clipped to the map), ring slot of y_lo.
struct BandDesc {
    int y_lo, y_hi, slot_lo, v_lo;
};

// One (pixel, group) item of a band step, sampled by one lane: the item's
// taps read their corners from the staged band (or, for taps that leave it,
// from global memory), accumulate in float32 and store the item's 16 outputs.
// off_s / mask_s: shared addresses of the item's K offset pairs and K
// modulations (or logits), as T (staged from the tensors) or float (computed
// in-kernel).
// Lanes with active = false compute but store nothing.
template <typename T, typename OT, bool SOFTMAX, int KF, int LPI>
__device__ __forceinline__ void band_item(const BandArgs& a, const BandDesc& dsc,
                                          uint32_t ring_s, int n, int oy, int item, bool active,
                                          uint32_t off_s, uint32_t mask_s, int lane) {
    constexpr uint32_t OB = sizeof(OT);
    constexpr int UNROLL = KF ? KF * KF : 1;
    constexpr int NH = 2 / LPI;            // 16-byte halves of the group per lane
    const int kh = KF ? KF : a.kh;
    const int kw = KF ? KF : a.kw;
    const int K = kh * kw;
    const int row_items = a.Wo * a.G;
    const int ox = (int)a.div_G.div((uint32_t)item);
    const int g = item - ox * a.G;
    const int bx = ox * a.stride - a.pad;
    const int by = oy * a.stride - a.pad;
    // byte offsets, inside the group's 32 bytes, of the halves this lane reads
    // in order: one lane per item reads both, lanes 4-7 of every eight in the
    // opposite order; two lanes per item read one half each
    uint32_t hb[NH];
    if constexpr (LPI == 1) {
        const int rot = (lane >> 2) & 1;
        hb[0] = (uint32_t)(rot * 16);
        hb[NH - 1] = (uint32_t)((rot ^ 1) * 16);
    } else {
        hb[0] = (uint32_t)((lane & 1) * 16);
    }
    // shared address of this lane's first half in ring slot 0, pixel 0, and
    // the step from the first half to the second
    const uint32_t lane_s = ring_s + (uint32_t)(g * 32) + hb[0];
    const uint32_t dh = hb[NH - 1] - hb[0];
    const int span = dsc.y_hi - dsc.y_lo;
    const int slot_lo = dsc.slot_lo;
    const char* xg = static_cast<const char*>(a.x) +
                     (long long)n * a.H * a.row_bytes + g * 32;

    float zmax = 0.f, inv_sum = 1.f;
    if constexpr (SOFTMAX) {
        zmax = lds_one<OT>(mask_s);
        for (int k = 1; k < K; ++k) zmax = fmaxf(zmax, lds_one<OT>(mask_s + k * OB));
        float s = 0.f;
        for (int k = 0; k < K; ++k) s += expf(lds_one<OT>(mask_s + k * OB) - zmax);
        inv_sum = 1.f / s;
    }

    float acc[8 * NH];
#pragma unroll
    for (int i = 0; i < 8 * NH; ++i) acc[i] = 0.f;

    // Tap geometry: corner weights (zero outside the map, m folded in),
    // shared addresses of the four corners' halves, and whether a row
    // inside the map lies outside the band (then all four corners come
    // from global memory).
    struct Tap {
        uint32_t s[4];       // shared address of corner c, first half
        float w[4];
        int x0, y0;          // for the global fallback
        bool fb;
    };
    int nix = 0, niy = 0;
    auto geometry = [&]() {
        const int k = nix * kh + niy;
        float dx, dy;
        lds_pair<OT>(off_s + 2 * k * OB, dx, dy);
        float m = lds_one<OT>(mask_s + k * OB);
        if constexpr (SOFTMAX) m = expf(m - zmax) * inv_sum;
        Tap t;
        float fx = floorf(dx), fy = floorf(dy);
        const float ax = dx - fx, ay = dy - fy;
        fx = fminf(fmaxf(fx, -kBandBigCoord), kBandBigCoord);
        fy = fminf(fmaxf(fy, -kBandBigCoord), kBandBigCoord);
        const int x0 = bx + nix * a.dil + (int)fx;
        const int y0 = by + niy * a.dil + (int)fy;
        const bool vx0 = (unsigned)x0 < (unsigned)a.W, vx1 = (unsigned)(x0 + 1) < (unsigned)a.W;
        const bool vy0 = (unsigned)y0 < (unsigned)a.H, vy1 = (unsigned)(y0 + 1) < (unsigned)a.H;
        const float wx0 = vx0 ? 1.f - ax : 0.f, wx1 = vx1 ? ax : 0.f;
        const float wy0 = vy0 ? (1.f - ay) * m : 0.f, wy1 = vy1 ? ay * m : 0.f;
        t.w[0] = wx0 * wy0;
        t.w[1] = wx1 * wy0;
        t.w[2] = wx0 * wy1;
        t.w[3] = wx1 * wy1;
        // rows relative to the band; a row inside the map but outside the
        // band sends the tap to global memory
        const int r0 = y0 - dsc.y_lo;
        const bool in0 = (unsigned)r0 <= (unsigned)span;
        const bool in1 = (unsigned)(r0 + 1) <= (unsigned)span;
        t.fb = (vy0 && !in0) || (vy1 && !in1);
        // rows clamped into the band, columns into the map: every
        // shared read is of a staged row
        int s0 = slot_lo + min(max(r0, 0), span);
        int s1 = slot_lo + min(max(r0 + 1, 0), span);
        if (s0 >= a.ring_rows) s0 -= a.ring_rows;
        if (s1 >= a.ring_rows) s1 -= a.ring_rows;
        const uint32_t c0 = (uint32_t)(vx0 ? x0 : 0) * a.pix_bytes;
        const uint32_t c1 = (uint32_t)(vx1 ? x0 + 1 : 0) * a.pix_bytes;
        const uint32_t b0 = lane_s + (uint32_t)s0 * a.row_bytes;
        const uint32_t b1 = lane_s + (uint32_t)s1 * a.row_bytes;
        t.s[0] = b0 + c0;
        t.s[1] = b0 + c1;
        t.s[2] = b1 + c0;
        t.s[3] = b1 + c1;
        t.x0 = x0;
        t.y0 = y0;
        if (++niy == kh) {
            niy = 0;
            ++nix;
        }
        return t;
    };
    // the four corners of tap t into v (shared memory, then the global
    // fallback for lanes whose tap leaves the band)
    uint32_t v[4][4 * NH];
    auto load_shared = [&](const Tap& t, int c) {
#pragma unroll
        for (int h = 0; h < NH; ++h) {
            const uint32_t ad = h ? t.s[c] + dh : t.s[c];
            if (DCN_IN_BOUNDS(ad >= ring_s && ad + 16 <= ring_s + a.ring_bytes, a.flags)) {
                lds128(ad, &v[c][4 * h]);
            } else {
#pragma unroll
                for (int i = 0; i < 4; ++i) v[c][4 * h + i] = 0u;
            }
        }
    };
    auto load_fallback = [&](const Tap& t) {
        if (__any_sync(0xffffffffu, t.fb) && t.fb) {
            const bool vx0 = (unsigned)t.x0 < (unsigned)a.W;
            const bool vx1 = (unsigned)(t.x0 + 1) < (unsigned)a.W;
            const bool vy0 = (unsigned)t.y0 < (unsigned)a.H;
            const bool vy1 = (unsigned)(t.y0 + 1) < (unsigned)a.H;
            const long long c0 = (long long)(vx0 ? t.x0 : 0) * a.pix_bytes;
            const long long c1 = (long long)(vx1 ? t.x0 + 1 : 0) * a.pix_bytes;
            const long long r0 = (long long)(vy0 ? t.y0 : 0) * a.row_bytes;
            const long long r1 = (long long)(vy1 ? t.y0 + 1 : 0) * a.row_bytes;
            const long long offs[4] = {r0 + c0, r0 + c1, r1 + c0, r1 + c1};
#pragma unroll
            for (int c = 0; c < 4; ++c)
#pragma unroll
                for (int h = 0; h < NH; ++h) {
                    const char* src = xg + offs[c] + hb[h];
                    const char* x0p = static_cast<const char*>(a.x);
                    if (DCN_IN_BOUNDS(src >= x0p && src + 16 <= x0p + a.x_bytes, a.flags)) {
                        load_vec<16>(src, &v[c][4 * h]);
                    } else {
#pragma unroll
                        for (int i = 0; i < 4; ++i) v[c][4 * h + i] = 0u;
                    }
                }
        }
    };

    float w[4];
    {
        const Tap t0 = geometry();
#pragma unroll
        for (int c = 0; c < 4; ++c) {
            load_shared(t0, c);
            w[c] = t0.w[c];
        }
        load_fallback(t0);
    }
#if DCN_BAND_AHEAD == 2
    // geometry two taps ahead of the math: tap k + 2's chain of dependent
    // instructions runs while tap k is accumulated and tap k + 1 loads
    Tap tn;
    if (K > 1) tn = geometry();
#pragma unroll UNROLL
    for (int k = 0; k < K; ++k) {
        const bool more = k + 1 < K;
        Tap tnn;
        if (k + 2 < K) tnn = geometry();
#pragma unroll
        for (int c = 0; c < 4; ++c) {
#pragma unroll
            for (int h = 0; h < NH; ++h) {
                float f[8];
                widen<T, 8>(&v[c][4 * h], f);
                axpy<8>(acc + 8 * h, w[c], f);
            }
            if (more) load_shared(tn, c);
        }
        if (more) {
            load_fallback(tn);
#pragma unroll
            for (int c = 0; c < 4; ++c) w[c] = tn.w[c];
        }
        tn = tnn;
    }
#else
#pragma unroll UNROLL
    for (int k = 0; k < K; ++k) {
        const bool more = k + 1 < K;
        Tap tn;
        if (more) tn = geometry();
#pragma unroll
        for (int c = 0; c < 4; ++c) {
#pragma unroll
            for (int h = 0; h < NH; ++h) {
                float f[8];
                widen<T, 8>(&v[c][4 * h], f);
                axpy<8>(acc + 8 * h, w[c], f);
            }
            if (more) load_shared(tn, c);
        }
        if (more) {
            load_fallback(tn);
#pragma unroll
            for (int c = 0; c < 4; ++c) w[c] = tn.w[c];
        }
    }
#endif

    // acc[8h .. 8h + 7] holds the half at byte hb[h] of the group
    char* ob = static_cast<char*>(a.out) +
               (((long long)n * a.Ho + oy) * row_items + item) * 32;
#pragma unroll
    for (int h = 0; h < NH; ++h) {
        uint32_t o[4];
        narrow<T, 8>(acc + 8 * h, o);
        char* dst = ob + hb[h];
        const char* o0p = static_cast<const char*>(a.out);
        if (active && DCN_IN_BOUNDS(dst >= o0p && dst + 16 <= o0p + a.out_bytes, a.flags))
            store_vec<16>(dst, o);
    }
}

// --------------------------------------------------------------- kernel ----

template <typename T, bool SOFTMAX, int KF>
__global__ void __launch_bounds__(kBandMaxThreads, 1) dcn_band_kernel(const BandArgs a) {
    constexpr int LPI = kBandLanesPerItem;
    constexpr int RUN = 32 / LPI;          // items per warp run
    static_assert(sizeof(T) == 2, "the band kernel handles 16-bit data");
    extern __shared__ __align__(128) unsigned char band_smem[];
    const int NS = a.stages;
    unsigned char* ring = band_smem;
    unsigned char* stages = band_smem + a.ring_bytes;
    uint64_t* full = reinterpret_cast<uint64_t*>(stages + NS * a.stage_bytes);
    uint64_t* empty = full + NS;
    int* descs = reinterpret_cast<int*>(empty + NS);

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    const int nc = a.consumer_warps;
    if (threadIdx.x == 0) {
        for (int s = 0; s < NS; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&empty[s], (uint32_t)nc);
        }
        mbar_fence_init();
    }
    __syncthreads();

    const int r_begin = (int)(((long long)a.rows_total * blockIdx.x) / gridDim.x);
    const int r_end = (int)(((long long)a.rows_total * (blockIdx.x + 1)) / gridDim.x);

    // ------------------------------------------------------------ producer
    if (warp == nc) {
        if (lane != 0) return;
        const char* xg = static_cast<const char*>(a.x);
        const char* offg = static_cast<const char*>(a.offset);
        const char* mg = static_cast<const char*>(a.mask);
        const int RB = a.ring_rows;
        int prev_n = -1, prev_ylo = 0, prev_yhi = -1, prev_vlo = 0;
        int next_v = 0;
        int done = -1;          // every step <= done has been released by all consumers
        int step = 0;
        for (int cur = r_begin; cur < r_end; ++step) {
            const BandStep st = band_step(a, cur, r_end);
            const int y_lo = max(0, st.o * a.stride - a.pad - a.margin);
            const int y_hi = min(a.H - 1, (st.o + st.nrows - 1) * a.stride - a.pad +
                                              (a.kh - 1) * a.dil + a.margin);
            int v_lo, first_new;
            if (st.n == prev_n && y_lo >= prev_ylo && y_lo <= prev_yhi + 1) {
                v_lo = prev_vlo + (y_lo - prev_ylo);        // the band continues
                first_new = max(y_lo, prev_yhi + 1);
            } else {
                v_lo = next_v;                              // a fresh band
                first_new = y_lo;
            }
            const int v_hi = v_lo + (y_hi - y_lo);
            const int v_first_new = v_lo + (first_new - y_lo);
            // free the stage buffer (step - NS) and every ring slot
            // that the new rows overwrite (steps whose band starts at or below
            // v_hi - RB)
            while (done < step - 1) {
                const int t = done + 1;
                const BandDesc* dt =
                    reinterpret_cast<const BandDesc*>(descs + (t % NS) * kBandDescInts);
                const bool must = t <= step - NS ||
                                  (first_new <= y_hi && dt->v_lo <= v_hi - RB);
                if (!must) break;
                if (!mbar_wait(&empty[t % NS], (uint32_t)((t / NS) & 1),
                               a.flags))
                    return;
                done = t;
            }
            const int sb = step % NS;
            BandDesc* d = reinterpret_cast<BandDesc*>(descs + sb * kBandDescInts);
            d->y_lo = y_lo;
            d->y_hi = y_hi;
            d->slot_lo = v_lo % RB;
            d->v_lo = v_lo;
            const int new_rows = y_hi >= first_new ? y_hi - first_new + 1 : 0;
            const uint32_t off_bytes = (uint32_t)st.nrows * a.off_row_bytes;
            const uint32_t m_bytes = (uint32_t)st.nrows * a.mask_row_bytes;
            mbar_arrive_expect_tx(&full[sb], (uint32_t)new_rows * a.row_bytes + off_bytes + m_bytes);
            // new rows: contiguous in global memory; in the ring up to the wrap
            if (new_rows > 0) {
                const char* src = xg + ((long long)st.n * a.H + first_new) * a.row_bytes;
                int slot = v_first_new % RB;
                int left = new_rows;
                while (left > 0) {
                    const int cnt = min(left, RB - slot);
                    bulk_g2s(ring + (uint32_t)slot * a.row_bytes, src, (uint32_t)cnt * a.row_bytes,
                             &full[sb]);
                    src += (long long)cnt * a.row_bytes;
                    left -= cnt;
                    slot = 0;
                }
            }
            const long long orow = (long long)st.n * a.Ho + st.o;
            unsigned char* sbuf = stages + sb * a.stage_bytes;
            bulk_g2s(sbuf, offg + orow * a.off_row_bytes, off_bytes, &full[sb]);
            bulk_g2s(sbuf + (uint32_t)a.th * a.off_row_bytes, mg + orow * a.mask_row_bytes, m_bytes,
                     &full[sb]);
            prev_n = st.n;
            prev_ylo = y_lo;
            prev_yhi = y_hi;
            prev_vlo = v_lo;
            next_v = max(next_v, v_hi + 1);
            cur += st.nrows;
        }
        // leave only once the copies of the last stages have landed
        for (int t = max(0, step - NS); t < step; ++t)
            if (!mbar_wait(&full[t % NS], (uint32_t)((t / NS) & 1), a.flags))
                return;
        return;
    }

    // ----------------------------------------------------------- consumers
    const int K = KF ? KF * KF : a.K;
    const uint32_t ring_s = smem_u32(ring);
    const int row_items = a.Wo * a.G;

    // runs are dealt to the consumer warps round-robin over the CTA's whole
    // range (run j of the range to warp j mod nc), so that when a step has
    // fewer runs than there are warps, the rest start on the next step
    int step = 0;
    int j0 = 0;                 // index in the range of this step's first run
    for (int cur = r_begin; cur < r_end; ++step) {
        const BandStep st = band_step(a, cur, r_end);
        cur += st.nrows;
        const int sb = step % NS;
        if (!mbar_wait(&full[sb], (uint32_t)((step / NS) & 1), a.flags)) return;
        const BandDesc dsc = *reinterpret_cast<const BandDesc*>(descs + sb * kBandDescInts);
        const uint32_t sbuf_s = smem_u32(stages + sb * a.stage_bytes);
        const int runs = st.nrows * a.runs_per_row;
        const int r_first = (warp - j0 % nc + nc) % nc;
        j0 += runs;
        for (int r = r_first; r < runs; r += nc) {
            const int row_local = (int)a.div_runs.div((uint32_t)r);
            const int run_in_row = r - row_local * a.runs_per_row;
            // lanes past the end of the row compute a copy of the row's last
            // item and store nothing (every lane takes part in the warp votes)
            const bool active = run_in_row * RUN + lane / LPI < row_items;
            const int item = active ? run_in_row * RUN + lane / LPI : row_items - 1;
            const int oy = st.o + row_local;
            const uint32_t off_s = sbuf_s + row_local * a.off_row_bytes +
                                   (uint32_t)(item * K * 2 * (int)sizeof(T));
            const uint32_t mask_s = sbuf_s + a.th * a.off_row_bytes +
                                    row_local * a.mask_row_bytes +
                                    (uint32_t)(item * K * (int)sizeof(T));
            band_item<T, T, SOFTMAX, KF, LPI>(a, dsc, ring_s, st.n, oy, item, active, off_s,
                                              mask_s, lane);
        }
        __syncwarp();
        if (lane == 0) mbar_arrive(&empty[sb]);
    }
}

}  // namespace dcnb
