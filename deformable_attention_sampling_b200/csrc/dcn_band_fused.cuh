// DCNv4 forward with its merged offset / mask linear on the tensor cores
// (tcgen05, accumulators in TMEM) feeding the band sampler (sm_100a).
//
// "DCNv4" note, "1. Remove Softmax": one linear layer gives every location its
// G*K offset pairs and G*K modulation scalars, used without a softmax; the
// sampling core is that of dcn_band.cuh.  For every output pixel p (stride 1,
// same-size window, so output pixel p reads input pixel p):
//   om[p][j] = sum_c x[p][c] w_om[j][c] + b_om[j],   j < J = 3 G K
//   offsets = om[p][0 .. 2GK) in [G][K][2] order, masks = om[p][2GK .. 3GK)
// The offsets and masks never leave the SM and are never rounded to 16 bits.
//
// Per step of `th` output rows (th * W <= 128 pixels) of one image:
//   producer  (one thread)  bulk-copies the ring rows the step adds (as in
//             dcn_band.cuh) and, with a tensor-map load (cp.async.bulk.tensor,
//             128-byte swizzle), the step's pixels as the A tile [128 rows][C]
//             of the product; the weight matrix (B tile [NJ rows][C]) is loaded
//             the same way once per CTA;
//   MMA       (one thread of the MMA warp) issues C / 16 tcgen05.mma (kind::f16,
//             M = 128, N = NJ, K = 16, float32 accumulation) into one of two
//             TMEM accumulator stages and commits them to an mbarrier;
//   epilogue  (four warps, one per TMEM lane quarter) reads the accumulators
//             with tcgen05.ld (thread = pixel), adds the bias and writes the
//             step's offsets and masks, float32, into one of two shared buffers;
//   samplers  wait for the ring rows and that buffer and run band_item with
//             float32 offsets and masks.
// Each hand-over is an mbarrier; every wait is bounded (as in dcn_band.cuh).
// A role whose wait runs out records the timeout and stops its loop; all
// threads then meet at the final CTA barrier, after which the MMA warp frees
// the TMEM it allocated.
#pragma once

#include <cuda.h>

#include "dcn_band.cuh"

namespace dcnb {

constexpr int kFusedEpilogueWarps = 4;
// Warps per CTA: 10 samplers, the producer, the MMA warp and 4 epilogue
// warps.  Measured on the 64 x 56 x 56 x 64 fp16 front end with the tap loop
// not unrolled, us per launch: 114.0 with 10 samplers, 120.8 with 12, 117.6
// with 14, 128.2 with 18 (with the taps unrolled: 137.6 / 137.7 / 133.8 /
// 142.3).
#ifndef DCN_FUSED_WARPS
#define DCN_FUSED_WARPS 16
#endif
constexpr int kFusedMaxThreads = 32 * DCN_FUSED_WARPS;

struct BandFusedArgs {
    CUtensorMap tmap_x;        // x viewed as [N*H*W rows][C], box {64, a_rows}, 128-byte swizzle
    CUtensorMap tmap_w;        // w_om viewed as [J rows][C], box {64, NJ}, 128-byte swizzle
    BandArgs b;                // sampler geometry (offset / mask unused)
    const void* b_om;          // bias [J] or null
    int J;                     // 3 * G * K
    int NJ;                    // J rounded up to a multiple of 16: the MMA's N
    int kchunks;               // C / 64: 128-byte K slices of the A and B tiles
    int a_rows;                // th * W: pixels (rows) of one A tile load
    int consumer_warps;        // sampler warps
    uint32_t tmem_cols;        // TMEM columns allocated (power of 2 >= 2 * NJ)
    uint32_t a_bytes;          // one A stage: kchunks * 128-byte K slices of a_stage_rows rows
    uint32_t a_box_bytes;      // bytes one step's A loads deliver: kchunks * a_rows * 128
    uint32_t w_bytes;          // kchunks * NJ * 128 B
    uint32_t om_stride;        // floats per pixel in the om buffer (J rounded up to 4)
    uint32_t om_bytes;         // one om buffer: th * W * om_stride * 4, 16-byte multiple
};

// ------------------------------------------------------ tcgen05 helpers ----

// Shared-memory matrix descriptor of a K-major tile with the 128-byte swizzle:
// 8-row groups 1024 bytes apart (stride byte offset), 16-byte leading offset,
// descriptor version 1, layout type 2 (SWIZZLE_128B).
__device__ __forceinline__ uint64_t umma_desc_k128(uint32_t smem_addr) {
    return (uint64_t)((smem_addr >> 4) & 0x3FFFu) | ((uint64_t)1u << 16) |
           ((uint64_t)(1024u >> 4) << 32) | ((uint64_t)1u << 46) | ((uint64_t)2u << 61);
}

// Instruction descriptor of tcgen05.mma kind::f16: float32 accumulator, A and
// B both f16 (or both bf16), both K-major, N = n, M = 128.
template <typename T>
__device__ __forceinline__ uint32_t umma_idesc_f16(int n) {
    constexpr uint32_t ab = std::is_same<T, __nv_bfloat16>::value ? 1u : 0u;
    return (1u << 4) | (ab << 7) | (ab << 10) | ((uint32_t)(n >> 3) << 17) |
           ((uint32_t)(128 >> 4) << 24);
}

__device__ __forceinline__ void umma_f16(uint32_t tmem_d, uint64_t adesc, uint64_t bdesc,
                                         uint32_t idesc, uint32_t accumulate) {
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}"
        :: "r"(tmem_d), "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate) : "memory");
}

__device__ __forceinline__ void umma_commit(uint64_t* bar) {
    asm volatile(
        "tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];"
        :: "r"(smem_u32(bar)) : "memory");
}

__device__ __forceinline__ void tmem_fence_before() {
    asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
}

__device__ __forceinline__ void tmem_fence_after() {
    asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
}

// 16 consecutive 32-bit TMEM columns of this thread's lane.
__device__ __forceinline__ void tmem_ld16(uint32_t taddr, uint32_t* r) {
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x16.b32 "
        "{%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15}, [%16];"
        : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
          "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]),
          "=r"(r[13]), "=r"(r[14]), "=r"(r[15])
        : "r"(taddr));
}

__device__ __forceinline__ void tmem_wait_ld() {
    asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
}

// 2-D tensor-map tile load (no multicast) into this CTA's shared memory,
// completing on `bar`: box origin (c0 = column, c1 = row).
__device__ __forceinline__ void tma_load_2d(void* dst, const CUtensorMap* map, int c0, int c1,
                                            uint64_t* bar) {
    asm volatile(
        "cp.async.bulk.tensor.2d.shared::cluster.global.tile.mbarrier::complete_tx::bytes "
        "[%0], [%1, {%2, %3}], [%4];"
        :: "r"(smem_u32(dst)), "l"(map), "r"(c0), "r"(c1), "r"(smem_u32(bar)) : "memory");
}

// ------------------------------------------------------------------ kernel --

template <typename T, int KF>
__global__ void __launch_bounds__(kFusedMaxThreads, 1)
    dcn_band_fused_kernel(const __grid_constant__ BandFusedArgs f) {
    constexpr int LPI = kBandLanesPerItem;
    constexpr int RUN = 32 / LPI;          // items per warp run
    const BandArgs& a = f.b;
    const int NS = a.stages;               // steps in flight: A tiles, accumulators, om buffers
    extern __shared__ __align__(128) unsigned char fused_smem[];
    // 1024-byte aligned base for the swizzled tiles (the allocation has 1 KB of slack)
    const uint32_t raw = smem_u32(fused_smem);
    unsigned char* base = fused_smem + ((1024u - (raw & 1023u)) & 1023u);
    unsigned char* wtile = base;                                     // w_bytes
    unsigned char* atile = wtile + f.w_bytes;                        // NS x a_bytes
    unsigned char* ring = atile + NS * f.a_bytes;          // ring_bytes
    float* om = reinterpret_cast<float*>(ring + a.ring_bytes);       // NS x om_bytes
    uint64_t* bars = reinterpret_cast<uint64_t*>(reinterpret_cast<unsigned char*>(om) +
                                                 NS * f.om_bytes);
    uint64_t* full = bars;                          // ring rows + A tile of a step
    uint64_t* empty = full + NS;           // samplers done with a step
    uint64_t* mma_done = empty + NS;       // accumulator stage written
    uint64_t* tmem_free = mma_done + NS;  // accumulator stage read
    uint64_t* om_full = tmem_free + NS;   // om buffer written
    uint64_t* om_free = om_full + NS;     // om buffer read
    uint64_t* w_full = om_free + NS;      // weight tile landed
    int* descs = reinterpret_cast<int*>(w_full + 1);
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(descs + NS * kBandDescInts);
    float* bias_s = reinterpret_cast<float*>(tmem_slot + 4);       // NJ floats

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    const int nc = f.consumer_warps;
    const int w_prod = nc, w_mma = nc + 1, w_epi = nc + 2;

    if (threadIdx.x == 0) {
        for (int s = 0; s < NS; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&empty[s], (uint32_t)nc);
        }
        for (int s = 0; s < NS; ++s) {
            mbar_init(&mma_done[s], 1);
            mbar_init(&tmem_free[s], kFusedEpilogueWarps);
            mbar_init(&om_full[s], kFusedEpilogueWarps);
            mbar_init(&om_free[s], (uint32_t)nc);
        }
        mbar_init(w_full, 1);
        mbar_fence_init();
    }
    for (int j = threadIdx.x; j < f.NJ; j += blockDim.x)
        bias_s[j] = (f.b_om && j < f.J) ? Elem<T>::one(static_cast<const T*>(f.b_om) + j) : 0.f;
    if (warp == w_mma) {   // the whole warp allocates the accumulators
        asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;"
                     :: "r"(smem_u32(tmem_slot)), "r"(f.tmem_cols) : "memory");
        asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
    }
    tmem_fence_before();
    __syncthreads();
    tmem_fence_after();
    const uint32_t tmem_base = *tmem_slot;

    const int r_begin = (int)(((long long)a.rows_total * blockIdx.x) / gridDim.x);
    const int r_end = (int)(((long long)a.rows_total * (blockIdx.x + 1)) / gridDim.x);
    const int K = KF ? KF * KF : a.K;
    const int GK = a.G * K;

    if (warp == w_prod) {
        // ---------------------------------------------------------- producer
        if (lane == 0) {
            mbar_arrive_expect_tx(w_full, f.w_bytes);
            for (int kc = 0; kc < f.kchunks; ++kc)
                tma_load_2d(wtile + kc * (f.w_bytes / f.kchunks), &f.tmap_w, kc * 64, 0, w_full);
            const char* xg = static_cast<const char*>(a.x);
            const int RB = a.ring_rows;
            int prev_n = -1, prev_ylo = 0, prev_yhi = -1, prev_vlo = 0, next_v = 0;
            int done = -1, step = 0;
            bool ok = true;
            for (int cur = r_begin; cur < r_end && ok; ++step) {
                const BandStep st = band_step(a, cur, r_end);
                const int y_lo = max(0, st.o - a.pad - a.margin);
                const int y_hi = min(a.H - 1, st.o + st.nrows - 1 - a.pad + (a.kh - 1) * a.dil +
                                                  a.margin);
                int v_lo, first_new;
                if (st.n == prev_n && y_lo >= prev_ylo && y_lo <= prev_yhi + 1) {
                    v_lo = prev_vlo + (y_lo - prev_ylo);
                    first_new = max(y_lo, prev_yhi + 1);
                } else {
                    v_lo = next_v;
                    first_new = y_lo;
                }
                const int v_hi = v_lo + (y_hi - y_lo);
                const int v_first_new = v_lo + (first_new - y_lo);
                while (done < step - 1) {
                    const int t = done + 1;
                    const BandDesc* dt = reinterpret_cast<const BandDesc*>(
                        descs + (t % NS) * kBandDescInts);
                    const bool must = t <= step - NS ||
                                      (first_new <= y_hi && dt->v_lo <= v_hi - RB);
                    if (!must) break;
                    if (!mbar_wait(&empty[t % NS], (uint32_t)((t / NS) & 1),
                                   a.flags)) {
                        ok = false;
                        break;
                    }
                    done = t;
                }
                if (!ok) break;
                const int sb = step % NS;
                BandDesc* d = reinterpret_cast<BandDesc*>(descs + sb * kBandDescInts);
                d->y_lo = y_lo;
                d->y_hi = y_hi;
                d->slot_lo = v_lo % RB;
                d->v_lo = v_lo;
                const int new_rows = y_hi >= first_new ? y_hi - first_new + 1 : 0;
                mbar_arrive_expect_tx(&full[sb], (uint32_t)new_rows * a.row_bytes + f.a_box_bytes);
                if (new_rows > 0) {
                    const char* src = xg + ((long long)st.n * a.H + first_new) * a.row_bytes;
                    int slot = v_first_new % RB;
                    int left = new_rows;
                    while (left > 0) {
                        const int cnt = min(left, RB - slot);
                        bulk_g2s(ring + (uint32_t)slot * a.row_bytes, src,
                                 (uint32_t)cnt * a.row_bytes, &full[sb]);
                        src += (long long)cnt * a.row_bytes;
                        left -= cnt;
                        slot = 0;
                    }
                }
                // the step's pixels: rows (n H + o) W ... of the 2-D view of x
                const int prow = (st.n * a.H + st.o) * a.W;
                unsigned char* adst = atile + (step % NS) * f.a_bytes;
                for (int kc = 0; kc < f.kchunks; ++kc)
                    tma_load_2d(adst + kc * (f.a_bytes / f.kchunks), &f.tmap_x, kc * 64, prow,
                                &full[sb]);
                prev_n = st.n;
                prev_ylo = y_lo;
                prev_yhi = y_hi;
                prev_vlo = v_lo;
                next_v = max(next_v, v_hi + 1);
                cur += st.nrows;
            }
            // leave the loop only once the last stages' copies have landed
            for (int t = max(0, step - NS); t < step; ++t)
                (void)mbar_wait(&full[t % NS], (uint32_t)((t / NS) & 1),
                                a.flags);
            (void)mbar_wait(w_full, 0, a.flags);
        }
    } else if (warp == w_mma) {
        // --------------------------------------------------------------- MMA
        if (lane == 0) {
            bool ok = mbar_wait(w_full, 0, a.flags);
            const uint32_t idesc = umma_idesc_f16<T>(f.NJ);
            const uint32_t w_s = smem_u32(wtile);
            int step = 0;
            for (int cur = r_begin; cur < r_end && ok; ++step) {
                const BandStep st = band_step(a, cur, r_end);
                cur += st.nrows;
                const int sb = step % NS, fs = step % NS;
                if (!mbar_wait(&full[sb], (uint32_t)((step / NS) & 1), a.flags)) break;
                if (step >= NS &&
                    !mbar_wait(&tmem_free[fs], (uint32_t)(((step / NS) - 1) & 1),
                               a.flags))
                    break;
                tmem_fence_after();
                const uint32_t a_s = smem_u32(atile + fs * f.a_bytes);
                const uint32_t d_t = tmem_base + (uint32_t)(fs * f.NJ);
                for (int kc = 0; kc < f.kchunks; ++kc) {
                    const uint32_t a_k = a_s + kc * (f.a_bytes / f.kchunks);
                    const uint32_t b_k = w_s + kc * (f.w_bytes / f.kchunks);
#pragma unroll
                    for (int k16 = 0; k16 < 4; ++k16)
                        umma_f16(d_t, umma_desc_k128(a_k + 32 * k16),
                                 umma_desc_k128(b_k + 32 * k16), idesc,
                                 (kc | k16) != 0 ? 1u : 0u);
                }
                umma_commit(&mma_done[fs]);
            }
        }
        __syncwarp();
    } else if (warp >= w_epi) {
        // ---------------------------------------------------------- epilogue
        const int quarter = warp & 3;            // TMEM lanes 32 quarter .. + 31
        const int pix = quarter * 32 + lane;     // this thread's pixel of the step
        int step = 0;
        for (int cur = r_begin; cur < r_end; ++step) {
            const BandStep st = band_step(a, cur, r_end);
            cur += st.nrows;
            const int fs = step % NS;
            if (!mbar_wait(&mma_done[fs], (uint32_t)((step / NS) & 1), a.flags)) break;
            if (step >= NS &&
                !mbar_wait(&om_free[fs], (uint32_t)(((step / NS) - 1) & 1), a.flags))
                break;
            tmem_fence_after();
            float* dst = om + (size_t)fs * (f.om_bytes / 4) + (size_t)pix * f.om_stride;
            const bool valid = pix < st.nrows * a.W;
            const uint32_t t_row = tmem_base + ((uint32_t)(quarter * 32) << 16) +
                                   (uint32_t)(fs * f.NJ);
            for (int j0 = 0; j0 < f.NJ; j0 += 16) {
                uint32_t r[16];
                tmem_ld16(t_row + (uint32_t)j0, r);
                tmem_wait_ld();
                if (valid) {
#pragma unroll
                    for (int e = 0; e < 16; e += 4) {
                        const int j = j0 + e;
                        if (j < (int)f.om_stride) {   // columns up to NJ are zero-padded
                            float4 v;
                            v.x = __uint_as_float(r[e]) + bias_s[j];
                            v.y = __uint_as_float(r[e + 1]) + bias_s[j + 1];
                            v.z = __uint_as_float(r[e + 2]) + bias_s[j + 2];
                            v.w = __uint_as_float(r[e + 3]) + bias_s[j + 3];
                            *reinterpret_cast<float4*>(dst + j) = v;
                        }
                    }
                }
            }
            tmem_fence_before();
            __syncwarp();
            if (lane == 0) {
                mbar_arrive(&tmem_free[fs]);
                mbar_arrive(&om_full[fs]);
            }
        }
    } else {
        // ---------------------------------------------------------- samplers
        const uint32_t ring_s = smem_u32(ring);
        const int row_items = a.Wo * a.G;
        int step = 0, j0 = 0;
        for (int cur = r_begin; cur < r_end; ++step) {
            const BandStep st = band_step(a, cur, r_end);
            cur += st.nrows;
            const int sb = step % NS, fs = step % NS;
            if (!mbar_wait(&full[sb], (uint32_t)((step / NS) & 1), a.flags)) break;
            if (!mbar_wait(&om_full[fs], (uint32_t)((step / NS) & 1), a.flags)) break;
            const BandDesc dsc = *reinterpret_cast<const BandDesc*>(descs + sb * kBandDescInts);
            const uint32_t omb_s = smem_u32(om) + (uint32_t)fs * f.om_bytes;
            const int runs = st.nrows * a.runs_per_row;
            const int r_first = (warp - j0 % nc + nc) % nc;
            j0 += runs;
            for (int r = r_first; r < runs; r += nc) {
                const int row_local = (int)a.div_runs.div((uint32_t)r);
                const int run_in_row = r - row_local * a.runs_per_row;
                const bool active = run_in_row * RUN + lane / LPI < row_items;
                const int item = active ? run_in_row * RUN + lane / LPI : row_items - 1;
                const int ox = (int)a.div_G.div((uint32_t)item);
                const int g = item - ox * a.G;
                const uint32_t prow =
                    omb_s + (uint32_t)((row_local * a.W + ox) * f.om_stride) * 4u;
                band_item<T, float, false, KF, LPI>(a, dsc, ring_s, st.n, st.o + row_local,
                                                    item, active, prow + (uint32_t)(g * 2 * K) * 4u,
                                                    prow + (uint32_t)(2 * GK + g * K) * 4u, lane);
            }
            __syncwarp();
            if (lane == 0) {
                mbar_arrive(&empty[sb]);
                mbar_arrive(&om_free[fs]);
            }
        }
    }

    // every role has left its loop: free the accumulators
    tmem_fence_before();
    __syncthreads();
    if (warp == w_mma) {
        tmem_fence_after();
        asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;"
                     :: "r"(tmem_base), "r"(f.tmem_cols) : "memory");
    }
}

}  // namespace dcnb
