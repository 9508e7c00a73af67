// Device helpers shared by the sampling-aggregation kernels (sm_100a).
//
// - 2..32-byte vector loads through the read-only path and matching stores
//   (32 bytes = one ld/st .v8.b32, one full L1/L2 sector per lane);
// - exact widening of f16 / bf16 / f32 words to float32;
// - packed float32x2 FMA (FFMA2) for the weighted sums;
// - division by a runtime constant with a precomputed multiplier;
// - cooperative copy of a contiguous global span into shared memory.
#pragma once

#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <stdint.h>

namespace dcnb {

// ------------------------------------------------------------ status word --

// Bits of the per-device status word (dcn_device_flags in the C interface).
constexpr unsigned int kFlagWaitTimeout = 1u;   // a bounded pipeline wait gave up
constexpr unsigned int kFlagOutOfBounds = 2u;   // debug library: an access outside its buffer
constexpr unsigned int kFlagBadLevels = 4u;     // debug library: an inconsistent MSDA level table

__device__ __forceinline__ void set_flag(unsigned int* word, unsigned int bit) {
    if (word) atomicOr(word, bit);
}

// In the debug library (DCN_DEBUG), `cond` states that an access lies inside
// its buffer; when it does not, the access is reported in the status word and
// the caller skips it.  In the release library the check compiles away.
#ifdef DCN_DEBUG
#define DCN_IN_BOUNDS(cond, word) \
    ((cond) ? true : (::dcnb::set_flag((word), ::dcnb::kFlagOutOfBounds), false))
#else
#define DCN_IN_BOUNDS(cond, word) (true || (cond))
#endif

// ---------------------------------------------------------------- vectors --

// Load VB bytes from global memory (read-only for the kernel's lifetime) into
// 32-bit words.  VB = 2 leaves the value in the low half of w[0].
template <int VB>
__device__ __forceinline__ void load_vec(const void* p, uint32_t* w);

template <>
__device__ __forceinline__ void load_vec<32>(const void* p, uint32_t* w) {
    asm("ld.global.nc.v8.b32 {%0,%1,%2,%3,%4,%5,%6,%7}, [%8];"
        : "=r"(w[0]), "=r"(w[1]), "=r"(w[2]), "=r"(w[3]), "=r"(w[4]), "=r"(w[5]),
          "=r"(w[6]), "=r"(w[7])
        : "l"(p));
}
template <>
__device__ __forceinline__ void load_vec<16>(const void* p, uint32_t* w) {
    asm("ld.global.nc.v4.b32 {%0,%1,%2,%3}, [%4];"
        : "=r"(w[0]), "=r"(w[1]), "=r"(w[2]), "=r"(w[3])
        : "l"(p));
}
template <>
__device__ __forceinline__ void load_vec<8>(const void* p, uint32_t* w) {
    asm("ld.global.nc.v2.b32 {%0,%1}, [%2];" : "=r"(w[0]), "=r"(w[1]) : "l"(p));
}
template <>
__device__ __forceinline__ void load_vec<4>(const void* p, uint32_t* w) {
    asm("ld.global.nc.b32 %0, [%1];" : "=r"(w[0]) : "l"(p));
}
template <>
__device__ __forceinline__ void load_vec<2>(const void* p, uint32_t* w) {
    unsigned short h;
    asm("ld.global.nc.b16 %0, [%1];" : "=h"(h) : "l"(p));
    w[0] = h;
}

// Store VB bytes (streaming: the output is not read again by the kernel).
template <int VB>
__device__ __forceinline__ void store_vec(void* p, const uint32_t* w);

template <>
__device__ __forceinline__ void store_vec<32>(void* p, const uint32_t* w) {
    asm volatile("st.global.cs.v8.b32 [%0], {%1,%2,%3,%4,%5,%6,%7,%8};"
                 :: "l"(p), "r"(w[0]), "r"(w[1]), "r"(w[2]), "r"(w[3]), "r"(w[4]),
                    "r"(w[5]), "r"(w[6]), "r"(w[7])
                 : "memory");
}
template <>
__device__ __forceinline__ void store_vec<16>(void* p, const uint32_t* w) {
    asm volatile("st.global.cs.v4.b32 [%0], {%1,%2,%3,%4};"
                 :: "l"(p), "r"(w[0]), "r"(w[1]), "r"(w[2]), "r"(w[3]) : "memory");
}
template <>
__device__ __forceinline__ void store_vec<8>(void* p, const uint32_t* w) {
    asm volatile("st.global.cs.v2.b32 [%0], {%1,%2};" :: "l"(p), "r"(w[0]), "r"(w[1])
                 : "memory");
}
template <>
__device__ __forceinline__ void store_vec<4>(void* p, const uint32_t* w) {
    asm volatile("st.global.cs.b32 [%0], %1;" :: "l"(p), "r"(w[0]) : "memory");
}
template <>
__device__ __forceinline__ void store_vec<2>(void* p, const uint32_t* w) {
    unsigned short h = (unsigned short)w[0];
    asm volatile("st.global.cs.b16 [%0], %1;" :: "l"(p), "h"(h) : "memory");
}

// ------------------------------------------------------ element widening --

// Element traits: exact widening of stored words to float32 and rounding of
// float32 results back to the storage type (round to nearest even; `from`
// rounds one value).
template <typename T>
struct Elem;

template <>
struct Elem<float> {
    static constexpr int kBytes = 4;
    // word i holds element i
    static __device__ __forceinline__ float lo(uint32_t w) { return __uint_as_float(w); }
    static __device__ __forceinline__ float one(const float* p) { return *p; }
    static __device__ __forceinline__ uint32_t pack2(float a, float) { return __float_as_uint(a); }
    static __device__ __forceinline__ uint32_t pack1(float a) { return __float_as_uint(a); }
    static __device__ __forceinline__ float from(float a) { return a; }
};

template <>
struct Elem<__half> {
    static constexpr int kBytes = 2;
    static __device__ __forceinline__ float lo(uint32_t w) {
        return __half2float(__ushort_as_half((unsigned short)(w & 0xffffu)));
    }
    static __device__ __forceinline__ float hi(uint32_t w) {
        return __half2float(__ushort_as_half((unsigned short)(w >> 16)));
    }
    static __device__ __forceinline__ float one(const __half* p) { return __half2float(*p); }
    static __device__ __forceinline__ uint32_t pack2(float a, float b) {
        __half2 h = __floats2half2_rn(a, b);   // a -> low half
        return *reinterpret_cast<uint32_t*>(&h);
    }
    static __device__ __forceinline__ uint32_t pack1(float a) {
        return (uint32_t)__half_as_ushort(__float2half_rn(a));
    }
    static __device__ __forceinline__ __half from(float a) { return __float2half_rn(a); }
};

template <>
struct Elem<__nv_bfloat16> {
    static constexpr int kBytes = 2;
    // bf16 is the upper half of a float32: widening is a shift or a mask
    static __device__ __forceinline__ float lo(uint32_t w) { return __uint_as_float(w << 16); }
    static __device__ __forceinline__ float hi(uint32_t w) {
        return __uint_as_float(w & 0xffff0000u);
    }
    static __device__ __forceinline__ float one(const __nv_bfloat16* p) {
        return __bfloat162float(*p);
    }
    static __device__ __forceinline__ uint32_t pack2(float a, float b) {
        __nv_bfloat162 h = __floats2bfloat162_rn(a, b);
        return *reinterpret_cast<uint32_t*>(&h);
    }
    static __device__ __forceinline__ uint32_t pack1(float a) {
        return (uint32_t)__bfloat16_as_ushort(__float2bfloat16_rn(a));
    }
    static __device__ __forceinline__ __nv_bfloat16 from(float a) {
        return __float2bfloat16_rn(a);
    }
};

// Widen the CPT elements held in w[] to float32.
template <typename T, int CPT>
__device__ __forceinline__ void widen(const uint32_t* w, float* f) {
    if constexpr (sizeof(T) == 4) {
#pragma unroll
        for (int i = 0; i < CPT; ++i) f[i] = Elem<T>::lo(w[i]);
    } else if constexpr (CPT == 1) {
        f[0] = Elem<T>::lo(w[0]);
    } else {
#pragma unroll
        for (int i = 0; i < CPT / 2; ++i) {
            f[2 * i] = Elem<T>::lo(w[i]);
            f[2 * i + 1] = Elem<T>::hi(w[i]);
        }
    }
}

// Round CPT float32 results to T and pack them into words.
template <typename T, int CPT>
__device__ __forceinline__ void narrow(const float* f, uint32_t* w) {
    if constexpr (sizeof(T) == 4) {
#pragma unroll
        for (int i = 0; i < CPT; ++i) w[i] = __float_as_uint(f[i]);
    } else if constexpr (CPT == 1) {
        w[0] = Elem<T>::pack1(f[0]);
    } else {
#pragma unroll
        for (int i = 0; i < CPT / 2; ++i) w[i] = Elem<T>::pack2(f[2 * i], f[2 * i + 1]);
    }
}

// acc[i] += wt * v[i] for i < CPT, two lanes per FFMA2 where possible.
template <int CPT>
__device__ __forceinline__ void axpy(float* acc, float wt, const float* v) {
#pragma unroll
    for (int i = 0; i + 1 < CPT; i += 2) {
        float2 r = __ffma2_rn(make_float2(wt, wt), make_float2(v[i], v[i + 1]),
                              make_float2(acc[i], acc[i + 1]));
        acc[i] = r.x;
        acc[i + 1] = r.y;
    }
    if constexpr (CPT % 2 == 1) acc[CPT - 1] = fmaf(wt, v[CPT - 1], acc[CPT - 1]);
}

// Two consecutive elements (an (x, y) pair) from shared memory, widened.
template <typename T>
__device__ __forceinline__ void load_pair(const T* p, float& x, float& y) {
    if constexpr (sizeof(T) == 4) {
        const float2 v = *reinterpret_cast<const float2*>(p);
        x = v.x;
        y = v.y;
    } else {
        const uint32_t w = *reinterpret_cast<const uint32_t*>(p);
        x = Elem<T>::lo(w);
        y = Elem<T>::hi(w);
    }
}

// ---------------------------------------------------------- fast division --

// n / d and n % d for 0 <= n < 2^31 with a runtime divisor 1 <= d < 2^31:
// q = (umulhi(n, mul) + n) >> shift with shift = ceil(log2 d) and
// mul = floor(2^32 (2^shift - d) / d) + 1 (computed on the host).
struct FastDiv {
    uint32_t d;
    uint32_t mul;
    uint32_t shift;
    __device__ __forceinline__ uint32_t div(uint32_t n) const {
        return (__umulhi(n, mul) + n) >> shift;
    }
};

// ------------------------------------------------------ shared staging ----

// Copy nbytes (a multiple of 2) from global src to shared dst with all threads
// of the block, using the widest access both addresses and the size allow.
// Streaming loads: the span is read once.
__device__ __forceinline__ void stage_span(void* dst, const void* src, int nbytes) {
    const uintptr_t a = (uintptr_t)src | (uintptr_t)dst | (uintptr_t)nbytes;
    if ((a & 15) == 0) {
        const uint4* s = reinterpret_cast<const uint4*>(src);
        uint4* d = reinterpret_cast<uint4*>(dst);
        for (int i = threadIdx.x; i < (nbytes >> 4); i += blockDim.x) {
            uint4 v;
            asm("ld.global.nc.L1::no_allocate.v4.u32 {%0,%1,%2,%3}, [%4];"
                : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w) : "l"(s + i));
            d[i] = v;
        }
    } else if ((a & 3) == 0) {
        const uint32_t* s = reinterpret_cast<const uint32_t*>(src);
        uint32_t* d = reinterpret_cast<uint32_t*>(dst);
        for (int i = threadIdx.x; i < (nbytes >> 2); i += blockDim.x) d[i] = __ldg(s + i);
    } else {
        const unsigned short* s = reinterpret_cast<const unsigned short*>(src);
        unsigned short* d = reinterpret_cast<unsigned short*>(dst);
        for (int i = threadIdx.x; i < (nbytes >> 1); i += blockDim.x) d[i] = __ldg(s + i);
    }
}

}  // namespace dcnb
