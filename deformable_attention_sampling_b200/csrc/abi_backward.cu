// C interface of libdcn_b200.so: dcn_backward, msda_backward, their workspace
// sizes, and dcn_backward_static_scratch (the backward with a library-owned
// accumulator).
#include <mutex>

#include "abi_common.cuh"
#include "dcn_bwd.cuh"
#include "msda_bwd.cuh"

using namespace dcnb_abi;

namespace {

template <typename T, int VB, bool PAIR = false>
const void* dcn_bwd_kernel_for(int softmax, int kh, int kw) {
    using namespace dcnb;
    if (kh == 3 && kw == 3)
        return softmax ? (const void*)dcn_bwd_kernel<T, VB, true, 3, PAIR>
                       : (const void*)dcn_bwd_kernel<T, VB, false, 3, PAIR>;
    return softmax ? (const void*)dcn_bwd_kernel<T, VB, true, 0, PAIR>
                   : (const void*)dcn_bwd_kernel<T, VB, false, 0, PAIR>;
}

template <typename T>
const void* dcn_bwd_kernel_vb(int vb, int kh, int kw, int softmax, int pair) {
    if (pair) {   // 8 channels per lane
        if (vb == 8 * (int)sizeof(T))
            return dcn_bwd_kernel_for<T, 8 * sizeof(T), true>(softmax, kh, kw);
        return nullptr;
    }
    switch (vb) {
        case 32: return dcn_bwd_kernel_for<T, 32>(softmax, kh, kw);
        case 16: return dcn_bwd_kernel_for<T, 16>(softmax, kh, kw);
        case 8: return dcn_bwd_kernel_for<T, 8>(softmax, kh, kw);
        case 4: return dcn_bwd_kernel_for<T, 4>(softmax, kh, kw);
        default: break;
    }
    if constexpr (sizeof(T) == 2) {
        if (vb == 2) return dcn_bwd_kernel_for<T, 2>(softmax, kh, kw);
    }
    return nullptr;
}

template <typename T>
const void* msda_bwd_kernel_vb(int vb, int pair) {
    using namespace dcnb;
    if (pair) {   // 8 channels per lane
        if (vb == 8 * (int)sizeof(T)) return (const void*)msda_bwd_kernel<T, 8 * sizeof(T), true>;
        return nullptr;
    }
    switch (vb) {
        case 32: return (const void*)msda_bwd_kernel<T, 32>;
        case 16: return (const void*)msda_bwd_kernel<T, 16>;
        case 8: return (const void*)msda_bwd_kernel<T, 8>;
        case 4: return (const void*)msda_bwd_kernel<T, 4>;
        default: break;
    }
    if constexpr (sizeof(T) == 2) {
        if (vb == 2) return (const void*)msda_bwd_kernel<T, 2>;
    }
    return nullptr;
}

// Widest float32 reduction (4, 2 or 1 floats) whose every address is aligned:
// the accumulator base, the pixel stride (floats) and the lane's channel
// chunk (cpt floats) must all be multiples of it.
int pick_red_vec(const void* acc, long long pix_floats, int cpt) {
    for (int rv = 4; rv > 1; rv >>= 1) {
        if ((uintptr_t)acc % (uintptr_t)(4 * rv) == 0 && pix_floats % rv == 0 && cpt % rv == 0)
            return rv;
    }
    return 1;
}

// Per-lane vector width of a backward kernel.  Where a group's (head's)
// channels split into an even number of 8-channel lanes and the accumulator's
// 32-byte sectors line up with them, 8 channels per lane (one float32 sector)
// so that lane pairs reduce whole sectors (*pair = 1); otherwise the forward's
// widest vector.
int pick_bwd_vector_bytes(int es, int D, uintptr_t bases, const void* acc,
                          long long pix_floats, int* pair) {
    *pair = 0;
    const int vb8 = 8 * es;
    if (D % 16 == 0 && bases % (uintptr_t)vb8 == 0 && (uintptr_t)acc % 32 == 0 &&
        pix_floats % 8 == 0) {
        *pair = 1;
        return vb8;
    }
    return pick_vector_bytes(es, D, bases);
}

// The accumulator set-up and wrap-up launches around a backward kernel.
int launch_zero(float* p, long long n, void* stream) {
    if (n <= 0) return DCN_OK;
    const long long blocks = (n / 4 + dcnb::kUtilThreads - 1) / dcnb::kUtilThreads + 1;
    return launch((const void*)dcnb::zero_f32_kernel, dcnb::ZeroArgs{p, n},
                  (int)std::min(blocks, 1LL << 20), dcnb::kUtilThreads, 0, stream);
}

template <typename T>
int launch_round(const float* src, void* dst, long long n, void* stream) {
    if (n <= 0) return DCN_OK;
    const int vec4 = ((uintptr_t)dst % (4 * sizeof(T))) == 0 ? 1 : 0;
    const long long blocks = (n / 4 + dcnb::kUtilThreads - 1) / dcnb::kUtilThreads + 1;
    return launch((const void*)dcnb::round_f32_kernel<T>,
                  dcnb::RoundArgs<T>{src, static_cast<T*>(dst), n, vec4},
                  (int)std::min(blocks, 1LL << 20), dcnb::kUtilThreads, 0, stream);
}

int launch_round_dtype(int dtype, const float* src, void* dst, long long n, void* stream) {
    switch (dtype) {
        case DCN_F16: return launch_round<__half>(src, dst, n, stream);
        case DCN_BF16: return launch_round<__nv_bfloat16>(src, dst, n, stream);
        default: return DCN_OK;   // float32 accumulates in place
    }
}


}  // namespace

extern "C" {

long long dcn_backward_workspace_size(int N, int H, int W, int C, int dtype) {
    const int es = elem_bytes(dtype);
    if (es == 0 || N < 0 || H <= 0 || W <= 0 || C <= 0) return DCN_ERR_INVALID_ARG;
    if (dtype == DCN_F32) return 0;
    return (long long)N * H * W * C * 4;
}

int dcn_backward(const void* x, const void* offset, const void* mask, const void* grad_out,
                 void* grad_x, void* grad_offset, void* grad_mask, void* workspace,
                 long long workspace_bytes, int N, int H, int W, int C, int G, int kh, int kw,
                 int stride, int pad, int dil, int softmax_flag, int dtype, void* stream) {
    const int es = elem_bytes(dtype);
    if (es == 0 || N < 0 || H <= 0 || W <= 0 || C <= 0 || G <= 0 || C % G != 0 || kh <= 0 ||
        kw <= 0 || stride <= 0 || pad < 0 || dil <= 0 || (softmax_flag != 0 && softmax_flag != 1))
        return DCN_ERR_INVALID_ARG;
    if (H > kMaxDim || W > kMaxDim || pad > kMaxDim || stride > kMaxDim || dil > kMaxDim ||
        kh > kMaxDim || kw > kMaxDim || (long long)kh * kw > kMaxTaps)
        return DCN_ERR_UNSUPPORTED;
    const int Ho = dcn_output_size(H, kh, stride, pad, dil);
    const int Wo = dcn_output_size(W, kw, stride, pad, dil);
    if (Ho <= 0 || Wo <= 0) return DCN_ERR_INVALID_ARG;
    const int D = C / G;
    const int K = kh * kw;
    const long long img_bytes = (long long)H * W * C * es;
    const long long out_img_bytes = (long long)Ho * Wo * C * es;
    const long long items = (long long)N * Ho * Wo * G;
    if (img_bytes > kInt31 || out_img_bytes > kInt31 || items > kInt31 ||
        (long long)N * Ho * Wo > kInt31)
        return DCN_ERR_UNSUPPORTED;
    if (N == 0) return DCN_OK;
    if (!x || !offset || !mask || !grad_out || !grad_x || !grad_offset || !grad_mask)
        return DCN_ERR_INVALID_ARG;
    if ((((uintptr_t)x | (uintptr_t)offset | (uintptr_t)mask | (uintptr_t)grad_out |
          (uintptr_t)grad_x | (uintptr_t)grad_offset | (uintptr_t)grad_mask) % es) != 0)
        return DCN_ERR_MISALIGNED;
    const long long need_ws = dcn_backward_workspace_size(N, H, W, C, dtype);
    if (need_ws > 0) {
        if (!workspace || workspace_bytes < need_ws) return DCN_ERR_INVALID_ARG;
        if ((uintptr_t)workspace % 16 != 0) return DCN_ERR_MISALIGNED;
    }
    const long long x_bytes = img_bytes * N;
    const long long go_bytes = out_img_bytes * N;
    const long long off_bytes = items * K * 2 * es;
    const long long m_bytes = items * K * es;
    {
        const void* in_p[4] = {x, offset, mask, grad_out};
        const long long in_b[4] = {x_bytes, off_bytes, m_bytes, go_bytes};
        const void* out_p[4] = {grad_x, grad_offset, grad_mask, workspace};
        const long long out_b[4] = {x_bytes, off_bytes, m_bytes, need_ws > 0 ? need_ws : 0};
        for (int i = 0; i < 4; ++i) {
            if (out_b[i] == 0) continue;
            for (int j = 0; j < 4; ++j)
                if (overlaps(out_p[i], out_b[i], in_p[j], in_b[j])) return DCN_ERR_INVALID_ARG;
            for (int j = 0; j < i; ++j)
                if (out_b[j] > 0 && overlaps(out_p[i], out_b[i], out_p[j], out_b[j]))
                    return DCN_ERR_INVALID_ARG;
        }
    }

    float* acc = dtype == DCN_F32 ? static_cast<float*>(grad_x) : static_cast<float*>(workspace);
    int pair = 0;
    const int vb = pick_bwd_vector_bytes(es, D, (uintptr_t)x | (uintptr_t)grad_out, acc, C,
                                         &pair);
    if (vb == 0) return DCN_ERR_MISALIGNED;
    const int cpt = vb / es;
    const int tpi = D / cpt;
    if (tpi > 32) return DCN_ERR_UNSUPPORTED;
    const int run_items = 32 / tpi;
    const int slice = dcnb::bwd_slice(run_items, K, es, softmax_flag != 0).total();
    if (slice > kMaxBwdSliceBytes) return DCN_ERR_UNSUPPORTED;
    int cap = kMaxBwdSmemBytes / slice;
    if (cap > dcnb::kDcnBwdMaxWarps) cap = dcnb::kDcnBwdMaxWarps;
    const int row_items = Wo * G;
    const int runs_per_row = (row_items + run_items - 1) / run_items;
    int sms = 148;
    {
        int device = 0;
        if (cudaGetDevice(&device) == cudaSuccess)
            (void)cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, device);
        (void)cudaGetLastError();
    }
    // 128 registers per thread: 16 warps per SM
    const TileShape ts = choose_tile(N, Ho, runs_per_row, kh * dil, sms, cap, 16);
    const int warps = ts.h * ts.w;
    const int tiles_x = (runs_per_row + ts.w - 1) / ts.w;
    const long long tiles_per_image = (long long)((Ho + ts.h - 1) / ts.h) * tiles_x;
    const long long num_tiles = tiles_per_image * N;
    if (num_tiles > kInt31) return DCN_ERR_UNSUPPORTED;

    dcnb::DcnBwdArgs b;
    dcnb::DcnArgs& a = b.f;
    a.x = x;
    a.offset = offset;
    a.mask = mask;
    a.out = nullptr;
    a.H = H;
    a.W = W;
    a.C = C;
    a.G = G;
    a.D = D;
    a.kh = kh;
    a.kw = kw;
    a.K = K;
    a.stride = stride;
    a.pad = pad;
    a.dil = dil;
    a.Ho = Ho;
    a.Wo = Wo;
    a.tpi = tpi;
    a.run_items = run_items;
    a.runs_per_row = runs_per_row;
    a.tile_h = ts.h;
    a.tile_w = ts.w;
    a.tiles_x = tiles_x;
    a.tiles_per_image = (int)tiles_per_image;
    a.num_tiles = (int)num_tiles;
    a.stage_elems = run_items * K;
    a.prefetch = (((uintptr_t)x | (uintptr_t)(C * es)) % 16) == 0 ? 1 : 0;
    a.div_G = make_div((uint32_t)G);
    a.div_tpi = make_div((uint32_t)tpi);
    a.div_tile_w = make_div((uint32_t)ts.w);
    a.div_tiles_x = make_div((uint32_t)tiles_x);
    a.div_tiles_per_image = make_div((uint32_t)tiles_per_image);
    a.pix_bytes = (uint32_t)(C * es);
    a.row_bytes = (uint32_t)((long long)W * C * es);
    a.img_bytes = img_bytes;
    a.w_om = nullptr;
    a.b_om = nullptr;
    a.J = 0;
    a.flags = device_flags_word();
    a.x_bytes = img_bytes * N;
    a.out_bytes = out_img_bytes * N;
    b.grad_out = grad_out;
    b.grad_offset = grad_offset;
    b.grad_mask = grad_mask;
    b.gx_acc = acc;
    b.red_vec = pick_red_vec(acc, C, cpt);

    const void* fn = nullptr;
    switch (dtype) {
        case DCN_F32: fn = dcn_bwd_kernel_vb<float>(vb, kh, kw, softmax_flag, pair); break;
        case DCN_F16: fn = dcn_bwd_kernel_vb<__half>(vb, kh, kw, softmax_flag, pair); break;
        case DCN_BF16:
            fn = dcn_bwd_kernel_vb<__nv_bfloat16>(vb, kh, kw, softmax_flag, pair);
            break;
        default: break;
    }
    if (!fn) return DCN_ERR_UNSUPPORTED;
    const long long acc_elems = (long long)N * H * W * C;
    int rc = launch_zero(acc, acc_elems, stream);
    if (rc != DCN_OK) return rc;
    rc = launch(fn, b, a.num_tiles, 32 * warps, slice * warps, stream);
    if (rc != DCN_OK) return rc;
    return launch_round_dtype(dtype, acc, grad_x, acc_elems, stream);
}

long long msda_backward_workspace_size(int N, int S, int M, int D, int dtype) {
    const int es = elem_bytes(dtype);
    if (es == 0 || N < 0 || S <= 0 || M <= 0 || D <= 0) return DCN_ERR_INVALID_ARG;
    if (dtype == DCN_F32) return 0;
    return (long long)N * S * M * D * 4;
}

int msda_backward(const void* value, const int64_t* spatial_shapes, const int64_t* level_start,
                  const void* sampling_loc, const void* attn_w, const void* grad_out,
                  void* grad_value, void* grad_loc, void* grad_attn, void* workspace,
                  long long workspace_bytes, int N, int S, int Lq, int M, int D, int L, int K,
                  int dtype, void* stream) {
    const int es = elem_bytes(dtype);
    if (es == 0 || N < 0 || S <= 0 || Lq < 0 || M <= 0 || D <= 0 || L <= 0 || K <= 0)
        return DCN_ERR_INVALID_ARG;
    if (L > dcnb::kMsdaMaxLevels || K > 64) return DCN_ERR_UNSUPPORTED;
    const long long items = (long long)N * Lq * M;
    if (items > kInt31 || (long long)M * D * es > kInt31) return DCN_ERR_UNSUPPORTED;
    if (N == 0) return DCN_OK;
    if (!value || !spatial_shapes || !level_start || !grad_value) return DCN_ERR_INVALID_ARG;
    if (items > 0 && (!sampling_loc || !attn_w || !grad_out || !grad_loc || !grad_attn))
        return DCN_ERR_INVALID_ARG;
    if ((((uintptr_t)value | (uintptr_t)sampling_loc | (uintptr_t)attn_w | (uintptr_t)grad_out |
          (uintptr_t)grad_value | (uintptr_t)grad_loc | (uintptr_t)grad_attn) % es) != 0 ||
        (((uintptr_t)spatial_shapes | (uintptr_t)level_start) % 8) != 0)
        return DCN_ERR_MISALIGNED;
    const long long need_ws = msda_backward_workspace_size(N, S, M, D, dtype);
    if (need_ws > 0) {
        if (!workspace || workspace_bytes < need_ws) return DCN_ERR_INVALID_ARG;
        if ((uintptr_t)workspace % 16 != 0) return DCN_ERR_MISALIGNED;
    }
    const int LK = L * K;
    const long long v_bytes = (long long)N * S * M * D * es;
    {
        const void* in_p[6] = {value, spatial_shapes, level_start, sampling_loc, attn_w, grad_out};
        const long long in_b[6] = {v_bytes, (long long)L * 16, (long long)L * 8,
                                   items * LK * 2 * es, items * LK * es, items * D * es};
        const void* out_p[4] = {grad_value, grad_loc, grad_attn, workspace};
        const long long out_b[4] = {v_bytes, items * LK * 2 * es, items * LK * es,
                                    need_ws > 0 ? need_ws : 0};
        for (int i = 0; i < 4; ++i) {
            if (out_b[i] == 0) continue;
            for (int j = 0; j < 6; ++j)
                if (in_b[j] > 0 && overlaps(out_p[i], out_b[i], in_p[j], in_b[j]))
                    return DCN_ERR_INVALID_ARG;
            for (int j = 0; j < i; ++j)
                if (out_b[j] > 0 && overlaps(out_p[i], out_b[i], out_p[j], out_b[j]))
                    return DCN_ERR_INVALID_ARG;
        }
    }

    float* acc =
        dtype == DCN_F32 ? static_cast<float*>(grad_value) : static_cast<float*>(workspace);
    int pair = 0;
    const int vb = pick_bwd_vector_bytes(es, D, (uintptr_t)value | (uintptr_t)grad_out, acc,
                                         (long long)M * D, &pair);
    if (vb == 0) return DCN_ERR_MISALIGNED;
    const int cpt = vb / es;
    const int tpi = D / cpt;
    if (tpi > 32) return DCN_ERR_UNSUPPORTED;
    const int run_items = 32 / tpi;
    const int loc_stride = staged_row_stride(run_items, LK * 2, 2, es);
    const int w_stride = staged_row_stride(run_items, LK, 1, es);
    const int slice = dcnb::msda_bwd_slice(run_items, loc_stride, w_stride, es).total();
    if (slice > kMaxBwdSliceBytes || slice * dcnb::kMsdaWarps > kMaxBwdSmemBytes)
        return DCN_ERR_UNSUPPORTED;

    const long long acc_elems = (long long)N * S * M * D;
    dcnb::MsdaBwdArgs b;
    dcnb::MsdaArgs& a = b.f;
    a.value = value;
    a.shapes = spatial_shapes;
    a.level_start = level_start;
    a.loc = sampling_loc;
    a.attn = attn_w;
    a.out = nullptr;
    a.Lq = Lq;
    a.M = M;
    a.D = D;
    a.L = L;
    a.K = K;
    a.tpi = tpi;
    a.run_items = run_items;
    a.total_items = (int)items;
    a.num_runs = (int)((items + run_items - 1) / run_items);
    a.stage_elems = run_items * LK;
    a.loc_stride = loc_stride;
    a.w_stride = w_stride;
    a.div_M = make_div((uint32_t)M);
    a.div_Lq = make_div((uint32_t)(Lq > 0 ? Lq : 1));
    a.div_tpi = make_div((uint32_t)tpi);
    a.ref = nullptr;
    a.vr = nullptr;
    a.flags = device_flags_word();
    b.grad_out = grad_out;
    b.grad_loc = grad_loc;
    b.grad_attn = grad_attn;
    b.gv_acc = acc;
    b.S = S;
    b.red_vec = pick_red_vec(acc, (long long)M * D, cpt);

    const void* fn = nullptr;
    switch (dtype) {
        case DCN_F32: fn = msda_bwd_kernel_vb<float>(vb, pair); break;
        case DCN_F16: fn = msda_bwd_kernel_vb<__half>(vb, pair); break;
        case DCN_BF16: fn = msda_bwd_kernel_vb<__nv_bfloat16>(vb, pair); break;
        default: break;
    }
    if (!fn) return DCN_ERR_UNSUPPORTED;
    int rc = launch_zero(acc, acc_elems, stream);
    if (rc != DCN_OK) return rc;
    if (items > 0) {
        const int num_ctas = (a.num_runs + dcnb::kMsdaWarps - 1) / dcnb::kMsdaWarps;
        rc = launch(fn, b, num_ctas, dcnb::kMsdaThreads, slice * dcnb::kMsdaWarps, stream);
        if (rc != DCN_OK) return rc;
    }
    return launch_round_dtype(dtype, acc, grad_value, acc_elems, stream);
}

}  // extern "C"

// ------------------------------------------- backward without caller scratch
//
// dcn_backward needs a float32 accumulator for grad_x of 16-bit data, and it
// takes it from the caller.  Some callers have no device memory to hand over
// at call time: a plain C host program that has no allocator of its own, or
// code that must not allocate once it has started (a fixed device-memory
// budget set at initialisation).  For them this file keeps one statically
// sized accumulator per device, placed in the module's global memory when the
// library's device code is loaded, and dcn_backward_static_scratch runs the
// unchanged dcn_backward path with it.  Nothing is allocated per call.

namespace {

constexpr long long kStaticScratchBytes = DCN_STATIC_SCRATCH_BYTES;   // 16 MiB
constexpr int kMaxScratchDevices = 64;

static __device__ __align__(256) float g_static_scratch[kStaticScratchBytes / 4];

std::mutex g_scratch_mutex;
void* g_scratch_ptr[kMaxScratchDevices] = {};

// Device address of the static accumulator on the current device, looked up
// (cudaGetSymbolAddress) the first time a device asks and cached after that.
int static_scratch(void** out) {
    int device = 0;
    cudaError_t err = cudaGetDevice(&device);
    if (err != cudaSuccess) {
        g_last_cuda_error = (int)err;
        (void)cudaGetLastError();
        return DCN_ERR_CUDA;
    }
    if (device < 0 || device >= kMaxScratchDevices) return DCN_ERR_UNSUPPORTED;
    std::lock_guard<std::mutex> lock(g_scratch_mutex);
    if (g_scratch_ptr[device] == nullptr) {
        void* p = nullptr;
        err = cudaGetSymbolAddress(&p, g_static_scratch);
        if (err != cudaSuccess || p == nullptr) {
            g_last_cuda_error = (int)(err != cudaSuccess ? err : cudaErrorInvalidSymbol);
            (void)cudaGetLastError();
            return DCN_ERR_CUDA;
        }
        g_scratch_ptr[device] = p;
    }
    *out = g_scratch_ptr[device];
    return DCN_OK;
}

}  // namespace

extern "C" {

int dcn_backward_static_scratch(const void* x, const void* offset, const void* mask,
                                const void* grad_out, void* grad_x, void* grad_offset,
                                void* grad_mask, int N, int H, int W, int C, int G, int kh,
                                int kw, int stride, int pad, int dil, int softmax_flag,
                                int dtype, void* stream) {
    const long long need = dcn_backward_workspace_size(N, H, W, C, dtype);
    if (need < 0) return DCN_ERR_INVALID_ARG;
    if (need > kStaticScratchBytes) return DCN_ERR_UNSUPPORTED;
    void* ws = nullptr;
    if (need > 0) {
        const int rc = static_scratch(&ws);
        if (rc != DCN_OK) return rc;
    }
    return dcn_backward(x, offset, mask, grad_out, grad_x, grad_offset, grad_mask, ws,
                        need > 0 ? kStaticScratchBytes : 0, N, H, W, C, G, kh, kw, stride, pad,
                        dil, softmax_flag, dtype, stream);
}

}  // extern "C"
