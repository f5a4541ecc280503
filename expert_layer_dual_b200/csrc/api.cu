// api.cu -- the C ABI of include/moe.h: argument validation, workspace
// carving, TMA descriptor creation and the stage sequence of moe_forward.
// Host code only; every stage of the layer runs in the kernels of
// routing.cu, router.cu, gemm_bf16.cu and gemm_fp8.cu.
#include <mutex>

#include "common.cuh"
#include "launch.h"

namespace moe {

// ------------------------------------------------------------------ device
const DevInfo& current_device_info() {
    static DevInfo infos[64];
    static bool ready[64] = {false};
    static std::mutex mu;
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) dev = 0;
    std::lock_guard<std::mutex> lock(mu);
    if (!ready[dev]) {
        DevInfo& d = infos[dev];
        d.device = dev;
        d.num_sms = 0;
        d.cc_major = d.cc_minor = 0;
        cudaDeviceGetAttribute(&d.num_sms, cudaDevAttrMultiProcessorCount, dev);
        cudaDeviceGetAttribute(&d.cc_major, cudaDevAttrComputeCapabilityMajor, dev);
        cudaDeviceGetAttribute(&d.cc_minor, cudaDevAttrComputeCapabilityMinor, dev);
        ready[dev] = true;
    }
    return infos[dev];
}

// ------------------------------------------------------------------ TMA maps
typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                  const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                  const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                  CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

static EncodeTiledFn encode_tiled() {
    static std::once_flag once;
    static EncodeTiledFn fn = nullptr;
    std::call_once(once, [] {
        void* p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) ==
                cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<EncodeTiledFn>(p);
    });
    return fn;
}

bool make_tmap_2d(CUtensorMap* map, const void* base, int elem_bytes, uint64_t rows,
                  uint64_t cols, uint32_t box_rows, uint32_t box_cols) {
    EncodeTiledFn fn = encode_tiled();
    if (fn == nullptr || base == nullptr || rows == 0 || cols == 0) return false;
    const CUtensorMapDataType dt =
        elem_bytes == 2 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16 : CU_TENSOR_MAP_DATA_TYPE_UINT8;
    const cuuint64_t dims[2] = {cols, rows};
    const cuuint64_t strides[1] = {cols * (cuuint64_t)elem_bytes};
    const cuuint32_t box[2] = {box_cols, box_rows};
    const cuuint32_t estr[2] = {1, 1};
    return fn(map, dt, 2, const_cast<void*>(base), dims, strides, box, estr,
              CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
              CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

}  // namespace moe

using namespace moe;

namespace {

inline size_t round_up(size_t v, size_t a) { return (v + a - 1) / a * a; }

struct WsLayout {
    size_t logits, part, ids, w, counts, offsets, perm, inv, seg, xq, xs, h, hs, o, xin, yout, total;
    int ksplit;
};

WsLayout ws_layout(const moe_shape& s) {
    WsLayout L{};
    size_t off = kWsHeader;
    auto take = [&](size_t bytes) {
        const size_t at = off;
        off += round_up(bytes, 256);
        return at;
    };
    const size_t T = (size_t)s.T, d = (size_t)s.d, E = (size_t)s.E, k = (size_t)s.k,
                 I = (size_t)s.I;
    const size_t R = T * k + (s.I_shared > 0 ? T : 0);
    L.logits = take(T * E * 4);
    L.ksplit = router_ksplit(s.T, s.d, s.E);
    L.part = L.ksplit > 1 ? take(2 * (size_t)L.ksplit * T * E * 4) : 0;  // split-K router partials
    L.ids = take(T * k * 4);
    L.w = take(T * k * 4);
    L.counts = take(E * 4);
    L.offsets = take((E + 1) * 4);
    L.perm = take(T * k * 4);
    L.inv = take(T * k * 4);
    L.seg = take((size_t)permute_segments((int64_t)(T * k)) * E * 4);
    if (s.wdtype == MOE_WDTYPE_FP8_BLOCK128) {
        L.xq = take(R * d);                               // quantised x in permuted row order
        L.xs = take(R * (d / 128) * 4);
        L.h = take(R * I);
        L.hs = take(R * (I / 128) * 4);
    } else if (s.wdtype == MOE_WDTYPE_FP8_TENSOR) {
        L.xq = take(R * d);                               // e4m3 x, permuted rows
        L.xs = L.hs = 0;                                  // static scales
        L.h = take(R * I);
    } else if (s.wdtype == MOE_WDTYPE_MXFP8) {
        L.xq = take(R * d);                               // e4m3 x, permuted rows
        L.xs = take(R * (d / 32));                        // E8M0 byte per 1x32 block
        L.h = take(R * I);
        L.hs = take(R * (I / 32));
    } else {
        L.xq = L.xs = L.hs = 0;
        L.h = take(R * I * 2);
    }
    L.o = take(R * d * 2);                                // FP16 rows of the down GEMM
    L.xin = take(T * d * 2);
    L.yout = take(T * d * 2);
    L.total = off;
    return L;
}

bool device_ok() {
    const DevInfo& d = current_device_info();
    return d.cc_major == 10 && d.num_sms > 0;
}

moe_status check_shape(const moe_shape* s) {
    if (s == nullptr) return MOE_ERR_INVALID_ARG;
    if (s->T < 0 || s->d <= 0 || s->E <= 0 || s->k <= 0 || s->I <= 0 || s->I_shared < 0)
        return MOE_ERR_INVALID_ARG;
    if (s->d % 128 != 0 || s->I % 128 != 0 || s->E > 256 || s->k > 8 || s->k > s->E)
        return MOE_ERR_UNSUPPORTED;
    if (s->I_shared != 0 && s->I_shared != s->I) return MOE_ERR_UNSUPPORTED;
    if (s->wdtype != MOE_WDTYPE_BF16 && s->wdtype != MOE_WDTYPE_FP8_BLOCK128 &&
        s->wdtype != MOE_WDTYPE_MXFP8 && s->wdtype != MOE_WDTYPE_FP8_TENSOR)
        return MOE_ERR_UNSUPPORTED;
    if ((int64_t)s->T * s->k + s->T >= (int64_t)1 << 31) return MOE_ERR_UNSUPPORTED;
    if ((int64_t)s->E * 2 * s->I >= (int64_t)1 << 31 || (int64_t)s->E * s->d >= (int64_t)1 << 31)
        return MOE_ERR_UNSUPPORTED;
    return MOE_OK;
}

moe_status check_weights(const moe_shape* s, const moe_weights* w, bool need_gateup,
                         bool need_down, bool need_router) {
    if (w == nullptr) return MOE_ERR_INVALID_ARG;
    const bool fp8 = s->wdtype != MOE_WDTYPE_BF16;  // scaled weights (FP8 or MXFP8)
    const bool sh = s->I_shared > 0;
    if (need_gateup && (w->w_gu == nullptr || (fp8 && w->w_gu_scale == nullptr) ||
                        (sh && (w->ws_gu == nullptr || (fp8 && w->ws_gu_scale == nullptr)))))
        return MOE_ERR_INVALID_ARG;
    if (need_down && (w->w_d == nullptr || (fp8 && w->w_d_scale == nullptr) ||
                      (sh && (w->ws_d == nullptr || (fp8 && w->ws_d_scale == nullptr)))))
        return MOE_ERR_INVALID_ARG;
    if (need_router && (w->router_hi == nullptr || w->router_lo == nullptr))
        return MOE_ERR_INVALID_ARG;
    if (s->wdtype == MOE_WDTYPE_FP8_TENSOR &&
        (!(w->act_scale_x > 0.0f) || !(w->act_scale_h > 0.0f) || !isfinite(w->act_scale_x) ||
         !isfinite(w->act_scale_h)))
        return MOE_ERR_INVALID_ARG;
    return MOE_OK;
}

inline moe_status cuda_status(cudaError_t e) { return e == cudaSuccess ? MOE_OK : MOE_ERR_CUDA; }

inline cudaStream_t as_stream(void* s) { return static_cast<cudaStream_t>(s); }

inline bool aligned256(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 255u) == 0; }

moe_status check_ws(void* ws, size_t have, size_t need) {
    if (ws == nullptr || !aligned256(ws)) return MOE_ERR_INVALID_ARG;
    if (have < need) return MOE_ERR_WORKSPACE_TOO_SMALL;
    return MOE_OK;
}

GroupedGemmArgs gemm_args(const moe_shape* s, const int32_t* offsets, const int32_t* perm,
                          int32_t* status) {
    GroupedGemmArgs a;
    a.T = s->T;
    a.d = s->d;
    a.E = s->E;
    a.k = s->k;
    a.I = s->I;
    a.has_shared = s->I_shared > 0 ? 1 : 0;
    a.offsets = offsets;
    a.perm = perm;
    a.status = status;
    a.tile_counter = status + kWsTileCounter;
    a.timeout_ns = kDefaultTimeoutNs;
    return a;
}

template <typename P>
inline P* at(void* ws, size_t off) {
    return reinterpret_cast<P*>(static_cast<uint8_t*>(ws) + off);
}

moe_status run_gateup(const moe_shape* s, const moe_weights* w, const void* x, const void* xs,
                      const int32_t* perm, const int32_t* offsets, void* h, void* hs,
                      int32_t* status, cudaStream_t st) {
    const GroupedGemmArgs a = gemm_args(s, offsets, perm, status);
    if (s->wdtype == MOE_WDTYPE_BF16)
        return cuda_status((use_wide_gateup(s->T, s->E, s->k) ? launch_gateup_bf16_wide
                                                              : launch_gateup_bf16)(
            a, static_cast<const uint16_t*>(x), static_cast<const uint16_t*>(w->w_gu),
            static_cast<const uint16_t*>(w->ws_gu), static_cast<uint16_t*>(h), st));
    if (s->wdtype == MOE_WDTYPE_FP8_TENSOR)
        return cuda_status(launch_gateup_f8t(
            a, static_cast<const uint8_t*>(x), w->act_scale_x, w->act_scale_h,
            static_cast<const uint8_t*>(w->w_gu), static_cast<const float*>(w->w_gu_scale),
            static_cast<const uint8_t*>(w->ws_gu), static_cast<const float*>(w->ws_gu_scale),
            static_cast<uint8_t*>(h), st));
    if (s->wdtype == MOE_WDTYPE_MXFP8)
        return cuda_status(launch_gateup_mx(
            a, static_cast<const uint8_t*>(x), static_cast<const uint8_t*>(xs),
            static_cast<const uint8_t*>(w->w_gu), static_cast<const uint8_t*>(w->w_gu_scale),
            static_cast<const uint8_t*>(w->ws_gu), static_cast<const uint8_t*>(w->ws_gu_scale),
            static_cast<uint8_t*>(h), static_cast<uint8_t*>(hs), st));
    return cuda_status(launch_gateup_fp8(
        a, static_cast<const uint8_t*>(x), static_cast<const float*>(xs),
        static_cast<const uint8_t*>(w->w_gu), static_cast<const float*>(w->w_gu_scale),
        static_cast<const uint8_t*>(w->ws_gu), static_cast<const float*>(w->ws_gu_scale),
        static_cast<uint8_t*>(h), static_cast<float*>(hs), st));
}

moe_status run_down(const moe_shape* s, const moe_weights* w, const void* h, const void* hs,
                    const int32_t* offsets, __half* o, int32_t* status, cudaStream_t st) {
    const GroupedGemmArgs a = gemm_args(s, offsets, nullptr, status);
    if (s->wdtype == MOE_WDTYPE_BF16)
        return cuda_status((use_pair_tiles(s->T, s->E, s->k) ? launch_down_bf16_2sm
                                                             : launch_down_bf16)(
            a, static_cast<const uint16_t*>(h), static_cast<const uint16_t*>(w->w_d),
            static_cast<const uint16_t*>(w->ws_d), o, st));
    if (s->wdtype == MOE_WDTYPE_FP8_TENSOR)
        return cuda_status(launch_down_f8t(
            a, static_cast<const uint8_t*>(h), w->act_scale_h, static_cast<const uint8_t*>(w->w_d),
            static_cast<const float*>(w->w_d_scale), static_cast<const uint8_t*>(w->ws_d),
            static_cast<const float*>(w->ws_d_scale), o, st));
    if (s->wdtype == MOE_WDTYPE_MXFP8)
        return cuda_status(launch_down_mx(
            a, static_cast<const uint8_t*>(h), static_cast<const uint8_t*>(hs),
            static_cast<const uint8_t*>(w->w_d), static_cast<const uint8_t*>(w->w_d_scale),
            static_cast<const uint8_t*>(w->ws_d), static_cast<const uint8_t*>(w->ws_d_scale), o, st));
    return cuda_status(launch_down_fp8(
        a, static_cast<const uint8_t*>(h), static_cast<const float*>(hs),
        static_cast<const uint8_t*>(w->w_d), static_cast<const float*>(w->w_d_scale),
        static_cast<const uint8_t*>(w->ws_d), static_cast<const float*>(w->ws_d_scale), o, st));
}

// Records events[i] (when given) at the stage boundaries: 0 start, 1 router
// logits, 2 top-k, 3 permute, 4 activation quantisation (FP8; else = 3),
// 5 gate-up, 6 down, 7 combine.
moe_status forward_device(const moe_shape* s, const moe_weights* w, const uint16_t* x, uint16_t* y,
                          void* ws, cudaStream_t st, void* const* events = nullptr) {
    auto mark = [&](int i) {
        return events == nullptr ||
               cudaEventRecord(static_cast<cudaEvent_t>(events[i]), st) == cudaSuccess;
    };
    const WsLayout L = ws_layout(*s);
    int32_t* status = at<int32_t>(ws, 0);
    float* logits = at<float>(ws, L.logits);
    int32_t* ids = at<int32_t>(ws, L.ids);
    float* rw = at<float>(ws, L.w);
    int32_t* counts = at<int32_t>(ws, L.counts);
    int32_t* offsets = at<int32_t>(ws, L.offsets);
    int32_t* perm = at<int32_t>(ws, L.perm);
    int32_t* inv = at<int32_t>(ws, L.inv);
    int32_t* seg = at<int32_t>(ws, L.seg);
    const bool fp8 = s->wdtype == MOE_WDTYPE_FP8_BLOCK128;
    const bool mx = s->wdtype == MOE_WDTYPE_MXFP8;
    const bool f8t = s->wdtype == MOE_WDTYPE_FP8_TENSOR;
    moe_status r;
    if (cudaMemsetAsync(status, 0, sizeof(int32_t), st) != cudaSuccess) return MOE_ERR_CUDA;
    if (!mark(0)) return MOE_ERR_CUDA;
    if (L.ksplit == 1) {
        if ((r = cuda_status(launch_router_logits(x, w->router_hi, w->router_lo, w->router_bias,
                                                  logits, s->T, s->d, s->E, status, st))) != MOE_OK)
            return r;
        if (!mark(1)) return MOE_ERR_CUDA;
        if ((r = cuda_status(launch_route_topk(logits, s->T, s->E, s->k, s->renormalize, ids, rw,
                                               st))) != MOE_OK)
            return r;
    } else {
        // few tokens: K split across CTAs, partials combined inside the top-k kernel
        float* ph = at<float>(ws, L.part);
        float* pl = ph + (size_t)L.ksplit * s->T * s->E;
        if ((r = cuda_status(launch_router_partials(x, w->router_hi, w->router_lo, ph, pl, L.ksplit,
                                                    s->T, s->d, s->E, status, st))) != MOE_OK)
            return r;
        if (!mark(1)) return MOE_ERR_CUDA;
        if ((r = cuda_status(launch_route_topk_partials(ph, pl, L.ksplit, w->router_bias, logits,
                                                        s->T, s->E, s->k, s->renormalize, ids, rw,
                                                        st))) != MOE_OK)
            return r;
    }
    if (!mark(2)) return MOE_ERR_CUDA;
    if ((r = cuda_status(launch_permute(ids, s->T, s->E, s->k, counts, offsets, perm, inv, seg,
                                        status, st))) != MOE_OK)
        return r;
    if (!mark(3)) return MOE_ERR_CUDA;
    const void* a_in = x;
    const void* a_scale = nullptr;
    if (f8t) {
        const int64_t R = (int64_t)s->T * s->k + (s->I_shared > 0 ? s->T : 0);
        if ((r = cuda_status(launch_quant_act_fp8_static(x, perm, s->T, s->k, R, s->d,
                                                         w->act_scale_x, at<uint8_t>(ws, L.xq),
                                                         st))) != MOE_OK)
            return r;
        a_in = at<uint8_t>(ws, L.xq);
    }
    if (mx) {
        if ((r = cuda_status(launch_quant_mx_permuted(x, perm, s->T, s->k, s->I_shared > 0 ? 1 : 0,
                                                      s->d, at<uint8_t>(ws, L.xq),
                                                      at<uint8_t>(ws, L.xs), st))) != MOE_OK)
            return r;
        a_in = at<uint8_t>(ws, L.xq);
        a_scale = at<uint8_t>(ws, L.xs);
    }
    if (fp8) {
        if ((r = cuda_status(launch_quant_act_fp8_permuted(x, perm, s->T, s->k, s->I_shared > 0 ? 1 : 0,
                                                           s->d, at<uint8_t>(ws, L.xq),
                                                           at<float>(ws, L.xs), st))) != MOE_OK)
            return r;
        a_in = at<uint8_t>(ws, L.xq);
        a_scale = at<float>(ws, L.xs);
    }
    if (!mark(4)) return MOE_ERR_CUDA;
    void* h = at<uint8_t>(ws, L.h);
    void* hs = (fp8 || mx) ? at<uint8_t>(ws, L.hs) : nullptr;
    __half* o = at<__half>(ws, L.o);
    if ((r = run_gateup(s, w, a_in, a_scale, perm, offsets, h, hs, status, st)) != MOE_OK) return r;
    if (!mark(5)) return MOE_ERR_CUDA;
    if ((r = run_down(s, w, h, hs, offsets, o, status, st)) != MOE_OK) return r;
    if (!mark(6)) return MOE_ERR_CUDA;
    if ((r = cuda_status(launch_combine(o, inv, rw, y, s->T, s->d, s->k, s->I_shared > 0 ? 1 : 0,
                                        st))) != MOE_OK)
        return r;
    return mark(7) ? MOE_OK : MOE_ERR_CUDA;
}

}  // namespace

extern "C" {

const char* moe_status_string(moe_status s) {
    switch (s) {
        case MOE_OK: return "ok";
        case MOE_ERR_INVALID_ARG: return "invalid argument";
        case MOE_ERR_UNSUPPORTED: return "unsupported shape, type or device";
        case MOE_ERR_CUDA: return "CUDA launch or runtime error";
        case MOE_ERR_WORKSPACE_TOO_SMALL: return "workspace too small";
        case MOE_ERR_DEVICE_TIMEOUT: return "a bounded device wait ran out";
        case MOE_ERR_DEVICE_BAD_INDEX: return "an expert id was out of range";
        default: return "unknown status";
    }
}

size_t moe_workspace_bytes(const moe_shape* shape) {
    if (check_shape(shape) != MOE_OK) return 0;
    return ws_layout(*shape).total;
}

size_t moe_permute_workspace_bytes(int32_t T, int32_t E, int32_t k) {
    if (T < 0 || E <= 0 || k <= 0) return 0;
    return kWsHeader + round_up((size_t)permute_segments((int64_t)T * k) * (size_t)E * 4, 256);
}

moe_status moe_router_split(const float* W, uint16_t* hi, uint16_t* lo, int64_t n, void* stream) {
    if (n < 0 || (n > 0 && (W == nullptr || hi == nullptr || lo == nullptr)))
        return MOE_ERR_INVALID_ARG;
    if (!device_ok()) return MOE_ERR_UNSUPPORTED;
    return cuda_status(launch_router_split(W, hi, lo, n, as_stream(stream)));
}

moe_status moe_quantize_weights_fp8(const uint16_t* W, int64_t batch, int32_t rows, int32_t cols,
                                    uint8_t* q, float* scale, void* stream) {
    if (batch < 0 || rows < 0 || cols < 0) return MOE_ERR_INVALID_ARG;
    if (rows % 128 != 0 || cols % 128 != 0) return MOE_ERR_UNSUPPORTED;
    if (batch * rows * (int64_t)cols == 0) return MOE_OK;
    if (W == nullptr || q == nullptr || scale == nullptr) return MOE_ERR_INVALID_ARG;
    if (!device_ok()) return MOE_ERR_UNSUPPORTED;
    if (batch * (rows / 128) * (int64_t)(cols / 128) >= ((int64_t)1 << 31)) return MOE_ERR_UNSUPPORTED;
    return cuda_status(launch_quant_weights_fp8(W, batch, rows, cols, q, scale, as_stream(stream)));
}

moe_status moe_quantize_act_fp8(const uint16_t* x, int64_t rows, int32_t cols, uint8_t* q,
                                float* scale, void* stream) {
    if (rows < 0 || cols < 0) return MOE_ERR_INVALID_ARG;
    if (cols % 128 != 0) return MOE_ERR_UNSUPPORTED;
    if (rows * (int64_t)cols == 0) return MOE_OK;
    if (x == nullptr || q == nullptr || scale == nullptr) return MOE_ERR_INVALID_ARG;
    if (!device_ok()) return MOE_ERR_UNSUPPORTED;
    return cuda_status(launch_quant_act_fp8(x, rows, cols, q, scale, as_stream(stream)));
}

moe_status moe_quantize_weights_fp8_tensor(const uint16_t* W, int64_t batch, int32_t rows,
                                           int32_t cols, uint8_t* q, float* scale, void* stream) {
    if (batch < 0 || rows < 0 || cols < 0) return MOE_ERR_INVALID_ARG;
    if (cols % 8 != 0) return MOE_ERR_UNSUPPORTED;
    if (batch * rows * (int64_t)cols == 0) return MOE_OK;
    if (W == nullptr || q == nullptr || scale == nullptr) return MOE_ERR_INVALID_ARG;
    if (batch >= 65536) return MOE_ERR_UNSUPPORTED;
    if (!device_ok()) return MOE_ERR_UNSUPPORTED;
    return cuda_status(launch_quant_weights_fp8_tensor(W, batch, rows, cols, q, scale, as_stream(stream)));
}

moe_status moe_quantize_act_fp8_static(const uint16_t* x, int64_t rows, int32_t cols, float scale,
                                       uint8_t* q, void* stream) {
    if (rows < 0 || cols <= 0 || !(scale > 0.0f) || !isfinite(scale)) return MOE_ERR_INVALID_ARG;
    if (cols % 8 != 0) return MOE_ERR_UNSUPPORTED;
    if (rows == 0) return MOE_OK;
    if (x == nullptr || q == nullptr) return MOE_ERR_INVALID_ARG;
    if (!device_ok()) return MOE_ERR_UNSUPPORTED;
    return cuda_status(launch_quant_act_fp8_static(x, nullptr, 0, 1, rows, cols, scale, q,
                                                   as_stream(stream)));
}

moe_status moe_quantize_act_fp8_static_permuted(const uint16_t* x, const int32_t* perm, int32_t T,
                                                int32_t k, int32_t with_shared, int32_t d,
                                                float scale, uint8_t* q, void* stream) {
    if (T < 0 || k <= 0 || d <= 0 || !(scale > 0.0f) || !isfinite(scale)) return MOE_ERR_INVALID_ARG;
    if (d % 8 != 0 || (int64_t)T * k + T >= ((int64_t)1 << 31)) return MOE_ERR_UNSUPPORTED;
    if (T == 0) return MOE_OK;
    if (x == nullptr || perm == nullptr || q == nullptr) return MOE_ERR_INVALID_ARG;
    if (!device_ok()) return MOE_ERR_UNSUPPORTED;
    const int64_t R = (int64_t)T * k + (with_shared ? T : 0);
    return cuda_status(launch_quant_act_fp8_static(x, perm, T, k, R, d, scale, q, as_stream(stream)));
}

moe_status moe_quantize_weights_mxfp8(const uint16_t* W, int64_t batch, int32_t rows, int32_t cols,
                                      uint8_t* q, uint8_t* scale, void* stream) {
    if (batch < 0 || rows < 0 || cols < 0) return MOE_ERR_INVALID_ARG;
    if (cols % 128 != 0 || rows % 128 != 0) return MOE_ERR_UNSUPPORTED;
    if (batch * rows * (int64_t)cols == 0) return MOE_OK;
    if (W == nullptr || q == nullptr || scale == nullptr) return MOE_ERR_INVALID_ARG;
    if (!device_ok()) return MOE_ERR_UNSUPPORTED;
    return cuda_status(launch_quant_mx_weights(W, batch, rows, cols, q, scale, as_stream(stream)));
}

moe_status moe_quantize_act_mxfp8(const uint16_t* x, int64_t rows, int32_t cols, uint8_t* q,
                                  uint8_t* scale, void* stream) {
    if (rows < 0 || cols <= 0) return MOE_ERR_INVALID_ARG;
    if (cols % 128 != 0) return MOE_ERR_UNSUPPORTED;
    if (rows == 0) return MOE_OK;
    if (x == nullptr || q == nullptr || scale == nullptr) return MOE_ERR_INVALID_ARG;
    if (!device_ok()) return MOE_ERR_UNSUPPORTED;
    return cuda_status(launch_quant_mx_rows(x, rows, cols, q, scale, as_stream(stream)));
}

moe_status moe_quantize_act_mxfp8_permuted(const uint16_t* x, const int32_t* perm, int32_t T,
                                           int32_t k, int32_t with_shared, int32_t d, uint8_t* q,
                                           uint8_t* scale, void* stream) {
    if (T < 0 || k <= 0 || d <= 0) return MOE_ERR_INVALID_ARG;
    if (d % 128 != 0 || (int64_t)T * k + T >= ((int64_t)1 << 31)) return MOE_ERR_UNSUPPORTED;
    if (T == 0) return MOE_OK;
    if (x == nullptr || perm == nullptr || q == nullptr || scale == nullptr) return MOE_ERR_INVALID_ARG;
    if (!device_ok()) return MOE_ERR_UNSUPPORTED;
    return cuda_status(launch_quant_mx_permuted(x, perm, T, k, with_shared ? 1 : 0, d, q, scale,
                                                as_stream(stream)));
}

moe_status moe_quantize_act_fp8_permuted(const uint16_t* x, const int32_t* perm, int32_t T,
                                         int32_t k, int32_t with_shared, int32_t d, uint8_t* q,
                                         float* scale, void* stream) {
    if (T < 0 || k <= 0 || d <= 0) return MOE_ERR_INVALID_ARG;
    if (d % 128 != 0 || (int64_t)T * k + T >= ((int64_t)1 << 31)) return MOE_ERR_UNSUPPORTED;
    if (T == 0) return MOE_OK;
    if (x == nullptr || perm == nullptr || q == nullptr || scale == nullptr) return MOE_ERR_INVALID_ARG;
    if (!device_ok()) return MOE_ERR_UNSUPPORTED;
    return cuda_status(launch_quant_act_fp8_permuted(x, perm, T, k, with_shared ? 1 : 0, d, q, scale,
                                                     as_stream(stream)));
}

moe_status moe_router_logits(const uint16_t* x, const uint16_t* hi, const uint16_t* lo,
                             const float* bias, float* logits, int32_t T, int32_t d, int32_t E,
                             void* stream) {
    if (T < 0 || d <= 0 || E <= 0) return MOE_ERR_INVALID_ARG;
    if (d % 128 != 0 || E > 256) return MOE_ERR_UNSUPPORTED;
    if (T == 0) return MOE_OK;
    if (x == nullptr || hi == nullptr || lo == nullptr || logits == nullptr) return MOE_ERR_INVALID_ARG;
    if (!device_ok()) return MOE_ERR_UNSUPPORTED;
    return cuda_status(launch_router_logits(x, hi, lo, bias, logits, T, d, E, nullptr,
                                            as_stream(stream)));
}

moe_status moe_route_topk(const float* logits, int32_t T, int32_t E, int32_t k, int32_t renormalize,
                          int32_t* ids, float* w, void* stream) {
    if (T < 0 || E <= 0 || k <= 0) return MOE_ERR_INVALID_ARG;
    if (E > 256 || k > 8 || k > E) return MOE_ERR_UNSUPPORTED;
    if (T == 0) return MOE_OK;
    if (logits == nullptr || ids == nullptr || w == nullptr) return MOE_ERR_INVALID_ARG;
    if (!device_ok()) return MOE_ERR_UNSUPPORTED;
    return cuda_status(launch_route_topk(logits, T, E, k, renormalize, ids, w, as_stream(stream)));
}

moe_status moe_permute(const int32_t* ids, int32_t T, int32_t E, int32_t k, int32_t* counts,
                       int32_t* offsets, int32_t* perm, int32_t* inv, void* ws, size_t ws_bytes,
                       void* stream) {
    if (T < 0 || E <= 0 || k <= 0) return MOE_ERR_INVALID_ARG;
    if (E > 256 || (int64_t)T * k >= ((int64_t)1 << 31)) return MOE_ERR_UNSUPPORTED;
    if (counts == nullptr || offsets == nullptr) return MOE_ERR_INVALID_ARG;
    if (T > 0 && (ids == nullptr || perm == nullptr || inv == nullptr)) return MOE_ERR_INVALID_ARG;
    moe_status r = check_ws(ws, ws_bytes, moe_permute_workspace_bytes(T, E, k));
    if (r != MOE_OK) return r;
    if (!device_ok()) return MOE_ERR_UNSUPPORTED;
    cudaStream_t st = as_stream(stream);
    int32_t* status = at<int32_t>(ws, 0);
    if (cudaMemsetAsync(status, 0, sizeof(int32_t), st) != cudaSuccess) return MOE_ERR_CUDA;
    return cuda_status(launch_permute(ids, T, E, k, counts, offsets, perm, inv,
                                      at<int32_t>(ws, kWsHeader), status, st));
}

moe_status moe_gemm_gateup(const moe_shape* shape, const moe_weights* weights, const void* x,
                           const void* x_scale, const int32_t* perm, const int32_t* offsets,
                           void* h, void* h_scale, void* ws, size_t ws_bytes, void* stream) {
    moe_status r = check_shape(shape);
    if (r != MOE_OK) return r;
    if ((r = check_weights(shape, weights, true, false, false)) != MOE_OK) return r;
    if (shape->T == 0) return MOE_OK;
    const bool fp8 = shape->wdtype != MOE_WDTYPE_BF16;  // permuted e4m3 rows
    const bool scaled = fp8 && shape->wdtype != MOE_WDTYPE_FP8_TENSOR;  // per-row scales
    if (x == nullptr || offsets == nullptr || h == nullptr || (!fp8 && perm == nullptr) ||
        (scaled && (x_scale == nullptr || h_scale == nullptr)))
        return MOE_ERR_INVALID_ARG;
    if ((r = check_ws(ws, ws_bytes, kWsHeader)) != MOE_OK) return r;
    if (!device_ok()) return MOE_ERR_UNSUPPORTED;
    cudaStream_t st = as_stream(stream);
    int32_t* status = at<int32_t>(ws, 0);
    if (cudaMemsetAsync(status, 0, sizeof(int32_t), st) != cudaSuccess) return MOE_ERR_CUDA;
    return run_gateup(shape, weights, x, x_scale, perm, offsets, h, h_scale, status, st);
}

moe_status moe_gemm_down(const moe_shape* shape, const moe_weights* weights, const void* h,
                         const void* h_scale, const int32_t* offsets, void* o, void* ws,
                         size_t ws_bytes, void* stream) {
    moe_status r = check_shape(shape);
    if (r != MOE_OK) return r;
    if ((r = check_weights(shape, weights, false, true, false)) != MOE_OK) return r;
    if (shape->T == 0) return MOE_OK;
    const bool scaled = shape->wdtype == MOE_WDTYPE_FP8_BLOCK128 || shape->wdtype == MOE_WDTYPE_MXFP8;
    if (h == nullptr || offsets == nullptr || o == nullptr || (scaled && h_scale == nullptr))
        return MOE_ERR_INVALID_ARG;
    if ((r = check_ws(ws, ws_bytes, kWsHeader)) != MOE_OK) return r;
    if (!device_ok()) return MOE_ERR_UNSUPPORTED;
    cudaStream_t st = as_stream(stream);
    int32_t* status = at<int32_t>(ws, 0);
    if (cudaMemsetAsync(status, 0, sizeof(int32_t), st) != cudaSuccess) return MOE_ERR_CUDA;
    return run_down(shape, weights, h, h_scale, offsets, static_cast<__half*>(o), status, st);
}

moe_status moe_combine(const moe_shape* shape, const void* o, const int32_t* inv,
                       const float* w, uint16_t* y, void* stream) {
    moe_status r = check_shape(shape);
    if (r != MOE_OK) return r;
    if (shape->T == 0) return MOE_OK;
    if (o == nullptr || inv == nullptr || w == nullptr || y == nullptr) return MOE_ERR_INVALID_ARG;
    if (!device_ok()) return MOE_ERR_UNSUPPORTED;
    return cuda_status(launch_combine(static_cast<const __half*>(o), inv, w, y, shape->T, shape->d,
                                      shape->k, shape->I_shared > 0 ? 1 : 0, as_stream(stream)));
}

moe_status moe_forward(const moe_shape* shape, const moe_weights* weights, const uint16_t* x,
                       uint16_t* y, void* ws, size_t ws_bytes, void* stream) {
    moe_status r = check_shape(shape);
    if (r != MOE_OK) return r;
    if ((r = check_weights(shape, weights, true, true, true)) != MOE_OK) return r;
    if (shape->T == 0) return MOE_OK;
    if (x == nullptr || y == nullptr) return MOE_ERR_INVALID_ARG;
    if ((r = check_ws(ws, ws_bytes, ws_layout(*shape).total)) != MOE_OK) return r;
    if (!device_ok()) return MOE_ERR_UNSUPPORTED;
    return forward_device(shape, weights, x, y, ws, as_stream(stream));
}

moe_status moe_forward_profiled(const moe_shape* shape, const moe_weights* weights,
                                const uint16_t* x, uint16_t* y, void* ws, size_t ws_bytes,
                                void* stream, void* const* events, int32_t n_events) {
    if (events == nullptr || n_events != MOE_PROFILE_EVENTS) return MOE_ERR_INVALID_ARG;
    for (int i = 0; i < n_events; ++i)
        if (events[i] == nullptr) return MOE_ERR_INVALID_ARG;
    moe_status r = check_shape(shape);
    if (r != MOE_OK) return r;
    if ((r = check_weights(shape, weights, true, true, true)) != MOE_OK) return r;
    if (shape->T == 0) return MOE_OK;
    if (x == nullptr || y == nullptr) return MOE_ERR_INVALID_ARG;
    if ((r = check_ws(ws, ws_bytes, ws_layout(*shape).total)) != MOE_OK) return r;
    if (!device_ok()) return MOE_ERR_UNSUPPORTED;
    return forward_device(shape, weights, x, y, ws, as_stream(stream), events);
}

moe_status moe_forward_host_async(const moe_shape* shape, const moe_weights* weights,
                                  const uint16_t* x_host, uint16_t* y_host, void* ws,
                                  size_t ws_bytes, void* stream) {
    moe_status r = check_shape(shape);
    if (r != MOE_OK) return r;
    if ((r = check_weights(shape, weights, true, true, true)) != MOE_OK) return r;
    if (shape->T == 0) return MOE_OK;
    if (x_host == nullptr || y_host == nullptr) return MOE_ERR_INVALID_ARG;
    const WsLayout L = ws_layout(*shape);
    if ((r = check_ws(ws, ws_bytes, L.total)) != MOE_OK) return r;
    if (!device_ok()) return MOE_ERR_UNSUPPORTED;
    cudaStream_t st = as_stream(stream);
    const size_t bytes = (size_t)shape->T * shape->d * 2;
    uint16_t* xin = at<uint16_t>(ws, L.xin);
    uint16_t* yout = at<uint16_t>(ws, L.yout);
    if (cudaMemcpyAsync(xin, x_host, bytes, cudaMemcpyHostToDevice, st) != cudaSuccess)
        return MOE_ERR_CUDA;
    if ((r = forward_device(shape, weights, xin, yout, ws, st)) != MOE_OK) return r;
    if (cudaMemcpyAsync(y_host, yout, bytes, cudaMemcpyDeviceToHost, st) != cudaSuccess)
        return MOE_ERR_CUDA;
    return MOE_OK;
}

moe_status moe_forward_host(const moe_shape* shape, const moe_weights* weights,
                            const uint16_t* x_host, uint16_t* y_host, void* ws, size_t ws_bytes,
                            void* stream) {
    moe_status r = check_shape(shape);
    if (r != MOE_OK) return r;
    if ((r = check_weights(shape, weights, true, true, true)) != MOE_OK) return r;
    if (shape->T == 0) return MOE_OK;
    if (x_host == nullptr || y_host == nullptr) return MOE_ERR_INVALID_ARG;
    const WsLayout L = ws_layout(*shape);
    if ((r = check_ws(ws, ws_bytes, L.total)) != MOE_OK) return r;
    if (!device_ok()) return MOE_ERR_UNSUPPORTED;
    cudaStream_t st = as_stream(stream);
    const size_t bytes = (size_t)shape->T * shape->d * 2;
    uint16_t* xin = at<uint16_t>(ws, L.xin);
    uint16_t* yout = at<uint16_t>(ws, L.yout);
    if (cudaMemcpyAsync(xin, x_host, bytes, cudaMemcpyHostToDevice, st) != cudaSuccess)
        return MOE_ERR_CUDA;
    if ((r = forward_device(shape, weights, xin, yout, ws, st)) != MOE_OK) return r;
    if (cudaMemcpyAsync(y_host, yout, bytes, cudaMemcpyDeviceToHost, st) != cudaSuccess)
        return MOE_ERR_CUDA;
    return cuda_status(cudaStreamSynchronize(st));
}

moe_status moe_read_device_status(const void* ws, void* stream) {
    if (ws == nullptr) return MOE_ERR_INVALID_ARG;
    cudaStream_t st = as_stream(stream);
    if (cudaStreamSynchronize(st) != cudaSuccess) return MOE_ERR_CUDA;
    int32_t v = 0;
    if (cudaMemcpy(&v, ws, sizeof(v), cudaMemcpyDeviceToHost) != cudaSuccess) return MOE_ERR_CUDA;
    return v;
}

moe_status moe_selftest_timeout(void* ws, int32_t limit_us, void* stream) {
    if (ws == nullptr || limit_us < 0) return MOE_ERR_INVALID_ARG;
    if (!device_ok()) return MOE_ERR_UNSUPPORTED;
    cudaStream_t st = as_stream(stream);
    int32_t* status = at<int32_t>(ws, 0);
    if (cudaMemsetAsync(status, 0, sizeof(int32_t), st) != cudaSuccess) return MOE_ERR_CUDA;
    return cuda_status(launch_selftest_timeout(status, (uint64_t)limit_us * 1000ull, st));
}

}  // extern "C"
