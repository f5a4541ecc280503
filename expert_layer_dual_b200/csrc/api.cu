// api.cu -- the C ABI of include/moe.h: argument validation, workspace
// carving, TMA descriptor creation and the stage sequence of moe_forward.
// Host code only; every stage of the layer runs in the kernels of
// routing.cu, router.cu, gemm_bf16.cu and gemm_fp8.cu.
#include <cstring>
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
    size_t logits, part, rtk, ids, w, counts, offsets, perm, inv, seg, xq, xs, h, hs, o, xin, yout, total;
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
    L.rtk = L.ksplit == 1 && router_fuses_topk(s.E) ? take(router_topk_scratch_bytes(s.T, s.E))
                                                     : 0;  // fused top-k scratch
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
        // x's routed rows in permuted order (bf16) when the gate-up runs on CTA pairs
        L.xq = use_pair_gateup(s.T, s.E, s.k) ? take(T * k * d * 2) : 0;
        L.xs = L.hs = 0;
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

// Row buffers and weight matrices are read by TMA (whose base must be 16-byte
// aligned) or with 16-byte vector accesses.
inline bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

moe_status check_weights(const moe_shape* s, const moe_weights* w, bool need_gateup,
                         bool need_down, bool need_router) {
    if (w == nullptr) return MOE_ERR_INVALID_ARG;
    // the weight matrices are TMA sources
    if (!aligned16(w->w_gu) || !aligned16(w->w_d) || !aligned16(w->ws_gu) || !aligned16(w->ws_d) ||
        !aligned16(w->router_hi) || !aligned16(w->router_lo))
        return MOE_ERR_INVALID_ARG;
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

// Tile counters of the grouped GEMMs' dynamic schedules, in the workspace
// header after the status word: one per GEMM of a forward, so that the down
// GEMM, launched while the gate-up drains, never shares one with it.
constexpr int kGateupCounter = kWsTileCounter, kDownCounter = kWsTileCounter + 1;
constexpr size_t kHeaderZeroBytes = (kDownCounter + 1) * sizeof(int32_t);

GroupedGemmArgs gemm_args(const moe_shape* s, const int32_t* offsets, const int32_t* perm,
                          int32_t* status, int counter, bool counter_zeroed) {
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
    a.tile_counter = status + counter;
    a.timeout_ns = kDefaultTimeoutNs;
    a.counter_zeroed = counter_zeroed ? 1 : 0;
    return a;
}

template <typename P>
inline P* at(void* ws, size_t off) {
    return reinterpret_cast<P*>(static_cast<uint8_t*>(ws) + off);
}

// BF16 with `xp` (the forward's copy of x's routed rows in the permuted row
// order): the gate-up runs on CTA pairs; otherwise the kernels gather x
// through perm.
moe_status run_gateup(const moe_shape* s, const moe_weights* w, const void* x, const void* xs,
                      const int32_t* perm, const int32_t* offsets, void* h, void* hs,
                      int32_t* status, cudaStream_t st, bool counter_zeroed = false,
                      const uint16_t* xp = nullptr) {
    const GroupedGemmArgs a = gemm_args(s, offsets, perm, status, kGateupCounter, counter_zeroed);
    if (s->wdtype == MOE_WDTYPE_BF16 && xp != nullptr)
        return cuda_status(launch_gateup_bf16_2sm(
            a, xp, static_cast<const uint16_t*>(x), static_cast<const uint16_t*>(w->w_gu),
            static_cast<const uint16_t*>(w->ws_gu), static_cast<uint16_t*>(h), st));
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
                    const int32_t* offsets, __half* o, int32_t* status, cudaStream_t st,
                    bool counter_zeroed = false) {
    const GroupedGemmArgs a = gemm_args(s, offsets, nullptr, status, kDownCounter, counter_zeroed);
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

// Records events[i] (when given) on `st`; inside a stream capture the record
// becomes an event node of the graph (timed on every replay).
bool record_event(void* const* events, int i, cudaStream_t st) {
    if (events == nullptr) return true;
    cudaStreamCaptureStatus cap = cudaStreamCaptureStatusNone;
    if (cudaStreamIsCapturing(st, &cap) != cudaSuccess) return false;
    cudaEvent_t ev = static_cast<cudaEvent_t>(events[i]);
    const cudaError_t e = cap == cudaStreamCaptureStatusActive
                              ? cudaEventRecordWithFlags(ev, st, cudaEventRecordExternal)
                              : cudaEventRecord(ev, st);
    return e == cudaSuccess;
}

// The routing stages (router logits, top-k, permute) into the workspace
// regions of L; events 1..3 as in forward_device.
moe_status route_device(const moe_shape* s, const moe_weights* w, const uint16_t* x, void* ws,
                        const WsLayout& L, cudaStream_t st, void* const* events) {
    int32_t* status = at<int32_t>(ws, 0);
    float* logits = at<float>(ws, L.logits);
    int32_t* ids = at<int32_t>(ws, L.ids);
    float* rw = at<float>(ws, L.w);
    moe_status r;
    if (L.ksplit == 1 && router_fuses_topk(s->E)) {
        // router logits with the top-k fused into the same kernel
        if ((r = cuda_status(launch_router_topk(x, w->router_hi, w->router_lo, w->router_bias,
                                                logits, s->T, s->d, s->E, s->k, s->renormalize,
                                                ids, rw, at<uint8_t>(ws, L.rtk), status, st))) !=
            MOE_OK)
            return r;
        if (!record_event(events, 1, st)) return MOE_ERR_CUDA;
    } else if (L.ksplit == 1) {
        if ((r = cuda_status(launch_router_logits(x, w->router_hi, w->router_lo, w->router_bias,
                                                  logits, s->T, s->d, s->E, status, st))) != MOE_OK)
            return r;
        if (!record_event(events, 1, st)) return MOE_ERR_CUDA;
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
        if (!record_event(events, 1, st)) return MOE_ERR_CUDA;
        if ((r = cuda_status(launch_route_topk_partials(ph, pl, L.ksplit, w->router_bias, logits,
                                                        s->T, s->E, s->k, s->renormalize, ids, rw,
                                                        st))) != MOE_OK)
            return r;
    }
    if (!record_event(events, 2, st)) return MOE_ERR_CUDA;
    if ((r = cuda_status(launch_permute(ids, s->T, s->E, s->k, at<int32_t>(ws, L.counts),
                                        at<int32_t>(ws, L.offsets), at<int32_t>(ws, L.perm),
                                        at<int32_t>(ws, L.inv), at<int32_t>(ws, L.seg), status,
                                        st))) != MOE_OK)
        return r;
    return record_event(events, 3, st) ? MOE_OK : MOE_ERR_CUDA;
}

// Records events[i] (when given) at the stage boundaries: 0 start, 1 router
// logits, 2 top-k, 3 permute, 4 activation quantisation (FP8; else = 3),
// 5 gate-up, 6 down, 7 combine.
moe_status forward_device(const moe_shape* s, const moe_weights* w, const uint16_t* x, uint16_t* y,
                          void* ws, cudaStream_t st, void* const* events = nullptr) {
    auto mark = [&](int i) { return record_event(events, i, st); };
    const WsLayout L = ws_layout(*s);
    int32_t* status = at<int32_t>(ws, 0);
    float* rw = at<float>(ws, L.w);
    int32_t* offsets = at<int32_t>(ws, L.offsets);
    int32_t* perm = at<int32_t>(ws, L.perm);
    int32_t* inv = at<int32_t>(ws, L.inv);
    const bool fp8 = s->wdtype == MOE_WDTYPE_FP8_BLOCK128;
    const bool mx = s->wdtype == MOE_WDTYPE_MXFP8;
    const bool f8t = s->wdtype == MOE_WDTYPE_FP8_TENSOR;
    moe_status r;
    // the status word and both GEMM tile counters, zeroed before the first kernel so
    // that no memset separates the kernels of the chain (each may start early)
    if (cudaMemsetAsync(status, 0, kHeaderZeroBytes, st) != cudaSuccess) return MOE_ERR_CUDA;
    if (!mark(0)) return MOE_ERR_CUDA;
    if ((r = route_device(s, w, x, ws, L, st, events)) != MOE_OK) return r;
    const void* a_in = x;
    const void* a_scale = nullptr;
    const uint16_t* xp = nullptr;
    if (s->wdtype == MOE_WDTYPE_BF16 && use_pair_gateup(s->T, s->E, s->k)) {
        // the routed rows only: the pair gate-up reads the shared expert's rows from x
        if ((r = cuda_status(launch_permute_rows_bf16(x, inv, s->T, s->k, 0, s->d,
                                                      at<uint16_t>(ws, L.xq), st))) != MOE_OK)
            return r;
        xp = at<uint16_t>(ws, L.xq);
    }
    if (f8t) {
        if ((r = cuda_status(launch_quant_act_fp8_static_scatter(
                 x, inv, s->T, s->k, s->I_shared > 0 ? 1 : 0, s->d, w->act_scale_x,
                 at<uint8_t>(ws, L.xq), st))) != MOE_OK)
            return r;
        a_in = at<uint8_t>(ws, L.xq);
    }
    if (mx) {
        if ((r = cuda_status(launch_quant_mx_scatter(x, inv, s->T, s->k, s->I_shared > 0 ? 1 : 0,
                                                     s->d, at<uint8_t>(ws, L.xq),
                                                     at<uint8_t>(ws, L.xs), st))) != MOE_OK)
            return r;
        a_in = at<uint8_t>(ws, L.xq);
        a_scale = at<uint8_t>(ws, L.xs);
    }
    if (fp8) {
        if ((r = cuda_status(launch_quant_act_fp8_scatter(x, inv, s->T, s->k,
                                                          s->I_shared > 0 ? 1 : 0, s->d,
                                                          at<uint8_t>(ws, L.xq),
                                                          at<float>(ws, L.xs), st))) != MOE_OK)
            return r;
        a_in = at<uint8_t>(ws, L.xq);
        a_scale = at<float>(ws, L.xs);
    }
    if (!mark(4)) return MOE_ERR_CUDA;
    void* h = at<uint8_t>(ws, L.h);
    void* hs = (fp8 || mx) ? at<uint8_t>(ws, L.hs) : nullptr;
    __half* o = at<__half>(ws, L.o);
    if ((r = run_gateup(s, w, a_in, a_scale, perm, offsets, h, hs, status, st, true, xp)) != MOE_OK)
        return r;
    if (!mark(5)) return MOE_ERR_CUDA;
    if ((r = run_down(s, w, h, hs, offsets, o, status, st, true)) != MOE_OK) return r;
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
    if (W == nullptr || q == nullptr || scale == nullptr || !aligned16(W) || !aligned16(q))
        return MOE_ERR_INVALID_ARG;
    if (!device_ok()) return MOE_ERR_UNSUPPORTED;
    if (batch * (rows / 128) * (int64_t)(cols / 128) >= ((int64_t)1 << 31)) return MOE_ERR_UNSUPPORTED;
    return cuda_status(launch_quant_weights_fp8(W, batch, rows, cols, q, scale, as_stream(stream)));
}

moe_status moe_quantize_act_fp8(const uint16_t* x, int64_t rows, int32_t cols, uint8_t* q,
                                float* scale, void* stream) {
    if (rows < 0 || cols < 0) return MOE_ERR_INVALID_ARG;
    if (cols % 128 != 0) return MOE_ERR_UNSUPPORTED;
    if (rows * (int64_t)cols == 0) return MOE_OK;
    if (x == nullptr || q == nullptr || scale == nullptr || !aligned16(x) || !aligned16(q))
        return MOE_ERR_INVALID_ARG;
    if (!device_ok()) return MOE_ERR_UNSUPPORTED;
    return cuda_status(launch_quant_act_fp8(x, rows, cols, q, scale, as_stream(stream)));
}

moe_status moe_quantize_weights_fp8_tensor(const uint16_t* W, int64_t batch, int32_t rows,
                                           int32_t cols, uint8_t* q, float* scale, void* stream) {
    if (batch < 0 || rows < 0 || cols < 0) return MOE_ERR_INVALID_ARG;
    if (cols % 8 != 0) return MOE_ERR_UNSUPPORTED;
    if (batch * rows * (int64_t)cols == 0) return MOE_OK;
    if (W == nullptr || q == nullptr || scale == nullptr || !aligned16(W) || !aligned16(q))
        return MOE_ERR_INVALID_ARG;
    if (batch >= 65536) return MOE_ERR_UNSUPPORTED;
    if (!device_ok()) return MOE_ERR_UNSUPPORTED;
    return cuda_status(launch_quant_weights_fp8_tensor(W, batch, rows, cols, q, scale, as_stream(stream)));
}

moe_status moe_quantize_act_fp8_static(const uint16_t* x, int64_t rows, int32_t cols, float scale,
                                       uint8_t* q, void* stream) {
    if (rows < 0 || cols <= 0 || !(scale > 0.0f) || !isfinite(scale)) return MOE_ERR_INVALID_ARG;
    if (cols % 8 != 0) return MOE_ERR_UNSUPPORTED;
    if (rows == 0) return MOE_OK;
    if (x == nullptr || q == nullptr || !aligned16(x) || !aligned16(q)) return MOE_ERR_INVALID_ARG;
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
    if (x == nullptr || perm == nullptr || q == nullptr || !aligned16(x) || !aligned16(q))
        return MOE_ERR_INVALID_ARG;
    if (!device_ok()) return MOE_ERR_UNSUPPORTED;
    const int64_t R = (int64_t)T * k + (with_shared ? T : 0);
    return cuda_status(launch_quant_act_fp8_static(x, perm, T, k, R, d, scale, q, as_stream(stream)));
}

moe_status moe_quantize_weights_mxfp8(const uint16_t* W, int64_t batch, int32_t rows, int32_t cols,
                                      uint8_t* q, uint8_t* scale, void* stream) {
    if (batch < 0 || rows < 0 || cols < 0) return MOE_ERR_INVALID_ARG;
    if (cols % 128 != 0 || rows % 128 != 0) return MOE_ERR_UNSUPPORTED;
    if (batch * rows * (int64_t)cols == 0) return MOE_OK;
    if (W == nullptr || q == nullptr || scale == nullptr || !aligned16(W) || !aligned16(q))
        return MOE_ERR_INVALID_ARG;
    if (!device_ok()) return MOE_ERR_UNSUPPORTED;
    return cuda_status(launch_quant_mx_weights(W, batch, rows, cols, q, scale, as_stream(stream)));
}

moe_status moe_quantize_act_mxfp8(const uint16_t* x, int64_t rows, int32_t cols, uint8_t* q,
                                  uint8_t* scale, void* stream) {
    if (rows < 0 || cols <= 0) return MOE_ERR_INVALID_ARG;
    if (cols % 128 != 0) return MOE_ERR_UNSUPPORTED;
    if (rows == 0) return MOE_OK;
    if (x == nullptr || q == nullptr || scale == nullptr || !aligned16(x) || !aligned16(q))
        return MOE_ERR_INVALID_ARG;
    if (!device_ok()) return MOE_ERR_UNSUPPORTED;
    return cuda_status(launch_quant_mx_rows(x, rows, cols, q, scale, as_stream(stream)));
}

moe_status moe_quantize_act_mxfp8_permuted(const uint16_t* x, const int32_t* perm, int32_t T,
                                           int32_t k, int32_t with_shared, int32_t d, uint8_t* q,
                                           uint8_t* scale, void* stream) {
    if (T < 0 || k <= 0 || d <= 0) return MOE_ERR_INVALID_ARG;
    if (d % 128 != 0 || (int64_t)T * k + T >= ((int64_t)1 << 31)) return MOE_ERR_UNSUPPORTED;
    if (T == 0) return MOE_OK;
    if (x == nullptr || perm == nullptr || q == nullptr || scale == nullptr || !aligned16(x) ||
        !aligned16(q))
        return MOE_ERR_INVALID_ARG;
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
    if (x == nullptr || perm == nullptr || q == nullptr || scale == nullptr || !aligned16(x) ||
        !aligned16(q))
        return MOE_ERR_INVALID_ARG;
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
    if (x == nullptr || hi == nullptr || lo == nullptr || logits == nullptr || !aligned16(x) ||
        !aligned16(hi) || !aligned16(lo) || !aligned16(logits))
        return MOE_ERR_INVALID_ARG;
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
        (scaled && (x_scale == nullptr || h_scale == nullptr)) || !aligned16(x) || !aligned16(h))
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
    if (h == nullptr || offsets == nullptr || o == nullptr || (scaled && h_scale == nullptr) ||
        !aligned16(h) || !aligned16(o))
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
    if (o == nullptr || inv == nullptr || w == nullptr || y == nullptr || !aligned16(o) ||
        !aligned16(y))
        return MOE_ERR_INVALID_ARG;
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
    if (x == nullptr || y == nullptr || !aligned16(x) || !aligned16(y)) return MOE_ERR_INVALID_ARG;
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
    if (x == nullptr || y == nullptr || !aligned16(x) || !aligned16(y)) return MOE_ERR_INVALID_ARG;
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

moe_status moe_workspace_offsets(const moe_shape* shape, moe_workspace_map* map) {
    if (map == nullptr) return MOE_ERR_INVALID_ARG;
    const moe_status r = check_shape(shape);
    if (r != MOE_OK) return r;
    const WsLayout L = ws_layout(*shape);
    map->logits = L.logits;
    map->ids = L.ids;
    map->w = L.w;
    map->counts = L.counts;
    map->offsets = L.offsets;
    map->perm = L.perm;
    map->inv = L.inv;
    map->xq = L.xq;
    map->xs = L.xs;
    map->h = L.h;
    map->total = L.total;
    return MOE_OK;
}

moe_status moe_calibrate_fp8_static(const moe_shape* shape, const moe_weights* weights,
                                    const uint16_t* x, float* scales, void* ws, size_t ws_bytes,
                                    void* stream) {
    moe_status r = check_shape(shape);
    if (r != MOE_OK) return r;
    if (shape->wdtype != MOE_WDTYPE_BF16) return MOE_ERR_UNSUPPORTED;
    if ((r = check_weights(shape, weights, true, false, true)) != MOE_OK) return r;
    if (shape->T == 0 || x == nullptr || scales == nullptr || !aligned16(x))
        return MOE_ERR_INVALID_ARG;
    const WsLayout L = ws_layout(*shape);
    if ((r = check_ws(ws, ws_bytes, L.total)) != MOE_OK) return r;
    if (!device_ok()) return MOE_ERR_UNSUPPORTED;
    cudaStream_t st = as_stream(stream);
    int32_t* status = at<int32_t>(ws, 0);
    if (cudaMemsetAsync(status, 0, kHeaderZeroBytes, st) != cudaSuccess) return MOE_ERR_CUDA;
    if ((r = route_device(shape, weights, x, ws, L, st, nullptr)) != MOE_OK) return r;
    uint16_t* h = at<uint16_t>(ws, L.h);
    if ((r = run_gateup(shape, weights, x, nullptr, at<int32_t>(ws, L.perm),
                        at<int32_t>(ws, L.offsets), h, nullptr, status, st, true)) != MOE_OK)
        return r;
    const int64_t R = (int64_t)shape->T * shape->k + (shape->I_shared > 0 ? shape->T : 0);
    if ((r = cuda_status(launch_amax_scale(x, (int64_t)shape->T * shape->d, scales, st))) != MOE_OK)
        return r;
    return cuda_status(launch_amax_scale(h, R * shape->I, scales + 1, st));
}

moe_status moe_route(const moe_shape* shape, const moe_weights* weights, const uint16_t* x,
                     void* ws, size_t ws_bytes, void* stream) {
    moe_status r = check_shape(shape);
    if (r != MOE_OK) return r;
    if (shape->wdtype != MOE_WDTYPE_BF16 && shape->wdtype != MOE_WDTYPE_FP8_BLOCK128 &&
        shape->wdtype != MOE_WDTYPE_MXFP8 && shape->wdtype != MOE_WDTYPE_FP8_TENSOR)
        return MOE_ERR_UNSUPPORTED;
    if ((r = check_weights(shape, weights, false, false, true)) != MOE_OK) return r;
    if (shape->T == 0) return MOE_OK;
    if (x == nullptr || !aligned16(x)) return MOE_ERR_INVALID_ARG;
    const WsLayout L = ws_layout(*shape);
    if ((r = check_ws(ws, ws_bytes, L.total)) != MOE_OK) return r;
    if (!device_ok()) return MOE_ERR_UNSUPPORTED;
    cudaStream_t st = as_stream(stream);
    if (cudaMemsetAsync(ws, 0, kHeaderZeroBytes, st) != cudaSuccess) return MOE_ERR_CUDA;
    return route_device(shape, weights, x, ws, L, st, nullptr);
}

moe_status moe_ep_dispatch(const uint16_t* x, const int32_t* ids, const int32_t* perm, int32_t T,
                           int32_t d, int32_t k, int32_t E_local, uint16_t* send_rows,
                           int32_t* send_ids, void* stream) {
    if (T < 0 || d <= 0 || k <= 0 || E_local <= 0) return MOE_ERR_INVALID_ARG;
    if (d % 8 != 0 || (int64_t)T * k >= ((int64_t)1 << 31)) return MOE_ERR_UNSUPPORTED;
    if (T == 0) return MOE_OK;
    if (x == nullptr || ids == nullptr || perm == nullptr || send_rows == nullptr ||
        send_ids == nullptr || (reinterpret_cast<uintptr_t>(x) & 15u) != 0 ||
        (reinterpret_cast<uintptr_t>(send_rows) & 15u) != 0)
        return MOE_ERR_INVALID_ARG;
    if (!device_ok()) return MOE_ERR_UNSUPPORTED;
    return cuda_status(launch_ep_dispatch(x, ids, perm, (int64_t)T * k, d, k, E_local, send_rows,
                                          send_ids, as_stream(stream)));
}

moe_status moe_gather_rows(const void* src, const int32_t* index, int64_t n, int32_t row_bytes,
                           void* dst, void* stream) {
    if (n < 0 || row_bytes <= 0) return MOE_ERR_INVALID_ARG;
    if (row_bytes % 16 != 0) return MOE_ERR_UNSUPPORTED;
    if (n == 0) return MOE_OK;
    if (src == nullptr || index == nullptr || dst == nullptr ||
        (reinterpret_cast<uintptr_t>(src) & 15u) != 0 || (reinterpret_cast<uintptr_t>(dst) & 15u) != 0)
        return MOE_ERR_INVALID_ARG;
    if (!device_ok()) return MOE_ERR_UNSUPPORTED;
    return cuda_status(launch_gather_rows(src, index, n, row_bytes, dst, as_stream(stream)));
}

size_t moe_lamport_buffer_bytes(int32_t G, int32_t T_max, int32_t d) {
    if (G < 1 || G > kArMaxRanks || T_max < 0 || d <= 0) return 0;
    return lamport_buffer_bytes(G, T_max, d);
}

moe_status moe_lamport_init(void* buf, size_t bytes, void* stream) {
    if (bytes == 0) return MOE_OK;
    if (buf == nullptr || (reinterpret_cast<uintptr_t>(buf) & 15u) != 0 || bytes % 16 != 0)
        return MOE_ERR_INVALID_ARG;
    if (!device_ok()) return MOE_ERR_UNSUPPORTED;
    return cuda_status(launch_lamport_init(buf, bytes, as_stream(stream)));
}

moe_status moe_peer_buffer_alloc(size_t bytes, void** ptr, void* ipc_handle) {
    if (ptr == nullptr || ipc_handle == nullptr || bytes == 0) return MOE_ERR_INVALID_ARG;
    if (!device_ok()) return MOE_ERR_UNSUPPORTED;
    *ptr = nullptr;
    if (cudaMalloc(ptr, bytes) != cudaSuccess) return MOE_ERR_CUDA;
    cudaIpcMemHandle_t h;
    if (cudaIpcGetMemHandle(&h, *ptr) != cudaSuccess) {
        cudaFree(*ptr);
        *ptr = nullptr;
        return MOE_ERR_CUDA;
    }
    memcpy(ipc_handle, &h, sizeof(h));
    return MOE_OK;
}

moe_status moe_peer_buffer_open(const void* ipc_handle, void** ptr) {
    if (ptr == nullptr || ipc_handle == nullptr) return MOE_ERR_INVALID_ARG;
    cudaIpcMemHandle_t h;
    memcpy(&h, ipc_handle, sizeof(h));
    *ptr = nullptr;
    return cuda_status(cudaIpcOpenMemHandle(ptr, h, cudaIpcMemLazyEnablePeerAccess));
}

moe_status moe_peer_buffer_close(void* ptr) {
    if (ptr == nullptr) return MOE_ERR_INVALID_ARG;
    return cuda_status(cudaIpcCloseMemHandle(ptr));
}

moe_status moe_peer_buffer_free(void* ptr) {
    if (ptr == nullptr) return MOE_ERR_INVALID_ARG;
    return cuda_status(cudaFree(ptr));
}

namespace {
moe_status check_ar(int32_t G, int32_t T_max, int32_t T, int32_t d, const void* gamma) {
    if (G < 1 || T < 0 || T_max < 0 || d <= 0) return MOE_ERR_INVALID_ARG;
    if (G > kArMaxRanks || d % 8 != 0 || d > allreduce_norm_max_d() || T > T_max)
        return MOE_ERR_UNSUPPORTED;
    if (T > 0 && (gamma == nullptr || !aligned16(gamma))) return MOE_ERR_INVALID_ARG;
    return MOE_OK;
}
}  // namespace

moe_status moe_allreduce_rmsnorm(void* const* bufs, int32_t G, int32_t rank, uint32_t call,
                                 int32_t T_max, const uint16_t* x, const uint16_t* residual,
                                 const uint16_t* gamma, float eps, int32_t T, int32_t d,
                                 uint16_t* out, uint16_t* residual_out, void* ws, size_t ws_bytes,
                                 void* stream) {
    moe_status r = check_ar(G, T_max, T, d, gamma);
    if (r != MOE_OK) return r;
    if (rank < 0 || rank >= G || bufs == nullptr || !(eps >= 0.0f)) return MOE_ERR_INVALID_ARG;
    if (T == 0) return MOE_OK;
    if ((r = check_ws(ws, ws_bytes, kWsHeader)) != MOE_OK) return r;
    for (int p = 0; p < G; ++p)
        if (bufs[p] == nullptr || !aligned16(bufs[p])) return MOE_ERR_INVALID_ARG;
    if (x == nullptr || out == nullptr || !aligned16(x) || !aligned16(out) ||
        (residual != nullptr && !aligned16(residual)) ||
        (residual_out != nullptr && !aligned16(residual_out)))
        return MOE_ERR_INVALID_ARG;
    if (!device_ok()) return MOE_ERR_UNSUPPORTED;
    ArNormArgs a{};
    for (int p = 0; p < G; ++p) a.bufs[p] = static_cast<uint16_t*>(bufs[p]);
    a.x[0] = x;
    a.residual[0] = residual;
    a.out[0] = out;
    a.res_out[0] = residual_out;
    a.gamma = gamma;
    a.G = G;
    a.T = T;
    a.T_max = T_max;
    a.d = d;
    a.rank0 = rank;
    a.call = call;
    a.eps = eps;
    a.status = at<int32_t>(ws, 0);
    a.timeout_ns = kDefaultTimeoutNs;
    return cuda_status(launch_allreduce_rmsnorm(a, 1, false, as_stream(stream)));
}

moe_status moe_allreduce_rmsnorm_emulated(void* const* bufs, int32_t G, int32_t ranks,
                                          uint32_t call, int32_t T_max, const uint16_t* const* x,
                                          const uint16_t* const* residual, const uint16_t* gamma,
                                          float eps, int32_t T, int32_t d, uint16_t* const* out,
                                          uint16_t* const* residual_out, int32_t timeout_us,
                                          void* ws, size_t ws_bytes, void* stream) {
    moe_status r = check_ar(G, T_max, T, d, gamma);
    if (r != MOE_OK) return r;
    if (ranks < 1 || ranks > G || bufs == nullptr || x == nullptr || out == nullptr ||
        timeout_us <= 0 || !(eps >= 0.0f))
        return MOE_ERR_INVALID_ARG;
    if ((r = check_ws(ws, ws_bytes, kWsHeader)) != MOE_OK) return r;
    for (int p = 0; p < G; ++p)
        if (bufs[p] == nullptr || !aligned16(bufs[p])) return MOE_ERR_INVALID_ARG;
    for (int p = 0; p < ranks; ++p)
        if (x[p] == nullptr || out[p] == nullptr || !aligned16(x[p]) || !aligned16(out[p]) ||
            (residual != nullptr && residual[p] != nullptr && !aligned16(residual[p])) ||
            (residual_out != nullptr && residual_out[p] != nullptr && !aligned16(residual_out[p])))
            return MOE_ERR_INVALID_ARG;
    if (!device_ok()) return MOE_ERR_UNSUPPORTED;
    cudaStream_t st = as_stream(stream);
    int32_t* status = at<int32_t>(ws, 0);
    if (cudaMemsetAsync(status, 0, sizeof(int32_t), st) != cudaSuccess) return MOE_ERR_CUDA;
    if (T == 0) return MOE_OK;
    ArNormArgs a{};
    for (int p = 0; p < G; ++p) a.bufs[p] = static_cast<uint16_t*>(bufs[p]);
    for (int p = 0; p < ranks; ++p) {
        a.x[p] = x[p];
        a.residual[p] = residual != nullptr ? residual[p] : nullptr;
        a.out[p] = out[p];
        a.res_out[p] = residual_out != nullptr ? residual_out[p] : nullptr;
    }
    a.gamma = gamma;
    a.G = G;
    a.T = T;
    a.T_max = T_max;
    a.d = d;
    a.rank0 = 0;
    a.call = call;
    a.eps = eps;
    a.status = status;
    a.timeout_ns = (uint64_t)timeout_us * 1000ull;
    return cuda_status(launch_allreduce_rmsnorm(a, ranks, true, st));
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
