// gemm_f8t.cu -- grouped expert GEMMs with per-tensor FP8: e4m3 operands, one
// FP32 scale per weight matrix and static (calibrated) activation scales.
//
// "HPC-Ops - 騰訊混元開源的工業級高性能大模型推理算子庫", section HPC-Ops的主要功能,
// "GroupGEMM FP8" (per-tensor and block-wise FP8); "腾讯混元大模型：从多场景适配到
// 高效部署的全栈技术解析", section 量化压缩技术实践 / FP8量化方案 (static FP8
// quantisation of weights and activations with precomputed scales).
//
// With one scale per operand the product needs no promotion: the whole K
// accumulates in TMEM (kind::f8f6f4) and the epilogue applies s_a * s_w once.
// The kernels have the shape of the BF16 down GEMM: one CTA per SM on the
// dynamic tile schedule, 128 x 256 tiles, 128-byte k-blocks (128 e4m3 values:
// four MMAs of K = 32), a 4-stage TMA ring for both operands (the gate-up A
// rows are the static quantisation's output, already in permuted order), two
// 256-column TMEM accumulators so a tile's epilogue overlaps the next tile's
// MMAs, and 4 epilogue warps:
//  - gate-up: h = silu(s g) * (s u), s = s_x * s_w[e], quantised with the
//    static scale of h (e4m3 of fp32(h / s_h), saturating);
//  - down: o = s_h * s_w[e] * acc, stored as FP16 rows.
// Every wait is bounded, as in the other kernels.
#include "common.cuh"
#include "grouped_common.cuh"
#include "launch.h"

namespace moe {
namespace {

constexpr int BM = 128, BK = 128, BN = 256, STAGES = 4;
constexpr int A_BYTES = BM * BK;       // 16 KB
constexpr int B_HALF = 128 * BK;       // 16 KB
constexpr int B_BYTES = 2 * B_HALF;    // 32 KB
constexpr int STAGE_BYTES = A_BYTES + B_BYTES;
constexpr uint32_t TMEM_COLS = 512;    // two 256-column accumulators
constexpr int EPI_WARPS = 4, MMA_WARP = 4, TMA_WARP = 5;
constexpr int THREADS = 32 * (TMA_WARP + 1);  // 192

struct Bars {
    uint64_t full[STAGES];   // TMA arrival + transaction bytes
    uint64_t empty[STAGES];  // MMA commit
    uint64_t tfull[2];       // accumulator ready (MMA commit)
    uint64_t tempty[2];      // accumulator drained (one arrival per epilogue warp)
    TileRing ring;
    uint32_t tmem_slot;
    int abort_flag;
};

constexpr size_t SMEM_BYTES = 1024 + STAGES * STAGE_BYTES + sizeof(Bars) + sizeof(TileTable) + 64;

struct Smem {
    uint8_t* stages;
    Bars* bars;
    TileTable* tt;
};

__device__ __forceinline__ Smem carve(uint8_t* raw) {
    Smem s;
    s.stages = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(raw) + 1023) &
                                          ~static_cast<uintptr_t>(1023));
    s.bars = reinterpret_cast<Bars*>(s.stages + STAGES * STAGE_BYTES);
    s.tt = reinterpret_cast<TileTable*>(s.bars + 1);
    return s;
}

__device__ __forceinline__ void fail(Bars* b, int32_t* status) {
    report_status(status, MOE_ERR_DEVICE_TIMEOUT);
    *reinterpret_cast<volatile int*>(&b->abort_flag) = 1;
}

__device__ __forceinline__ void warp_arrive(uint64_t* bar) {
    __syncwarp();
    if ((threadIdx.x & 31) == 0) mbar_arrive(bar);
}

__device__ __forceinline__ uint32_t prologue(Smem& sm, const GroupedGemmArgs& a) {
    const int warp = threadIdx.x >> 5;
    Bars* b = sm.bars;
    if (threadIdx.x == 0) {
        for (int s = 0; s < STAGES; ++s) {
            mbar_init(&b->full[s], 1);
            mbar_init(&b->empty[s], 1);
        }
        for (int i = 0; i < 2; ++i) {
            mbar_init(&b->tfull[i], 1);
            mbar_init(&b->tempty[i], EPI_WARPS);
        }
        tile_ring_init(&b->ring, 1 + EPI_WARPS);  // the MMA thread and the epilogue warps
        b->abort_flag = 0;
        fence_barrier_init();
    }
    if (warp == MMA_WARP) tmem_alloc(&b->tmem_slot, TMEM_COLS);
    pdl_wait();  // offsets and the A operand come from the previous kernels
    if (warp == 0) build_tile_table(sm.tt, a.offsets, a.E, a.T, a.k, a.has_shared, BM);
    tc_fence_before_sync();
    __syncthreads();
    pdl_trigger();
    tc_fence_after_sync();
    return b->tmem_slot;
}

__device__ __forceinline__ void teardown(uint32_t tmem) {
    tc_fence_before_sync();
    __syncthreads();
    if ((threadIdx.x >> 5) == MMA_WARP) {
        tc_fence_after_sync();
        tmem_dealloc(tmem, TMEM_COLS);
    }
}

// B rows of a tile: half 0 at rb0, half 1 at rb1 (`two` false: past the matrix).
struct BRows {
    const CUtensorMap* map;
    int rb0, rb1;
    bool two;
};

template <typename RowsOf>
__device__ __forceinline__ void tma_role(Smem& sm, const GroupedGemmArgs& a, const CUtensorMap* tm_a,
                                         int G, int n_tiles, int nk, RowsOf rows_of) {
    Bars* b = sm.bars;
    const volatile int* ab = &b->abort_flag;
    const int total = sm.tt->mstart[G] * n_tiles;
    uint32_t it = 0, issued = 0;
    bool ok = true;
    for (uint32_t ti = 0; ok; ++ti) {
        const int tile = tile_ring_push(&b->ring, ti, a.tile_counter, total, a.timeout_ns, ab, ok);
        if (tile < 0) {
            if (!ok) fail(b, a.status);
            break;
        }
        const Tile t = decode_tile(sm.tt, G, n_tiles, tile, BM);
        const BRows L = rows_of(t);
        for (int kb = 0; kb < nk; ++kb, ++it) {
            const int s = it % STAGES;
            const uint32_t ph = (it / STAGES) & 1;
            if (!mbar_wait(&b->empty[s], ph ^ 1, a.timeout_ns, ab)) {
                fail(b, a.status);
                ok = false;
                break;
            }
            uint8_t* st = sm.stages + s * STAGE_BYTES;
            mbar_arrive_expect_tx(&b->full[s], A_BYTES + (L.two ? B_BYTES : B_HALF));
            tma_load_2d(st, tm_a, &b->full[s], kb * BK, t.row0);
            tma_load_2d(st + A_BYTES, L.map, &b->full[s], kb * BK, L.rb0);
            if (L.two) tma_load_2d(st + A_BYTES + B_HALF, L.map, &b->full[s], kb * BK, L.rb1);
            ++issued;
        }
    }
    if (*ab) {
        for (uint32_t i = (issued > STAGES ? issued - STAGES : 0); i < issued; ++i)
            mbar_wait(&b->full[i % STAGES], (i / STAGES) & 1, a.timeout_ns, nullptr);
    }
}

__device__ __forceinline__ void mma_role(Smem& sm, const GroupedGemmArgs& a, uint32_t tmem, int nk) {
    Bars* b = sm.bars;
    const volatile int* ab = &b->abort_flag;
    constexpr uint32_t idesc = idesc_e4m3(BM, BN);
    uint32_t it = 0;
    bool ok = true;
    for (uint32_t lt = 0; ok; ++lt) {
        if (tile_ring_pop(&b->ring, lt, a.timeout_ns, ab, ok) < 0) {
            if (!ok) fail(b, a.status);
            break;
        }
        const uint32_t buf = lt & 1, tph = (lt >> 1) & 1;
        if (!mbar_wait(&b->tempty[buf], tph ^ 1, a.timeout_ns, ab)) {
            fail(b, a.status);
            break;
        }
        tc_fence_after_sync();
        const uint32_t d_tmem = tmem + buf * BN;
        for (int kb = 0; kb < nk; ++kb, ++it) {
            const int s = it % STAGES;
            const uint32_t ph = (it / STAGES) & 1;
            if (!mbar_wait(&b->full[s], ph, a.timeout_ns, ab)) {
                fail(b, a.status);
                ok = false;
                break;
            }
            tc_fence_after_sync();
            const uint32_t sa = smem_u32(sm.stages + s * STAGE_BYTES);
            const uint32_t sb = sa + A_BYTES;
#pragma unroll
            for (int kk = 0; kk < BK / 32; ++kk)
                umma_e4m3(d_tmem, sdesc_k_sw128(sa + kk * 32), sdesc_k_sw128(sb + kk * 32), idesc,
                          (kb | kk) != 0);
            umma_commit(&b->empty[s]);
        }
        umma_commit(&b->tfull[buf]);  // also after an abort: arrives when issued MMAs finish
    }
}

__device__ __forceinline__ uint32_t q4_static(const float* v, float s) {
    const __nv_fp8x2_storage_t lo = __nv_cvt_float2_to_fp8x2(
        make_float2(__fdiv_rn(v[0], s), __fdiv_rn(v[1], s)), __NV_SATFINITE, __NV_E4M3);
    const __nv_fp8x2_storage_t hi = __nv_cvt_float2_to_fp8x2(
        make_float2(__fdiv_rn(v[2], s), __fdiv_rn(v[3], s)), __NV_SATFINITE, __NV_E4M3);
    return (uint32_t)lo | ((uint32_t)hi << 16);
}

// ---------------------------------------------------------------------------
// Gate-Up: h = silu(x Wg^T) * (x Wu^T) with per-tensor scales; e4m3 h with
// the static scale s_h.
// ---------------------------------------------------------------------------
__global__ void __launch_bounds__(THREADS, 1)
    k_gateup_f8t(const __grid_constant__ CUtensorMap tm_a, const __grid_constant__ CUtensorMap tm_w,
                 const __grid_constant__ CUtensorMap tm_ws, GroupedGemmArgs a, float sx, float sh,
                 const float* __restrict__ wsc, const float* __restrict__ wssc,
                 uint8_t* __restrict__ hq) {
    extern __shared__ uint8_t smem_raw[];
    Smem sm = carve(smem_raw);
    Bars* b = sm.bars;
    const volatile int* ab = &b->abort_flag;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const uint32_t tmem = prologue(sm, a);
    const int G = a.E + a.has_shared;
    const int n_tiles = a.I / 128;
    const int nk = a.d / BK;
    if (warp == TMA_WARP) {
        if (lane == 0) {
            tma_prefetch_desc(&tm_a);
            tma_prefetch_desc(&tm_w);
            tma_prefetch_desc(&tm_ws);
            tma_role(sm, a, &tm_a, G, n_tiles, nk, [&](const Tile& t) {
                const bool shared = t.g >= a.E;
                const int r0 = (shared ? 0 : t.g * 2 * a.I) + t.n * 128;
                return BRows{shared ? &tm_ws : &tm_w, r0, r0 + a.I, true};
            });
        }
    } else if (warp == MMA_WARP) {
        if (lane == 0) mma_role(sm, a, tmem, nk);
    } else {
        const int row = warp * 32 + lane;
        bool ok = true;
        for (uint32_t lt = 0;; ++lt) {
            const int tile = tile_ring_pop_warp(&b->ring, lt, a.timeout_ns, ab, ok);
            if (tile < 0) {
                if (!ok && lane == 0) fail(b, a.status);
                break;
            }
            const Tile t = decode_tile(sm.tt, G, n_tiles, tile, BM);
            const uint32_t buf = lt & 1, tph = (lt >> 1) & 1;
            if (!warp_wait(&b->tfull[buf], tph, a.timeout_ns, ab)) {
                if (lane == 0) fail(b, a.status);
                break;
            }
            tc_fence_after_sync();
            const float f = sx * (t.g >= a.E ? wssc[0] : wsc[t.g]);
            const uint32_t taddr = tmem + (static_cast<uint32_t>(warp * 32) << 16) + buf * BN;
            uint8_t* dst = hq + (int64_t)(t.row0 + row) * a.I + t.n * 128;
#pragma unroll 1
            for (int c = 0; c < 4; ++c) {
                float gv[32], uv[32];
                tmem_load32x2(taddr + c * 32, taddr + 128 + c * 32, gv, uv);
                if (row < t.nrows) {
#pragma unroll
                    for (int i = 0; i < 32; ++i) gv[i] = silu_f(gv[i] * f) * (uv[i] * f);
#pragma unroll
                    for (int q = 0; q < 2; ++q)
                        st_global_v4(dst + c * 32 + q * 16, q4_static(gv + 16 * q, sh),
                                     q4_static(gv + 16 * q + 4, sh), q4_static(gv + 16 * q + 8, sh),
                                     q4_static(gv + 16 * q + 12, sh));
                }
            }
            tc_fence_before_sync();
            warp_arrive(&b->tempty[buf]);
        }
    }
    teardown(tmem);
}

// ---------------------------------------------------------------------------
// Down: o = s_h * s_w[e] * (hq . Wq), stored as FP16 rows.
// ---------------------------------------------------------------------------
__global__ void __launch_bounds__(THREADS, 1)
    k_down_f8t(const __grid_constant__ CUtensorMap tm_a, const __grid_constant__ CUtensorMap tm_w,
               const __grid_constant__ CUtensorMap tm_ws, GroupedGemmArgs a, float sh,
               const float* __restrict__ wsc, const float* __restrict__ wssc, __half* __restrict__ o) {
    extern __shared__ uint8_t smem_raw[];
    Smem sm = carve(smem_raw);
    Bars* b = sm.bars;
    const volatile int* ab = &b->abort_flag;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const uint32_t tmem = prologue(sm, a);
    const int G = a.E + a.has_shared;
    const int n_tiles = (a.d + BN - 1) / BN;
    const int nk = a.I / BK;
    if (warp == TMA_WARP) {
        if (lane == 0) {
            tma_prefetch_desc(&tm_a);
            tma_prefetch_desc(&tm_w);
            tma_prefetch_desc(&tm_ws);
            tma_role(sm, a, &tm_a, G, n_tiles, nk, [&](const Tile& t) {
                const bool shared = t.g >= a.E;
                const int r0 = (shared ? 0 : t.g * a.d) + t.n * BN;
                return BRows{shared ? &tm_ws : &tm_w, r0, r0 + 128, t.n * BN + 128 < a.d};
            });
        }
    } else if (warp == MMA_WARP) {
        if (lane == 0) mma_role(sm, a, tmem, nk);
    } else {
        const int row = warp * 32 + lane;
        bool ok = true;
        for (uint32_t lt = 0;; ++lt) {
            const int tile = tile_ring_pop_warp(&b->ring, lt, a.timeout_ns, ab, ok);
            if (tile < 0) {
                if (!ok && lane == 0) fail(b, a.status);
                break;
            }
            const Tile t = decode_tile(sm.tt, G, n_tiles, tile, BM);
            const uint32_t buf = lt & 1, tph = (lt >> 1) & 1;
            if (!warp_wait(&b->tfull[buf], tph, a.timeout_ns, ab)) {
                if (lane == 0) fail(b, a.status);
                break;
            }
            tc_fence_after_sync();
            const float f = sh * (t.g >= a.E ? wssc[0] : wsc[t.g]);
            const uint32_t taddr = tmem + (static_cast<uint32_t>(warp * 32) << 16) + buf * BN;
            const int ncols = min(BN, a.d - t.n * BN);
            __half* dst = o + (int64_t)(t.row0 + row) * a.d + t.n * BN;
#pragma unroll 1
            for (int c = 0; c < BN / 32; ++c) {
                if (c * 32 >= ncols) break;  // uniform across the warp
                float v[32];
                tmem_load32(taddr + c * 32, v);
                if (row < t.nrows) st_f16x32(dst + c * 32, v, f);
            }
            tc_fence_before_sync();
            warp_arrive(&b->tempty[buf]);
        }
    }
    teardown(tmem);
}

template <typename K>
cudaError_t set_smem_once(K kernel, bool* flags) {
    const int dev = current_device_info().device;
    if (dev < 0 || dev >= 64) return cudaErrorInvalidDevice;
    if (flags[dev]) return cudaSuccess;
    cudaError_t e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         (int)SMEM_BYTES);
    if (e == cudaSuccess) flags[dev] = true;
    return e;
}

}  // namespace

cudaError_t launch_gateup_f8t(const GroupedGemmArgs& a, const uint8_t* xq, float sx, float sh,
                              const uint8_t* w_gu, const float* w_gu_s, const uint8_t* ws_gu,
                              const float* ws_gu_s, uint8_t* hq, cudaStream_t s) {
    if (a.T == 0) return cudaSuccess;
    const uint64_t R = (uint64_t)a.T * a.k + (a.has_shared ? a.T : 0);
    CUtensorMap ta, tw, tws;
    if (!make_tmap_2d(&ta, xq, 1, R, (uint64_t)a.d, BM, BK) ||
        !make_tmap_2d(&tw, w_gu, 1, (uint64_t)a.E * 2 * a.I, (uint64_t)a.d, 128, BK) ||
        !make_tmap_2d(&tws, a.has_shared ? ws_gu : w_gu, 1, (uint64_t)2 * a.I, (uint64_t)a.d, 128,
                      BK))
        return cudaErrorInvalidValue;
    static bool flags[64] = {false};
    cudaError_t e = set_smem_once(k_gateup_f8t, flags);
    if (e != cudaSuccess) return e;
    if (!a.counter_zeroed &&
        (e = cudaMemsetAsync(a.tile_counter, 0, sizeof(int32_t), s)) != cudaSuccess)
        return e;
    {
        const cudaError_t le = launch_pdl(k_gateup_f8t, dim3(current_device_info().num_sms),
                                          dim3(THREADS), SMEM_BYTES, s, ta, tw, tws, a, sx, sh,
                                          w_gu_s, a.has_shared ? ws_gu_s : w_gu_s, hq);
        if (le != cudaSuccess) return le;
    }
    return cudaGetLastError();
}

cudaError_t launch_down_f8t(const GroupedGemmArgs& a, const uint8_t* hq, float sh,
                            const uint8_t* w_d, const float* w_d_s, const uint8_t* ws_d,
                            const float* ws_d_s, __half* o, cudaStream_t s) {
    if (a.T == 0) return cudaSuccess;
    const uint64_t R = (uint64_t)a.T * a.k + (a.has_shared ? a.T : 0);
    CUtensorMap ta, tw, tws;
    if (!make_tmap_2d(&ta, hq, 1, R, (uint64_t)a.I, BM, BK) ||
        !make_tmap_2d(&tw, w_d, 1, (uint64_t)a.E * a.d, (uint64_t)a.I, 128, BK) ||
        !make_tmap_2d(&tws, a.has_shared ? ws_d : w_d, 1, (uint64_t)a.d, (uint64_t)a.I, 128, BK))
        return cudaErrorInvalidValue;
    static bool flags[64] = {false};
    cudaError_t e = set_smem_once(k_down_f8t, flags);
    if (e != cudaSuccess) return e;
    if (!a.counter_zeroed &&
        (e = cudaMemsetAsync(a.tile_counter, 0, sizeof(int32_t), s)) != cudaSuccess)
        return e;
    {
        const cudaError_t le = launch_pdl(k_down_f8t, dim3(current_device_info().num_sms),
                                          dim3(THREADS), SMEM_BYTES, s, ta, tw, tws, a, sh, w_d_s,
                                          a.has_shared ? ws_d_s : w_d_s, o);
        if (le != cudaSuccess) return le;
    }
    return cudaGetLastError();
}

}  // namespace moe
