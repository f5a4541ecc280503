// gemm_bf16.cu -- grouped expert GEMMs of the MoE layer on sm_100a tensor
// cores, BF16 operands, FP32 accumulation in TMEM.
//
// "HPC-Ops - 騰訊混元開源的工業級高性能大模型推理算子庫", section HPC-Ops的主要功能,
// "FusedMoE" (Gate-Up GEMM, Down GEMM) and section HPC-Ops的技術原理,
// "FusedMoE 流水線重構": Gate-Up reads the original input through the routing
// index, with no separate gather pass.
//
// B200 design (the pages' Hopper kernel drops warp specialisation and relies
// on cross-CTA scheduling; on sm_100a the MMA is issued by one thread and
// runs asynchronously from its operand loads, so the kernel is warp
// specialised instead):
//  - persistent: one CTA per SM takes tiles from the dynamic schedule of
//    grouped_common.cuh (m-tiles that share a weight tile start together);
//  - tile 128 rows x 256 columns x 64-wide k-blocks, 4-stage shared-memory
//    ring, 128-byte swizzled K-major operands;
//  - gate-up: the 256 B columns are 128 gate rows and the matching 128 up
//    rows of W_gu, so one N=256 MMA yields both halves of h's 128 columns;
//    the A rows are gathered from x by the routing permutation with
//    cp.async (4 warps, 8 lanes per 128-byte row slice), the weights arrive
//    by TMA;
//  - down: A (contiguous permuted rows of h) and B by TMA;
//  - one thread issues tcgen05.mma into one of two 256-column TMEM
//    accumulators, so the epilogue of a tile overlaps the next tile's MMAs;
//  - 4 epilogue warps read TMEM (tcgen05.ld), apply SiLU*mul (gate-up) and
//    store rows (h in bf16, the MMA operand of the down GEMM; o in FP16);
// Every wait is bounded; a timeout sets the device status word and all roles
// stop, drain their copies in flight and free TMEM.
#include "common.cuh"
#include "grouped_common.cuh"
#include "launch.h"

namespace moe {
namespace {

constexpr int BM = 128, BK = 64, BN = 256, STAGES = 4;
constexpr int A_BYTES = BM * BK * 2;      // 16 KB
constexpr int B_HALF = 128 * BK * 2;      // 16 KB
constexpr int B_BYTES = 2 * B_HALF;       // 32 KB
constexpr int STAGE_BYTES = A_BYTES + B_BYTES;
constexpr uint32_t TMEM_COLS = 512;       // two 256-column accumulators
constexpr int EPI_WARPS = 4, MMA_WARP = 4, TMA_WARP = 5, GATHER_WARP0 = 6, GATHER_WARPS = 4;
constexpr int GATEUP_THREADS = 32 * (GATHER_WARP0 + GATHER_WARPS);  // 320
constexpr int DOWN_THREADS = 32 * (TMA_WARP + 1);                    // 192

struct Bars {
    uint64_t full_a[STAGES];  // gate-up: one arrival per gather warp; down: unused
    uint64_t full_b[STAGES];  // TMA arrival + transaction bytes
    uint64_t empty[STAGES];   // MMA commit
    uint64_t tfull[2];        // accumulator ready (MMA commit)
    uint64_t tempty[2];       // accumulator drained (one arrival per epilogue warp)
    TileRing ring;            // tile numbers from the producer to the other roles
    uint32_t tmem_slot;
    int abort_flag;
};

constexpr size_t SMEM_BYTES = 1024 + STAGES * STAGE_BYTES + sizeof(Bars) + sizeof(TileTable) + 64;

struct Smem {
    uint8_t* stages;
    Bars* bars;
    TileTable* tt;
};

__device__ __forceinline__ Smem carve_smem(uint8_t* raw) {
    Smem s;
    s.stages = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(raw) + 1023) &
                                          ~static_cast<uintptr_t>(1023));
    s.bars = reinterpret_cast<Bars*>(s.stages + STAGES * STAGE_BYTES);
    s.tt = reinterpret_cast<TileTable*>(s.bars + 1);
    return s;
}

// All lanes of the warp are done with their part: one lane arrives for it.
__device__ __forceinline__ void warp_arrive(uint64_t* bar) {
    __syncwarp();
    if ((threadIdx.x & 31) == 0) mbar_arrive(bar);
}

__device__ __forceinline__ void fail(Bars* b, int32_t* status) {
    report_status(status, MOE_ERR_DEVICE_TIMEOUT);
    *reinterpret_cast<volatile int*>(&b->abort_flag) = 1;
}

// Shared prologue: barriers, tile table, TMEM.  full_a_count = 0 means the
// A operand also arrives by TMA (full_a unused); `consumers` is the number of
// arrivals that release a tile-ring slot.
__device__ __forceinline__ uint32_t prologue(Smem& sm, const GroupedGemmArgs& a, int full_a_count,
                                             uint32_t consumers) {
    const int warp = threadIdx.x >> 5;
    Bars* b = sm.bars;
    if (threadIdx.x == 0) {
        for (int s = 0; s < STAGES; ++s) {
            mbar_init(&b->full_a[s], full_a_count > 0 ? full_a_count : 1);
            mbar_init(&b->full_b[s], 1);
            mbar_init(&b->empty[s], 1);
        }
        for (int i = 0; i < 2; ++i) {
            mbar_init(&b->tfull[i], 1);
            mbar_init(&b->tempty[i], EPI_WARPS);
        }
        tile_ring_init(&b->ring, consumers);
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

__device__ __forceinline__ void teardown(Smem& sm, uint32_t tmem) {
    tc_fence_before_sync();
    __syncthreads();
    if ((threadIdx.x >> 5) == MMA_WARP) {
        tc_fence_after_sync();
        tmem_dealloc(tmem, TMEM_COLS);
    }
}

// The MMA role: identical for both GEMMs.  `wait_a` says whether the A
// operand has its own barrier (gathered rows).
__device__ __forceinline__ void mma_role(Smem& sm, const GroupedGemmArgs& a, uint32_t tmem,
                                         int G, int n_tiles, bool wait_a) {
    Bars* b = sm.bars;
    const volatile int* ab = &b->abort_flag;
    constexpr uint32_t idesc = idesc_bf16(BM, BN);
    const int nk = (wait_a ? a.d : a.I) / BK;
    uint32_t it = 0, lt = 0;
    bool ok = true;
    for (;; ++lt) {
        if (tile_ring_pop(&b->ring, lt, a.timeout_ns, ab, ok) < 0) {
            if (!ok) fail(b, a.status);
            break;
        }
        const uint32_t buf = lt & 1, tph = (lt >> 1) & 1;
        if (!mbar_wait(&b->tempty[buf], tph ^ 1, a.timeout_ns, ab)) { fail(b, a.status); break; }
        tc_fence_after_sync();
        const uint32_t d_tmem = tmem + buf * BN;
        for (int kb = 0; kb < nk; ++kb, ++it) {
            const int s = it % STAGES;
            const uint32_t ph = (it / STAGES) & 1;
            if ((wait_a && !mbar_wait(&b->full_a[s], ph, a.timeout_ns, ab)) ||
                !mbar_wait(&b->full_b[s], ph, a.timeout_ns, ab)) {
                fail(b, a.status);
                ok = false;
                break;
            }
            tc_fence_after_sync();
            const uint32_t sa = smem_u32(sm.stages + s * STAGE_BYTES);
            const uint32_t sb = sa + A_BYTES;
#pragma unroll
            for (int kk = 0; kk < BK / 16; ++kk)
                umma_bf16(d_tmem, sdesc_k_sw128(sa + kk * 32), sdesc_k_sw128(sb + kk * 32), idesc,
                          (kb | kk) != 0);
            umma_commit(&b->empty[s]);
        }
        umma_commit(&b->tfull[buf]);  // also after an abort: arrives when issued MMAs finish
        if (!ok) break;
    }
}

// ---------------------------------------------------------------------------
// Gate-Up: h[p][n0 + j] = silu(x_t . Wg[n0 + j]) * (x_t . Wu[n0 + j])
// ---------------------------------------------------------------------------
__global__ void __launch_bounds__(GATEUP_THREADS, 1)
    k_gateup_bf16(const __grid_constant__ CUtensorMap tm_w, const __grid_constant__ CUtensorMap tm_ws,
                  GroupedGemmArgs a, const uint16_t* __restrict__ x, uint16_t* __restrict__ h) {
    extern __shared__ uint8_t smem_raw[];
    Smem sm = carve_smem(smem_raw);
    Bars* b = sm.bars;
    const volatile int* ab = &b->abort_flag;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    // ring consumers: the MMA thread, 4 epilogue warps, 4 gather warps
    const uint32_t tmem = prologue(sm, a, GATHER_WARPS, 1 + EPI_WARPS + GATHER_WARPS);
    const int G = a.E + a.has_shared;
    const int n_tiles = a.I / 128;
    const int total = sm.tt->mstart[G] * n_tiles;
    const int nk = a.d / BK;
    const int Tk = a.T * a.k;

    if (warp == TMA_WARP) {
        if (lane == 0) {
            // ---------------- weights by TMA: 128 gate rows + 128 up rows
            tma_prefetch_desc(&tm_w);
            tma_prefetch_desc(&tm_ws);
            uint32_t it = 0, issued = 0;
            bool ok = true;
            // weight rows of a tile: 128 gate rows and the matching 128 up rows
            auto rows_of = [&](const Tile& t, const CUtensorMap*& map, int& rg, int& ru) {
                const bool shared = t.g >= a.E;
                map = shared ? &tm_ws : &tm_w;
                const int rbase = shared ? 0 : t.g * 2 * a.I;
                rg = rbase + t.n * 128;
                ru = rbase + a.I + t.n * 128;
            };
            for (uint32_t ti = 0; ok; ++ti) {
                const int tile = tile_ring_push(&b->ring, ti, a.tile_counter, total, a.timeout_ns,
                                                ab, ok);
                if (tile < 0) {
                    if (!ok) fail(b, a.status);
                    break;
                }
                const Tile t = decode_tile(sm.tt, G, n_tiles, tile, BM);
                const CUtensorMap* map;
                int rg, ru;
                rows_of(t, map, rg, ru);
                for (int kb = 0; kb < nk; ++kb, ++it) {
                    const int s = it % STAGES;
                    const uint32_t ph = (it / STAGES) & 1;
                    if (!mbar_wait(&b->empty[s], ph ^ 1, a.timeout_ns, ab)) {
                        fail(b, a.status);
                        ok = false;
                        break;
                    }
                    uint8_t* sb = sm.stages + s * STAGE_BYTES + A_BYTES;
                    mbar_arrive_expect_tx(&b->full_b[s], B_BYTES);
                    tma_load_2d(sb, map, &b->full_b[s], kb * BK, rg);
                    tma_load_2d(sb + B_HALF, map, &b->full_b[s], kb * BK, ru);
                    ++issued;
                }
            }
            if (*ab) {
                for (uint32_t i = (issued > STAGES ? issued - STAGES : 0); i < issued; ++i)
                    mbar_wait(&b->full_b[i % STAGES], (i / STAGES) & 1, a.timeout_ns, nullptr);
            }
        }
    } else if (warp >= GATHER_WARP0) {
        // ---------------- A rows gathered from x through the permutation.
        // Eight consecutive lanes copy the eight 16-byte chunks of one row's
        // 128-byte k-slice, so each warp instruction reads four whole lines;
        // thread j owns chunk j % 8 of rows j / 8 + 16 i, i = 0..7.  A stage
        // is published (proxy fence + arrive) once its copies have landed,
        // two stages behind the newest, so three stages are in flight.
        const int j = threadIdx.x - GATHER_WARP0 * 32;
        const uint32_t chunk = static_cast<uint32_t>(j & 7);
        const int rr = j >> 3;
        const uint32_t swz_off = ((chunk ^ static_cast<uint32_t>(rr & 7)) << 4);
        uint32_t it = 0;
        int pend0 = -1, pend1 = -1;  // stages issued but not yet published, oldest first
        bool ok = true;
        for (uint32_t ti = 0; ok; ++ti) {
            const int tile = tile_ring_pop_warp(&b->ring, ti, a.timeout_ns, ab, ok);
            if (tile < 0) {
                if (!ok && lane == 0) fail(b, a.status);
                break;
            }
            const Tile t = decode_tile(sm.tt, G, n_tiles, tile, BM);
            const uint16_t* src[8];
            uint32_t valid = 0;
#pragma unroll
            for (int i = 0; i < 8; ++i) {
                const int r = rr + 16 * i;
                int64_t tok = 0;
                if (r < t.nrows) {
                    const int p = t.row0 + r;
                    tok = (t.g < a.E) ? (int64_t)(a.perm[p] / a.k) : (int64_t)(p - Tk);
                    valid |= 1u << i;
                }
                src[i] = x + tok * a.d + chunk * 8;
            }
            for (int kb = 0; kb < nk; ++kb, ++it) {
                const int s = it % STAGES;
                const uint32_t ph = (it / STAGES) & 1;
                if (!warp_wait(&b->empty[s], ph ^ 1, a.timeout_ns, ab)) {
                    fail(b, a.status);
                    ok = false;
                    break;
                }
                const uint32_t dst = smem_u32(sm.stages + s * STAGE_BYTES) + rr * 128 + swz_off;
#pragma unroll
                for (int i = 0; i < 8; ++i)
                    cp_async_16(dst + i * 16 * 128, src[i] + kb * BK, ((valid >> i) & 1u) ? 16u : 0u);
                cp_async_commit();
                if (pend0 >= 0) {
                    cp_async_wait<2>();  // the oldest of the three groups in flight is done
                    fence_proxy_async_smem();
                    warp_arrive(&b->full_a[pend0]);
                }
                pend0 = pend1;
                pend1 = s;
            }
        }
        cp_async_wait<0>();
        fence_proxy_async_smem();
        if (pend0 >= 0) warp_arrive(&b->full_a[pend0]);
        if (pend1 >= 0) warp_arrive(&b->full_a[pend1]);
    } else if (warp == MMA_WARP) {
        if (lane == 0) mma_role(sm, a, tmem, G, n_tiles, true);
    } else {
        // ---------------- epilogue warps 0-3: TMEM -> silu(g) * u -> bf16
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
            if (!warp_wait(&b->tfull[buf], tph, a.timeout_ns, ab)) { fail(b, a.status); break; }
            tc_fence_after_sync();
            const uint32_t taddr = tmem + (static_cast<uint32_t>(warp * 32) << 16) + buf * BN;
            uint16_t* dst = h + (int64_t)(t.row0 + row) * a.I + t.n * 128;
#pragma unroll 1
            for (int c = 0; c < 4; ++c) {
                float gv[32], uv[32];
                tmem_load32x2(taddr + c * 32, taddr + 128 + c * 32, gv, uv);
                if (row < t.nrows) {
                    uint32_t pk[16];
#pragma unroll
                    for (int i = 0; i < 16; ++i)
                        pk[i] = pack_bf16x2(silu_f(gv[2 * i]) * uv[2 * i],
                                            silu_f(gv[2 * i + 1]) * uv[2 * i + 1]);
#pragma unroll
                    for (int q = 0; q < 4; ++q)
                        st_global_v4(dst + c * 32 + q * 8, pk[4 * q], pk[4 * q + 1], pk[4 * q + 2],
                                     pk[4 * q + 3]);
                }
            }
            tc_fence_before_sync();
            warp_arrive(&b->tempty[buf]);
        }
    }
    teardown(sm, tmem);
}

// ---------------------------------------------------------------------------
// Down: o[p][n0 + j] = h[p] . Wd[n0 + j]
// ---------------------------------------------------------------------------
// o is stored FP16 [R][d] (saturating): its rounding (2^-11 relative) adds
// little to the layer output's own bf16 rounding, where a bf16 o would add a
// second rounding of the same size to every term of the weighted combine.
__global__ void __launch_bounds__(DOWN_THREADS, 1)
    k_down_bf16(const __grid_constant__ CUtensorMap tm_h, const __grid_constant__ CUtensorMap tm_w,
                const __grid_constant__ CUtensorMap tm_ws, GroupedGemmArgs a, __half* __restrict__ o) {
    extern __shared__ uint8_t smem_raw[];
    Smem sm = carve_smem(smem_raw);
    Bars* b = sm.bars;
    const volatile int* ab = &b->abort_flag;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    // ring consumers: the MMA thread and 4 epilogue warps
    const uint32_t tmem = prologue(sm, a, 0, 1 + EPI_WARPS);
    const int G = a.E + a.has_shared;
    const int n_tiles = (a.d + BN - 1) / BN;
    const int total = sm.tt->mstart[G] * n_tiles;
    const int nk = a.I / BK;

    if (warp == TMA_WARP) {
        if (lane == 0) {
            tma_prefetch_desc(&tm_h);
            tma_prefetch_desc(&tm_w);
            tma_prefetch_desc(&tm_ws);
            uint32_t it = 0, issued = 0;
            bool ok = true;
            for (uint32_t ti = 0; ok; ++ti) {
                const int tile = tile_ring_push(&b->ring, ti, a.tile_counter, total, a.timeout_ns,
                                                ab, ok);
                if (tile < 0) {
                    if (!ok) fail(b, a.status);
                    break;
                }
                const Tile t = decode_tile(sm.tt, G, n_tiles, tile, BM);
                const bool shared = t.g >= a.E;
                const CUtensorMap* map = shared ? &tm_ws : &tm_w;
                const int r0 = (shared ? 0 : t.g * a.d) + t.n * BN;
                const bool two = t.n * BN + 128 < a.d;  // second 128-row half inside this matrix
                for (int kb = 0; kb < nk; ++kb, ++it) {
                    const int s = it % STAGES;
                    const uint32_t ph = (it / STAGES) & 1;
                    if (!mbar_wait(&b->empty[s], ph ^ 1, a.timeout_ns, ab)) {
                        fail(b, a.status);
                        ok = false;
                        break;
                    }
                    uint8_t* st = sm.stages + s * STAGE_BYTES;
                    mbar_arrive_expect_tx(&b->full_b[s], A_BYTES + (two ? B_BYTES : B_HALF));
                    tma_load_2d(st, &tm_h, &b->full_b[s], kb * BK, t.row0);
                    tma_load_2d(st + A_BYTES, map, &b->full_b[s], kb * BK, r0);
                    if (two) tma_load_2d(st + A_BYTES + B_HALF, map, &b->full_b[s], kb * BK, r0 + 128);
                    ++issued;
                }
            }
            if (*ab) {
                for (uint32_t i = (issued > STAGES ? issued - STAGES : 0); i < issued; ++i)
                    mbar_wait(&b->full_b[i % STAGES], (i / STAGES) & 1, a.timeout_ns, nullptr);
            }
        }
    } else if (warp == MMA_WARP) {
        if (lane == 0) mma_role(sm, a, tmem, G, n_tiles, false);
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
            if (!warp_wait(&b->tfull[buf], tph, a.timeout_ns, ab)) { fail(b, a.status); break; }
            tc_fence_after_sync();
            const uint32_t taddr = tmem + (static_cast<uint32_t>(warp * 32) << 16) + buf * BN;
            const int ncols = min(BN, a.d - t.n * BN);
            __half* dst = o + (int64_t)(t.row0 + row) * a.d + t.n * BN;
#pragma unroll 1
            for (int c = 0; c < BN / 32; ++c) {
                if (c * 32 >= ncols) break;  // uniform across the warp
                float v[32];
                tmem_load32(taddr + c * 32, v);
                if (row < t.nrows) st_f16x32(dst + c * 32, v);
            }
            tc_fence_before_sync();
            warp_arrive(&b->tempty[buf]);
        }
    }
    teardown(sm, tmem);
}

template <typename K>
cudaError_t set_smem_once(K kernel, bool* flags) {
    const int dev = current_device_info().device;
    if (dev >= 64 || flags[dev]) return cudaSuccess;
    cudaError_t e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         (int)SMEM_BYTES);
    if (e == cudaSuccess) flags[dev] = true;
    return e;
}

}  // namespace

cudaError_t launch_gateup_bf16(const GroupedGemmArgs& a, const uint16_t* x, const uint16_t* w_gu,
                               const uint16_t* ws_gu, uint16_t* h, cudaStream_t s) {
    if (a.T == 0) return cudaSuccess;
    CUtensorMap tw, tws;
    if (!make_tmap_2d(&tw, w_gu, 2, (uint64_t)a.E * 2 * a.I, (uint64_t)a.d, 128, BK))
        return cudaErrorInvalidValue;
    if (!make_tmap_2d(&tws, a.has_shared ? ws_gu : w_gu, 2, (uint64_t)2 * a.I, (uint64_t)a.d, 128, BK))
        return cudaErrorInvalidValue;
    static bool flags[64] = {false};
    cudaError_t e = set_smem_once(k_gateup_bf16, flags);
    if (e != cudaSuccess) return e;
    if (!a.counter_zeroed &&
        (e = cudaMemsetAsync(a.tile_counter, 0, sizeof(int32_t), s)) != cudaSuccess)
        return e;
    {
        const cudaError_t le = launch_pdl(k_gateup_bf16, dim3(current_device_info().num_sms),
                                          dim3(GATEUP_THREADS), SMEM_BYTES, s, tw, tws, a, x, h);
        if (le != cudaSuccess) return le;
    }
    return cudaGetLastError();
}

cudaError_t launch_down_bf16(const GroupedGemmArgs& a, const uint16_t* h, const uint16_t* w_d,
                             const uint16_t* ws_d, __half* o, cudaStream_t s) {
    if (a.T == 0) return cudaSuccess;
    const uint64_t R = (uint64_t)a.T * a.k + (a.has_shared ? a.T : 0);
    CUtensorMap th, tw, tws;
    if (!make_tmap_2d(&th, h, 2, R, (uint64_t)a.I, BM, BK) ||
        !make_tmap_2d(&tw, w_d, 2, (uint64_t)a.E * a.d, (uint64_t)a.I, 128, BK) ||
        !make_tmap_2d(&tws, a.has_shared ? ws_d : w_d, 2, (uint64_t)a.d, (uint64_t)a.I, 128, BK))
        return cudaErrorInvalidValue;
    static bool flags[64] = {false};
    cudaError_t e = set_smem_once(k_down_bf16, flags);
    if (e != cudaSuccess) return e;
    if (!a.counter_zeroed &&
        (e = cudaMemsetAsync(a.tile_counter, 0, sizeof(int32_t), s)) != cudaSuccess)
        return e;
    {
        const cudaError_t le = launch_pdl(k_down_bf16, dim3(current_device_info().num_sms),
                                          dim3(DOWN_THREADS), SMEM_BYTES, s, th, tw, tws, a, o);
        if (le != cudaSuccess) return le;
    }
    return cudaGetLastError();
}

}  // namespace moe
