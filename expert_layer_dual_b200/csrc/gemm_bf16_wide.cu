// gemm_bf16_wide.cu -- the grouped Gate-Up GEMM with 256-row tiles, for
// workloads with many tiles.
//
// Same computation as k_gateup_bf16 ("HPC-Ops - 騰訊混元開源的工業級高性能大模型推理算子庫",
// section HPC-Ops的主要功能, "FusedMoE": Gate-Up GEMM, and section HPC-Ops的技術原理,
// "FusedMoE 流水線重構": x read through the routing index, no separate gather
// pass):  h[p][j] = silu(x_t . Wg[j]) * (x_t . Wu[j]).
//
// A tile is 256 permuted rows x 128 columns j of h: two M = 128 MMAs per
// 16-wide k-step share each stage of weights (the 128 gate rows and the
// matching 128 up rows of W_gu, N = 256), one per 128-row half of the tile,
// into two 256-column TMEM accumulators.  A 64-wide k-block moves 64 KB into
// shared memory for twice the MMA work of the one-CTA kernel's 48 KB, so
// 1.5x fewer bytes per FLOP; the two accumulators fill TMEM, so a tile's
// epilogue does not overlap the next tile's MMAs, and 256-row tiles leave
// more of the last wave idle.  Measured on B200 with the bench's CUDA-graph
// timing, against the 128-row kernel, both with the fast SiLU: 4-7% faster
// per step at prefill (~256 rows per expert), 3% on the skewed workload,
// 2-3% with ~512 rows per expert, 1-7% on a dense 16384-row problem; so it
// serves shapes with at least 256 rows per expert on average when x is
// gathered through the permutation (the stage entry point moe_gemm_gateup);
// the forward at those shapes copies x into the permuted order and runs the
// CTA-pair gate-up of gemm_bf16_2sm.cu instead (~2% faster per step).
//  - persistent, one CTA per SM, tiles from the dynamic schedule of
//    grouped_common.cuh;
//  - three 64 KB stages: 256 rows gathered from x through the permutation by
//    eight warps with cp.async (128-byte swizzle, K-major), the weights by TMA;
//  - eight epilogue warps: warps 0-3 drain the first accumulator (rows
//    0-127), warps 4-7 the second (rows 128-255, skipped for a tile of at
//    most 128 rows, whose second MMA is not issued).
// Every wait is bounded; a timeout sets the device status word and all roles
// stop, drain their copies in flight and free TMEM.
#include "common.cuh"
#include "grouped_common.cuh"
#include "launch.h"

namespace moe {
namespace {

constexpr int BM = 256, BK = 64, BN = 256, STAGES = 3;
constexpr int A_HALF = 128 * BK * 2;  // 16 KB: 128 rows
constexpr int A_BYTES = 2 * A_HALF;   // 32 KB: the tile's 256 rows
constexpr int B_HALF = 128 * BK * 2;  // 16 KB: 128 weight rows
constexpr int B_BYTES = 2 * B_HALF;   // 32 KB: gate + up rows
constexpr int STAGE_BYTES = A_BYTES + B_BYTES;
constexpr uint32_t TMEM_COLS = 512;   // two 256-column accumulators
constexpr int EPI_WARPS = 8, MMA_WARP = 8, TMA_WARP = 9, GATHER_WARP0 = 10, GATHER_WARPS = 8;
constexpr int THREADS = 32 * (GATHER_WARP0 + GATHER_WARPS);  // 576

struct Bars {
    uint64_t full_a[STAGES];  // one arrival per gather warp
    uint64_t full_b[STAGES];  // TMA arrival + transaction bytes
    uint64_t empty[STAGES];   // MMA commit
    uint64_t tfull;           // accumulators ready (MMA commit)
    uint64_t tempty;          // accumulators drained (one arrival per epilogue warp)
    TileRing ring;
    uint32_t tmem_slot;
    int abort_flag;
};

constexpr size_t SMEM_BYTES = 1024 + STAGES * STAGE_BYTES + sizeof(Bars) + sizeof(TileTable) + 64;

__device__ __forceinline__ void fail(Bars* b, int32_t* status) {
    report_status(status, MOE_ERR_DEVICE_TIMEOUT);
    *reinterpret_cast<volatile int*>(&b->abort_flag) = 1;
}

__device__ __forceinline__ void warp_arrive(uint64_t* bar) {
    __syncwarp();
    if ((threadIdx.x & 31) == 0) mbar_arrive(bar);
}

__global__ void __launch_bounds__(THREADS, 1)
    k_gateup_bf16_wide(const __grid_constant__ CUtensorMap tm_w,
                       const __grid_constant__ CUtensorMap tm_ws, GroupedGemmArgs a,
                       const uint16_t* __restrict__ x, uint16_t* __restrict__ h) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t* stages = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                                 ~static_cast<uintptr_t>(1023));
    Bars* b = reinterpret_cast<Bars*>(stages + STAGES * STAGE_BYTES);
    TileTable* tt = reinterpret_cast<TileTable*>(b + 1);
    const volatile int* ab = &b->abort_flag;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

    if (threadIdx.x == 0) {
        for (int s = 0; s < STAGES; ++s) {
            mbar_init(&b->full_a[s], GATHER_WARPS);
            mbar_init(&b->full_b[s], 1);
            mbar_init(&b->empty[s], 1);
        }
        mbar_init(&b->tfull, 1);
        mbar_init(&b->tempty, EPI_WARPS);
        // ring consumers: the MMA thread, the epilogue warps, the gather warps
        tile_ring_init(&b->ring, 1 + EPI_WARPS + GATHER_WARPS);
        b->abort_flag = 0;
        fence_barrier_init();
    }
    if (warp == MMA_WARP) tmem_alloc(&b->tmem_slot, TMEM_COLS);
    pdl_wait();  // offsets and the A operand come from the previous kernels
    if (warp == 0) build_tile_table(tt, a.offsets, a.E, a.T, a.k, a.has_shared, BM);
    tc_fence_before_sync();
    __syncthreads();
    pdl_trigger();
    tc_fence_after_sync();
    const uint32_t tmem = b->tmem_slot;
    const int G = a.E + a.has_shared;
    const int n_tiles = a.I / 128;
    const int total = tt->mstart[G] * n_tiles;
    const int nk = a.d / BK;
    const int Tk = a.T * a.k;

    if (warp == TMA_WARP) {
        if (lane == 0) {
            // ---------------- weights by TMA: 128 gate rows + the matching 128 up rows
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
                const Tile t = decode_tile(tt, G, n_tiles, tile, BM);
                const bool shared = t.g >= a.E;
                const CUtensorMap* map = shared ? &tm_ws : &tm_w;
                const int rg = (shared ? 0 : t.g * 2 * a.I) + t.n * 128;
                for (int kb = 0; kb < nk; ++kb, ++it) {
                    const int s = it % STAGES;
                    const uint32_t ph = (it / STAGES) & 1;
                    if (!mbar_wait(&b->empty[s], ph ^ 1, a.timeout_ns, ab)) {
                        fail(b, a.status);
                        ok = false;
                        break;
                    }
                    uint8_t* sb = stages + s * STAGE_BYTES + A_BYTES;
                    mbar_arrive_expect_tx(&b->full_b[s], B_BYTES);
                    tma_load_2d(sb, map, &b->full_b[s], kb * BK, rg);
                    tma_load_2d(sb + B_HALF, map, &b->full_b[s], kb * BK, rg + a.I);
                    ++issued;
                }
            }
            if (*ab) {
                for (uint32_t i = (issued > STAGES ? issued - STAGES : 0); i < issued; ++i)
                    mbar_wait(&b->full_b[i % STAGES], (i / STAGES) & 1, a.timeout_ns, nullptr);
            }
        }
    } else if (warp >= GATHER_WARP0) {
        // ---------------- the tile's 256 rows gathered from x through the
        // permutation: eight consecutive lanes copy the eight 16-byte chunks of
        // one row's 128-byte k-slice; thread j owns chunk j % 8 of rows
        // j / 8 + 32 i.  A stage is published (proxy fence + arrive) once its
        // copies have landed, one stage behind the newest.
        const int j = threadIdx.x - GATHER_WARP0 * 32;
        const uint32_t chunk = static_cast<uint32_t>(j & 7);
        const int rr = j >> 3;
        const uint32_t swz_off = ((chunk ^ static_cast<uint32_t>(rr & 7)) << 4);
        uint32_t it = 0;
        int pend = -1;  // stage issued but not yet published
        bool ok = true;
        for (uint32_t ti = 0; ok; ++ti) {
            const int tile = tile_ring_pop_warp(&b->ring, ti, a.timeout_ns, ab, ok);
            if (tile < 0) {
                if (!ok && lane == 0) fail(b, a.status);
                break;
            }
            const Tile t = decode_tile(tt, G, n_tiles, tile, BM);
            const uint16_t* src[8];
            uint32_t valid = 0;
#pragma unroll
            for (int i = 0; i < 8; ++i) {
                const int r = rr + 32 * i;
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
                    if (lane == 0) fail(b, a.status);
                    ok = false;
                    break;
                }
                const uint32_t dst = smem_u32(stages + s * STAGE_BYTES) + rr * 128 + swz_off;
#pragma unroll
                for (int i = 0; i < 8; ++i)
                    cp_async_16(dst + i * 32 * 128, src[i] + kb * BK, ((valid >> i) & 1u) ? 16u : 0u);
                cp_async_commit();
                if (pend >= 0) {
                    cp_async_wait<1>();  // the older of the two groups in flight has landed
                    fence_proxy_async_smem();
                    warp_arrive(&b->full_a[pend]);
                }
                pend = s;
            }
        }
        cp_async_wait<0>();
        fence_proxy_async_smem();
        if (pend >= 0) warp_arrive(&b->full_a[pend]);
    } else if (warp == MMA_WARP) {
        if (lane == 0) {
            // ---------------- the MMA issuer: both halves of the tile per k-step
            constexpr uint32_t idesc = idesc_bf16(128, BN);
            uint32_t it = 0;
            bool ok = true;
            for (uint32_t lt = 0; ok; ++lt) {
                const int tile = tile_ring_pop(&b->ring, lt, a.timeout_ns, ab, ok);
                if (tile < 0) {
                    if (!ok) fail(b, a.status);
                    break;
                }
                const Tile t = decode_tile(tt, G, n_tiles, tile, BM);
                const bool two = t.nrows > 128;
                if (!mbar_wait(&b->tempty, (lt & 1) ^ 1, a.timeout_ns, ab)) {
                    fail(b, a.status);
                    break;
                }
                tc_fence_after_sync();
                for (int kb = 0; kb < nk; ++kb, ++it) {
                    const int s = it % STAGES;
                    const uint32_t ph = (it / STAGES) & 1;
                    if (!mbar_wait(&b->full_a[s], ph, a.timeout_ns, ab) ||
                        !mbar_wait(&b->full_b[s], ph, a.timeout_ns, ab)) {
                        fail(b, a.status);
                        ok = false;
                        break;
                    }
                    tc_fence_after_sync();
                    const uint32_t sa = smem_u32(stages + s * STAGE_BYTES);
                    const uint32_t sb = sa + A_BYTES;
#pragma unroll
                    for (int kk = 0; kk < BK / 16; ++kk) {
                        const uint64_t bd = sdesc_k_sw128(sb + kk * 32);
                        umma_bf16(tmem, sdesc_k_sw128(sa + kk * 32), bd, idesc, (kb | kk) != 0);
                        if (two)
                            umma_bf16(tmem + BN, sdesc_k_sw128(sa + A_HALF + kk * 32), bd, idesc,
                                      (kb | kk) != 0);
                    }
                    umma_commit(&b->empty[s]);
                }
                umma_commit(&b->tfull);  // also after an abort: arrives when issued MMAs finish
            }
        }
    } else {
        // ---------------- epilogue warps 0-7: TMEM -> silu(g) * u -> bf16 h
        const int quad = warp & 3, half = warp >> 2;
        const int row = half * 128 + quad * 32 + lane;
        bool ok = true;
        for (uint32_t lt = 0;; ++lt) {
            const int tile = tile_ring_pop_warp(&b->ring, lt, a.timeout_ns, ab, ok);
            if (tile < 0) {
                if (!ok && lane == 0) fail(b, a.status);
                break;
            }
            const Tile t = decode_tile(tt, G, n_tiles, tile, BM);
            if (!warp_wait(&b->tfull, lt & 1, a.timeout_ns, ab)) {
                if (lane == 0) fail(b, a.status);
                break;
            }
            tc_fence_after_sync();
            if (half == 0 || t.nrows > 128) {  // warp-uniform
                const uint32_t taddr = tmem + (static_cast<uint32_t>(quad * 32) << 16) + half * BN;
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
                            st_global_v4(dst + c * 32 + q * 8, pk[4 * q], pk[4 * q + 1],
                                         pk[4 * q + 2], pk[4 * q + 3]);
                    }
                }
            }
            tc_fence_before_sync();
            warp_arrive(&b->tempty);
        }
    }
    tc_fence_before_sync();
    __syncthreads();
    if (warp == MMA_WARP) {
        tc_fence_after_sync();
        tmem_dealloc(tmem, TMEM_COLS);
    }
}

bool g_smem_set[64] = {false};

}  // namespace

cudaError_t launch_gateup_bf16_wide(const GroupedGemmArgs& a, const uint16_t* x,
                                    const uint16_t* w_gu, const uint16_t* ws_gu, uint16_t* h,
                                    cudaStream_t s) {
    if (a.T == 0) return cudaSuccess;
    CUtensorMap tw, tws;
    if (!make_tmap_2d(&tw, w_gu, 2, (uint64_t)a.E * 2 * a.I, (uint64_t)a.d, 128, BK) ||
        !make_tmap_2d(&tws, a.has_shared ? ws_gu : w_gu, 2, (uint64_t)2 * a.I, (uint64_t)a.d, 128,
                      BK))
        return cudaErrorInvalidValue;
    const int dev = current_device_info().device;
    if (dev < 64 && !g_smem_set[dev]) {
        cudaError_t e = cudaFuncSetAttribute(k_gateup_bf16_wide,
                                             cudaFuncAttributeMaxDynamicSharedMemorySize,
                                             (int)SMEM_BYTES);
        if (e != cudaSuccess) return e;
        g_smem_set[dev] = true;
    }
    cudaError_t e =
        a.counter_zeroed ? cudaSuccess : cudaMemsetAsync(a.tile_counter, 0, sizeof(int32_t), s);
    if (e != cudaSuccess) return e;
    {
        const cudaError_t le = launch_pdl(k_gateup_bf16_wide, dim3(current_device_info().num_sms),
                                          dim3(THREADS), SMEM_BYTES, s, tw, tws, a, x, h);
        if (le != cudaSuccess) return le;
    }
    return cudaGetLastError();
}

}  // namespace moe
