// gemm_bf16_2sm.cu -- the grouped Down GEMM, and the Gate-Up GEMM over x
// already in permuted row order (below), on CTA pairs (tcgen05 cta_group::2),
// for workloads with many rows per expert.
//
// Same computation as the down kernel of gemm_bf16.cu ("HPC-Ops -
// 騰訊混元開源的工業級高性能大模型推理算子庫", section HPC-Ops的主要功能, "FusedMoE":
// Down GEMM), on a pair of CTAs (a cluster of two) per tile of 256 rows x 256
// output columns:
//  - each CTA holds its own 128 rows of h and the weights of 128 of the 256
//    output columns, so a 64-wide k-block is 32 KB of shared memory per CTA
//    instead of 48 KB (less shared-memory traffic per MMA, six stages);
//  - the pair leader (cluster rank 0) issues one M=256, N=256 MMA per 16-wide
//    k-step; the hardware reads A and B from both CTAs and leaves each CTA's
//    128 rows x 256 columns in its own TMEM (two accumulators, double
//    buffered across tiles);
//  - both CTAs' TMA loads complete on the leader's barrier (the leader arms
//    the pair's byte count); the leader's MMA commits arrive on the barriers
//    of both CTAs; the epilogue warps of the other CTA signal the leader's
//    accumulator barrier through cluster-mapped addresses.
// Measured on B200: +15% over the one-CTA kernel on a dense 16384-row problem,
// +8% on the skewed workload, +3% at ~256 rows per expert (prefill; with FP16
// expert outputs -- it was -10% with FP32 rows, where 256-row tiles pad more)
// and much slower at a few rows per expert (decode); so it serves >= 256 rows
// per expert on average.  Every wait is bounded, as in the one-CTA kernels.
#include "common.cuh"
#include "grouped_common.cuh"
#include "launch.h"

namespace moe {
namespace {

constexpr int BM = 128, PM = 256, BK = 64, BN = 256, STAGES = 6;
constexpr int A_BYTES = BM * BK * 2;         // 16 KB: this CTA's rows
constexpr int B_BYTES = 128 * BK * 2;        // 16 KB: this CTA's half of N
constexpr int STAGE_BYTES = A_BYTES + B_BYTES;
constexpr uint32_t TMEM_COLS = 512;          // two 256-column accumulators
constexpr int EPI_WARPS = 4, MMA_WARP = 4, TMA_WARP = 5;
constexpr int DOWN_THREADS = 32 * (TMA_WARP + 1);  // 192
constexpr uint16_t kPairMask = 0x3;

struct Bars {
    uint64_t full_b[STAGES];  // leader: its expect_tx arrival + both CTAs' bytes
    uint64_t empty[STAGES];   // each CTA: the leader's multicast MMA commit
    uint64_t tfull[2];        // each CTA: the leader's multicast commit
    uint64_t tempty[2];       // leader: epilogue warps of both CTAs (8 arrivals)
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

// One lane of the warp arrives (at cluster scope) on the leader's barrier.
__device__ __forceinline__ void warp_arrive_leader(uint64_t* bar) {
    __syncwarp();
    if ((threadIdx.x & 31) == 0) mbar_arrive_cluster(smem_in_rank(bar, 0));
}

__device__ __forceinline__ uint32_t prologue(Smem& sm, const GroupedGemmArgs& a, uint32_t rank) {
    const int warp = threadIdx.x >> 5;
    Bars* b = sm.bars;
    if (threadIdx.x == 0) {
        for (int s = 0; s < STAGES; ++s) {
            mbar_init(&b->full_b[s], 1);
            mbar_init(&b->empty[s], 1);
        }
        for (int i = 0; i < 2; ++i) {
            mbar_init(&b->tfull[i], 1);
            mbar_init(&b->tempty[i], 2 * EPI_WARPS);
        }
        b->abort_flag = 0;
        fence_barrier_init();
    }
    pdl_wait();  // offsets and the A operand come from the previous kernels
    if (warp == 0) build_tile_table(sm.tt, a.offsets, a.E, a.T, a.k, a.has_shared, PM);
    __syncthreads();
    pdl_trigger();
    cluster_sync();  // both CTAs' barriers exist before either signals the other
    if (warp == MMA_WARP) tmem_alloc_pair(&b->tmem_slot, TMEM_COLS);
    tc_fence_before_sync();
    __syncthreads();
    tc_fence_after_sync();
    (void)rank;
    return b->tmem_slot;
}

__device__ __forceinline__ void teardown(uint32_t tmem) {
    tc_fence_before_sync();
    __syncthreads();
    cluster_sync();  // neither CTA leaves while the other may still touch it
    if ((threadIdx.x >> 5) == MMA_WARP) {
        tc_fence_after_sync();
        tmem_dealloc_pair(tmem, TMEM_COLS);
    }
}

// This CTA's rows of a pair tile.
struct PairTile {
    Tile t;        // t.row0 / t.nrows: the pair's 256-row span
    int row0;      // first row of this CTA
    int nrows;     // valid rows of this CTA (0..128)
};

__device__ __forceinline__ PairTile decode_pair(const TileTable* tt, int G, int n_tiles, int tile,
                                                uint32_t rank) {
    PairTile p;
    p.t = decode_tile(tt, G, n_tiles, tile, PM);
    p.row0 = p.t.row0 + (int)rank * BM;
    p.nrows = min(BM, max(0, p.t.nrows - (int)rank * BM));
    return p;
}

// MMA issuer (pair leader only).
__device__ __forceinline__ void mma_role(Smem& sm, const GroupedGemmArgs& a, uint32_t tmem, int G,
                                         int n_tiles, int nk) {
    Bars* b = sm.bars;
    const volatile int* ab = &b->abort_flag;
    constexpr uint32_t idesc = idesc_bf16(PM, BN);
    const int total = sm.tt->mstart[G] * n_tiles;
    const int pair = blockIdx.x >> 1, npairs = gridDim.x >> 1;
    uint32_t it = 0, lt = 0;
    bool ok = true;
    for (int tile = pair; ok && tile < total; tile += npairs, ++lt) {
        const uint32_t buf = lt & 1, tph = (lt >> 1) & 1;
        if (!mbar_wait_cluster(&b->tempty[buf], tph ^ 1, a.timeout_ns, ab)) { fail(b, a.status); break; }
        tc_fence_after_sync();
        const uint32_t d_tmem = tmem + buf * BN;
        for (int kb = 0; kb < nk; ++kb, ++it) {
            const int s = it % STAGES;
            const uint32_t ph = (it / STAGES) & 1;
            if (!mbar_wait_cluster(&b->full_b[s], ph, a.timeout_ns, ab)) {
                fail(b, a.status);
                ok = false;
                break;
            }
            tc_fence_after_sync();
            const uint32_t sa = smem_u32(sm.stages + s * STAGE_BYTES);
            const uint32_t sb = sa + A_BYTES;
#pragma unroll
            for (int kk = 0; kk < BK / 16; ++kk)
                umma_bf16_pair(d_tmem, sdesc_k_sw128(sa + kk * 32), sdesc_k_sw128(sb + kk * 32),
                               idesc, (kb | kk) != 0);
            umma_commit_pair(&b->empty[s], kPairMask);
        }
        umma_commit_pair(&b->tfull[buf], kPairMask);
    }
}

// ---------------------------------------------------------------------------
// Down on a CTA pair: o rows = h rows . Wd^T, FP32
// ---------------------------------------------------------------------------
__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(DOWN_THREADS, 1)
    k_down_bf16_2sm(const __grid_constant__ CUtensorMap tm_h, const __grid_constant__ CUtensorMap tm_w,
                    const __grid_constant__ CUtensorMap tm_ws, GroupedGemmArgs a,
                    __half* __restrict__ o) {
    extern __shared__ uint8_t smem_raw[];
    Smem sm = carve(smem_raw);
    Bars* b = sm.bars;
    const volatile int* ab = &b->abort_flag;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const uint32_t rank = cluster_ctarank();
    const uint32_t tmem = prologue(sm, a, rank);
    const int G = a.E + a.has_shared;
    const int n_tiles = (a.d + BN - 1) / BN;
    const int total = sm.tt->mstart[G] * n_tiles;
    const int nk = a.I / BK;
    const int pair = blockIdx.x >> 1, npairs = gridDim.x >> 1;

    if (warp == TMA_WARP) {
        if (lane == 0) {
            tma_prefetch_desc(&tm_h);
            tma_prefetch_desc(&tm_w);
            tma_prefetch_desc(&tm_ws);
            const uint32_t full_b_leader = smem_in_rank(&b->full_b[0], 0);
            uint32_t it = 0;
            bool ok = true;
            for (int tile = pair; ok && tile < total; tile += npairs) {
                const PairTile p = decode_pair(sm.tt, G, n_tiles, tile, rank);
                const bool shared = p.t.g >= a.E;
                const CUtensorMap* map = shared ? &tm_ws : &tm_w;
                // this CTA's 128 output columns; the second half may lie beyond d
                const int c0 = p.t.n * BN + (int)rank * 128;
                const bool mine = c0 < a.d;
                const bool other = p.t.n * BN + (int)(rank ^ 1u) * 128 < a.d;
                const int rb = (shared ? 0 : p.t.g * a.d) + c0;
                for (int kb = 0; kb < nk; ++kb, ++it) {
                    const int s = it % STAGES;
                    const uint32_t ph = (it / STAGES) & 1;
                    if (!mbar_wait(&b->empty[s], ph ^ 1, a.timeout_ns, ab)) {
                        fail(b, a.status);
                        ok = false;
                        break;
                    }
                    if (rank == 0)
                        mbar_arrive_expect_tx(&b->full_b[s], 2 * A_BYTES + (mine ? B_BYTES : 0) +
                                                                 (other ? B_BYTES : 0));
                    uint8_t* st = sm.stages + s * STAGE_BYTES;
                    const uint32_t bar = full_b_leader + s * (uint32_t)sizeof(uint64_t);
                    tma_load_2d_pair(st, &tm_h, bar, kb * BK, p.row0);
                    if (mine) tma_load_2d_pair(st + A_BYTES, map, bar, kb * BK, rb);
                }
            }
        }
    } else if (warp == MMA_WARP) {
        if (lane == 0 && rank == 0) mma_role(sm, a, tmem, G, n_tiles, nk);
    } else if (warp < EPI_WARPS) {
        const int row = warp * 32 + lane;
        uint32_t lt = 0;
        for (int tile = pair; tile < total; tile += npairs, ++lt) {
            const PairTile p = decode_pair(sm.tt, G, n_tiles, tile, rank);
            const uint32_t buf = lt & 1, tph = (lt >> 1) & 1;
            if (!warp_wait(&b->tfull[buf], tph, a.timeout_ns, ab)) { fail(b, a.status); break; }
            tc_fence_after_sync();
            const uint32_t taddr = tmem + (static_cast<uint32_t>(warp * 32) << 16) + buf * BN;
            const int ncols = min(BN, a.d - p.t.n * BN);
            __half* dst = o + (int64_t)(p.row0 + row) * a.d + p.t.n * BN;
#pragma unroll 1
            for (int c = 0; c < BN / 32; ++c) {
                if (c * 32 >= ncols) break;  // uniform across the warp
                float v[32];
                tmem_load32(taddr + c * 32, v);
                if (row < p.nrows) st_f16x32(dst + c * 32, v);
            }
            tc_fence_before_sync();
            warp_arrive_leader(&b->tempty[buf]);
        }
    }
    teardown(tmem);
}

// ---------------------------------------------------------------------------
// Gate-Up on a CTA pair: h[p][j] = silu(x_t . Wg[j]) * (x_t . Wu[j]) for a tile
// of 256 permuted rows x 128 columns j of h.  Both operands arrive by TMA: the
// routed rows from xp, x already copied into the permuted row order, the shared
// expert's rows (token order) from x itself; CTA 0 loads the
// tile's 128 gate rows of W_gu and CTA 1 the matching 128 up rows, the two
// halves of the pair MMA's N = 256, so each CTA's accumulator holds its 128
// rows x [gate | up].  A CTA-pair MMA runs at the tensor core's full rate
// (8192 FLOP per SM cycle measured for M = 256, N = 256), the one-CTA M = 128
// MMA of k_gateup_bf16_wide at 75% of it, and each CTA's two 256-column
// accumulators alternate by tile, so a tile's epilogue overlaps the next
// tile's MMAs.
// ---------------------------------------------------------------------------
__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(DOWN_THREADS, 1)
    k_gateup_bf16_2sm(const __grid_constant__ CUtensorMap tm_x, const __grid_constant__ CUtensorMap tm_xt,
                      const __grid_constant__ CUtensorMap tm_w, const __grid_constant__ CUtensorMap tm_ws,
                      GroupedGemmArgs a, uint16_t* __restrict__ h) {
    extern __shared__ uint8_t smem_raw[];
    Smem sm = carve(smem_raw);
    Bars* b = sm.bars;
    const volatile int* ab = &b->abort_flag;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const uint32_t rank = cluster_ctarank();
    const uint32_t tmem = prologue(sm, a, rank);
    const int G = a.E + a.has_shared;
    const int n_tiles = a.I / 128;
    const int total = sm.tt->mstart[G] * n_tiles;
    const int nk = a.d / BK;
    const int pair = blockIdx.x >> 1, npairs = gridDim.x >> 1;

    if (warp == TMA_WARP) {
        if (lane == 0) {
            tma_prefetch_desc(&tm_x);
            tma_prefetch_desc(&tm_xt);
            tma_prefetch_desc(&tm_w);
            tma_prefetch_desc(&tm_ws);
            const uint32_t full_b_leader = smem_in_rank(&b->full_b[0], 0);
            const int Tk = a.T * a.k;
            uint32_t it = 0;
            bool ok = true;
            for (int tile = pair; ok && tile < total; tile += npairs) {
                const PairTile p = decode_pair(sm.tt, G, n_tiles, tile, rank);
                const bool shared = p.t.g >= a.E;
                const CUtensorMap* map = shared ? &tm_ws : &tm_w;
                // rows: the routed ones from the permuted copy, the shared expert's from x
                const CUtensorMap* amap = shared ? &tm_xt : &tm_x;
                const int arow = shared ? p.row0 - Tk : p.row0;
                // CTA 0: the tile's gate rows, CTA 1: the matching up rows
                const int rb = (shared ? 0 : p.t.g * 2 * a.I) + (int)rank * a.I + p.t.n * 128;
                for (int kb = 0; kb < nk; ++kb, ++it) {
                    const int s = it % STAGES;
                    const uint32_t ph = (it / STAGES) & 1;
                    if (!mbar_wait(&b->empty[s], ph ^ 1, a.timeout_ns, ab)) {
                        fail(b, a.status);
                        ok = false;
                        break;
                    }
                    if (rank == 0) mbar_arrive_expect_tx(&b->full_b[s], 2 * (A_BYTES + B_BYTES));
                    uint8_t* st = sm.stages + s * STAGE_BYTES;
                    const uint32_t bar = full_b_leader + s * (uint32_t)sizeof(uint64_t);
                    tma_load_2d_pair(st, amap, bar, kb * BK, arow);
                    tma_load_2d_pair(st + A_BYTES, map, bar, kb * BK, rb);
                }
            }
        }
    } else if (warp == MMA_WARP) {
        if (lane == 0 && rank == 0) mma_role(sm, a, tmem, G, n_tiles, nk);
    } else if (warp < EPI_WARPS) {
        const int row = warp * 32 + lane;
        uint32_t lt = 0;
        for (int tile = pair; tile < total; tile += npairs, ++lt) {
            const PairTile p = decode_pair(sm.tt, G, n_tiles, tile, rank);
            const uint32_t buf = lt & 1, tph = (lt >> 1) & 1;
            if (!warp_wait(&b->tfull[buf], tph, a.timeout_ns, ab)) { fail(b, a.status); break; }
            tc_fence_after_sync();
            const uint32_t taddr = tmem + (static_cast<uint32_t>(warp * 32) << 16) + buf * BN;
            uint16_t* dst = h + (int64_t)(p.row0 + row) * a.I + p.t.n * 128;
#pragma unroll 1
            for (int c = 0; c < 4; ++c) {
                float gv[32], uv[32];
                tmem_load32x2(taddr + c * 32, taddr + 128 + c * 32, gv, uv);
                if (row < p.nrows) {
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
            warp_arrive_leader(&b->tempty[buf]);
        }
    }
    teardown(tmem);
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

int pair_grid() { return (current_device_info().num_sms / 2) * 2; }

}  // namespace

cudaError_t launch_gateup_bf16_2sm(const GroupedGemmArgs& a, const uint16_t* xp, const uint16_t* x,
                                   const uint16_t* w_gu, const uint16_t* ws_gu, uint16_t* h,
                                   cudaStream_t s) {
    if (a.T == 0) return cudaSuccess;
    CUtensorMap tx, txt, tw, tws;
    if (!make_tmap_2d(&tx, xp, 2, (uint64_t)a.T * a.k, (uint64_t)a.d, BM, BK) ||
        !make_tmap_2d(&txt, x, 2, (uint64_t)a.T, (uint64_t)a.d, BM, BK) ||
        !make_tmap_2d(&tw, w_gu, 2, (uint64_t)a.E * 2 * a.I, (uint64_t)a.d, 128, BK) ||
        !make_tmap_2d(&tws, a.has_shared ? ws_gu : w_gu, 2, (uint64_t)2 * a.I, (uint64_t)a.d, 128, BK))
        return cudaErrorInvalidValue;
    static bool flags[64] = {false};
    cudaError_t e = set_smem_once(k_gateup_bf16_2sm, flags);
    if (e != cudaSuccess) return e;
    {
        const cudaError_t le = launch_pdl(k_gateup_bf16_2sm, dim3(pair_grid()), dim3(DOWN_THREADS),
                                          SMEM_BYTES, s, tx, txt, tw, tws, a, h);
        if (le != cudaSuccess) return le;
    }
    return cudaGetLastError();
}

cudaError_t launch_down_bf16_2sm(const GroupedGemmArgs& a, const uint16_t* h, const uint16_t* w_d,
                                 const uint16_t* ws_d, __half* o, cudaStream_t s) {
    if (a.T == 0) return cudaSuccess;
    const uint64_t R = (uint64_t)a.T * a.k + (a.has_shared ? a.T : 0);
    CUtensorMap th, tw, tws;
    if (!make_tmap_2d(&th, h, 2, R, (uint64_t)a.I, BM, BK) ||
        !make_tmap_2d(&tw, w_d, 2, (uint64_t)a.E * a.d, (uint64_t)a.I, 128, BK) ||
        !make_tmap_2d(&tws, a.has_shared ? ws_d : w_d, 2, (uint64_t)a.d, (uint64_t)a.I, 128, BK))
        return cudaErrorInvalidValue;
    static bool flags[64] = {false};
    cudaError_t e = set_smem_once(k_down_bf16_2sm, flags);
    if (e != cudaSuccess) return e;
    {
        const cudaError_t le = launch_pdl(k_down_bf16_2sm, dim3(pair_grid()), dim3(DOWN_THREADS),
                                          SMEM_BYTES, s, th, tw, tws, a, o);
        if (le != cudaSuccess) return le;
    }
    return cudaGetLastError();
}

}  // namespace moe
