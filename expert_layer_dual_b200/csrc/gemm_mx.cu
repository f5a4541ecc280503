// gemm_mx.cu -- grouped expert GEMMs in MXFP8: e4m3 operands with one E8M0
// (power-of-two) scale per 32 consecutive K-elements of every row, for the
// weights and the activations alike.
//
// "PR #54160 完整报告", section 实现拆解 item 4 (the MXFP8 weight format beside
// FP8 block-wise 128x128); "HPC-Ops - 騰訊混元開源的工業級高性能大模型推理算子庫",
// section HPC-Ops的主要功能, "GroupGEMM FP8" and "FusedMoE" (grouped expert
// GEMMs, activation quantisation between Gate-Up and Down).
//
// Unlike the 128x128 FP32-scaled path (gemm_fp8.cu), MX scales are native to
// the sm_100 tensor core: tcgen05.mma.kind::mxf8f6f4.block_scale multiplies
// every 32-wide K slice of A and B by its 2^e scales inside the MMA and
// accumulates the whole K in TMEM, so there is no software promotion:
//  - tile 128 rows x 256 columns x 128-wide k-blocks (4 MMAs of K = 32), one
//    256-column FP32 accumulator; the rest of TMEM holds the scale factors;
//  - operands by TMA into a 4-stage ring (128-byte swizzle), as in the other
//    grouped GEMMs, tiles from the dynamic schedule of grouped_common.cuh;
//  - each k-block needs 4 scale bytes (one per MMA) for each of the tile's
//    128 A rows and 256 B rows, in shared memory in the layout tcgen05.cp
//    reads: 32 rows of 16 bytes, byte 4g + j of row l = scale j of tile row
//    32g + l.  Weight scales are stored offline in exactly that image (512
//    bytes per k-block and 128-row block), so the TMA thread fetches them
//    with two 1-D bulk copies beside the operand tiles; activation scales are
//    k-block-major ([K/128][rows][4], written that way by the quantiser and
//    by the gate-up epilogue) and a scale warp gathers the tile's 128 records
//    with coalesced 4-byte cp.async copies (the tile's first row is arbitrary,
//    so its 512 bytes are not 16-byte aligned for a bulk copy);
//  - the MMA thread copies them into TMEM with tcgen05.cp (32x128b.warpx4:
//    the 32 rows go to every 32-lane subpartition, as the block-scaled MMA
//    expects), then issues the 4 MMAs, MMA j reading byte j of the 32-bit
//    scale cells (the scale-factor id of its descriptor);
//  - 16 epilogue warps drain the accumulator: gate-up computes
//    h = silu(g) * u for 32 columns per thread -- exactly one MX block -- and
//    writes e4m3 h with its E8M0 scale (no cross-thread amax); down writes
//    o in FP16.  The accumulator is handed back as soon as it has been read.
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
constexpr int SFA_BYTES = 512;         // 128 rows x 4 scale bytes
constexpr int SF_STAGE = SFA_BYTES + 1024;  // + 256 B rows x 4 bytes
constexpr uint32_t TMEM_COLS = 512;
constexpr uint32_t SF_COL = 256;       // two 16-column scale buffers after the accumulator
constexpr int EPI_WARPS = 16, MMA_WARP = 16, TMA_WARP = 17, SCALE_WARP = 18;
constexpr int THREADS = 32 * (SCALE_WARP + 1);  // 608

struct Bars {
    uint64_t full[STAGES];     // TMA arrival + transaction bytes
    uint64_t sf_full[STAGES];  // the stage's scale bytes landed (32 cp.async arrivals)
    uint64_t empty[STAGES];    // MMA commit (operands and scales consumed)
    uint64_t tfull;            // accumulator ready (MMA commit)
    uint64_t tempty;           // accumulator read (one arrival per epilogue warp)
    TileRing ring;
    uint32_t tmem_slot;
    int abort_flag;
};

constexpr size_t SMEM_BYTES =
    1024 + STAGES * STAGE_BYTES + STAGES * SF_STAGE + sizeof(Bars) + sizeof(TileTable) + 64;

struct Smem {
    uint8_t* stages;
    uint8_t* sf;  // [STAGES][SF_STAGE]
    Bars* bars;
    TileTable* tt;
};

__device__ __forceinline__ Smem carve(uint8_t* raw) {
    Smem s;
    s.stages = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(raw) + 1023) &
                                          ~static_cast<uintptr_t>(1023));
    s.sf = s.stages + STAGES * STAGE_BYTES;
    s.bars = reinterpret_cast<Bars*>(s.sf + STAGES * SF_STAGE);
    s.tt = reinterpret_cast<TileTable*>(s.bars + 1);
    return s;
}

__device__ __forceinline__ void fail(Bars* b, int32_t* status) {
    report_status(status, MOE_ERR_DEVICE_TIMEOUT);
    *reinterpret_cast<volatile int*>(&b->abort_flag) = 1;
}

__device__ __forceinline__ uint32_t prologue(Smem& sm, const GroupedGemmArgs& a) {
    const int warp = threadIdx.x >> 5;
    Bars* b = sm.bars;
    if (threadIdx.x == 0) {
        for (int s = 0; s < STAGES; ++s) {
            mbar_init(&b->full[s], 1);
            mbar_init(&b->sf_full[s], 32);  // one cp.async arrival per scale-warp lane
            mbar_init(&b->empty[s], 1);
        }
        mbar_init(&b->tfull, 1);
        mbar_init(&b->tempty, EPI_WARPS);
        // ring consumers: the MMA thread, the epilogue warps, the scale warp
        tile_ring_init(&b->ring, 1 + EPI_WARPS + 1);
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

// Weight rows of a tile's B operand: half 0 rows rb0.., half 1 rows rb1..
// (`two` false: the second half lies past the matrix and is not loaded).
// Their scales: the matrix's scale image, 128-row blocks lb0 / lb1 of the
// matrix's mrows rows.
struct BRows {
    const CUtensorMap* map;
    const uint8_t* scale;
    int rb0, rb1;
    int lb0, lb1, mrows;
    bool two;
};

// TMA producer (one thread).
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
            uint8_t* sf = sm.sf + s * SF_STAGE + SFA_BYTES;
            const uint8_t* img = L.scale + (int64_t)kb * (L.mrows / 128) * 512;
            mbar_arrive_expect_tx(&b->full[s], L.two ? B_BYTES + A_BYTES + 1024 : B_HALF + A_BYTES + 512);
            tma_load_2d(st, tm_a, &b->full[s], kb * BK, t.row0);
            tma_load_2d(st + A_BYTES, L.map, &b->full[s], kb * BK, L.rb0);
            bulk_load(sf, img + L.lb0 * 512, 512, &b->full[s]);
            if (L.two) {
                tma_load_2d(st + A_BYTES + B_HALF, L.map, &b->full[s], kb * BK, L.rb1);
                bulk_load(sf + 512, img + L.lb1 * 512, 512, &b->full[s]);
            }
            ++issued;
        }
    }
    if (*ab) {
        for (uint32_t i = (issued > STAGES ? issued - STAGES : 0); i < issued; ++i)
            mbar_wait(&b->full[i % STAGES], (i / STAGES) & 1, a.timeout_ns, nullptr);
    }
}

// All lanes of the warp are done with their part: one lane arrives for it.
__device__ __forceinline__ void warp_arrive(uint64_t* bar) {
    __syncwarp();
    if ((threadIdx.x & 31) == 0) mbar_arrive(bar);
}

// Byte offset, inside a stage's scale area, of the 4 scale bytes of tile row
// r (A: r < 128; B: r < 256, after the A part): the tcgen05.cp source layout.
__device__ __forceinline__ uint32_t sf_offset(int r) {
    return static_cast<uint32_t>((r >> 7) * 512 + (r & 31) * 16 + ((r >> 5) & 3) * 4);
}

// Scale warp: per k-block, the 128 A rows' 4-byte scale records (k-block-
// major: contiguous across rows, so each warp copy reads 128 contiguous
// bytes), 4 cp.async per lane; rows past the tile are zero-filled.  Each lane then arms an arrival on the
// stage's sf_full barrier (32 arrivals) that fires when its copies land, so a
// stage is published as soon as its bytes are in shared memory and the warp
// never waits for its own copies.  (Publishing a stage only after waiting
// for it, one or three stages later, starved the MMA: measured 1.72 and
// 2.39 ms for the FP8-sized gate-up.)  The MMA thread orders the landed
// bytes before its async-proxy reads with fence.proxy.async.
__device__ __forceinline__ void scale_role(Smem& sm, const GroupedGemmArgs& a, int G, int n_tiles,
                                           int nk, const uint8_t* __restrict__ act_scale,
                                           int64_t R) {
    Bars* b = sm.bars;
    const volatile int* ab = &b->abort_flag;
    const int lane = threadIdx.x & 31;
    uint32_t it = 0;
    bool ok = true;
    for (uint32_t lt = 0; ok; ++lt) {
        const int tile = tile_ring_pop_warp(&b->ring, lt, a.timeout_ns, ab, ok);
        if (tile < 0) break;
        const Tile t = decode_tile(sm.tt, G, n_tiles, tile, BM);
        for (int kb = 0; kb < nk; ++kb, ++it) {
            const int s = it % STAGES;
            const uint32_t ph = (it / STAGES) & 1;
            if (!warp_wait(&b->empty[s], ph ^ 1, a.timeout_ns, ab)) {
                ok = false;
                break;
            }
            const uint32_t dst = smem_u32(sm.sf + s * SF_STAGE);
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                const int r = lane + 32 * i;
                const bool in = r < t.nrows;
                cp_async_4(dst + sf_offset(r),
                           act_scale + (in ? ((int64_t)kb * R + t.row0 + r) * 4 : 0), in ? 4u : 0u);
            }
            cp_async_mbar_arrive_noinc(&b->sf_full[s]);
        }
    }
    cp_async_wait<0>();
    if (!ok && lane == 0) fail(b, a.status);
}

// MMA issuer (one thread): per k-block, the stage's scale bytes into a TMEM
// scale buffer (three tcgen05.cp: A, then B rows 0-127 and 128-255), then four
// block-scaled MMAs into the tile's accumulator.  The two scale buffers
// alternate by k-block; tcgen05.cp and tcgen05.mma of one thread run in issue
// order, so a buffer is rewritten only after the MMAs that read it.
__device__ __forceinline__ void mma_role(Smem& sm, const GroupedGemmArgs& a, uint32_t tmem, int nk) {
    Bars* b = sm.bars;
    const volatile int* ab = &b->abort_flag;
    constexpr uint32_t idesc = idesc_mx_e4m3(BM, BN);
    uint32_t it = 0;
    bool ok = true;
    for (uint32_t lt = 0; ok; ++lt) {
        if (tile_ring_pop(&b->ring, lt, a.timeout_ns, ab, ok) < 0) {
            if (!ok) fail(b, a.status);
            break;
        }
        if (!mbar_wait(&b->tempty, (lt & 1) ^ 1, a.timeout_ns, ab)) {
            fail(b, a.status);
            break;
        }
        tc_fence_after_sync();
        for (int kb = 0; kb < nk; ++kb, ++it) {
            const int s = it % STAGES;
            const uint32_t ph = (it / STAGES) & 1;
            if (!mbar_wait(&b->full[s], ph, a.timeout_ns, ab) ||
                !mbar_wait(&b->sf_full[s], ph, a.timeout_ns, ab)) {
                fail(b, a.status);
                ok = false;
                break;
            }
            tc_fence_after_sync();
            fence_proxy_async_smem();  // the cp.async scale bytes before tcgen05.cp reads them
            const uint32_t sa = smem_u32(sm.stages + s * STAGE_BYTES);
            const uint32_t sb = sa + A_BYTES;
            const uint32_t sfs = smem_u32(sm.sf + s * SF_STAGE);
            const uint32_t sfc = tmem + SF_COL + (it & 1) * 16;
            tmem_cp_32x128b_warpx4(sfc, sdesc_k_noswizzle(sfs, 128));
            tmem_cp_32x128b_warpx4(sfc + 4, sdesc_k_noswizzle(sfs + SFA_BYTES, 128));
            tmem_cp_32x128b_warpx4(sfc + 8, sdesc_k_noswizzle(sfs + SFA_BYTES + 512, 128));
#pragma unroll
            for (uint32_t kk = 0; kk < BK / 32; ++kk)
                umma_mx_e4m3(tmem, sdesc_k_sw128(sa + kk * 32), sdesc_k_sw128(sb + kk * 32),
                             idesc_with_sf_id(idesc, kk), sfc | (kk << 30), (sfc + 4) | (kk << 30),
                             (kb | kk) != 0);
            umma_commit(&b->empty[s]);
        }
        umma_commit(&b->tfull);  // also after an abort: arrives when issued work finishes
    }
}

// ---------------------------------------------------------------------------
// Gate-Up: h = silu(x Wg^T) * (x Wu^T) for 128 h columns per tile; each
// thread's 32 columns are one MX block of h: e4m3 codes and an E8M0 scale.
// ---------------------------------------------------------------------------
__global__ void __launch_bounds__(THREADS, 1)
    k_gateup_mx(const __grid_constant__ CUtensorMap tm_a, const __grid_constant__ CUtensorMap tm_w,
                const __grid_constant__ CUtensorMap tm_ws, GroupedGemmArgs a,
                const uint8_t* __restrict__ xs, const uint8_t* __restrict__ wsc,
                const uint8_t* __restrict__ wssc, uint8_t* __restrict__ hq,
                uint8_t* __restrict__ hs) {
    extern __shared__ uint8_t smem_raw[];
    Smem sm = carve(smem_raw);
    Bars* b = sm.bars;
    const volatile int* ab = &b->abort_flag;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const uint32_t tmem = prologue(sm, a);
    const int G = a.E + a.has_shared;
    const int n_tiles = a.I / 128;
    const int nk = a.d / BK;
    const int64_t R = (int64_t)a.T * a.k + (a.has_shared ? a.T : 0);
    auto rows_of = [&](const Tile& t) {
        const bool shared = t.g >= a.E;
        const int r0 = (shared ? 0 : t.g * 2 * a.I) + t.n * 128;
        const uint8_t* img = shared ? wssc : wsc + (int64_t)t.g * 2 * a.I * (a.d / 32);
        return BRows{shared ? &tm_ws : &tm_w, img, r0, r0 + a.I, t.n, a.I / 128 + t.n, 2 * a.I, true};
    };
    if (warp == TMA_WARP) {
        if (lane == 0) {
            tma_prefetch_desc(&tm_a);
            tma_prefetch_desc(&tm_w);
            tma_prefetch_desc(&tm_ws);
            tma_role(sm, a, &tm_a, G, n_tiles, nk, rows_of);
        }
    } else if (warp == MMA_WARP) {
        if (lane == 0) mma_role(sm, a, tmem, nk);
    } else if (warp == SCALE_WARP) {
        scale_role(sm, a, G, n_tiles, nk, xs, R);
    } else if (warp < EPI_WARPS) {
        const int quad = warp & 3, qtr = warp >> 2;
        const int row = quad * 32 + lane;
        const uint32_t base = tmem + (static_cast<uint32_t>(quad * 32) << 16);
        bool rok = true;
        for (uint32_t lt = 0;; ++lt) {
            const int tile = tile_ring_pop_warp(&b->ring, lt, a.timeout_ns, ab, rok);
            if (tile < 0) {
                if (!rok && lane == 0) fail(b, a.status);
                break;
            }
            const Tile t = decode_tile(sm.tt, G, n_tiles, tile, BM);
            if (!warp_wait(&b->tfull, lt & 1, a.timeout_ns, ab)) {
                if (lane == 0) fail(b, a.status);
                break;
            }
            tc_fence_after_sync();
            float h[32];
#pragma unroll
            for (int c = 0; c < 2; ++c) {
                float g[16], u[16];
                tmem_load16x2(base + qtr * 32 + c * 16, base + 128 + qtr * 32 + c * 16, g, u);
#pragma unroll
                for (int i = 0; i < 16; ++i) h[c * 16 + i] = silu_f(g[i]) * u[i];
            }
            tc_fence_before_sync();
            warp_arrive(&b->tempty);  // the accumulator is free for the next tile
            float amax = 0.0f;
#pragma unroll
            for (int i = 0; i < 32; ++i) amax = fmaxf(amax, fabsf(h[i]));
            const uint32_t sb = mx_scale_byte(amax);
            const float inv = __uint_as_float((254u - sb) << 23);
            if (row < t.nrows) {
                const int64_t p = t.row0 + row;
                uint8_t* dst = hq + p * a.I + t.n * 128 + qtr * 32;
#pragma unroll
                for (int q = 0; q < 2; ++q)
                    st_global_v4(dst + 16 * q, mx_quant4(h + 16 * q, inv),
                                 mx_quant4(h + 16 * q + 4, inv), mx_quant4(h + 16 * q + 8, inv),
                                 mx_quant4(h + 16 * q + 12, inv));
                hs[((int64_t)t.n * R + p) * 4 + qtr] = static_cast<uint8_t>(sb);  // k-block-major
            }
        }
    }
    teardown(tmem);
}

// ---------------------------------------------------------------------------
// Down: o[p][n0 + j] = (MX h)[p] . (MX Wd)[n0 + j], FP32 sums stored as FP16 rows.
// ---------------------------------------------------------------------------
__global__ void __launch_bounds__(THREADS, 1)
    k_down_mx(const __grid_constant__ CUtensorMap tm_a, const __grid_constant__ CUtensorMap tm_w,
              const __grid_constant__ CUtensorMap tm_ws, GroupedGemmArgs a,
              const uint8_t* __restrict__ hs, const uint8_t* __restrict__ wsc,
              const uint8_t* __restrict__ wssc, __half* __restrict__ o) {
    extern __shared__ uint8_t smem_raw[];
    Smem sm = carve(smem_raw);
    Bars* b = sm.bars;
    const volatile int* ab = &b->abort_flag;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const uint32_t tmem = prologue(sm, a);
    const int G = a.E + a.has_shared;
    const int n_tiles = (a.d + BN - 1) / BN;
    const int nk = a.I / BK;
    const int64_t R = (int64_t)a.T * a.k + (a.has_shared ? a.T : 0);
    auto rows_of = [&](const Tile& t) {
        const bool shared = t.g >= a.E;
        const int r0 = (shared ? 0 : t.g * a.d) + t.n * BN;
        const uint8_t* img = shared ? wssc : wsc + (int64_t)t.g * a.d * (a.I / 32);
        return BRows{shared ? &tm_ws : &tm_w, img, r0, r0 + 128, 2 * t.n, 2 * t.n + 1, a.d,
                     t.n * BN + 128 < a.d};
    };
    if (warp == TMA_WARP) {
        if (lane == 0) {
            tma_prefetch_desc(&tm_a);
            tma_prefetch_desc(&tm_w);
            tma_prefetch_desc(&tm_ws);
            tma_role(sm, a, &tm_a, G, n_tiles, nk, rows_of);
        }
    } else if (warp == MMA_WARP) {
        if (lane == 0) mma_role(sm, a, tmem, nk);
    } else if (warp == SCALE_WARP) {
        scale_role(sm, a, G, n_tiles, nk, hs, R);
    } else if (warp < EPI_WARPS) {
        const int quad = warp & 3, qtr = warp >> 2;
        const int row = quad * 32 + lane;
        const uint32_t base = tmem + (static_cast<uint32_t>(quad * 32) << 16);
        bool rok = true;
        for (uint32_t lt = 0;; ++lt) {
            const int tile = tile_ring_pop_warp(&b->ring, lt, a.timeout_ns, ab, rok);
            if (tile < 0) {
                if (!rok && lane == 0) fail(b, a.status);
                break;
            }
            const Tile t = decode_tile(sm.tt, G, n_tiles, tile, BM);
            if (!warp_wait(&b->tfull, lt & 1, a.timeout_ns, ab)) {
                if (lane == 0) fail(b, a.status);
                break;
            }
            tc_fence_after_sync();
            float v[64];
            tmem_load32x2(base + qtr * 64, base + qtr * 64 + 32, v, v + 32);
            tc_fence_before_sync();
            warp_arrive(&b->tempty);
            const int col = t.n * BN + qtr * 64;
            if (row < t.nrows && col < a.d) {
                __half* dst = o + (int64_t)(t.row0 + row) * a.d + col;
                st_f16x32(dst, v);
                st_f16x32(dst + 32, v + 32);
            }
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

cudaError_t launch_gateup_mx(const GroupedGemmArgs& a, const uint8_t* xq, const uint8_t* xs,
                             const uint8_t* w_gu, const uint8_t* w_gu_s, const uint8_t* ws_gu,
                             const uint8_t* ws_gu_s, uint8_t* hq, uint8_t* hs, cudaStream_t s) {
    if (a.T == 0) return cudaSuccess;
    const uint64_t R = (uint64_t)a.T * a.k + (a.has_shared ? a.T : 0);
    CUtensorMap ta, tw, tws;
    if (!make_tmap_2d(&ta, xq, 1, R, (uint64_t)a.d, BM, BK) ||
        !make_tmap_2d(&tw, w_gu, 1, (uint64_t)a.E * 2 * a.I, (uint64_t)a.d, 128, BK) ||
        !make_tmap_2d(&tws, a.has_shared ? ws_gu : w_gu, 1, (uint64_t)2 * a.I, (uint64_t)a.d, 128,
                      BK))
        return cudaErrorInvalidValue;
    static bool flags[64] = {false};
    cudaError_t e = set_smem_once(k_gateup_mx, flags);
    if (e != cudaSuccess) return e;
    if (!a.counter_zeroed &&
        (e = cudaMemsetAsync(a.tile_counter, 0, sizeof(int32_t), s)) != cudaSuccess)
        return e;
    {
        const cudaError_t le = launch_pdl(k_gateup_mx, dim3(current_device_info().num_sms),
                                          dim3(THREADS), SMEM_BYTES, s, ta, tw, tws, a, xs, w_gu_s,
                                          a.has_shared ? ws_gu_s : w_gu_s, hq, hs);
        if (le != cudaSuccess) return le;
    }
    return cudaGetLastError();
}

cudaError_t launch_down_mx(const GroupedGemmArgs& a, const uint8_t* hq, const uint8_t* hs,
                           const uint8_t* w_d, const uint8_t* w_d_s, const uint8_t* ws_d,
                           const uint8_t* ws_d_s, __half* o, cudaStream_t s) {
    if (a.T == 0) return cudaSuccess;
    const uint64_t R = (uint64_t)a.T * a.k + (a.has_shared ? a.T : 0);
    CUtensorMap ta, tw, tws;
    if (!make_tmap_2d(&ta, hq, 1, R, (uint64_t)a.I, BM, BK) ||
        !make_tmap_2d(&tw, w_d, 1, (uint64_t)a.E * a.d, (uint64_t)a.I, 128, BK) ||
        !make_tmap_2d(&tws, a.has_shared ? ws_d : w_d, 1, (uint64_t)a.d, (uint64_t)a.I, 128, BK))
        return cudaErrorInvalidValue;
    static bool flags[64] = {false};
    cudaError_t e = set_smem_once(k_down_mx, flags);
    if (e != cudaSuccess) return e;
    if (!a.counter_zeroed &&
        (e = cudaMemsetAsync(a.tile_counter, 0, sizeof(int32_t), s)) != cudaSuccess)
        return e;
    {
        const cudaError_t le = launch_pdl(k_down_mx, dim3(current_device_info().num_sms),
                                          dim3(THREADS), SMEM_BYTES, s, ta, tw, tws, a, hs, w_d_s,
                                          a.has_shared ? ws_d_s : w_d_s, o);
        if (le != cudaSuccess) return le;
    }
    return cudaGetLastError();
}

}  // namespace moe
