// gemm_fp8.cu -- grouped expert GEMMs with FP8 e4m3 operands: weights with
// one FP32 scale per 128x128 block, activations with one FP32 scale per row
// per 128 columns.
//
// "HPC-Ops - 騰訊混元開源的工業級高性能大模型推理算子庫", section HPC-Ops的主要功能,
// "GroupGEMM FP8" (grouped expert GEMM, block-wise FP8) and "FusedMoE"
// (activation quantisation between Gate-Up and Down); "PR #54160 完整报告",
// section 实现拆解 item 4 (FP8 block-wise 128x128 weight scales).
//
// Block scaling with arbitrary FP32 scales has no native tcgen05 form (the
// native block-scaled kinds take power-of-two or e4m3 scales per 16/32
// elements), so it is promoted in software:
//  - one k-block is 128 wide, exactly one scale block of both operands;
//  - one thread issues four kind::f8f6f4 MMAs (K = 32 each) that write a
//    fresh partial product of the k-block into one of two 256-column TMEM
//    buffers, so the next k-block's MMAs run while this one is promoted;
//  - sixteen epilogue warps (four per TMEM lane quadrant, each owning a
//    quarter of the columns, so four warps per scheduler hide the TMEM load
//    latency) read the partial with tcgen05.ld and accumulate
//    s_a[row] * s_w * P into 64 FP32 values per thread, held as 32 pairs for
//    the paired FMA (fma.rn.f32x2), which halves the promotion's FMA count;
//  - operands arrive by TMA into a 4-stage ring (128-byte swizzle).  The
//    gate-up A rows are the activation quantisation's output, already
//    written in permuted row order, so both operands are plain tiles;
//  - tiles come from the dynamic schedule of grouped_common.cuh, so the
//    m-tiles of one expert read its weight tile from DRAM once (with the
//    static round-robin order the FP8 gate-up read 1.4x its weight bytes);
//  - gate-up: a scale warp stages the tile's activation and weight scales in
//    shared memory, 16 k-blocks per chunk, double-buffered and issued as
//    cp.async copies, so the promotion never waits on a global load (a
//    per-k-block register prefetch left the epilogue warps stalled on those
//    loads a third of the time).  Down has one chunk per tile, where the
//    staging latency would fall on every tile start, so its epilogue keeps
//    the one-k-block-ahead register prefetch.
// Gate-up's tile is 128 rows x (128 gate + 128 up) columns: each row's 128
// h values form exactly one 1x128 quantisation group, so the epilogue
// computes h = silu(g) * u, the group's amax (combining the four column
// quarters through shared memory) and writes e4m3 h with its scale.  Down's
// tile is 128 rows x 256 output columns (two weight scale blocks) and writes
// o in FP16.  Every wait is bounded, as in the BF16 kernels.
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
constexpr uint32_t TMEM_COLS = 512;    // two 256-column partial buffers
constexpr int EPI_WARPS = 16, MMA_WARP = 16, TMA_WARP = 17, SCALE_WARP = 18;
constexpr int THREADS = 32 * (SCALE_WARP + 1);  // 608
// Scales are staged in chunks of SC_KB k-blocks: activation scales [k][row]
// with a padded row pitch (conflict-free reads by the 32 rows of a warp),
// then the chunk's scales of weight block 0 and weight block 1.
constexpr int SC_KB = 16, SA_PITCH = BM + 1;
constexpr int SC_FLOATS = SC_KB * SA_PITCH + 2 * SC_KB;  // one chunk buffer

struct Bars {
    uint64_t full[STAGES];   // TMA arrival + transaction bytes
    uint64_t empty[STAGES];  // MMA commit
    uint64_t pfull[2];       // partial ready (MMA commit)
    uint64_t pempty[2];      // partial consumed (one arrival per epilogue warp)
    uint64_t amax_bar[2];    // gate-up: the four quarters' amax written (one per warp)
    uint64_t sfull[2];       // scale chunk staged (scale warp)
    uint64_t sempty[2];      // scale chunk read (one arrival per epilogue warp)
    TileRing ring;           // tile numbers from the producer to the other roles
    uint32_t tmem_slot;
    int abort_flag;
    float amax[2][4][BM];    // [tile parity][column quarter][row]
};

constexpr size_t SMEM_BYTES = 1024 + STAGES * STAGE_BYTES + 2 * SC_FLOATS * sizeof(float) +
                              sizeof(Bars) + sizeof(TileTable) + 64;

struct Smem {
    uint8_t* stages;
    float* scales;  // two chunk buffers of SC_FLOATS
    Bars* bars;
    TileTable* tt;
};

__device__ __forceinline__ Smem carve(uint8_t* raw) {
    Smem s;
    s.stages = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(raw) + 1023) &
                                          ~static_cast<uintptr_t>(1023));
    s.scales = reinterpret_cast<float*>(s.stages + STAGES * STAGE_BYTES);
    s.bars = reinterpret_cast<Bars*>(s.scales + 2 * SC_FLOATS);
    s.tt = reinterpret_cast<TileTable*>(s.bars + 1);
    return s;
}

__device__ __forceinline__ void fail(Bars* b, int32_t* status) {
    report_status(status, MOE_ERR_DEVICE_TIMEOUT);
    *reinterpret_cast<volatile int*>(&b->abort_flag) = 1;
}

__device__ __forceinline__ uint32_t prologue(Smem& sm, const GroupedGemmArgs& a,
                                             uint32_t ring_consumers) {
    const int warp = threadIdx.x >> 5;
    Bars* b = sm.bars;
    if (threadIdx.x == 0) {
        for (int s = 0; s < STAGES; ++s) {
            mbar_init(&b->full[s], 1);
            mbar_init(&b->empty[s], 1);
        }
        for (int i = 0; i < 2; ++i) {
            mbar_init(&b->pfull[i], 1);
            mbar_init(&b->pempty[i], EPI_WARPS);
            mbar_init(&b->amax_bar[i], EPI_WARPS);
            mbar_init(&b->sfull[i], 1);
            mbar_init(&b->sempty[i], EPI_WARPS);
        }
        tile_ring_init(&b->ring, ring_consumers);
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

// TMA producer: A tile rows row0.. of `tm_a`, B rows rb0.. (and rb1.. when
// two halves) of `map`, k-block kb.
struct Loads {
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
        const Loads L = rows_of(t);
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

// MMA issuer: one fresh partial per k-block into TMEM buffer it % 2.
__device__ __forceinline__ void mma_role(Smem& sm, const GroupedGemmArgs& a, uint32_t tmem, int G,
                                         int n_tiles, int nk) {
    Bars* b = sm.bars;
    const volatile int* ab = &b->abort_flag;
    constexpr uint32_t idesc = idesc_e4m3(BM, BN);
    uint32_t it = 0;
    bool ok = true;
    for (uint32_t ti = 0; ok; ++ti) {
        if (tile_ring_pop(&b->ring, ti, a.timeout_ns, ab, ok) < 0) {
            if (!ok) fail(b, a.status);
            break;
        }
        for (int kb = 0; kb < nk; ++kb, ++it) {
            const int s = it % STAGES;
            const uint32_t ph = (it / STAGES) & 1;
            const uint32_t pb = it & 1, pph = (it >> 1) & 1;
            if (!mbar_wait(&b->full[s], ph, a.timeout_ns, ab) ||
                !mbar_wait(&b->pempty[pb], pph ^ 1, a.timeout_ns, ab)) {
                fail(b, a.status);
                ok = false;
                break;
            }
            tc_fence_after_sync();
            const uint32_t sa = smem_u32(sm.stages + s * STAGE_BYTES);
            const uint32_t sb = sa + A_BYTES;
#pragma unroll
            for (int kk = 0; kk < BK / 32; ++kk)
                umma_e4m3(tmem + pb * BN, sdesc_k_sw128(sa + kk * 32), sdesc_k_sw128(sb + kk * 32),
                          idesc, kk != 0);
            umma_commit(&b->empty[s]);
            umma_commit(&b->pfull[pb]);
        }
    }
}

// Scale warp: for every tile (from the ring), stages its scales chunk by
// chunk into the two chunk buffers, SC_KB k-blocks at a time.  The
// activation scales of rows row0 .. row0+127 are one contiguous run of
// 128 * nk floats in global memory (consecutive rows); each chunk reads
// 16-float row segments coalesced and writes them transposed.  Rows past the
// tile's valid rows get 0.  `weight_rows(t, w0, w1)` gives the nk scales of
// the tile's two weight blocks.
template <typename WeightRows>
__device__ __forceinline__ void scale_role(Smem& sm, const GroupedGemmArgs& a, int G, int n_tiles,
                                           int nk, const float* __restrict__ act_scale,
                                           WeightRows weight_rows) {
    Bars* b = sm.bars;
    const volatile int* ab = &b->abort_flag;
    const int lane = threadIdx.x & 31;
    uint32_t cc = 0;  // chunks staged so far
    bool ok = true;
    for (uint32_t lt = 0; ok; ++lt) {
        const int tile = tile_ring_pop_warp(&b->ring, lt, a.timeout_ns, ab, ok);
        if (tile < 0) break;
        const Tile t = decode_tile(sm.tt, G, n_tiles, tile, BM);
        const float* src = act_scale + (int64_t)t.row0 * nk;
        const float* w0;
        const float* w1;
        weight_rows(t, w0, w1);
        for (int k0 = 0; k0 < nk; k0 += SC_KB, ++cc) {
            const int buf = cc & 1;
            if (!warp_wait(&b->sempty[buf], ((cc >> 1) & 1) ^ 1, a.timeout_ns, ab)) {
                ok = false;
                break;
            }
            const int nkb = min(SC_KB, nk - k0);
            const uint32_t dst = smem_u32(sm.scales + buf * SC_FLOATS);
            // every copy of the chunk in flight at once (4-byte cp.async,
            // zero-filled past the valid rows), then one wait
            for (int idx = lane; idx < BM * SC_KB; idx += 32) {
                const int row = idx / SC_KB, kk = idx % SC_KB;
                if (kk < nkb) {
                    const bool in = row < t.nrows;
                    cp_async_4(dst + 4u * (kk * SA_PITCH + row),
                               src + (in ? (int64_t)row * nk + k0 + kk : 0), in ? 4u : 0u);
                }
            }
            if (lane < nkb) {
                cp_async_4(dst + 4u * (SC_KB * SA_PITCH + lane), w0 + k0 + lane, 4u);
                cp_async_4(dst + 4u * (SC_KB * SA_PITCH + SC_KB + lane), w1 + k0 + lane, 4u);
            }
            cp_async_commit();
            cp_async_wait<0>();
            __syncwarp();
            if (lane == 0) mbar_arrive(&b->sfull[buf]);
        }
    }
    if (!ok && lane == 0) fail(b, a.status);
}

// Epilogue side of the scale chunks: the scales of k-block kb (chunk cc
// counted over all of the CTA's tiles).  Waits for the chunk at its first
// k-block and releases it after its last.
struct ScaleReader {
    uint32_t cc = 0;
    const float* buf = nullptr;
    __device__ __forceinline__ bool fetch(Smem& sm, const GroupedGemmArgs& a, int kb, int nk,
                                          int row, float& sa, float& s0, float& s1) {
        Bars* b = sm.bars;
        const int kk = kb % SC_KB;
        if (kk == 0) {
            if (!warp_wait(&b->sfull[cc & 1], (cc >> 1) & 1, a.timeout_ns, &b->abort_flag))
                return false;
            buf = sm.scales + (cc & 1) * SC_FLOATS;
        }
        sa = buf[kk * SA_PITCH + row];
        s0 = buf[SC_KB * SA_PITCH + kk];
        s1 = buf[SC_KB * SA_PITCH + SC_KB + kk];
        if (kk == SC_KB - 1 || kb == nk - 1) {
            // the chunk's last k-block: its scales are in registers now
            __syncwarp();
            if ((threadIdx.x & 31) == 0) mbar_arrive(&b->sempty[cc & 1]);
            ++cc;
        }
        return true;
    }
};

__device__ __forceinline__ uint64_t f32x2_pack(float lo, float hi) {
    uint64_t r;
    asm("mov.b64 %0, {%1, %2};" : "=l"(r) : "f"(lo), "f"(hi));
    return r;
}
__device__ __forceinline__ void f32x2_unpack(uint64_t r, float& lo, float& hi) {
    asm("mov.b64 {%0, %1}, %2;" : "=f"(lo), "=f"(hi) : "l"(r));
}
__device__ __forceinline__ uint64_t f32x2_fma(uint64_t a, uint64_t b, uint64_t c) {
    uint64_t d;
    asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(d) : "l"(a), "l"(b), "l"(c));
    return d;
}
__device__ __forceinline__ void promote(uint32_t lane_base, int c0, int c1, float f0, float f1,
                                        uint64_t* acc) {
    const uint64_t ff0 = f32x2_pack(f0, f0), ff1 = f32x2_pack(f1, f1);
#pragma unroll
    for (int q = 0; q < 4; ++q) {
        float v[16];
        const int col = (q < 2 ? c0 : c1) + (q & 1) * 16;
        const uint64_t ff = q < 2 ? ff0 : ff1;
        tmem_load16(lane_base + col, v);
#pragma unroll
        for (int i = 0; i < 8; ++i)
            acc[q * 8 + i] = f32x2_fma(ff, f32x2_pack(v[2 * i], v[2 * i + 1]), acc[q * 8 + i]);
    }
}
__device__ __forceinline__ void unpack_acc(const uint64_t* acc2, float* acc) {
#pragma unroll
    for (int i = 0; i < 32; ++i) f32x2_unpack(acc2[i], acc[2 * i], acc[2 * i + 1]);
}

// All lanes of the warp are done with their part (TMEM loads waited for,
// shared-memory writes issued): one lane arrives for the warp.
__device__ __forceinline__ void warp_arrive(uint64_t* bar) {
    __syncwarp();
    if ((threadIdx.x & 31) == 0) mbar_arrive(bar);
}

__device__ __forceinline__ uint32_t quant4(float a, float b, float c, float d, float s) {
    const __nv_fp8x2_storage_t lo = __nv_cvt_float2_to_fp8x2(
        make_float2(__fdiv_rn(a, s), __fdiv_rn(b, s)), __NV_SATFINITE, __NV_E4M3);
    const __nv_fp8x2_storage_t hi = __nv_cvt_float2_to_fp8x2(
        make_float2(__fdiv_rn(c, s), __fdiv_rn(d, s)), __NV_SATFINITE, __NV_E4M3);
    return (uint32_t)lo | ((uint32_t)hi << 16);
}

// ---------------------------------------------------------------------------
// Gate-Up: h = silu(x Wg^T) * (x Wu^T) for 128 h columns per tile, quantised
// per row to e4m3 with one scale.
// ---------------------------------------------------------------------------
__global__ void __launch_bounds__(THREADS, 1)
    k_gateup_fp8(const __grid_constant__ CUtensorMap tm_a, const __grid_constant__ CUtensorMap tm_w,
                 const __grid_constant__ CUtensorMap tm_ws, GroupedGemmArgs a,
                 const float* __restrict__ xs, const float* __restrict__ wsc,
                 const float* __restrict__ wssc, uint8_t* __restrict__ hq, float* __restrict__ hs) {
    extern __shared__ uint8_t smem_raw[];
    Smem sm = carve(smem_raw);
    Bars* b = sm.bars;
    const volatile int* ab = &b->abort_flag;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    // ring consumers: the MMA thread, the epilogue warps, the scale warp
    const uint32_t tmem = prologue(sm, a, 1 + EPI_WARPS + 1);
    const int G = a.E + a.has_shared;
    const int n_tiles = a.I / 128;
    const int nk = a.d / BK;
    const int kbs = a.d / 128;         // scale blocks along K
    const int nbs = 2 * a.I / 128;     // scale blocks along the gate-up rows

    if (warp == TMA_WARP) {
        if (lane == 0) {
            tma_prefetch_desc(&tm_a);
            tma_prefetch_desc(&tm_w);
            tma_prefetch_desc(&tm_ws);
            tma_role(sm, a, &tm_a, G, n_tiles, nk, [&](const Tile& t) {
                const bool shared = t.g >= a.E;
                const int rbase = shared ? 0 : t.g * 2 * a.I;
                return Loads{shared ? &tm_ws : &tm_w, rbase + t.n * 128, rbase + a.I + t.n * 128, true};
            });
        }
    } else if (warp == MMA_WARP) {
        if (lane == 0) mma_role(sm, a, tmem, G, n_tiles, nk);
    } else if (warp == SCALE_WARP) {
        scale_role(sm, a, G, n_tiles, nk, xs, [&](const Tile& t, const float*& w0, const float*& w1) {
            const bool shared = t.g >= a.E;
            const float* base = shared ? wssc : wsc + (int64_t)t.g * nbs * kbs;
            w0 = base + (int64_t)t.n * kbs;
            w1 = base + (int64_t)(a.I / 128 + t.n) * kbs;
        });
    } else if (warp < EPI_WARPS) {
        // ---------------- 16 epilogue warps
        const int quad = warp & 3, qtr = warp >> 2;
        const int row = quad * 32 + lane;
        const uint32_t lane_off = static_cast<uint32_t>(quad * 32) << 16;
        uint32_t it = 0;
        ScaleReader sr;
        bool rok = true;
        for (uint32_t lt = 0;; ++lt) {
            const int tile = tile_ring_pop_warp(&b->ring, lt, a.timeout_ns, ab, rok);
            if (tile < 0) {
                if (!rok && lane == 0) fail(b, a.status);
                break;
            }
            const Tile t = decode_tile(sm.tt, G, n_tiles, tile, BM);
            const bool valid = row < t.nrows;
            uint64_t acc2[32];
#pragma unroll
            for (int i = 0; i < 32; ++i) acc2[i] = 0ull;
            bool ok = true;
            for (int kb = 0; kb < nk; ++kb, ++it) {
                const uint32_t pb = it & 1, pph = (it >> 1) & 1;
                float sa, sg, su;
                if (!sr.fetch(sm, a, kb, nk, row, sa, sg, su)) {
                    fail(b, a.status);
                    ok = false;
                    break;
                }
                const float fg = sa * sg, fu = sa * su;
                if (!warp_wait(&b->pfull[pb], pph, a.timeout_ns, ab)) {
                    fail(b, a.status);
                    ok = false;
                    break;
                }
                tc_fence_after_sync();
                const uint32_t base = tmem + lane_off + pb * BN;
                promote(base, qtr * 32, 128 + qtr * 32, fg, fu, acc2);
                tc_fence_before_sync();
                warp_arrive(&b->pempty[pb]);
            }
            if (!ok) break;
            float acc[64];
            unpack_acc(acc2, acc);
            float amax = 0.0f;
#pragma unroll
            for (int i = 0; i < 32; ++i) {
                acc[i] = silu_f(acc[i]) * acc[32 + i];
                amax = fmaxf(amax, fabsf(acc[i]));
            }
            // the four column quarters of a row meet in shared memory; the
            // exchange waits on an mbarrier (bounded), double-buffered by tile
            const int par = lt & 1;
            b->amax[par][qtr][row] = amax;
            warp_arrive(&b->amax_bar[par]);
            if (!warp_wait(&b->amax_bar[par], (lt >> 1) & 1, a.timeout_ns, ab)) {
                fail(b, a.status);
                break;
            }
            amax = fmaxf(fmaxf(b->amax[par][0][row], b->amax[par][1][row]),
                         fmaxf(b->amax[par][2][row], b->amax[par][3][row]));
            const float s = amax == 0.0f ? 1.0f : __fdiv_rn(amax, 448.0f);
            if (valid) {
                uint8_t* dst = hq + (int64_t)(t.row0 + row) * a.I + t.n * 128 + qtr * 32;
#pragma unroll
                for (int q = 0; q < 2; ++q)
                    st_global_v4(dst + q * 16, quant4(acc[16 * q], acc[16 * q + 1], acc[16 * q + 2], acc[16 * q + 3], s),
                                 quant4(acc[16 * q + 4], acc[16 * q + 5], acc[16 * q + 6], acc[16 * q + 7], s),
                                 quant4(acc[16 * q + 8], acc[16 * q + 9], acc[16 * q + 10], acc[16 * q + 11], s),
                                 quant4(acc[16 * q + 12], acc[16 * q + 13], acc[16 * q + 14], acc[16 * q + 15], s));
                if (qtr == 0) hs[(int64_t)(t.row0 + row) * (a.I / 128) + t.n] = s;
            }
        }
    }
    teardown(tmem);
}

// ---------------------------------------------------------------------------
// Down: o[p][n0 + j] = sum_kb s_h[p][kb] * s_w[n-block][kb] * (hq . Wq)_kb
// ---------------------------------------------------------------------------
__global__ void __launch_bounds__(THREADS, 1)
    k_down_fp8(const __grid_constant__ CUtensorMap tm_a, const __grid_constant__ CUtensorMap tm_w,
               const __grid_constant__ CUtensorMap tm_ws, GroupedGemmArgs a,
               const float* __restrict__ hs, const float* __restrict__ wsc,
               const float* __restrict__ wssc, __half* __restrict__ o) {
    extern __shared__ uint8_t smem_raw[];
    Smem sm = carve(smem_raw);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    Bars* b = sm.bars;
    const volatile int* ab = &b->abort_flag;
    // ring consumers: the MMA thread and the epilogue warps (the scale warp idles:
    // with one chunk per tile its staging latency would sit at every tile start)
    const uint32_t tmem = prologue(sm, a, 1 + EPI_WARPS);
    const int G = a.E + a.has_shared;
    const int n_tiles = (a.d + BN - 1) / BN;
    const int nk = a.I / BK;
    const int kbs = a.I / 128;   // scale blocks along K
    const int nbs = a.d / 128;   // scale blocks along the output rows of W_d

    if (warp == TMA_WARP) {
        if (lane == 0) {
            tma_prefetch_desc(&tm_a);
            tma_prefetch_desc(&tm_w);
            tma_prefetch_desc(&tm_ws);
            tma_role(sm, a, &tm_a, G, n_tiles, nk, [&](const Tile& t) {
                const bool shared = t.g >= a.E;
                const int r0 = (shared ? 0 : t.g * a.d) + t.n * BN;
                return Loads{shared ? &tm_ws : &tm_w, r0, r0 + 128, t.n * BN + 128 < a.d};
            });
        }
    } else if (warp == MMA_WARP) {
        if (lane == 0) mma_role(sm, a, tmem, G, n_tiles, nk);
    } else if (warp < EPI_WARPS) {
        const int quad = warp & 3, qtr = warp >> 2;
        const int row = quad * 32 + lane;
        const uint32_t lane_off = static_cast<uint32_t>(quad * 32) << 16;
        uint32_t it = 0;
        bool rok = true;
        for (uint32_t lt = 0;; ++lt) {
            const int tile = tile_ring_pop_warp(&b->ring, lt, a.timeout_ns, ab, rok);
            if (tile < 0) {
                if (!rok && lane == 0) fail(b, a.status);
                break;
            }
            const Tile t = decode_tile(sm.tt, G, n_tiles, tile, BM);
            const bool shared = t.g >= a.E;
            const int nb = 2 * t.n + (qtr >> 1);             // this quarter's weight scale block
            const bool live = nb < nbs;                       // inside d
            const float* sw = shared ? wssc + (int64_t)(live ? nb : 0) * kbs
                                     : wsc + ((int64_t)t.g * nbs + (live ? nb : 0)) * kbs;
            const bool valid = row < t.nrows;
            const float* sa_row = hs + (int64_t)(valid ? t.row0 + row : 0) * kbs;
            uint64_t acc2[32];
#pragma unroll
            for (int i = 0; i < 32; ++i) acc2[i] = 0ull;
            bool ok = true;
            const bool use = valid && live;
            // the next k-block's scale product loads while this one is promoted
            float f_n = use ? __ldg(sa_row) * __ldg(sw) : 0.0f;
            for (int kb = 0; kb < nk; ++kb, ++it) {
                const uint32_t pb = it & 1, pph = (it >> 1) & 1;
                const float f = f_n;
                if (kb + 1 < nk) f_n = use ? __ldg(sa_row + kb + 1) * __ldg(sw + kb + 1) : 0.0f;
                if (!warp_wait(&b->pfull[pb], pph, a.timeout_ns, ab)) {
                    fail(b, a.status);
                    ok = false;
                    break;
                }
                tc_fence_after_sync();
                const uint32_t base = tmem + lane_off + pb * BN;
                promote(base, qtr * 64, qtr * 64 + 32, f, f, acc2);
                tc_fence_before_sync();
                warp_arrive(&b->pempty[pb]);
            }
            if (!ok) break;
            if (valid && live) {
                float acc[64];
                unpack_acc(acc2, acc);
                __half* dst = o + (int64_t)(t.row0 + row) * a.d + t.n * BN + qtr * 64;
                st_f16x32(dst, acc);
                st_f16x32(dst + 32, acc + 32);
            }
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

}  // namespace

cudaError_t launch_gateup_fp8(const GroupedGemmArgs& a, const uint8_t* xq, const float* xs,
                              const uint8_t* w_gu, const float* w_gu_s, const uint8_t* ws_gu,
                              const float* ws_gu_s, uint8_t* hq, float* hs, cudaStream_t s) {
    if (a.T == 0) return cudaSuccess;
    const uint64_t R = (uint64_t)a.T * a.k + (a.has_shared ? a.T : 0);
    CUtensorMap ta, tw, tws;
    if (!make_tmap_2d(&ta, xq, 1, R, (uint64_t)a.d, BM, BK) ||
        !make_tmap_2d(&tw, w_gu, 1, (uint64_t)a.E * 2 * a.I, (uint64_t)a.d, 128, BK) ||
        !make_tmap_2d(&tws, a.has_shared ? ws_gu : w_gu, 1, (uint64_t)2 * a.I, (uint64_t)a.d, 128, BK))
        return cudaErrorInvalidValue;
    static bool flags[64] = {false};
    cudaError_t e = set_smem_once(k_gateup_fp8, flags);
    if (e != cudaSuccess) return e;
    if (!a.counter_zeroed &&
        (e = cudaMemsetAsync(a.tile_counter, 0, sizeof(int32_t), s)) != cudaSuccess)
        return e;
    {
        const cudaError_t le = launch_pdl(k_gateup_fp8, dim3(current_device_info().num_sms),
                                          dim3(THREADS), SMEM_BYTES, s, ta, tw, tws, a, xs, w_gu_s,
                                          a.has_shared ? ws_gu_s : w_gu_s, hq, hs);
        if (le != cudaSuccess) return le;
    }
    return cudaGetLastError();
}

cudaError_t launch_down_fp8(const GroupedGemmArgs& a, const uint8_t* hq, const float* hs,
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
    cudaError_t e = set_smem_once(k_down_fp8, flags);
    if (e != cudaSuccess) return e;
    if (!a.counter_zeroed &&
        (e = cudaMemsetAsync(a.tile_counter, 0, sizeof(int32_t), s)) != cudaSuccess)
        return e;
    {
        const cudaError_t le = launch_pdl(k_down_fp8, dim3(current_device_info().num_sms),
                                          dim3(THREADS), SMEM_BYTES, s, ta, tw, tws, a, hs, w_d_s,
                                          a.has_shared ? ws_d_s : w_d_s, o);
        if (le != cudaSuccess) return le;
    }
    return cudaGetLastError();
}

}  // namespace moe
