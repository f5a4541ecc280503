// router.cu -- dual-BF16 router GEMM on the sm_100a tensor cores.
//
// "HPC-Ops - 騰訊混元開源的工業級高性能大模型推理算子庫", section HPC-Ops的技術原理,
// paragraph "Router GEMM 雙 BF16 模擬 FP32": the FP32 router weight is split
// offline into hi (BF16) and lo (BF16 residual, scale 1/256); at inference two
// BF16 tensor-core GEMMs run in ONE kernel, the BF16 activations are moved
// once, two accumulators hold the partial results and the epilogue applies a
// single FMA (acc_hi + acc_lo / 256) before writing.
//
// B200 form: one CTA per tile of 128 tokens x 64 experts, or x 128 experts
// for an unsplit router over more than 64 experts that needs more than one
// wave of 64-expert tiles (every tcgen05.mma costs at least ~120 cycles, so an
// N = 64 MMA wastes half of an N = 128 one).  Two TMA warps (one loads x and
// hi, the other lo: one thread completes a TMA load only about every 300
// cycles) stream each 64-wide k-block into a 4-stage shared-memory ring
// (128-byte swizzle); one thread issues two tcgen05.mma per 16-wide k-step,
// sharing the A descriptor, into TMEM accumulators; four epilogue warps read
// them with tcgen05.ld and write FP32 logits.  Every wait is bounded.
//
// Accuracy: the tensor core's FP32 accumulation loses a little at every MMA
// step, in proportion to the running sum, and over d = 4096 (256 steps) that
// alone reaches ~1e-5 of a logit.  The hi product therefore accumulates in
// C = min(4, k-blocks) separate TMEM accumulators (3 with 128-expert tiles,
// where C + 1 accumulators fill TMEM), one per contiguous part of the
// k-blocks, summed in FP32 by the epilogue ((c0 + c1) + (c2 + c3), or
// (c0 + c1) + c2) before the single correcting FMA; lo (already scaled down by
// 256) keeps one accumulator.  TMEM columns: hi chunk c at c*W .. c*W+W-1, lo
// at C*W .. C*W+W-1, W the tile's expert count.
//
// Top-k fused into the epilogue (moe_forward, one CTA per tile): the routing
// step needs all E logits of a token, which span E/64 CTAs.  Each CTA's
// epilogue thread keeps the best 8 of its row's 64 logits in registers as
// packed (logit, expert) keys and writes them out; the CTA that completes an
// m-tile last (an arrival counter per m-tile; writers fence before arriving,
// so no CTA ever waits on another) merges the E/64 lists of each of its 128
// tokens and writes ids and weights.  The merge picks exactly what a full
// sort of the FP32 logits picks (descending, ties to the lower expert id), and
// the weights use the same exponentials, summed in the same order, as
// moe_route_topk, so both give the same bits.  The split-K form below keeps
// the top-k in its own kernel: there no CTA holds a complete logit.
//
// Few tokens (decode): one 128-token tile row gives only E/64 CTAs, so the
// K dimension is also split across CTAs (grid z = ksplit); each CTA then
// writes its partial hi and lo sums, and the top-k kernel adds the ksplit
// partials in a fixed pairwise order before the correcting FMA.
#include "common.cuh"
#include "launch.h"

namespace moe {
namespace {

constexpr int BM = 128, BN = 64, BK = 64, STAGES = 4;
// Wide tiles (128 experts, three hi chunks) for the unsplit router with more
// than 64 experts: a tcgen05.mma with N <= 128 takes about as long as one with
// N = 128 (measured: ~120 cycles each for N = 16 .. 128 at M = 128), so the
// 64-expert tile spends half its MMA time on the fixed cost.  Three hi chunks
// and lo fill the 512 TMEM columns.
constexpr int BN_WIDE = 128, CHUNKS_WIDE = 3;
constexpr int A_BYTES = BM * BK * 2;
template <int TN>
constexpr int stage_bytes() { return A_BYTES + 2 * TN * BK * 2; }
template <int TN>
constexpr size_t smem_bytes() { return 1024 + STAGES * stage_bytes<TN>() + 256; }
constexpr int THREADS = 224;  // warps 0-3 epilogue, 4 MMA + TMEM owner, 5 and 6 TMA
constexpr int MAX_CHUNKS = 4;
constexpr uint32_t TMEM_COLS = 512;  // (chunks + 1) * tile width: 320 or 512 used

constexpr int CAND = 8;  // candidates kept per token and 64-expert tile (k <= 8)

// Fused top-k: outputs, per-token candidate keys [T][E/64][CAND] and one
// arrival counter per m-tile (zeroed by the launcher).
struct TopkArgs {
    int32_t* ids;              // [T][k]; nullptr: logits only (no fused top-k)
    float* w;                  // [T][k]
    unsigned long long* cand;  // [T][ntiles][CAND]
    int32_t* arrive_m;         // [m-tiles]: CTAs of the m-tile done
    int k, renorm;
};

// A logit and its expert id packed so that a larger key is a better choice:
// the high word orders like the FP32 value, the low word is ~e, so equal
// logits rank the lower id first.  Every real key is > 0; 0 marks "none".
__device__ __forceinline__ unsigned long long topk_key(float v, int e) {
    const uint32_t b = __float_as_uint(v);
    const uint32_t ord = (b & 0x80000000u) ? ~b : (b | 0x80000000u);
    return ((unsigned long long)ord << 32) | (uint32_t)~e;
}

__device__ __forceinline__ float key_value(unsigned long long key) {
    const uint32_t ord = (uint32_t)(key >> 32);
    return __uint_as_float((ord & 0x80000000u) ? (ord & 0x7fffffffu) : ~ord);
}

__device__ __forceinline__ int key_expert(unsigned long long key) { return (int)~(uint32_t)key; }

// The best CAND of N keys, in order (keys are distinct: each carries its
// expert id).  Each round takes the maximum by a tree of independent max
// operations and knocks the winner out, so the rounds are short dependency
// chains rather than one long insertion chain.
template <int N>
__device__ __forceinline__ void best_keys(unsigned long long (&k)[N], unsigned long long (&best)[CAND]) {
#pragma unroll
    for (int j = 0; j < CAND; ++j) {
        unsigned long long m[N];
#pragma unroll
        for (int i = 0; i < N; ++i) m[i] = k[i];
#pragma unroll
        for (int w = 1; w < N; w <<= 1)
#pragma unroll
            for (int i = 0; i + w < N; i += 2 * w) m[i] = m[i] > m[i + w] ? m[i] : m[i + w];
        best[j] = m[0];
#pragma unroll
        for (int i = 0; i < N; ++i) k[i] = k[i] == m[0] ? 0ull : k[i];
    }
}

// Token t's routing from its candidate keys (read through L2: other CTAs
// wrote them): the k best in order, then the weights.  Softmax over the
// selected k (renorm) or over all E logits of the token (read back from
// `logits`); the exponentials and the order of their sum are those of
// moe_route_topk's warp reduction, so the weights agree to the bit.
__device__ void merge_topk(const TopkArgs& tk, const float* logits, int64_t t, int ntiles, int E) {
    unsigned long long k[4 * CAND], best[CAND];
#pragma unroll
    for (int i = 0; i < 4 * CAND; ++i)
        k[i] = i < ntiles * CAND ? __ldcg(tk.cand + t * ntiles * CAND + i) : 0ull;
    best_keys<4 * CAND>(k, best);
    float sv[CAND];
#pragma unroll
    for (int j = 0; j < CAND; ++j) sv[j] = key_value(best[j]);
    const float lmax = sv[0];
    float sum;
    if (tk.renorm) {
        float p[CAND];
#pragma unroll
        for (int j = 0; j < CAND; ++j) p[j] = j < tk.k ? expf(sv[j] - lmax) : 0.0f;
        // the xor-butterfly of a warp over lanes 0..7 (lanes >= k hold 0)
        sum = ((p[0] + p[4]) + (p[2] + p[6])) + ((p[1] + p[5]) + (p[3] + p[7]));
    } else {
        // lane L sums experts L, L+32, ... in order; the lanes then add in
        // pairs (L, L+16), (L, L+8), ... as the xor-butterfly does
        float part[32];
        const float* row = logits + t * E;
#pragma unroll
        for (int L = 0; L < 32; ++L) {
            float acc = 0.0f;
#pragma unroll
            for (int i = 0; i < 8; ++i)
                if (L + 32 * i < E) acc += expf(__ldcg(row + L + 32 * i) - lmax);
            part[L] = acc;
        }
#pragma unroll
        for (int off = 16; off > 0; off >>= 1)
#pragma unroll
            for (int L = 0; L < off; ++L) part[L] = part[L] + part[L + off];
        sum = part[0];
    }
#pragma unroll
    for (int j = 0; j < CAND; ++j)
        if (j < tk.k) {
            tk.ids[t * tk.k + j] = key_expert(best[j]);
            tk.w[t * tk.k + j] = expf(sv[j] - lmax) / sum;
        }
}

template <int TN, int MAXC>
__global__ void __launch_bounds__(THREADS, 1)
    k_router_dual(const __grid_constant__ CUtensorMap tm_x, const __grid_constant__ CUtensorMap tm_hi,
                  const __grid_constant__ CUtensorMap tm_lo, const float* __restrict__ bias,
                  float* __restrict__ logits, float* __restrict__ part_hi,
                  float* __restrict__ part_lo, int T, int d, int E, int32_t* status,
                  uint64_t timeout_ns, const TopkArgs tk) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
    constexpr int SB = stage_bytes<TN>(), TB = TN * BK * 2;
    uint64_t* full = reinterpret_cast<uint64_t*>(smem + STAGES * SB);
    uint64_t* empty = full + STAGES;
    uint64_t* done = empty + STAGES;
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(done + 1);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    // grid x runs over the expert tiles, so the CTAs that share a 128-token x tile
    // are launched together and read it from DRAM once
    const int m0 = blockIdx.y * BM, e0 = blockIdx.x * TN;
    const int ksplit = gridDim.z, ks = blockIdx.z;
    const int nk_all = d / BK;
    const int kb0 = ks * nk_all / ksplit;                // this CTA's k-blocks: kb0 .. kb0+nk-1
    const int nk = (ks + 1) * nk_all / ksplit - kb0;
    const int nchunks = nk < MAXC ? nk : MAXC;

    if (threadIdx.x == 0) {
        for (int s = 0; s < STAGES; ++s) {
            mbar_init(&full[s], 2);  // one arrival per TMA producer
            mbar_init(&empty[s], 1);
        }
        mbar_init(done, 1);
        *abort_flag = 0;
        fence_barrier_init();
    }
    if (warp == 4) tmem_alloc(tmem_slot, TMEM_COLS);
    tc_fence_before_sync();
    __syncthreads();
    tc_fence_after_sync();
    const uint32_t tmem = *tmem_slot;
    pdl_wait();  // x may come from the previous kernel in the stream
    pdl_trigger();

    if ((warp == 5 || warp == 6) && lane == 0) {
        // ---------------- TMA producers: warp 5 loads x and hi, warp 6 lo, each arming
        // the stage's barrier for its own bytes before issuing them (one thread
        // completes a TMA load only every ~300 cycles, so a stage's three loads from
        // one thread would bound the k-loop)
        const bool second = warp == 6;
        tma_prefetch_desc(second ? &tm_lo : &tm_x);
        if (!second) tma_prefetch_desc(&tm_hi);
        int issued = 0;
        for (int kb = 0; kb < nk; ++kb) {
            const int s = kb % STAGES;
            const uint32_t ph = (kb / STAGES) & 1;
            if (!mbar_wait(&empty[s], ph ^ 1, timeout_ns, abort_flag)) {
                report_status(status, MOE_ERR_DEVICE_TIMEOUT);
                *abort_flag = 1;
                break;
            }
            uint8_t* st = smem + s * SB;
            if (!second) {
                mbar_arrive_expect_tx(&full[s], A_BYTES + TB);
                tma_load_2d(st, &tm_x, &full[s], (kb0 + kb) * BK, m0);
                tma_load_2d(st + A_BYTES, &tm_hi, &full[s], (kb0 + kb) * BK, e0);
            } else {
                mbar_arrive_expect_tx(&full[s], TB);
                tma_load_2d(st + A_BYTES + TB, &tm_lo, &full[s], (kb0 + kb) * BK, e0);
            }
            ++issued;
        }
        if (*abort_flag) {  // let the copies still in flight land before the block exits
            for (int it = (issued > STAGES ? issued - STAGES : 0); it < issued; ++it)
                mbar_wait(&full[it % STAGES], (it / STAGES) & 1, timeout_ns, nullptr);
        }
    } else if (warp == 4 && lane == 0) {
        // ---------------- MMA issuer
        constexpr uint32_t idesc = idesc_bf16(BM, TN);
        for (int kb = 0; kb < nk; ++kb) {
            const int s = kb % STAGES;
            const uint32_t ph = (kb / STAGES) & 1;
            if (!mbar_wait(&full[s], ph, timeout_ns, abort_flag)) {
                report_status(status, MOE_ERR_DEVICE_TIMEOUT);
                *abort_flag = 1;
                break;
            }
            tc_fence_after_sync();
            const uint32_t a = smem_u32(smem + s * SB);
            const uint32_t bh = a + A_BYTES, bl = a + A_BYTES + TB;
            const int chunk = kb * nchunks / nk;
            const bool chunk_start = kb * nchunks % nk < nchunks;  // first k-block of its chunk
            const uint32_t d_hi = tmem + chunk * TN, d_lo = tmem + nchunks * TN;
#pragma unroll
            for (int kk = 0; kk < BK / 16; ++kk) {
                const uint64_t ad = sdesc_k_sw128(a + kk * 32);
                umma_bf16(d_hi, ad, sdesc_k_sw128(bh + kk * 32), idesc, !(chunk_start && kk == 0));
                umma_bf16(d_lo, ad, sdesc_k_sw128(bl + kk * 32), idesc, (kb | kk) != 0);
            }
            umma_commit(&empty[s]);
        }
        umma_commit(done);  // also on abort: arrives once the issued MMAs are done
    } else if (warp < 4) {
        // ---------------- epilogue: logit = fma(acc_lo, 1/256, acc_hi) + bias
        const bool ok = mbar_wait(done, 0, timeout_ns, abort_flag);
        if (!ok) {
            report_status(status, MOE_ERR_DEVICE_TIMEOUT);
            *abort_flag = 1;
        }
        tc_fence_after_sync();
        if (ok && !*abort_flag) {
            const int row = warp * 32 + lane;
            const int t = m0 + row;
            const uint32_t lane_base = tmem + (static_cast<uint32_t>(warp * 32) << 16);
            const bool fuse = tk.ids != nullptr && ksplit == 1;
            unsigned long long best[CAND];
#pragma unroll
            for (int j = 0; j < CAND; ++j) best[j] = 0ull;
#pragma unroll 1
            for (int c = 0; c < TN / 32; ++c) {
                float h[32], l[32], h2[32], h3[32];
                tmem_load32x2(lane_base + c * 32, lane_base + nchunks * TN + c * 32, h, l);
                if (nchunks >= 2) {
                    tmem_load32(lane_base + TN + c * 32, h2);
#pragma unroll
                    for (int i = 0; i < 32; ++i) h[i] += h2[i];
                }
                if (nchunks >= 3) {
                    tmem_load32(lane_base + 2 * TN + c * 32, h2);
                    if (nchunks == 4) tmem_load32(lane_base + 3 * TN + c * 32, h3);
#pragma unroll
                    for (int i = 0; i < 32; ++i) h[i] += (nchunks == 4) ? (h2[i] + h3[i]) : h2[i];
                }
                if (t < T && ksplit == 1) {
                    float* dst = logits + (int64_t)t * E;
                    unsigned long long keys[CAND + 32];
#pragma unroll
                    for (int i = 0; i < 32; ++i) {
                        const int e = e0 + c * 32 + i;
                        keys[CAND + i] = 0ull;
                        if (e < E) {
                            float v = fmaf(l[i], 0.00390625f, h[i]);
                            if (bias != nullptr) v += bias[e];
                            dst[e] = v;
                            keys[CAND + i] = topk_key(v, e);
                        }
                    }
                    if (fuse) {   // the best CAND of this row's logits so far
#pragma unroll
                        for (int j = 0; j < CAND; ++j) keys[j] = best[j];
                        best_keys<CAND + 32>(keys, best);
                    }
                } else if (t < T) {
                    float* dh = part_hi + ((int64_t)ks * T + t) * E;
                    float* dl = part_lo + ((int64_t)ks * T + t) * E;
#pragma unroll
                    for (int i = 0; i < 32; ++i) {
                        const int e = e0 + c * 32 + i;
                        if (e < E) {
                            dh[e] = h[i];
                            dl[e] = l[i];
                        }
                    }
                }
            }
            if (fuse && t < T) {
                ulonglong2* dst = reinterpret_cast<ulonglong2*>(
                    tk.cand + ((int64_t)t * gridDim.x + blockIdx.x) * CAND);
#pragma unroll
                for (int j = 0; j < CAND / 2; ++j) dst[j] = make_ulonglong2(best[2 * j], best[2 * j + 1]);
            }
        }
    }
    tc_fence_before_sync();
    __syncthreads();
    if (warp == 4) {
        tc_fence_after_sync();
        tmem_dealloc(tmem, TMEM_COLS);
    }
    if (tk.ids == nullptr || ksplit > 1 || *abort_flag) return;

    // ---------------- fused top-k: the last CTA of each tile row routes its 128 tokens
    __shared__ int s_last;
    const int ntiles = gridDim.x;
    __threadfence();
    __syncthreads();
    if (threadIdx.x == 0) s_last = atomicAdd(&tk.arrive_m[blockIdx.y], 1) == ntiles - 1;
    __syncthreads();
    if (!s_last) return;
    __threadfence();
    if (threadIdx.x < BM && m0 + (int)threadIdx.x < T)
        merge_topk(tk, logits, m0 + threadIdx.x, ntiles, E);
}

template <int TN, int MAXC>
cudaError_t launch_router_tiles(const uint16_t* x, const uint16_t* hi, const uint16_t* lo,
                                const float* bias, float* logits, float* part_hi, float* part_lo,
                                int ksplit, int T, int d, int E, int32_t* status, const TopkArgs& tk,
                                cudaStream_t s) {
    CUtensorMap tx, th, tl;
    if (!make_tmap_2d(&tx, x, 2, (uint64_t)T, (uint64_t)d, BM, BK) ||
        !make_tmap_2d(&th, hi, 2, (uint64_t)E, (uint64_t)d, TN, BK) ||
        !make_tmap_2d(&tl, lo, 2, (uint64_t)E, (uint64_t)d, TN, BK))
        return cudaErrorInvalidValue;
    static bool attr_set[64] = {false};
    const int dev = current_device_info().device;
    if (dev < 64 && !attr_set[dev]) {
        cudaError_t e = cudaFuncSetAttribute(k_router_dual<TN, MAXC>,
                                             cudaFuncAttributeMaxDynamicSharedMemorySize,
                                             (int)smem_bytes<TN>());
        if (e != cudaSuccess) return e;
        attr_set[dev] = true;
    }
    dim3 grid((E + TN - 1) / TN, (T + BM - 1) / BM, ksplit);
    if (tk.ids != nullptr) {
        cudaError_t e = cudaMemsetAsync(tk.arrive_m, 0, sizeof(int32_t) * grid.y, s);
        if (e != cudaSuccess) return e;
    }
    {
        const cudaError_t le = launch_pdl(k_router_dual<TN, MAXC>, dim3(grid), dim3(THREADS),
                                          smem_bytes<TN>(), s, tx, th, tl, bias, logits, part_hi,
                                          part_lo, T, d, E, status, kDefaultTimeoutNs, tk);
        if (le != cudaSuccess) return le;
    }
    return cudaGetLastError();
}

static cudaError_t launch_router_impl(const uint16_t* x, const uint16_t* hi, const uint16_t* lo,
                                      const float* bias, float* logits, float* part_hi,
                                      float* part_lo, int ksplit, int T, int d, int E,
                                      int32_t* status, const TopkArgs& tk, cudaStream_t s) {
    if (T == 0) return cudaSuccess;
    // the wide tile for an unsplit router over more than 64 experts without the
    // fused top-k (its merge assumes 64-expert tiles), when the 64-expert tiles
    // would take more than one wave of the GPU (fewer, wider CTAs lose below
    // that: 4096 tokens x 256 experts, 99.9 vs 94.7 us); the 64-expert tile otherwise
    const int narrow_ctas = ((T + BM - 1) / BM) * ((E + BN - 1) / BN);
    const bool wide = ksplit == 1 && E > BN && tk.ids == nullptr &&
                      narrow_ctas > current_device_info().num_sms;
    return wide ? launch_router_tiles<BN_WIDE, CHUNKS_WIDE>(x, hi, lo, bias, logits, part_hi, part_lo,
                                                            ksplit, T, d, E, status, tk, s)
                : launch_router_tiles<BN, MAX_CHUNKS>(x, hi, lo, bias, logits, part_hi, part_lo,
                                                      ksplit, T, d, E, status, tk, s);
}

}  // namespace

int router_ksplit(int T, int d, int E) {
    const int tiles = ((T + BM - 1) / BM) * ((E + BN - 1) / BN);
    const int nk = d / BK;
    int ks = 1;
    // split K while the grid fills less than half the SMs, keeping >= 4 k-blocks per CTA
    while (ks < 8 && tiles * ks * 2 <= 148 && nk / (ks * 2) >= 4) ks *= 2;
    return ks;
}

size_t router_topk_scratch_bytes(int T, int E) {
    const size_t mt = (size_t)(T + BM - 1) / BM, nt = (size_t)(E + BN - 1) / BN;
    return (size_t)T * nt * CAND * 8 + mt * 4;
}

cudaError_t launch_router_logits(const uint16_t* x, const uint16_t* hi, const uint16_t* lo,
                                 const float* bias, float* logits, int T, int d, int E,
                                 int32_t* status, cudaStream_t s) {
    TopkArgs tk{};
    return launch_router_impl(x, hi, lo, bias, logits, nullptr, nullptr, 1, T, d, E, status, tk, s);
}

cudaError_t launch_router_partials(const uint16_t* x, const uint16_t* hi, const uint16_t* lo,
                                   float* part_hi, float* part_lo, int ksplit, int T, int d, int E,
                                   int32_t* status, cudaStream_t s) {
    TopkArgs tk{};
    return launch_router_impl(x, hi, lo, nullptr, nullptr, part_hi, part_lo, ksplit, T, d, E,
                              status, tk, s);
}

cudaError_t launch_router_topk(const uint16_t* x, const uint16_t* hi, const uint16_t* lo,
                               const float* bias, float* logits, int T, int d, int E, int k,
                               int renorm, int32_t* ids, float* w, void* scratch, int32_t* status,
                               cudaStream_t s) {
    const size_t nt = (size_t)(E + BN - 1) / BN;
    TopkArgs tk;
    tk.ids = ids;
    tk.w = w;
    tk.cand = static_cast<unsigned long long*>(scratch);
    tk.arrive_m = reinterpret_cast<int32_t*>(tk.cand + (size_t)T * nt * CAND);
    tk.k = k;
    tk.renorm = renorm;
    return launch_router_impl(x, hi, lo, bias, logits, nullptr, nullptr, 1, T, d, E, status, tk, s);
}

}  // namespace moe
