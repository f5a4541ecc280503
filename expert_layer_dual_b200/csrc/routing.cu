// routing.cu -- the non-GEMM stages of the MoE layer on sm_100a:
// router weight split, top-k routing, per-expert count / scan / permute,
// top-k weighted combine, FP8 quantisation of activations and weights.
// All of them are HBM- or latency-bound; they use coalesced 16-byte or
// warp-contiguous accesses and warp-level primitives, no tensor cores.
//
// Sources (page title -- section):
//  "HPC-Ops - 騰訊混元開源的工業級高性能大模型推理算子庫":
//    HPC-Ops的技術原理, "Router GEMM 雙 BF16 模擬 FP32" (the offline split);
//    HPC-Ops的技術原理, "FusedMoE 流水線重構" (shared-memory blocked per-expert
//      counting with one contiguous output interval per expert);
//    HPC-Ops的主要功能, "FusedMoE" (activation quantisation, Top-K weighted
//      aggregation) and "GroupGEMM FP8" (block-wise FP8).
//  "PR #54160 完整报告", 功能与动机 (top-8 of 256 experts + 1 shared expert);
//    实现拆解 item 4 (FP8 block-wise 128x128 scales).
#include "common.cuh"
#include "launch.h"

namespace moe {

// ---------------------------------------------------------------------------
// Router weight split: hi = RNE_bf16(W); lo = RNE_bf16((W - hi) * 256).
// W - hi is exact in FP32 and the scaling by 256 is exact, so both steps are
// a single rounding.
// ---------------------------------------------------------------------------
__global__ void k_router_split(const float* __restrict__ W, uint16_t* __restrict__ hi,
                               uint16_t* __restrict__ lo, int64_t n) {
    for (int64_t i = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; i < n;
         i += (int64_t)gridDim.x * blockDim.x) {
        const float w = W[i];
        const __nv_bfloat16 h = __float2bfloat16_rn(w);
        const float r = w - __bfloat162float(h);
        const __nv_bfloat16 l = __float2bfloat16_rn(r * 256.0f);
        hi[i] = __bfloat16_as_ushort(h);
        lo[i] = __bfloat16_as_ushort(l);
    }
}

cudaError_t launch_router_split(const float* W, uint16_t* hi, uint16_t* lo, int64_t n,
                                cudaStream_t s) {
    if (n == 0) return cudaSuccess;
    const int threads = 256;
    int64_t blocks = (n + threads - 1) / threads;
    const int cap = current_device_info().num_sms * 8;
    if (blocks > cap) blocks = cap;
    k_router_split<<<(unsigned)blocks, threads, 0, s>>>(W, hi, lo, n);
    return cudaGetLastError();
}

// ---------------------------------------------------------------------------
// Top-k routing: one warp selects for a token; lane l holds logits l, l+32,
// ... (E <= 256).  k rounds of a warp arg-max over (value desc, id asc) -- a
// total order, so every lane converges to the same winner -- select the
// experts in descending order with ties to the lower id.  Weights: softmax
// over the selected logits (or over all E when renorm == 0), in FP32.
// ---------------------------------------------------------------------------
constexpr int kTopkWarps = 8;

// Sum of the split-K router partials of one logit, in a fixed pairwise order.
__device__ __forceinline__ float sum_partials(const float* p, int64_t stride, int n) {
    if (n == 1) return p[0];
    if (n == 2) return p[0] + p[stride];
    if (n == 4) return (p[0] + p[stride]) + (p[2 * stride] + p[3 * stride]);
    return ((p[0] + p[stride]) + (p[2 * stride] + p[3 * stride])) +
           ((p[4 * stride] + p[5 * stride]) + (p[6 * stride] + p[7 * stride]));
}

// The warp's k selections from the logits v[i] of experts lane + 32 i (bits
// of `taken` mark absent experts), then the routing weights of token t.
__device__ __forceinline__ void select_topk(const float (&v)[8], uint32_t taken, int lane, int t,
                                            int E, int k, int renorm, int32_t* __restrict__ ids,
                                            float* __restrict__ w) {
    float my_v = 0.0f;
    int my_e = 0;
    for (int j = 0; j < k; ++j) {
        float bv = -INFINITY;
        int be = 0x7fffffff;
#pragma unroll
        for (int i = 0; i < 8; ++i) {
            if (!((taken >> i) & 1u)) {
                const int e = lane + 32 * i;
                if (be == 0x7fffffff || v[i] > bv) {  // ids ascend with i: first max wins ties
                    bv = v[i];
                    be = e;
                }
            }
        }
#pragma unroll
        for (int off = 16; off > 0; off >>= 1) {
            const float ov = __shfl_xor_sync(0xffffffffu, bv, off);
            const int oe = __shfl_xor_sync(0xffffffffu, be, off);
            const bool other_better = (oe != 0x7fffffff) &&
                                      (be == 0x7fffffff || ov > bv || (ov == bv && oe < be));
            if (other_better) {
                bv = ov;
                be = oe;
            }
        }
        if ((be & 31) == lane) taken |= 1u << (be >> 5);
        if (lane == j) {
            my_v = bv;
            my_e = be;
        }
    }
    const float lmax = __shfl_sync(0xffffffffu, my_v, 0);
    float part = 0.0f;
    if (renorm) {
        if (lane < k) part = expf(my_v - lmax);
    } else {
#pragma unroll
        for (int i = 0; i < 8; ++i)
            if (lane + 32 * i < E) part += expf(v[i] - lmax);
    }
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) part += __shfl_xor_sync(0xffffffffu, part, off);
    if (lane < k) {
        ids[(int64_t)t * k + lane] = my_e;
        w[(int64_t)t * k + lane] = expf(my_v - lmax) / part;
    }
}

// A warp per token: the logits in memory (one router pass), or the sums of
// the split-K router partials.
__global__ void __launch_bounds__(kTopkWarps * 32)
    k_route_topk(const float* __restrict__ logits_in, const float* __restrict__ part_hi,
                 const float* __restrict__ part_lo, int ksplit, const float* __restrict__ bias,
                 float* __restrict__ logits_out, int T, int E, int k, int renorm,
                 int32_t* __restrict__ ids, float* __restrict__ w) {
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int t = blockIdx.x * kTopkWarps + warp;
    if (t >= T) return;
    float v[8];
    uint32_t taken = 0;
    const int64_t pstride = (int64_t)T * E;
#pragma unroll
    for (int i = 0; i < 8; ++i) {
        const int e = lane + 32 * i;
        if (e < E) {
            if (part_hi != nullptr) {
                // split-K router: hi sums + lo sums / 256 (one FMA) + bias
                const int64_t off = (int64_t)t * E + e;
                float x = fmaf(sum_partials(part_lo + off, pstride, ksplit), 0.00390625f,
                               sum_partials(part_hi + off, pstride, ksplit));
                if (bias != nullptr) x += bias[e];
                logits_out[off] = x;
                v[i] = x;
            } else {
                v[i] = logits_in[(int64_t)t * E + e];
            }
        } else {
            v[i] = 0.0f;
            taken |= 1u << i;
        }
    }
    select_topk(v, taken, lane, t, E, k, renorm, ids, w);
}

// Split-K partials with few tokens: one block per token, one thread per
// expert, so each logit's partial loads are all in flight at once; the
// logits then go through shared memory to warp 0, which selects as above.
__global__ void __launch_bounds__(256)
    k_route_topk_sum(const float* __restrict__ part_hi, const float* __restrict__ part_lo,
                     int ksplit, const float* __restrict__ bias, float* __restrict__ logits_out,
                     int T, int E, int k, int renorm, int32_t* __restrict__ ids,
                     float* __restrict__ w) {
    __shared__ float lg[256];
    const int t = blockIdx.x, e = threadIdx.x;
    const int64_t pstride = (int64_t)T * E;
    if (e < E) {
        // hi sums + lo sums / 256 (one FMA) + bias
        const int64_t off = (int64_t)t * E + e;
        float x = fmaf(sum_partials(part_lo + off, pstride, ksplit), 0.00390625f,
                       sum_partials(part_hi + off, pstride, ksplit));
        if (bias != nullptr) x += bias[e];
        logits_out[off] = x;
        lg[e] = x;
    }
    __syncthreads();
    if (threadIdx.x >= 32) return;
    const int lane = threadIdx.x;
    float v[8];
    uint32_t taken = 0;
#pragma unroll
    for (int i = 0; i < 8; ++i) {
        const int ei = lane + 32 * i;
        if (ei < E) {
            v[i] = lg[ei];
        } else {
            v[i] = 0.0f;
            taken |= 1u << i;
        }
    }
    select_topk(v, taken, lane, t, E, k, renorm, ids, w);
}

cudaError_t launch_route_topk(const float* logits, int T, int E, int k, int renorm, int32_t* ids,
                              float* w, cudaStream_t s) {
    if (T == 0) return cudaSuccess;
    k_route_topk<<<(T + kTopkWarps - 1) / kTopkWarps, kTopkWarps * 32, 0, s>>>(
        logits, nullptr, nullptr, 1, nullptr, nullptr, T, E, k, renorm, ids, w);
    return cudaGetLastError();
}

cudaError_t launch_route_topk_partials(const float* part_hi, const float* part_lo, int ksplit,
                                       const float* bias, float* logits, int T, int E, int k,
                                       int renorm, int32_t* ids, float* w, cudaStream_t s) {
    if (T == 0) return cudaSuccess;
    // a block per token while a warp per token would leave most SMs idle
    if (T <= 512)
        k_route_topk_sum<<<T, 256, 0, s>>>(part_hi, part_lo, ksplit, bias, logits, T, E, k,
                                           renorm, ids, w);
    else
        k_route_topk<<<(T + kTopkWarps - 1) / kTopkWarps, kTopkWarps * 32, 0, s>>>(
            nullptr, part_hi, part_lo, ksplit, bias, logits, T, E, k, renorm, ids, w);
    return cudaGetLastError();
}

// ---------------------------------------------------------------------------
// Count / scan / permute.  The flat assignment list a = t*k + j is cut into
// segments of kSeg; (1) each block counts its segment's experts in a
// shared-memory histogram; (2) one block turns the per-segment counts into
// per-expert totals, the exclusive scan over experts (offsets) and, per
// segment, the first output row of each expert; (3) each segment is placed
// in order by one warp: __match_any_sync groups equal experts inside 32
// consecutive assignments, the rank inside the group keeps the order stable.
// No step depends on atomic ordering, so perm / inv are deterministic.  A
// single segment (at most kSeg assignments) runs all three in one block.
// ---------------------------------------------------------------------------
constexpr int kSeg = 1024;

int permute_segments(int64_t n) { return (int)((n + kSeg - 1) / kSeg); }

__global__ void __launch_bounds__(256)
    k_perm_count(const int32_t* __restrict__ ids, int64_t n, int E, int32_t* __restrict__ seg_hist,
                 int32_t* status) {
    pdl_wait();  // inputs come from the previous kernel of the forward
    pdl_trigger();
    __shared__ int32_t hist[256];
    for (int e = threadIdx.x; e < E; e += blockDim.x) hist[e] = 0;
    __syncthreads();
    const int64_t a0 = (int64_t)blockIdx.x * kSeg;
    const int64_t a1 = (a0 + kSeg < n) ? a0 + kSeg : n;
    for (int64_t a = a0 + threadIdx.x; a < a1; a += blockDim.x) {
        const int e = ids[a];
        if ((unsigned)e < (unsigned)E)
            atomicAdd(&hist[e], 1);
        else
            report_status(status, MOE_ERR_DEVICE_BAD_INDEX);
    }
    __syncthreads();
    for (int e = threadIdx.x; e < E; e += blockDim.x)
        seg_hist[(int64_t)blockIdx.x * E + e] = hist[e];
}

// One thread per expert walks the segments in order: seg_hist[s][e] becomes
// the number of expert-e assignments before segment s (loads issued 16 at a
// time, so the walk costs a few memory round trips, not one per segment);
// then the exclusive scan of the totals over the experts gives offsets.  The
// scatter adds offsets[e] to its segment's bases itself.
__global__ void __launch_bounds__(256)
    k_perm_scan(int32_t* __restrict__ seg_hist, int nseg, int E, int32_t* __restrict__ counts,
                int32_t* __restrict__ offsets) {
    pdl_wait();  // inputs come from the previous kernel of the forward
    pdl_trigger();
    __shared__ int32_t buf[2][256];
    const int e = threadIdx.x;
    int32_t run = 0;
    if (e < E) {
        for (int s0 = 0; s0 < nseg; s0 += 16) {
            int32_t c[16];
#pragma unroll
            for (int i = 0; i < 16; ++i)
                c[i] = s0 + i < nseg ? seg_hist[(int64_t)(s0 + i) * E + e] : 0;
#pragma unroll
            for (int i = 0; i < 16; ++i) {
                if (s0 + i < nseg) seg_hist[(int64_t)(s0 + i) * E + e] = run;
                run += c[i];
            }
        }
        counts[e] = run;
    }
    // inclusive Hillis-Steele scan of the totals over the 256 lanes
    int cur = 0;
    buf[0][e] = (e < E) ? run : 0;
    __syncthreads();
    for (int off = 1; off < 256; off <<= 1) {
        const int32_t x = buf[cur][e] + (e >= off ? buf[cur][e - off] : 0);
        buf[cur ^ 1][e] = x;
        cur ^= 1;
        __syncthreads();
    }
    const int32_t excl = buf[cur][e] - ((e < E) ? run : 0);
    if (e < E) {
        offsets[e] = excl;
        if (e == E - 1) offsets[E] = excl + run;
    }
}

__global__ void __launch_bounds__(32)
    k_perm_scatter(const int32_t* __restrict__ ids, int64_t n, int E,
                   const int32_t* __restrict__ seg_base, const int32_t* __restrict__ offsets,
                   int32_t* __restrict__ perm, int32_t* __restrict__ inv) {
    pdl_wait();  // inputs come from the previous kernel of the forward
    pdl_trigger();
    __shared__ int32_t cur[256];
    const int lane = threadIdx.x;
    for (int e = lane; e < E; e += 32) cur[e] = seg_base[(int64_t)blockIdx.x * E + e] + offsets[e];
    __syncwarp();
    const int64_t a0 = (int64_t)blockIdx.x * kSeg;
    const int64_t a1 = (a0 + kSeg < n) ? a0 + kSeg : n;
    for (int64_t base = a0; base < a1; base += 32) {
        const int64_t a = base + lane;
        const int e = (a < a1) ? ids[a] : -1;
        const bool ok = (unsigned)e < (unsigned)E;
        const unsigned peers = __match_any_sync(0xffffffffu, ok ? e : -1 - lane);
        int32_t start = 0;
        if (ok) {
            start = cur[e];
            const int32_t pos = start + __popc(peers & ((1u << lane) - 1u));
            perm[pos] = (int32_t)a;
            inv[a] = pos;
        }
        __syncwarp();
        if (ok && lane == __ffs(peers) - 1) cur[e] = start + __popc(peers);
        __syncwarp();
    }
}

// At most one segment (decode-sized batches): the three steps in one block --
// the segment's histogram, the scan over experts, then warp 0 places the
// assignments exactly as k_perm_scatter does, from the offsets.
__global__ void __launch_bounds__(256)
    k_perm_small(const int32_t* __restrict__ ids, int n, int E, int32_t* __restrict__ counts,
                 int32_t* __restrict__ offsets, int32_t* __restrict__ perm,
                 int32_t* __restrict__ inv, int32_t* status) {
    pdl_wait();  // inputs come from the previous kernel of the forward
    pdl_trigger();
    __shared__ int32_t hist[256];
    __shared__ int32_t buf[2][256];
    const int e = threadIdx.x;
    hist[e] = 0;
    __syncthreads();
    for (int a = threadIdx.x; a < n; a += blockDim.x) {
        const int ea = ids[a];
        if ((unsigned)ea < (unsigned)E)
            atomicAdd(&hist[ea], 1);
        else
            report_status(status, MOE_ERR_DEVICE_BAD_INDEX);
    }
    __syncthreads();
    const int32_t run = (e < E) ? hist[e] : 0;
    if (e < E) counts[e] = run;
    // inclusive Hillis-Steele scan of the totals over the 256 lanes
    int cur = 0;
    buf[0][e] = run;
    __syncthreads();
    for (int off = 1; off < 256; off <<= 1) {
        const int32_t x = buf[cur][e] + (e >= off ? buf[cur][e - off] : 0);
        buf[cur ^ 1][e] = x;
        cur ^= 1;
        __syncthreads();
    }
    const int32_t excl = buf[cur][e] - run;
    if (e < E) {
        offsets[e] = excl;
        if (e == E - 1) offsets[E] = excl + run;
    }
    hist[e] = excl;  // every thread read its count above, before the scan's barriers
    __syncthreads();
    if (threadIdx.x >= 32) return;
    const int lane = threadIdx.x;
    for (int base = 0; base < n; base += 32) {
        const int a = base + lane;
        const int ea = (a < n) ? ids[a] : -1;
        const bool ok = (unsigned)ea < (unsigned)E;
        const unsigned peers = __match_any_sync(0xffffffffu, ok ? ea : -1 - lane);
        int32_t start = 0;
        if (ok) {
            start = hist[ea];
            const int32_t pos = start + __popc(peers & ((1u << lane) - 1u));
            perm[pos] = a;
            inv[a] = pos;
        }
        __syncwarp();
        if (ok && lane == __ffs(peers) - 1) hist[ea] = start + __popc(peers);
        __syncwarp();
    }
}

cudaError_t launch_permute(const int32_t* ids, int T, int E, int k, int32_t* counts,
                           int32_t* offsets, int32_t* perm, int32_t* inv, int32_t* seg_hist,
                           int32_t* status, cudaStream_t s) {
    const int64_t n = (int64_t)T * k;
    const int nseg = permute_segments(n);
    if (nseg <= 1) {
        {
            const cudaError_t le = launch_pdl(k_perm_small, dim3(1), dim3(256), 0, s, ids, (int)n,
                                              E, counts, offsets, perm, inv, status);
            if (le != cudaSuccess) return le;
        }
        return cudaGetLastError();
    }
    {
        const cudaError_t le = launch_pdl(k_perm_count, dim3(nseg), dim3(256), 0, s, ids, n, E,
                                          seg_hist, status);
        if (le != cudaSuccess) return le;
    }
    {
        const cudaError_t le = launch_pdl(k_perm_scan, dim3(1), dim3(256), 0, s, seg_hist, nseg, E,
                                          counts, offsets);
        if (le != cudaSuccess) return le;
    }
    {
        const cudaError_t le = launch_pdl(k_perm_scatter, dim3(nseg), dim3(32), 0, s, ids, n, E,
                                          seg_hist, offsets, perm, inv);
        if (le != cudaSuccess) return le;
    }
    return cudaGetLastError();
}

// ---------------------------------------------------------------------------
// Combine: y[t] = sum_j w[t][j] * o[inv[t*k+j]] + o[T*k+t], FP16 rows from
// the down GEMM (widened exactly), FP32 sum in the order j = 0..k-1 then the
// shared row, one bf16 rounding.  One block per token, 16-byte loads along d.
// ---------------------------------------------------------------------------
__device__ __forceinline__ void bf16x8_to_f32(const uint4& u, float* f) {
    const uint32_t r[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        f[2 * i] = __uint_as_float(r[i] << 16);
        f[2 * i + 1] = __uint_as_float(r[i] & 0xffff0000u);
    }
}

// acc[i] += wj * row[i] for the 8 FP16 values of one 16-byte load u.
__device__ __forceinline__ void add8(float* acc, const uint4 u, float wj) {
    const uint32_t r[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        const float2 f = __half22float2(*reinterpret_cast<const __half2*>(&r[i]));
        acc[2 * i] = fmaf(wj, f.x, acc[2 * i]);
        acc[2 * i + 1] = fmaf(wj, f.y, acc[2 * i + 1]);
    }
}

__global__ void __launch_bounds__(128)
    k_combine(const __half* __restrict__ o, const int32_t* __restrict__ inv,
              const float* __restrict__ w, uint16_t* __restrict__ y, int T, int d, int k,
              int has_shared) {
    pdl_wait();  // inputs come from the previous kernel of the forward
    pdl_trigger();
    __shared__ int32_t rows[8];
    __shared__ float wts[8];
    const int t = blockIdx.x;
    if (threadIdx.x < k) {
        rows[threadIdx.x] = inv[(int64_t)t * k + threadIdx.x];
        wts[threadIdx.x] = w[(int64_t)t * k + threadIdx.x];
    }
    __syncthreads();
    const int64_t shared_row = (int64_t)T * k + t;
    // blockIdx.y splits the columns when there are few tokens
    for (int c = (blockIdx.y * blockDim.x + threadIdx.x) * 8; c < d; c += gridDim.y * blockDim.x * 8) {
        // all k (+1) rows' loads first, so they are in flight together
        uint4 u[9];
#pragma unroll
        for (int j = 0; j < 8; ++j)
            if (j < k) u[j] = __ldg(reinterpret_cast<const uint4*>(o + (int64_t)rows[j] * d + c));
        if (has_shared) u[8] = __ldg(reinterpret_cast<const uint4*>(o + shared_row * d + c));
        float acc[8];
#pragma unroll
        for (int i = 0; i < 8; ++i) acc[i] = 0.0f;
#pragma unroll
        for (int j = 0; j < 8; ++j)
            if (j < k) add8(acc, u[j], wts[j]);
        if (has_shared) {
            float sh[8];
#pragma unroll
            for (int i = 0; i < 8; ++i) sh[i] = 0.0f;
            add8(sh, u[8], 1.0f);
#pragma unroll
            for (int i = 0; i < 8; ++i) acc[i] += sh[i];
        }
        uint4 out;
        out.x = pack_bf16x2(acc[0], acc[1]);
        out.y = pack_bf16x2(acc[2], acc[3]);
        out.z = pack_bf16x2(acc[4], acc[5]);
        out.w = pack_bf16x2(acc[6], acc[7]);
        *reinterpret_cast<uint4*>(y + (int64_t)t * d + c) = out;
    }
}

cudaError_t launch_combine(const __half* o, const int32_t* inv, const float* w, uint16_t* y, int T,
                           int d, int k, int has_shared, cudaStream_t s) {
    if (T == 0) return cudaSuccess;
    // with few tokens, several blocks per token (each a share of the 1024-column
    // passes) so that about two blocks per SM have their loads in flight
    const int passes = (d + 1023) / 1024;
    const int want = (2 * current_device_info().num_sms + T - 1) / T;
    const int ysplit = want < passes ? want : passes;
    {
        const cudaError_t le = launch_pdl(k_combine, dim3(T, ysplit > 1 ? ysplit : 1), dim3(128), 0,
                                          s, o, inv, w, y, T, d, k, has_shared);
        if (le != cudaSuccess) return le;
    }
    return cudaGetLastError();
}

// ---------------------------------------------------------------------------
// FP8 e4m3 quantisation.  One group (1x128 of an activation row, or a 128x128
// weight block): s = fp32(amax) / 448 (amax == 0 -> 1); q = e4m3 of
// fp32(v / s), round to nearest even, saturating to +-448.  The divisions are
// IEEE round-to-nearest (__fdiv_rn), the conversion is the hardware
// cvt.rn.satfinite: the same decision the oracle takes in FP32.
// ---------------------------------------------------------------------------
__device__ __forceinline__ uint32_t quant4_e4m3(float a, float b, float c, float d, float s) {
    const __nv_fp8x2_storage_t lo = __nv_cvt_float2_to_fp8x2(
        make_float2(__fdiv_rn(a, s), __fdiv_rn(b, s)), __NV_SATFINITE, __NV_E4M3);
    const __nv_fp8x2_storage_t hi = __nv_cvt_float2_to_fp8x2(
        make_float2(__fdiv_rn(c, s), __fdiv_rn(d, s)), __NV_SATFINITE, __NV_E4M3);
    return (uint32_t)lo | ((uint32_t)hi << 16);
}

__device__ __forceinline__ float group_scale(float amax) {
    return amax == 0.0f ? 1.0f : __fdiv_rn(amax, 448.0f);
}

// The permuted rows that hold token t in the grouped GEMMs' row order: row
// inv[t*k + j] for each of its k assignments (j < k <= 8), and row T*k + t for
// the shared expert.  Every lane of the warp gets all of them (rows[j], j < k;
// rows[8] the shared row).  Used by the token-major quantisers below: a
// token's row is quantised once and its codes stored to each of these rows,
// instead of quantising each permuted row on its own.
struct TokenRows {
    int64_t row[9];
    int k;
    bool shared;
};

__device__ __forceinline__ TokenRows token_rows(const int32_t* __restrict__ inv, int64_t t, int T,
                                                int k, int has_shared) {
    const int lane = threadIdx.x & 31;
    const int32_t mine = lane < k ? inv[t * k + lane] : 0;
    TokenRows r;
#pragma unroll
    for (int j = 0; j < 8; ++j) r.row[j] = __shfl_sync(0xffffffffu, mine, j);
    r.row[8] = (int64_t)T * k + t;
    r.k = k;
    r.shared = has_shared != 0;
    return r;
}

// The token-major quantisers give each warp one chunk of kScatterCols columns
// of one token (more warps in flight than one per token; the chunk is a whole
// number of every format's 256-column step).
constexpr int kScatterCols = 1024;

__device__ __forceinline__ int scatter_chunks(int cols) {
    return (cols + kScatterCols - 1) / kScatterCols;
}

inline unsigned scatter_blocks(int T, int cols) {
    const int64_t warps = (int64_t)T * ((cols + kScatterCols - 1) / kScatterCols);
    return (unsigned)((warps + 7) / 8);
}

// f(row) for every row of the token, with indices known at compile time.
template <typename F>
__device__ __forceinline__ void for_token_rows(const TokenRows& r, F f) {
#pragma unroll
    for (int j = 0; j < 8; ++j)
        if (j < r.k) f(r.row[j]);
    if (r.shared) f(r.row[8]);
}

// One warp quantises one row: each step covers two 128-column groups, lanes
// 0-15 the first and 16-31 the second, 8 values (16 bytes) per lane; the
// group amax is a 16-lane shuffle reduction.
__device__ __forceinline__ void quant_row(const uint16_t* __restrict__ src, int cols,
                                          uint8_t* __restrict__ qrow, float* __restrict__ srow) {
    const int lane = threadIdx.x & 31;
    const int groups = cols / 128;
    const int half = lane >> 4, l16 = lane & 15;
    for (int g0 = 0; g0 < groups; g0 += 2) {
        const int g = g0 + half;
        const bool active = g < groups;
        uint4 u = make_uint4(0, 0, 0, 0);
        if (active) u = *reinterpret_cast<const uint4*>(src + g * 128 + l16 * 8);
        float f[8];
        bf16x8_to_f32(u, f);
        float amax = 0.0f;
#pragma unroll
        for (int i = 0; i < 8; ++i) amax = fmaxf(amax, fabsf(f[i]));
#pragma unroll
        for (int o = 8; o > 0; o >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, o));
        const float s = group_scale(amax);
        if (active) {
            uint2 q;
            q.x = quant4_e4m3(f[0], f[1], f[2], f[3], s);
            q.y = quant4_e4m3(f[4], f[5], f[6], f[7], s);
            *reinterpret_cast<uint2*>(qrow + g * 128 + l16 * 8) = q;
            if (l16 == 0) srow[g] = s;
        }
    }
}

__global__ void __launch_bounds__(256)
    k_quant_act(const uint16_t* __restrict__ x, int64_t rows, int cols, uint8_t* __restrict__ q,
                float* __restrict__ scale) {
    const int64_t r = (blockIdx.x * (int64_t)blockDim.x + threadIdx.x) >> 5;
    if (r >= rows) return;
    quant_row(x + r * cols, cols, q + r * cols, scale + r * (cols / 128));
}

// Same quantisation, written in the permuted row order of the grouped GEMMs:
// row p < T*k holds token perm[p] / k, row T*k + t holds token t.  The FP8
// gate-up GEMM then reads its A operand as plain TMA tiles; the gather
// rides on this pass, which has to read x anyway.
__global__ void __launch_bounds__(256)
    k_quant_act_permuted(const uint16_t* __restrict__ x, const int32_t* __restrict__ perm, int T,
                         int k, int64_t rows, int cols, uint8_t* __restrict__ q,
                         float* __restrict__ scale) {
    pdl_wait();  // inputs come from the previous kernel of the forward
    pdl_trigger();
    const int64_t p = (blockIdx.x * (int64_t)blockDim.x + threadIdx.x) >> 5;
    if (p >= rows) return;
    const int64_t Tk = (int64_t)T * k;
    const int64_t tok = p < Tk ? (int64_t)(perm[p] / k) : p - Tk;
    quant_row(x + tok * cols, cols, q + p * cols, scale + p * (cols / 128));
}

cudaError_t launch_quant_act_fp8_permuted(const uint16_t* x, const int32_t* perm, int T, int k,
                                          int has_shared, int cols, uint8_t* q, float* scale,
                                          cudaStream_t s) {
    const int64_t rows = (int64_t)T * k + (has_shared ? T : 0);
    if (rows == 0) return cudaSuccess;
    {
        const cudaError_t le = launch_pdl(k_quant_act_permuted, dim3((unsigned)((rows + 7) / 8)),
                                          dim3(256), 0, s, x, perm, T, k, rows, cols, q, scale);
        if (le != cudaSuccess) return le;
    }
    return cudaGetLastError();
}

// The same codes and scales as k_quant_act_permuted, token-major: one warp per
// token quantises its row once (the same quant_row arithmetic, so the same
// bits) and stores the codes and scales to each of its k (+1) permuted rows.
// The permuted kernel repeats the row's divisions for every copy; here each
// value is divided once and only the stores are repeated.
__global__ void __launch_bounds__(256)
    k_quant_act_scatter(const uint16_t* __restrict__ x, const int32_t* __restrict__ inv, int T,
                        int k, int has_shared, int cols, uint8_t* __restrict__ q,
                        float* __restrict__ scale) {
    pdl_wait();  // inputs come from the previous kernel of the forward
    pdl_trigger();
    const int64_t wid = (blockIdx.x * (int64_t)blockDim.x + threadIdx.x) >> 5;
    const int nch = scatter_chunks(cols);
    const int64_t t = wid / nch;
    if (t >= T) return;
    const int ch = (int)(wid - t * nch);
    const TokenRows tr = token_rows(inv, t, T, k, has_shared);
    const uint16_t* src = x + t * cols;
    const int lane = threadIdx.x & 31;
    const int groups = cols / 128;
    const int half = lane >> 4, l16 = lane & 15;
    const int g_end = min(groups, (ch + 1) * (kScatterCols / 128));
    for (int g0 = ch * (kScatterCols / 128); g0 < g_end; g0 += 2) {
        const int g = g0 + half;
        const bool active = g < g_end;
        uint4 u = make_uint4(0, 0, 0, 0);
        if (active) u = *reinterpret_cast<const uint4*>(src + g * 128 + l16 * 8);
        float f[8];
        bf16x8_to_f32(u, f);
        float amax = 0.0f;
#pragma unroll
        for (int i = 0; i < 8; ++i) amax = fmaxf(amax, fabsf(f[i]));
#pragma unroll
        for (int o = 8; o > 0; o >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, o));
        const float sc = group_scale(amax);
        if (active) {
            uint2 c;
            c.x = quant4_e4m3(f[0], f[1], f[2], f[3], sc);
            c.y = quant4_e4m3(f[4], f[5], f[6], f[7], sc);
            for_token_rows(tr, [&](int64_t p) {
                *reinterpret_cast<uint2*>(q + p * cols + g * 128 + l16 * 8) = c;
                if (l16 == 0) scale[p * groups + g] = sc;
            });
        }
    }
}

cudaError_t launch_quant_act_fp8_scatter(const uint16_t* x, const int32_t* inv, int T, int k,
                                         int has_shared, int cols, uint8_t* q, float* scale,
                                         cudaStream_t s) {
    if (T == 0) return cudaSuccess;
    {
        const cudaError_t le = launch_pdl(k_quant_act_scatter, dim3(scatter_blocks(T, cols)),
                                          dim3(256), 0, s, x, inv, T, k, has_shared, cols, q, scale);
        if (le != cudaSuccess) return le;
    }
    return cudaGetLastError();
}

cudaError_t launch_quant_act_fp8(const uint16_t* x, int64_t rows, int cols, uint8_t* q,
                                 float* scale, cudaStream_t s) {
    if (rows == 0) return cudaSuccess;
    k_quant_act<<<(unsigned)((rows + 7) / 8), 256, 0, s>>>(x, rows, cols, q, scale);
    return cudaGetLastError();
}

// ---------------------------------------------------------------------------
// MXFP8 quantisation (OCP microscaling): each block of 32 consecutive values
// along a row shares one E8M0 scale X = 2^(b - 127).  For the block's FP32
// amax, b = (exponent field of amax) - 8, i.e. shared_exp = floor(log2 amax)
// - 8 (8 = exponent of e4m3's largest normal), clamped to [0, 254] (0 for a
// zero or subnormal amax).  q = e4m3 cvt.rn.satfinite of v * 2^(127 - b): a
// power-of-two scaling, exact in FP32, so the decision is the oracle's.
// ---------------------------------------------------------------------------
// Where the scale byte of block j (32 columns) of row r goes.  Activations:
// k-block-major, [cols/128][rows][4] (byte j % 4 of row r's record for
// k-block j / 4), so the GEMM's gathers of one k-block's rows are contiguous.
// Weights: per matrix of `rows` rows, the image the block-scaled MMA's scale
// copy reads: for each k-block and 128-row block, 512 bytes where row r of
// the block is at (r % 32) * 16 + (r / 32) * 4 (+ j % 4).
struct MxScaleLayout {
    int64_t rows;  // rows of the k-block-major matrix, or of one weight matrix
    int cols;
    bool tiled;    // weights
    __device__ __forceinline__ int64_t at(int64_t r, int j) const {
        const int kb = j >> 2, kk = j & 3;
        if (!tiled) return ((int64_t)kb * rows + r) * 4 + kk;
        const int64_t m = r / rows, rl = r - m * rows;
        return m * rows * (cols / 32) + ((int64_t)kb * (rows / 128) + rl / 128) * 512 +
               (rl & 31) * 16 + ((rl & 127) >> 5) * 4 + kk;
    }
};

// One warp quantises one row: each step covers 256 columns (8 blocks), 8
// values (16 bytes) per lane; a block's amax is a 4-lane shuffle reduction.
__device__ __forceinline__ void mx_row(const uint16_t* __restrict__ src, int cols,
                                       uint8_t* __restrict__ qrow, uint8_t* __restrict__ scale,
                                       const MxScaleLayout& lay, int64_t r) {
    const int lane = threadIdx.x & 31;
    for (int c0 = 0; c0 < cols; c0 += 256) {
        const int c = c0 + lane * 8;
        const bool active = c < cols;
        uint4 u = make_uint4(0, 0, 0, 0);
        if (active) u = *reinterpret_cast<const uint4*>(src + c);
        float f[8];
        bf16x8_to_f32(u, f);
        float amax = 0.0f;
#pragma unroll
        for (int i = 0; i < 8; ++i) amax = fmaxf(amax, fabsf(f[i]));
        amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, 1));
        amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, 2));
        const uint32_t b = mx_scale_byte(amax);
        const float inv = __uint_as_float((254u - b) << 23);  // 2^(127 - b), b <= 253 here
        if (active) {
            uint2 q;
            q.x = mx_quant4(f, inv);
            q.y = mx_quant4(f + 4, inv);
            *reinterpret_cast<uint2*>(qrow + c) = q;
            if ((lane & 3) == 0) scale[lay.at(r, c / 32)] = static_cast<uint8_t>(b);
        }
    }
}

__global__ void __launch_bounds__(256)
    k_quant_mx_rows(const uint16_t* __restrict__ x, int64_t rows, int cols, uint8_t* __restrict__ q,
                    uint8_t* __restrict__ scale, MxScaleLayout lay) {
    const int64_t r = (blockIdx.x * (int64_t)blockDim.x + threadIdx.x) >> 5;
    if (r >= rows) return;
    mx_row(x + r * cols, cols, q + r * cols, scale, lay, r);
}

// Same, written in the permuted row order of the grouped GEMMs (row p < T*k
// holds token perm[p] / k, row T*k + t holds token t).
__global__ void __launch_bounds__(256)
    k_quant_mx_permuted(const uint16_t* __restrict__ x, const int32_t* __restrict__ perm, int T,
                        int k, int64_t rows, int cols, uint8_t* __restrict__ q,
                        uint8_t* __restrict__ scale) {
    pdl_wait();  // inputs come from the previous kernel of the forward
    pdl_trigger();
    const int64_t p = (blockIdx.x * (int64_t)blockDim.x + threadIdx.x) >> 5;
    if (p >= rows) return;
    const int64_t Tk = (int64_t)T * k;
    const int64_t tok = p < Tk ? (int64_t)(perm[p] / k) : p - Tk;
    mx_row(x + tok * cols, cols, q + p * cols, scale, MxScaleLayout{rows, cols, false}, p);
}

// The same codes and scale bytes as k_quant_mx_permuted, token-major (one warp
// per token, its row quantised once by mx_row's arithmetic, the results stored
// to each of its k (+1) permuted rows).  rows = T*k (+T): the scale layout's
// row count.
__global__ void __launch_bounds__(256)
    k_quant_mx_scatter(const uint16_t* __restrict__ x, const int32_t* __restrict__ inv, int T,
                       int k, int has_shared, int64_t rows, int cols, uint8_t* __restrict__ q,
                       uint8_t* __restrict__ scale) {
    pdl_wait();  // inputs come from the previous kernel of the forward
    pdl_trigger();
    const int64_t wid = (blockIdx.x * (int64_t)blockDim.x + threadIdx.x) >> 5;
    const int nch = scatter_chunks(cols);
    const int64_t t = wid / nch;
    if (t >= T) return;
    const int ch = (int)(wid - t * nch);
    const TokenRows tr = token_rows(inv, t, T, k, has_shared);
    const MxScaleLayout lay{rows, cols, false};
    const uint16_t* src = x + t * cols;
    const int lane = threadIdx.x & 31;
    const int c_end = min(cols, (ch + 1) * kScatterCols);
    for (int c0 = ch * kScatterCols; c0 < c_end; c0 += 256) {
        const int c = c0 + lane * 8;
        const bool active = c < c_end;
        uint4 u = make_uint4(0, 0, 0, 0);
        if (active) u = *reinterpret_cast<const uint4*>(src + c);
        float f[8];
        bf16x8_to_f32(u, f);
        float amax = 0.0f;
#pragma unroll
        for (int i = 0; i < 8; ++i) amax = fmaxf(amax, fabsf(f[i]));
        amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, 1));
        amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, 2));
        const uint32_t b = mx_scale_byte(amax);
        const float inv2 = __uint_as_float((254u - b) << 23);  // 2^(127 - b), b <= 253 here
        if (active) {
            uint2 cq;
            cq.x = mx_quant4(f, inv2);
            cq.y = mx_quant4(f + 4, inv2);
            for_token_rows(tr, [&](int64_t p) {
                *reinterpret_cast<uint2*>(q + p * cols + c) = cq;
                if ((lane & 3) == 0) scale[lay.at(p, c / 32)] = static_cast<uint8_t>(b);
            });
        }
    }
}

cudaError_t launch_quant_mx_scatter(const uint16_t* x, const int32_t* inv, int T, int k,
                                    int has_shared, int cols, uint8_t* q, uint8_t* scale,
                                    cudaStream_t s) {
    const int64_t rows = (int64_t)T * k + (has_shared ? T : 0);
    if (T == 0) return cudaSuccess;
    {
        const cudaError_t le = launch_pdl(k_quant_mx_scatter, dim3(scatter_blocks(T, cols)),
                                          dim3(256), 0, s, x, inv, T, k, has_shared, rows, cols, q,
                                          scale);
        if (le != cudaSuccess) return le;
    }
    return cudaGetLastError();
}

cudaError_t launch_quant_mx_rows(const uint16_t* x, int64_t rows, int cols, uint8_t* q,
                                 uint8_t* scale, cudaStream_t s) {
    if (rows == 0) return cudaSuccess;
    k_quant_mx_rows<<<(unsigned)((rows + 7) / 8), 256, 0, s>>>(x, rows, cols, q, scale,
                                                               MxScaleLayout{rows, cols, false});
    return cudaGetLastError();
}

cudaError_t launch_quant_mx_weights(const uint16_t* W, int64_t batch, int rows, int cols,
                                    uint8_t* q, uint8_t* scale, cudaStream_t s) {
    const int64_t n = batch * rows;
    if (n == 0) return cudaSuccess;
    k_quant_mx_rows<<<(unsigned)((n + 7) / 8), 256, 0, s>>>(W, n, cols, q, scale,
                                                            MxScaleLayout{rows, cols, true});
    return cudaGetLastError();
}

cudaError_t launch_quant_mx_permuted(const uint16_t* x, const int32_t* perm, int T, int k,
                                     int has_shared, int cols, uint8_t* q, uint8_t* scale,
                                     cudaStream_t s) {
    const int64_t rows = (int64_t)T * k + (has_shared ? T : 0);
    if (rows == 0) return cudaSuccess;
    {
        const cudaError_t le = launch_pdl(k_quant_mx_permuted, dim3((unsigned)((rows + 7) / 8)),
                                          dim3(256), 0, s, x, perm, T, k, rows, cols, q, scale);
        if (le != cudaSuccess) return le;
    }
    return cudaGetLastError();
}

// ---------------------------------------------------------------------------
// Per-tensor FP8.  Weights: one scale per matrix, s = fp32(amax) / 448
// (amax == 0 -> 1), q = e4m3(fp32(W / s)); computed in three stream-ordered
// passes -- the matrix amax (an atomicMax on the FP32 bits, which order like
// the values for non-negative floats) into `scale`, the codes, then `scale`
// rewritten from amax to s.  Activations: a static scale s given by the
// caller, q = e4m3(fp32(v / s)), saturating.
// ---------------------------------------------------------------------------
__global__ void __launch_bounds__(256)
    k_amax_matrices(const uint16_t* __restrict__ W, int64_t per, uint32_t* __restrict__ amax_bits) {
    const int64_t m = blockIdx.y;
    const uint16_t* src = W + m * per;
    float amax = 0.0f;
    for (int64_t i = ((int64_t)blockIdx.x * blockDim.x + threadIdx.x) * 8; i < per;
         i += (int64_t)gridDim.x * blockDim.x * 8) {
        float f[8];
        bf16x8_to_f32(*reinterpret_cast<const uint4*>(src + i), f);
#pragma unroll
        for (int j = 0; j < 8; ++j) amax = fmaxf(amax, fabsf(f[j]));
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, o));
    if ((threadIdx.x & 31) == 0) atomicMax(amax_bits + m, __float_as_uint(amax));
}

__global__ void __launch_bounds__(256)
    k_quant_matrices(const uint16_t* __restrict__ W, int64_t per, const uint32_t* __restrict__ amax_bits,
                     uint8_t* __restrict__ q) {
    const int64_t m = blockIdx.y;
    const float s = group_scale(__uint_as_float(amax_bits[m]));
    for (int64_t i = ((int64_t)blockIdx.x * blockDim.x + threadIdx.x) * 8; i < per;
         i += (int64_t)gridDim.x * blockDim.x * 8) {
        float f[8];
        bf16x8_to_f32(*reinterpret_cast<const uint4*>(W + m * per + i), f);
        uint2 o;
        o.x = quant4_e4m3(f[0], f[1], f[2], f[3], s);
        o.y = quant4_e4m3(f[4], f[5], f[6], f[7], s);
        *reinterpret_cast<uint2*>(q + m * per + i) = o;
    }
}

__global__ void k_scale_from_amax(float* __restrict__ scale, int64_t batch) {
    const int64_t m = blockIdx.x * (int64_t)blockDim.x + threadIdx.x;
    if (m < batch) scale[m] = group_scale(scale[m]);
}

// amax (as float bits) -> the static scale, for one value.
static cudaError_t launch_one_scale(float* scale, cudaStream_t s) {
    k_scale_from_amax<<<1, 32, 0, s>>>(scale, 1);
    return cudaGetLastError();
}

cudaError_t launch_quant_weights_fp8_tensor(const uint16_t* W, int64_t batch, int rows, int cols,
                                            uint8_t* q, float* scale, cudaStream_t s) {
    const int64_t per = (int64_t)rows * cols;
    if (batch == 0 || per == 0) return cudaSuccess;
    cudaError_t e = cudaMemsetAsync(scale, 0, sizeof(float) * (size_t)batch, s);
    if (e != cudaSuccess) return e;
    const int64_t want = (per / 8 + 255) / 256;
    const unsigned bx = (unsigned)(want < 1024 ? want : 1024);
    const dim3 grid(bx, (unsigned)batch);
    k_amax_matrices<<<grid, 256, 0, s>>>(W, per, reinterpret_cast<uint32_t*>(scale));
    k_quant_matrices<<<grid, 256, 0, s>>>(W, per, reinterpret_cast<const uint32_t*>(scale), q);
    k_scale_from_amax<<<(unsigned)((batch + 255) / 256), 256, 0, s>>>(scale, batch);
    return cudaGetLastError();
}

cudaError_t launch_amax_scale(const uint16_t* v, int64_t n, float* scale, cudaStream_t s) {
    cudaError_t e = cudaMemsetAsync(scale, 0, sizeof(float), s);
    if (e != cudaSuccess || n == 0) return e == cudaSuccess ? launch_one_scale(scale, s) : e;
    const int64_t want = (n / 8 + 255) / 256;
    const unsigned bx = (unsigned)(want < 1024 ? want : 1024);
    k_amax_matrices<<<dim3(bx, 1), 256, 0, s>>>(v, n, reinterpret_cast<uint32_t*>(scale));
    return launch_one_scale(scale, s);
}

// v / s rounded to nearest in FP32 -- the IEEE quotient -- for a divisor that
// is the same for many values: with r the correctly rounded reciprocal of s,
// the product v * r is corrected twice by its FMA residual (Markstein's
// method).  It is used where every intermediate stays normal and finite:
// 2^-100 <= |v| <= 2^100 and 2^-26 <= s <= 2^26, so the quotient lies within
// [2^-126, 2^126]; elsewhere (and for NaN) the IEEE division itself.
__device__ __forceinline__ float div_by_fixed(float v, float s, float r, bool s_in_range) {
    const float a = fabsf(v);
    if (!(s_in_range && a >= 0x1p-100f && a <= 0x1p100f)) return __fdiv_rn(v, s);
    float q = v * r;
    float e = fmaf(-q, s, v);
    q = fmaf(e, r, q);
    e = fmaf(-q, s, v);
    return fmaf(e, r, q);
}

__device__ __forceinline__ uint32_t quant4_e4m3_fixed(float a, float b, float c, float d, float s,
                                                      float r, bool s_in_range) {
    const __nv_fp8x2_storage_t lo = __nv_cvt_float2_to_fp8x2(
        make_float2(div_by_fixed(a, s, r, s_in_range), div_by_fixed(b, s, r, s_in_range)),
        __NV_SATFINITE, __NV_E4M3);
    const __nv_fp8x2_storage_t hi = __nv_cvt_float2_to_fp8x2(
        make_float2(div_by_fixed(c, s, r, s_in_range), div_by_fixed(d, s, r, s_in_range)),
        __NV_SATFINITE, __NV_E4M3);
    return (uint32_t)lo | ((uint32_t)hi << 16);
}

// One warp per row, 8 values (16 bytes in, 8 bytes out) per lane per step.
// The scale is the same for every value, so the division is done by its
// reciprocal with the exact correction of div_by_fixed.
__global__ void __launch_bounds__(256)
    k_quant_static(const uint16_t* __restrict__ x, const int32_t* __restrict__ perm, int T, int k,
                   int64_t rows, int cols, float s, uint8_t* __restrict__ q) {
    pdl_wait();  // inputs come from the previous kernel of the forward
    pdl_trigger();
    const int64_t p = (blockIdx.x * (int64_t)blockDim.x + threadIdx.x) >> 5;
    if (p >= rows) return;
    const int lane = threadIdx.x & 31;
    const int64_t Tk = (int64_t)T * k;
    const int64_t src_row = perm == nullptr ? p : (p < Tk ? (int64_t)(perm[p] / k) : p - Tk);
    const uint16_t* src = x + src_row * cols;
    uint8_t* dst = q + p * cols;
    const float r = __frcp_rn(s);
    const bool s_in_range = s >= 0x1p-26f && s <= 0x1p26f;
    for (int c = lane * 8; c < cols; c += 256) {
        float f[8];
        bf16x8_to_f32(*reinterpret_cast<const uint4*>(src + c), f);
        uint2 o;
        o.x = quant4_e4m3_fixed(f[0], f[1], f[2], f[3], s, r, s_in_range);
        o.y = quant4_e4m3_fixed(f[4], f[5], f[6], f[7], s, r, s_in_range);
        *reinterpret_cast<uint2*>(dst + c) = o;
    }
}

// The same codes as k_quant_static over permuted rows, token-major: one warp
// per token divides its row once and stores the codes to each of its k (+1)
// permuted rows.
__global__ void __launch_bounds__(256)
    k_quant_static_scatter(const uint16_t* __restrict__ x, const int32_t* __restrict__ inv, int T,
                           int k, int has_shared, int cols, float s, uint8_t* __restrict__ q) {
    pdl_wait();  // inputs come from the previous kernel of the forward
    pdl_trigger();
    const int64_t wid = (blockIdx.x * (int64_t)blockDim.x + threadIdx.x) >> 5;
    const int nch = scatter_chunks(cols);
    const int64_t t = wid / nch;
    if (t >= T) return;
    const int ch = (int)(wid - t * nch);
    const TokenRows tr = token_rows(inv, t, T, k, has_shared);
    const int lane = threadIdx.x & 31;
    const uint16_t* src = x + t * cols;
    const float r = __frcp_rn(s);
    const bool s_in_range = s >= 0x1p-26f && s <= 0x1p26f;
    const int c_end = min(cols, (ch + 1) * kScatterCols);
    for (int c = ch * kScatterCols + lane * 8; c < c_end; c += 256) {
        float f[8];
        bf16x8_to_f32(*reinterpret_cast<const uint4*>(src + c), f);
        uint2 o;
        o.x = quant4_e4m3_fixed(f[0], f[1], f[2], f[3], s, r, s_in_range);
        o.y = quant4_e4m3_fixed(f[4], f[5], f[6], f[7], s, r, s_in_range);
        for_token_rows(tr, [&](int64_t p) { *reinterpret_cast<uint2*>(q + p * cols + c) = o; });
    }
}

cudaError_t launch_quant_act_fp8_static_scatter(const uint16_t* x, const int32_t* inv, int T,
                                                int k, int has_shared, int cols, float scale,
                                                uint8_t* q, cudaStream_t s) {
    if (T == 0) return cudaSuccess;
    {
        const cudaError_t le = launch_pdl(k_quant_static_scatter, dim3(scatter_blocks(T, cols)),
                                          dim3(256), 0, s, x, inv, T, k, has_shared, cols, scale, q);
        if (le != cudaSuccess) return le;
    }
    return cudaGetLastError();
}

// x copied into the grouped GEMMs' permuted row order, token-major (bf16
// rows; the CTA-pair gate-up then loads its A rows as TMA tiles): a warp per
// 1024 columns of a token reads them once and stores them to each of the
// token's k (+1) permuted rows.  The forward copies the routed rows only
// (has_shared = 0): the pair gate-up reads the shared expert's rows from x.
__global__ void __launch_bounds__(256)
    k_permute_rows_scatter(const uint16_t* __restrict__ x, const int32_t* __restrict__ inv, int T,
                           int k, int has_shared, int cols, uint16_t* __restrict__ xp) {
    pdl_wait();  // inputs come from the previous kernel of the forward
    pdl_trigger();
    const int64_t wid = (blockIdx.x * (int64_t)blockDim.x + threadIdx.x) >> 5;
    const int nch = scatter_chunks(cols);
    const int64_t t = wid / nch;
    if (t >= T) return;
    const int ch = (int)(wid - t * nch);
    const TokenRows tr = token_rows(inv, t, T, k, has_shared);
    const int lane = threadIdx.x & 31;
    const uint16_t* src = x + t * cols;
    const int c_end = min(cols, (ch + 1) * kScatterCols);
    for (int c = ch * kScatterCols + lane * 8; c < c_end; c += 256) {
        const uint4 v = *reinterpret_cast<const uint4*>(src + c);
        for_token_rows(tr, [&](int64_t p) { *reinterpret_cast<uint4*>(xp + p * cols + c) = v; });
    }
}

cudaError_t launch_permute_rows_bf16(const uint16_t* x, const int32_t* inv, int T, int k,
                                     int has_shared, int cols, uint16_t* xp, cudaStream_t s) {
    if (T == 0) return cudaSuccess;
    {
        const cudaError_t le = launch_pdl(k_permute_rows_scatter, dim3(scatter_blocks(T, cols)),
                                          dim3(256), 0, s, x, inv, T, k, has_shared, cols, xp);
        if (le != cudaSuccess) return le;
    }
    return cudaGetLastError();
}

cudaError_t launch_quant_act_fp8_static(const uint16_t* x, const int32_t* perm, int T, int k,
                                        int64_t rows, int cols, float scale, uint8_t* q,
                                        cudaStream_t s) {
    if (rows == 0) return cudaSuccess;
    {
        const cudaError_t le = launch_pdl(k_quant_static, dim3((unsigned)((rows + 7) / 8)),
                                          dim3(256), 0, s, x, perm, T, k, rows, cols, scale, q);
        if (le != cudaSuccess) return le;
    }
    return cudaGetLastError();
}

// one block of 256 threads per 128x128 block; thread = half a row (64 values)
__global__ void __launch_bounds__(256)
    k_quant_w(const uint16_t* __restrict__ W, int rows, int cols, uint8_t* __restrict__ q,
              float* __restrict__ scale) {
    __shared__ float red[8];
    const int rb = rows / 128, cb = cols / 128;
    const int64_t blk = blockIdx.x;
    const int64_t b = blk / ((int64_t)rb * cb);
    const int r0 = (int)((blk / cb) % rb) * 128, c0 = (int)(blk % cb) * 128;
    const int rr = threadIdx.x >> 1, half = threadIdx.x & 1;
    const int64_t off = (b * rows + r0 + rr) * (int64_t)cols + c0 + half * 64;
    uint4 u[8];
#pragma unroll
    for (int i = 0; i < 8; ++i) u[i] = *reinterpret_cast<const uint4*>(W + off + i * 8);
    float amax = 0.0f;
#pragma unroll
    for (int i = 0; i < 8; ++i) {
        float f[8];
        bf16x8_to_f32(u[i], f);
#pragma unroll
        for (int j = 0; j < 8; ++j) amax = fmaxf(amax, fabsf(f[j]));
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, o));
    if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = amax;
    __syncthreads();
    amax = red[0];
#pragma unroll
    for (int i = 1; i < 8; ++i) amax = fmaxf(amax, red[i]);
    const float s = group_scale(amax);
#pragma unroll
    for (int i = 0; i < 8; i += 2) {
        float f[16];
        bf16x8_to_f32(u[i], f);
        bf16x8_to_f32(u[i + 1], f + 8);
        uint4 o;
        o.x = quant4_e4m3(f[0], f[1], f[2], f[3], s);
        o.y = quant4_e4m3(f[4], f[5], f[6], f[7], s);
        o.z = quant4_e4m3(f[8], f[9], f[10], f[11], s);
        o.w = quant4_e4m3(f[12], f[13], f[14], f[15], s);
        *reinterpret_cast<uint4*>(q + off + i * 8) = o;
    }
    if (threadIdx.x == 0) scale[blk] = s;
}

cudaError_t launch_quant_weights_fp8(const uint16_t* W, int64_t batch, int rows, int cols,
                                     uint8_t* q, float* scale, cudaStream_t s) {
    const int64_t blocks = batch * (rows / 128) * (cols / 128);
    if (blocks == 0) return cudaSuccess;
    k_quant_w<<<(unsigned)blocks, 256, 0, s>>>(W, rows, cols, q, scale);
    return cudaGetLastError();
}

// ---------------------------------------------------------------------------
// Failure-path check: one thread waits on a barrier that nothing arrives at,
// gives up after limit_ns and records the timeout.
// ---------------------------------------------------------------------------
__global__ void k_selftest_timeout(int32_t* status, uint64_t limit_ns) {
    __shared__ __align__(8) uint64_t bar;
    if (threadIdx.x == 0) {
        mbar_init(&bar, 1);
        fence_barrier_init();
    }
    __syncthreads();
    if (threadIdx.x == 0) {
        if (!mbar_wait(&bar, 0, limit_ns, nullptr)) report_status(status, MOE_ERR_DEVICE_TIMEOUT);
    }
}

cudaError_t launch_selftest_timeout(int32_t* status, uint64_t limit_ns, cudaStream_t s) {
    k_selftest_timeout<<<1, 32, 0, s>>>(status, limit_ns);
    return cudaGetLastError();
}

}  // namespace moe
