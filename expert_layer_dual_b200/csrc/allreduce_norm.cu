// allreduce_norm.cu -- the tensor-parallel all-reduce of the G ranks' partial
// outputs fused with the residual add and RMSNorm, low-latency form:
//   s = sum_r x_r + residual;  residual_out = s;  out = s / sqrt(mean(s^2) + eps) * gamma.
//
// "HPC-Ops - 騰訊混元開源的工業級高性能大模型推理算子庫", section HPC-Ops的技術原理,
// "Fused AllReduce+Norm": RMSNorm(AllReduce(x) + residual, weight) as one
// NVLink operation; its low-latency (decode) version exchanges the data with
// Lamport-style P2P stores and overlaps with the previous kernel through
// programmatic dependent launch.  The high-throughput version of the page uses
// NVSwitch multicast; this file builds only the P2P one (no multicast).
//
// Protocol.  Every rank owns a Lamport buffer [3][G][T_max][d] bf16 that the
// other ranks can store into (peer memory: a CUDA IPC mapping); every element
// of it rests at the "empty" pattern 0x8000 (-0.0) between uses.  Call c uses
// slot c % 3.  Each block of rank r
//   1. stores its rows of x_r into slot c % 3, part r, of every rank's buffer
//      (its own included), with -0.0 sent as +0.0 so that a stored element
//      never looks empty -- the data is its own arrival flag;
//   2. for each of its rows, reads parts 0..G-1 of its own slot, polling each
//      16-byte vector until no element is empty (a bounded wait: after
//      timeout_ns the block records MOE_ERR_DEVICE_TIMEOUT and stops), sums
//      them in FP32 in rank order (so every rank computes the same bits), adds
//      the residual, writes residual_out and the normalised row;
//   3. stores the empty pattern back over what it consumed.  A rank writes
//      slot c % 3 again only at call c + 3, after it has received this rank's
//      data of calls c + 1 and c + 2, which this rank sends after this
//      kernel's stores are complete, so the reset never races a new store.
// Row t is handled by the block with the same index on every rank, and a block
// stores all its rows before it waits, so the wait of one block depends only on
// stores other ranks' same-index blocks make before their own waits; with the
// grid no larger than the GPU holds at once, no wait depends on a block that
// cannot run.  Emulation on one GPU: all G ranks' blocks in one cooperative
// launch (grid.y = rank), the peer buffers being local memory.
#include "common.cuh"
#include "launch.h"

namespace moe {
namespace {

constexpr uint16_t kEmpty = 0x8000;   // bf16 -0.0
constexpr int kThreads = 256;
constexpr int kMaxVec = 4;            // 16-byte vectors per thread and row: d <= 8192

__device__ __forceinline__ uint32_t positive_zero2(uint32_t v) {
    // an element -0.0 (0x8000) becomes +0.0; every other pattern is kept
    const uint32_t lo = (v & 0xffffu) == kEmpty ? 0u : (v & 0xffffu);
    const uint32_t hi = (v >> 16) == kEmpty ? 0u : (v >> 16);
    return lo | (hi << 16);
}

__device__ __forceinline__ bool has_empty2(uint32_t v) {
    return (v & 0xffffu) == kEmpty || (v >> 16) == kEmpty;
}

// Polling load: always fetches from memory (the value may be stored by another
// GPU or another block while this one waits).
__device__ __forceinline__ uint4 ld_poll(const uint4* p) {
    uint4 v;
    asm volatile("ld.volatile.global.v4.u32 {%0, %1, %2, %3}, [%4];"
                 : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
                 : "l"(p)
                 : "memory");
    return v;
}

__device__ __forceinline__ void st_vec(uint4* p, uint4 v) {
    asm volatile("st.volatile.global.v4.u32 [%0], {%1, %2, %3, %4};" ::"l"(p), "r"(v.x), "r"(v.y),
                 "r"(v.z), "r"(v.w)
                 : "memory");
}

__device__ __forceinline__ void add_bf16x8(float* acc, uint4 u) {
    const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        acc[2 * i] += __uint_as_float(w[i] << 16);
        acc[2 * i + 1] += __uint_as_float(w[i] & 0xffff0000u);
    }
}

__device__ __forceinline__ uint32_t pack_bf16x2(float a, float b) {
    const __nv_bfloat162 h = __floats2bfloat162_rn(a, b);
    return *reinterpret_cast<const uint32_t*>(&h);
}

__device__ __forceinline__ float block_sum(float v, float* red) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    __syncthreads();
    if (lane == 0) red[warp] = v;
    __syncthreads();
    float s = 0.0f;
#pragma unroll
    for (int w = 0; w < kThreads / 32; ++w) s += red[w];
    return s;
}

__global__ void __launch_bounds__(kThreads)
    k_allreduce_rmsnorm(const ArNormArgs a) {
    pdl_wait();  // x and the residual come from the previous kernels
    pdl_trigger();
    __shared__ float red[kThreads / 32];
    __shared__ volatile int stop;
    const int r = a.rank0 + blockIdx.y;                    // the rank this block works for
    const int G = a.G, d = a.d, nv = d / 8;
    const int64_t part = (int64_t)a.T_max * d;             // elements of one rank's part
    const int64_t slot_off = (int64_t)(a.call % 3) * G * part;
    const uint4* x = reinterpret_cast<const uint4*>(a.x[blockIdx.y]);
    if (threadIdx.x == 0) stop = 0;

    // 1. this rank's rows into every rank's buffer
    for (int t = blockIdx.x; t < a.T; t += gridDim.x) {
        for (int v = threadIdx.x; v < nv; v += kThreads) {
            uint4 u = x[(int64_t)t * nv + v];
            u.x = positive_zero2(u.x);
            u.y = positive_zero2(u.y);
            u.z = positive_zero2(u.z);
            u.w = positive_zero2(u.w);
            for (int p = 0; p < G; ++p) {
                uint4* dst = reinterpret_cast<uint4*>(a.bufs[p] + slot_off + r * part) +
                             (int64_t)t * nv + v;
                st_vec(dst, u);
            }
        }
    }

    // 2. sum the G parts of each row, residual, RMSNorm; 3. reset what was read
    uint4* mine = reinterpret_cast<uint4*>(a.bufs[r] + slot_off);
    const uint4* res = reinterpret_cast<const uint4*>(a.residual[blockIdx.y]);
    const uint16_t* gamma = a.gamma;
    const uint4 empty = make_uint4(0x80008000u, 0x80008000u, 0x80008000u, 0x80008000u);
    __syncthreads();
    for (int t = blockIdx.x; t < a.T; t += gridDim.x) {
        float acc[kMaxVec][8];
        float ss = 0.0f;
#pragma unroll
        for (int j = 0; j < kMaxVec; ++j) {
            const int v = threadIdx.x + j * kThreads;
#pragma unroll
            for (int e = 0; e < 8; ++e) acc[j][e] = 0.0f;
            if (v >= nv) continue;
            for (int p = 0; p < G; ++p) {
                const uint4* src = mine + p * (part / 8) + (int64_t)t * nv + v;
                uint4 u = ld_poll(src);
                if (has_empty2(u.x) || has_empty2(u.y) || has_empty2(u.z) || has_empty2(u.w)) {
                    const uint64_t t0 = global_timer_ns();
                    while (true) {
                        u = ld_poll(src);
                        if (!(has_empty2(u.x) || has_empty2(u.y) || has_empty2(u.z) ||
                              has_empty2(u.w)))
                            break;
                        if (stop || global_timer_ns() - t0 > a.timeout_ns) {
                            stop = 1;
                            break;
                        }
                    }
                }
                if (stop) break;
                add_bf16x8(acc[j], u);
            }
            if (stop) break;
            if (res != nullptr) add_bf16x8(acc[j], res[(int64_t)t * nv + v]);
#pragma unroll
            for (int e = 0; e < 8; ++e) ss += acc[j][e] * acc[j][e];
        }
        __syncthreads();
        if (stop) {
            if (threadIdx.x == 0) report_status(a.status, MOE_ERR_DEVICE_TIMEOUT);
            return;
        }
        const float inv = rsqrtf(block_sum(ss, red) / (float)d + a.eps);
        uint4* ro = reinterpret_cast<uint4*>(a.res_out[blockIdx.y]);
        uint4* out = reinterpret_cast<uint4*>(a.out[blockIdx.y]);
#pragma unroll
        for (int j = 0; j < kMaxVec; ++j) {
            const int v = threadIdx.x + j * kThreads;
            if (v >= nv) continue;
            const int64_t at = (int64_t)t * nv + v;
            if (ro != nullptr)
                ro[at] = make_uint4(pack_bf16x2(acc[j][0], acc[j][1]), pack_bf16x2(acc[j][2], acc[j][3]),
                                    pack_bf16x2(acc[j][4], acc[j][5]), pack_bf16x2(acc[j][6], acc[j][7]));
            const uint4 g = reinterpret_cast<const uint4*>(gamma)[v];
            const uint32_t gw[4] = {g.x, g.y, g.z, g.w};
            uint32_t o[4];
#pragma unroll
            for (int e = 0; e < 4; ++e)
                o[e] = pack_bf16x2(acc[j][2 * e] * inv * __uint_as_float(gw[e] << 16),
                                   acc[j][2 * e + 1] * inv * __uint_as_float(gw[e] & 0xffff0000u));
            out[at] = make_uint4(o[0], o[1], o[2], o[3]);
            for (int p = 0; p < G; ++p) st_vec(mine + p * (part / 8) + at, empty);
        }
    }
}

__global__ void k_fill_empty(uint4* buf, int64_t n16) {
    const uint4 empty = make_uint4(0x80008000u, 0x80008000u, 0x80008000u, 0x80008000u);
    for (int64_t i = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; i < n16;
         i += (int64_t)gridDim.x * blockDim.x)
        buf[i] = empty;
}

int max_resident_blocks() {
    static int per_sm[64] = {0};
    const DevInfo& di = current_device_info();
    const int dev = di.device < 64 ? di.device : 0;
    if (per_sm[dev] == 0) {
        int n = 0;
        if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&n, k_allreduce_rmsnorm, kThreads, 0) !=
                cudaSuccess ||
            n < 1)
            n = 1;
        per_sm[dev] = n;
    }
    return per_sm[dev] * di.num_sms;
}

}  // namespace

size_t lamport_buffer_bytes(int G, int T_max, int d) { return (size_t)3 * G * T_max * d * 2; }

cudaError_t launch_lamport_init(void* buf, size_t bytes, cudaStream_t s) {
    const int64_t n16 = (int64_t)(bytes / 16);
    if (n16 == 0) return cudaSuccess;
    k_fill_empty<<<(unsigned)(n16 < 148 * 64 ? (n16 + 255) / 256 : 148 * 16), 256, 0, s>>>(
        static_cast<uint4*>(buf), n16);
    return cudaGetLastError();
}

int allreduce_norm_max_d() { return kThreads * kMaxVec * 8; }

cudaError_t launch_allreduce_rmsnorm(const ArNormArgs& a, int ranks_in_launch, bool cooperative,
                                     cudaStream_t s) {
    if (a.T == 0 || ranks_in_launch == 0) return cudaSuccess;
    const int cap = max_resident_blocks() / ranks_in_launch;
    if (cap < 1) return cudaErrorCooperativeLaunchTooLarge;
    const int nb = a.T < cap ? a.T : cap;
    const dim3 grid(nb, ranks_in_launch);
    if (cooperative) {
        void* args[] = {const_cast<ArNormArgs*>(&a)};
        return cudaLaunchCooperativeKernel(reinterpret_cast<const void*>(k_allreduce_rmsnorm), grid,
                                           dim3(kThreads), args, 0, s);
    }
    return launch_pdl(k_allreduce_rmsnorm, grid, dim3(kThreads), 0, s, a);
}

}  // namespace moe
