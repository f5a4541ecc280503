// ep.cu -- the data movement of expert parallelism on sm_100a: the rows a
// rank sends to the ranks that own their experts, and the expert outputs
// it sends back.
//
// Sources (page title -- section): "HPC-Ops - 騰訊混元開源的工業級高性能大模型推理算子庫",
// HPC-Ops的主要功能, "GroupGEMM FP8" (the grouped expert GEMM suits expert
// parallelism); "PR #54160 完整报告", 实现拆解 (multi-GPU deployment of the
// 256-expert layer).
//
// Experts are partitioned in contiguous ranges, rank r owning experts
// r*E_local .. (r+1)*E_local-1.  The permutation of the routing step already
// groups the flat assignments by expert, so in its row order the rows bound
// for each rank are contiguous and in rank order: the send buffer is the
// gathered x in that order, with each row's expert id local to its owner.
// Both kernels are row copies: one warp per row, 16-byte accesses, bound by
// HBM bandwidth.
#include "common.cuh"
#include "launch.h"

namespace moe {
namespace {

// send_rows[p] = x[perm[p] / k]; send_ids[p] = ids[perm[p]] % E_local.
__global__ void __launch_bounds__(256)
    k_ep_dispatch(const uint16_t* __restrict__ x, const int32_t* __restrict__ ids,
                  const int32_t* __restrict__ perm, int64_t n, int d, int k, int E_local,
                  uint16_t* __restrict__ send_rows, int32_t* __restrict__ send_ids) {
    pdl_wait();
    pdl_trigger();
    const int64_t p = (blockIdx.x * (int64_t)blockDim.x + threadIdx.x) >> 5;
    if (p >= n) return;
    const int lane = threadIdx.x & 31;
    const int32_t a = perm[p];
    const uint4* src = reinterpret_cast<const uint4*>(x + (int64_t)(a / k) * d);
    uint4* dst = reinterpret_cast<uint4*>(send_rows + p * d);
    for (int i = lane; i < d / 8; i += 32) dst[i] = src[i];
    if (lane == 0) send_ids[p] = ids[a] % E_local;
}

// dst[i] = src[index[i]], rows of `row_bytes` (a multiple of 16) bytes.
__global__ void __launch_bounds__(256)
    k_gather_rows(const uint8_t* __restrict__ src, const int32_t* __restrict__ index, int64_t n,
                  int row_bytes, uint8_t* __restrict__ dst) {
    pdl_wait();
    pdl_trigger();
    const int64_t i = (blockIdx.x * (int64_t)blockDim.x + threadIdx.x) >> 5;
    if (i >= n) return;
    const int lane = threadIdx.x & 31;
    const uint4* s = reinterpret_cast<const uint4*>(src + (int64_t)index[i] * row_bytes);
    uint4* o = reinterpret_cast<uint4*>(dst + i * row_bytes);
    for (int j = lane; j < row_bytes / 16; j += 32) o[j] = s[j];
}

}  // namespace

cudaError_t launch_ep_dispatch(const uint16_t* x, const int32_t* ids, const int32_t* perm,
                               int64_t n, int d, int k, int E_local, uint16_t* send_rows,
                               int32_t* send_ids, cudaStream_t s) {
    if (n == 0) return cudaSuccess;
    return launch_pdl(k_ep_dispatch, dim3((unsigned)((n + 7) / 8)), dim3(256), 0, s, x, ids, perm,
                      n, d, k, E_local, send_rows, send_ids);
}

cudaError_t launch_gather_rows(const void* src, const int32_t* index, int64_t n, int row_bytes,
                               void* dst, cudaStream_t s) {
    if (n == 0) return cudaSuccess;
    return launch_pdl(k_gather_rows, dim3((unsigned)((n + 7) / 8)), dim3(256), 0, s,
                      static_cast<const uint8_t*>(src), index, n, row_bytes,
                      static_cast<uint8_t*>(dst));
}

}  // namespace moe
