// noalloc.cu -- moe_permute_noalloc: the count / scan / permute stage for
// callers that cannot allocate device memory.
//
// moe_permute needs a small scratch area (one expert histogram per segment
// of 1024 assignments) that its caller passes in as a workspace.  Some
// callers cannot provide one: code that runs where cudaMalloc is not allowed
// or not wanted (inside a framework that owns every allocation, a
// pre-reserved real-time loop, a plugin with no allocator handle).  This
// variant keeps that scratch in a file-scope device array instead, so the
// caller passes only its inputs and outputs.
//
// The array is a fixed 256 KiB (kScratchInts int32) that every GPU which
// loads this library holds until the process exits.  It bounds the problem
// size: permute_segments(T*k) * E <= kScratchInts, i.e. T*k <= 262144
// assignments at E = 256; larger calls are rejected on the host.
#include <mutex>

#include "common.cuh"
#include "launch.h"

namespace {

constexpr int64_t kScratchInts = 64 * 1024;  // 256 KiB of per-segment histograms

static __device__ __align__(256) int32_t g_permute_scratch[kScratchInts];

// Device address of g_permute_scratch on the current device.  In host code
// the array's name is only a host-side stand-in, so the address is looked up
// once per device (with that device current) and cached.
int32_t* scratch_on_current_device() {
    static std::mutex mu;
    static int32_t* ptrs[64] = {nullptr};
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return nullptr;
    std::lock_guard<std::mutex> lock(mu);
    if (ptrs[dev] == nullptr) {
        void* p = nullptr;
        if (cudaGetSymbolAddress(&p, g_permute_scratch) != cudaSuccess) return nullptr;
        ptrs[dev] = static_cast<int32_t*>(p);
    }
    return ptrs[dev];
}

}  // namespace

extern "C" moe_status moe_permute_noalloc(const int32_t* ids, int32_t T, int32_t E, int32_t k,
                                          int32_t* counts, int32_t* offsets, int32_t* perm,
                                          int32_t* inv, void* stream) {
    if (T < 0 || E <= 0 || k <= 0) return MOE_ERR_INVALID_ARG;
    if (E > 256 || (int64_t)T * k >= ((int64_t)1 << 31)) return MOE_ERR_UNSUPPORTED;
    if (counts == nullptr || offsets == nullptr) return MOE_ERR_INVALID_ARG;
    if (T > 0 && (ids == nullptr || perm == nullptr || inv == nullptr)) return MOE_ERR_INVALID_ARG;
    if ((int64_t)moe::permute_segments((int64_t)T * k) * E > kScratchInts)
        return MOE_ERR_WORKSPACE_TOO_SMALL;
    const moe::DevInfo& d = moe::current_device_info();
    if (d.cc_major != 10 || d.num_sms <= 0) return MOE_ERR_UNSUPPORTED;
    int32_t* scratch = scratch_on_current_device();
    if (scratch == nullptr) return MOE_ERR_CUDA;
    // Every histogram entry a call reads is written first by that call, so
    // nothing left over from the previous call needs clearing.  No status
    // word: an id outside [0, E) is skipped without being reported.
    const cudaError_t e = moe::launch_permute(ids, T, E, k, counts, offsets, perm, inv, scratch,
                                              nullptr, static_cast<cudaStream_t>(stream));
    return e == cudaSuccess ? MOE_OK : MOE_ERR_CUDA;
}
