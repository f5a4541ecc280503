// launch.h -- host-side launchers of the MoE kernels (internal to the
// library; the public ABI is include/moe.h).  Every launcher enqueues on
// `stream` and returns the launch error, if any.
#pragma once

#include <cuda.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>
#include <stddef.h>
#include <stdint.h>

namespace moe {

struct DevInfo {
    int device;
    int num_sms;
    int cc_major, cc_minor;
};

// Cached per-device properties of the current device.
const DevInfo& current_device_info();

// Launches `kernel` with programmatic dependent launch allowed: it may be
// scheduled while the previous kernel in `s` finishes, and must call
// pdl_wait() before reading anything that kernel (or one before it) wrote.
// Captured into a CUDA graph, the dependency becomes a programmatic edge.
template <typename... Params, typename... Args>
inline cudaError_t launch_pdl(void (*kernel)(Params...), dim3 grid, dim3 block, size_t smem,
                              cudaStream_t s, Args... args) {
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = grid;
    cfg.blockDim = block;
    cfg.dynamicSmemBytes = smem;
    cfg.stream = s;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, kernel, static_cast<Params>(args)...);
}

// ---- routing.cu
cudaError_t launch_router_split(const float* W, uint16_t* hi, uint16_t* lo, int64_t n,
                                cudaStream_t s);
cudaError_t launch_route_topk(const float* logits, int T, int E, int k, int renorm, int32_t* ids,
                              float* w, cudaStream_t s);
// Top-k on router partial sums (split-K router): logits = sum_ks part_hi (pairwise)
// + sum_ks part_lo / 256 + bias, also written to `logits`.
cudaError_t launch_route_topk_partials(const float* part_hi, const float* part_lo, int ksplit,
                                       const float* bias, float* logits, int T, int E, int k,
                                       int renorm, int32_t* ids, float* w, cudaStream_t s);
// Scratch: seg_hist [nseg][E] int32, nseg = permute_segments(T*k).
int permute_segments(int64_t n_assign);
cudaError_t launch_permute(const int32_t* ids, int T, int E, int k, int32_t* counts,
                           int32_t* offsets, int32_t* perm, int32_t* inv, int32_t* seg_hist,
                           int32_t* status, cudaStream_t s);
// o [R][d] FP16: routed rows then (has_shared) the shared expert's rows
cudaError_t launch_combine(const __half* o, const int32_t* inv, const float* w, uint16_t* y, int T,
                           int d, int k, int has_shared, cudaStream_t s);
cudaError_t launch_quant_act_fp8(const uint16_t* x, int64_t rows, int cols, uint8_t* q,
                                 float* scale, cudaStream_t s);
cudaError_t launch_quant_act_fp8_permuted(const uint16_t* x, const int32_t* perm, int T, int k,
                                          int has_shared, int cols, uint8_t* q, float* scale,
                                          cudaStream_t s);
// The same outputs token-major: each token's row quantised once and stored to
// its rows inv[t*k + j] (and T*k + t with the shared expert).
cudaError_t launch_quant_act_fp8_scatter(const uint16_t* x, const int32_t* inv, int T, int k,
                                         int has_shared, int cols, uint8_t* q, float* scale,
                                         cudaStream_t s);
cudaError_t launch_quant_weights_fp8(const uint16_t* W, int64_t batch, int rows, int cols,
                                     uint8_t* q, float* scale, cudaStream_t s);
// MXFP8 (e4m3 + E8M0 scale per 1x32 along the row): rows as they are, or in
// the permuted row order of the grouped GEMMs; scales k-block-major
// [cols/128][rows][4].  Weights (rows % 128 == 0): scales in the per-matrix
// image of the block-scaled MMA's scale copy (see routing.cu).
cudaError_t launch_quant_mx_rows(const uint16_t* x, int64_t rows, int cols, uint8_t* q,
                                 uint8_t* scale, cudaStream_t s);
cudaError_t launch_quant_mx_weights(const uint16_t* W, int64_t batch, int rows, int cols,
                                    uint8_t* q, uint8_t* scale, cudaStream_t s);
cudaError_t launch_quant_mx_permuted(const uint16_t* x, const int32_t* perm, int T, int k,
                                     int has_shared, int cols, uint8_t* q, uint8_t* scale,
                                     cudaStream_t s);
cudaError_t launch_quant_mx_scatter(const uint16_t* x, const int32_t* inv, int T, int k,
                                    int has_shared, int cols, uint8_t* q, uint8_t* scale,
                                    cudaStream_t s);
// Per-tensor FP8: weights with one scale per matrix (scale [batch]);
// activations with a static scale, rows as they are (perm NULL) or in the
// permuted order of the grouped GEMMs (rows = T*k + shared T).
cudaError_t launch_quant_weights_fp8_tensor(const uint16_t* W, int64_t batch, int rows, int cols,
                                            uint8_t* q, float* scale, cudaStream_t s);
cudaError_t launch_quant_act_fp8_static(const uint16_t* x, const int32_t* perm, int T, int k,
                                        int64_t rows, int cols, float scale, uint8_t* q,
                                        cudaStream_t s);
// x [T][cols] bf16 copied to the permuted row order (rows inv[t*k + j], and
// T*k + t with the shared expert): xp [T*k (+T)][cols].
cudaError_t launch_permute_rows_bf16(const uint16_t* x, const int32_t* inv, int T, int k,
                                     int has_shared, int cols, uint16_t* xp, cudaStream_t s);
cudaError_t launch_quant_act_fp8_static_scatter(const uint16_t* x, const int32_t* inv, int T,
                                                int k, int has_shared, int cols, float scale,
                                                uint8_t* q, cudaStream_t s);
// Static FP8 scale of n bf16 values (n % 8 == 0, v 16-byte aligned): *scale =
// fp32(max |v|) / 448 (1 when every value is zero).
cudaError_t launch_amax_scale(const uint16_t* v, int64_t n, float* scale, cudaStream_t s);
cudaError_t launch_selftest_timeout(int32_t* status, uint64_t limit_ns, cudaStream_t s);

// ---- router.cu (tcgen05 dual-BF16 GEMM)
cudaError_t launch_router_logits(const uint16_t* x, const uint16_t* hi, const uint16_t* lo,
                                 const float* bias, float* logits, int T, int d, int E,
                                 int32_t* status, cudaStream_t s);

// Router logits with the top-k fused into the kernel (moe_forward, one CTA per
// tile, i.e. router_ksplit(T, d, E) == 1): ids [T][k], w [T][k] as
// launch_route_topk writes them.  `scratch`: router_topk_scratch_bytes(T, E)
// bytes (16-byte aligned) of candidate keys and arrival counters, the
// counters zeroed here before the launch.
size_t router_topk_scratch_bytes(int T, int E);
// Whether moe_forward fuses the top-k into a one-CTA-per-tile router: with one
// 64-expert tile per token (E <= 64).  With more, the epilogue's per-row
// selection and the cross-CTA merge cost more than the separate top-k kernel
// (measured on the 256-expert workloads); there the top-k runs on its own.
inline bool router_fuses_topk(int E) { return E <= 64; }
cudaError_t launch_router_topk(const uint16_t* x, const uint16_t* hi, const uint16_t* lo,
                               const float* bias, float* logits, int T, int d, int E, int k,
                               int renorm, int32_t* ids, float* w, void* scratch, int32_t* status,
                               cudaStream_t s);

// K split of the router GEMM for T tokens (1 = one CTA per tile covers all of d).
int router_ksplit(int T, int d, int E);
// Partial sums [ksplit][T][E] of the hi and lo products (no bias, no combination).
cudaError_t launch_router_partials(const uint16_t* x, const uint16_t* hi, const uint16_t* lo,
                                   float* part_hi, float* part_lo, int ksplit, int T, int d, int E,
                                   int32_t* status, cudaStream_t s);

// ---- gemm_bf16.cu (tcgen05 grouped GEMMs)
struct GroupedGemmArgs {
    int T, d, E, k, I, has_shared;
    const int32_t* offsets;  // [E+1]
    const int32_t* perm;     // [T*k]
    int32_t* status;
    int32_t* tile_counter;   // next tile number of the dynamic schedule
    uint64_t timeout_ns;
    int counter_zeroed;      // 1: the caller zeroed tile_counter earlier in the stream;
                             // 0: the launcher zeroes it before the launch
};
cudaError_t launch_gateup_bf16(const GroupedGemmArgs& a, const uint16_t* x, const uint16_t* w_gu,
                               const uint16_t* ws_gu, uint16_t* h, cudaStream_t s);
cudaError_t launch_down_bf16(const GroupedGemmArgs& a, const uint16_t* h, const uint16_t* w_d,
                             const uint16_t* ws_d, __half* o, cudaStream_t s);

// ---- gemm_bf16_wide.cu (gate-up with 256-row tiles: two accumulators share each weight stage)
cudaError_t launch_gateup_bf16_wide(const GroupedGemmArgs& a, const uint16_t* x,
                                    const uint16_t* w_gu, const uint16_t* ws_gu, uint16_t* h,
                                    cudaStream_t s);
// Whether the 256-row gate-up serves this shape (>= 256 rows per expert on average).
inline bool use_wide_gateup(int T, int E, int k) { return (int64_t)T * k >= (int64_t)256 * E; }

// ---- gemm_bf16_2sm.cu (down GEMM on CTA-pair tiles of 256 rows)
// Gate-up on CTA pairs (256-row tiles, both operands by TMA): the routed rows
// from xp [T*k][d], x's routed copies in the permuted row order
// (launch_permute_rows_bf16 without the shared rows), the shared expert's rows
// from x [T][d].
cudaError_t launch_gateup_bf16_2sm(const GroupedGemmArgs& a, const uint16_t* xp, const uint16_t* x,
                                   const uint16_t* w_gu, const uint16_t* ws_gu, uint16_t* h,
                                   cudaStream_t s);
cudaError_t launch_down_bf16_2sm(const GroupedGemmArgs& a, const uint16_t* h, const uint16_t* w_d,
                                 const uint16_t* ws_d, __half* o, cudaStream_t s);
// Whether the CTA-pair down kernel serves this shape (>= 256 rows per expert on average).
inline bool use_pair_tiles(int T, int E, int k) { return (int64_t)T * k >= (int64_t)256 * E; }
// Whether the forward copies x into the permuted row order and runs the gate-up
// on CTA pairs (the same shapes).
inline bool use_pair_gateup(int T, int E, int k) { return use_pair_tiles(T, E, k); }

// ---- gemm_fp8.cu (tcgen05 grouped GEMMs, e4m3 with 128x128 block scales)
cudaError_t launch_gateup_fp8(const GroupedGemmArgs& a, const uint8_t* xq, const float* xs,
                              const uint8_t* w_gu, const float* w_gu_s, const uint8_t* ws_gu,
                              const float* ws_gu_s, uint8_t* hq, float* hs, cudaStream_t s);
cudaError_t launch_down_fp8(const GroupedGemmArgs& a, const uint8_t* hq, const float* hs,
                            const uint8_t* w_d, const float* w_d_s, const uint8_t* ws_d,
                            const float* ws_d_s, __half* o, cudaStream_t s);

// ---- gemm_mx.cu (tcgen05 block-scaled grouped GEMMs, MXFP8: e4m3 + E8M0 per 1x32)
// Scales are bytes [rows][K/32]; h / o as in the FP8 path.
cudaError_t launch_gateup_mx(const GroupedGemmArgs& a, const uint8_t* xq, const uint8_t* xs,
                             const uint8_t* w_gu, const uint8_t* w_gu_s, const uint8_t* ws_gu,
                             const uint8_t* ws_gu_s, uint8_t* hq, uint8_t* hs, cudaStream_t s);
cudaError_t launch_down_mx(const GroupedGemmArgs& a, const uint8_t* hq, const uint8_t* hs,
                           const uint8_t* w_d, const uint8_t* w_d_s, const uint8_t* ws_d,
                           const uint8_t* ws_d_s, __half* o, cudaStream_t s);

// ---- gemm_f8t.cu (tcgen05 grouped GEMMs, per-tensor FP8, static activation scales)
cudaError_t launch_gateup_f8t(const GroupedGemmArgs& a, const uint8_t* xq, float sx, float sh,
                              const uint8_t* w_gu, const float* w_gu_s, const uint8_t* ws_gu,
                              const float* ws_gu_s, uint8_t* hq, cudaStream_t s);
cudaError_t launch_down_f8t(const GroupedGemmArgs& a, const uint8_t* hq, float sh,
                            const uint8_t* w_d, const float* w_d_s, const uint8_t* ws_d,
                            const float* ws_d_s, __half* o, cudaStream_t s);

// ---- ep.cu (expert parallelism: the rows sent to the experts' owners and back)
cudaError_t launch_ep_dispatch(const uint16_t* x, const int32_t* ids, const int32_t* perm,
                               int64_t n, int d, int k, int E_local, uint16_t* send_rows,
                               int32_t* send_ids, cudaStream_t s);
cudaError_t launch_gather_rows(const void* src, const int32_t* index, int64_t n, int row_bytes,
                               void* dst, cudaStream_t s);

// ---- allreduce_norm.cu (tensor-parallel all-reduce + residual + RMSNorm, Lamport P2P)
constexpr int kArMaxRanks = 8;
struct ArNormArgs {
    uint16_t* bufs[kArMaxRanks];             // every rank's Lamport buffer, by rank
    const uint16_t* x[kArMaxRanks];          // per rank of this launch (grid.y): its input
    const uint16_t* residual[kArMaxRanks];   // or nullptr
    uint16_t* out[kArMaxRanks];
    uint16_t* res_out[kArMaxRanks];          // or nullptr
    const uint16_t* gamma;
    int G, T, T_max, d, rank0;               // rank of grid.y == 0
    uint32_t call;
    float eps;
    int32_t* status;
    uint64_t timeout_ns;
};
size_t lamport_buffer_bytes(int G, int T_max, int d);
int allreduce_norm_max_d();
cudaError_t launch_lamport_init(void* buf, size_t bytes, cudaStream_t s);
// One rank (ranks_in_launch = 1, PDL launch) or every rank of an emulated
// group on one GPU (cooperative launch, grid.y = rank).
cudaError_t launch_allreduce_rmsnorm(const ArNormArgs& a, int ranks_in_launch, bool cooperative,
                                     cudaStream_t s);

// ---- tensor maps (api.cu)
// 2-D row-major tensor [rows][cols] of `elem_bytes`-sized elements, box
// [box_rows][box_cols], 128-byte swizzle, zero fill out of bounds.
bool make_tmap_2d(CUtensorMap* map, const void* base, int elem_bytes, uint64_t rows,
                  uint64_t cols, uint32_t box_rows, uint32_t box_cols);

}  // namespace moe
