/* moe.h -- C ABI of the B200 (sm_100a) fused Mixture-of-Experts layer forward.
 *
 *   y = sum_{j<k} w[t][j] * E_{ids[t][j]}(x[t]) + S(x[t])
 *   E_e(x) = (silu(x Wg_e^T) * (x Wu_e^T)) Wd_e^T,  silu(z) = z / (1 + e^-z)
 *
 * Sources (page title -- section):
 *  [RG] "HPC-Ops - 騰訊混元開源的工業級高性能大模型推理算子庫", HPC-Ops的技術原理,
 *       "Router GEMM 雙 BF16 模擬 FP32": the FP32 router weight is split
 *       offline into a BF16 high part and a BF16 low residual with scale 1/256;
 *       inference runs both BF16 GEMMs in one kernel, the activations stay
 *       BF16 and are moved once, two accumulators, one FMA in the epilogue.
 *  [FM] same page, HPC-Ops的主要功能, "FusedMoE": routing index -> Gate-Up
 *       GEMM -> activation quantisation -> Down GEMM -> Top-K weighted
 *       aggregation.
 *  [FP] same page, HPC-Ops的技術原理, "FusedMoE 流水線重構": shared-memory
 *       blocked per-expert counting, one contiguous output interval per
 *       expert; Gate-Up reads the original input through the routing index.
 *  [G8] same page, HPC-Ops的主要功能, "GroupGEMM FP8": grouped expert GEMM with
 *       block-wise FP8 quantisation.
 *  [HY] "PR #54160 完整报告" ([Hy4] support Hy4-preview model), 功能与动机:
 *       256 routed experts, top-8, one shared expert; 实现拆解 item 4: FP8
 *       block-wise 128x128 weight scales.
 *
 * Conventions shared by every entry point
 *  - Pointers are DEVICE memory owned by the caller unless a comment says
 *    HOST.  The library never allocates, frees or synchronises, except where
 *    an entry point says so (moe_forward_host, moe_read_device_status).
 *  - Layouts are row-major and contiguous.  BF16 travels as uint16_t bits,
 *    FP8 e4m3 as uint8_t codes, scales as float.
 *  - `stream` is a cudaStream_t passed as void* (NULL = legacy default
 *    stream).  Work is enqueued asynchronously in stream order; nothing
 *    reads back counts, so a forward can be captured in a CUDA graph.
 *  - Row buffers (x, y, h, o, logits, FP8 codes q) and weight matrices
 *    (w_gu, w_d, ws_gu, ws_d, router_hi, router_lo, and the W of the weight
 *    quantisers) start on a 16-byte boundary: the kernels read them by TMA
 *    or with 16-byte vector accesses.  The workspace starts on a 256-byte
 *    boundary.
 *  - Arguments are validated on the host before any launch.  A failed check
 *    returns MOE_ERR_INVALID_ARG (null pointer, negative size, a pointer
 *    off the alignment above) or MOE_ERR_UNSUPPORTED (a shape outside the
 *    limits below, or no sm_100 device); nothing is launched then.  There is
 *    no fallback path.  T == 0 is a valid no-op.
 *  - Shape limits: d % 128 == 0, I % 128 == 0, I_shared in {0, I},
 *    1 <= E <= 256, 1 <= k <= min(E, 8), T*k + T < 2^31.
 *  - A launch failure returns MOE_ERR_CUDA.  Errors found on the device (an
 *    expert id out of range, a bounded wait that ran out) are written into a
 *    status word at the start of the workspace; moe_read_device_status()
 *    returns it.  Each entry point that takes a workspace clears that word
 *    first, so it reports the most recent such call.
 *  - Inputs must be finite; NaN logits give an unspecified but in-range
 *    routing.
 */
#ifndef MOE_B200_H
#define MOE_B200_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef int32_t moe_status;
#define MOE_OK 0
#define MOE_ERR_INVALID_ARG 1
#define MOE_ERR_UNSUPPORTED 2
#define MOE_ERR_CUDA 3
#define MOE_ERR_WORKSPACE_TOO_SMALL 4
#define MOE_ERR_DEVICE_TIMEOUT 5
#define MOE_ERR_DEVICE_BAD_INDEX 6

#define MOE_WDTYPE_BF16 0           /* expert weights bf16                         */
#define MOE_WDTYPE_FP8_BLOCK128 1   /* expert weights e4m3 + f32 scale per 128x128
                                       block; activations quantised per 1x128     */
#define MOE_WDTYPE_MXFP8 2          /* MXFP8: weights and activations e4m3 with one
                                       E8M0 (power-of-two) scale byte per 1x32
                                       block along K; native block-scaled MMA      */
#define MOE_WDTYPE_FP8_TENSOR 3     /* FP8 per tensor: e4m3 weights with one f32
                                       scale per matrix; activations e4m3 with
                                       static (calibrated) scales act_scale_x/h    */

/* Layer shape.  T tokens of hidden size d; E routed experts of intermediate
 * size I, top-k routing; I_shared = 0 (no shared expert) or I. */
typedef struct moe_shape {
    int32_t T, d, E, k, I, I_shared;
    int32_t wdtype;       /* MOE_WDTYPE_*                                     */
    int32_t renormalize;  /* 1: softmax over the selected k; 0: over all E    */
} moe_shape;

/* Layer weights (device).  Gate rows come first in every gate-up matrix.
 *   w_gu  [E][2I][d]   bf16 (wdtype 0) or e4m3 (wdtype 1, 2)
 *   w_d   [E][d][I]
 *   wdtype 1: w_gu_scale float [E][2I/128][d/128], w_d_scale float [E][d/128][I/128]
 *   wdtype 2: w_gu_scale, w_d_scale uint8 E8M0, one per 1x32 block along K, in
 *             the per-matrix image of moe_quantize_weights_mxfp8 (E matrices of
 *             2I x d, resp. d x I)
 *   wdtype 3: w_gu_scale, w_d_scale float [E] (one per matrix), ws_*_scale float
 *             [1]; act_scale_x, act_scale_h the static scales of x and of h
 *             (finite, > 0; q = e4m3_rne_satfinite(fp32(v / s)))
 *   ws_gu [2I][d], ws_d [d][I], ws_*_scale likewise  (when I_shared > 0)
 *   router_hi, router_lo [E][d] bf16 from moe_router_split; router_bias [E]
 *   or NULL (added to the logits, so it steers both selection and weights). */
typedef struct moe_weights {
    const void* w_gu;
    const void* w_d;
    const void* w_gu_scale;   /* float (wdtype 1) or uint8 E8M0 (wdtype 2) */
    const void* w_d_scale;
    const void* ws_gu;
    const void* ws_d;
    const void* ws_gu_scale;
    const void* ws_d_scale;
    const uint16_t* router_hi;
    const uint16_t* router_lo;
    const float* router_bias;
    float act_scale_x;        /* wdtype 3 only */
    float act_scale_h;        /* wdtype 3 only */
} moe_weights;

/* Human-readable name of a status code (static storage). */
const char* moe_status_string(moe_status s);

/* Workspace bytes that moe_forward / moe_forward_profiled / moe_forward_host
 * need for `shape` (0 on an invalid shape).  The workspace is
 * device memory, 256-byte aligned, owned by the caller, and may be reused
 * across calls that are ordered on one stream. */
size_t moe_workspace_bytes(const moe_shape* shape);

/* Where moe_forward (and moe_forward_profiled / moe_forward_host) leaves
 * the layer's intermediates in its workspace: byte offsets from the
 * workspace's start, each region 256-byte aligned.  After a forward on
 * `shape` returns and its stream has reached that point, until the
 * workspace is used again:
 *   logits float [T][E]   the router logits the routing was decided on
 *                         (bias included)
 *   ids int32 [T][k], w float [T][k]           moe_route_topk's outputs
 *   counts int32 [E], offsets int32 [E+1], perm, inv int32 [T*k]
 *                                              moe_permute's outputs
 *   xq, xs  the gate-up's A operand where the forward writes it in the permuted
 *           row order.  FP8 formats: the quantised activations, the outputs
 *           moe_quantize_act_fp8_permuted, moe_quantize_act_mxfp8_permuted or
 *           moe_quantize_act_fp8_static_permuted give for this routing's perm
 *           (xs: FP32 [R][d/128] for wdtype 1, the E8M0 bytes for wdtype 2,
 *           absent for wdtype 3).  wdtype 0 with T*k >= 256*E (the gate-up on
 *           CTA pairs): xq holds the bf16 routed rows of x [T*k][d] in that order
 *           (the shared expert's rows are read from x itself), no xs.
 *           0 where there is no such region
 *   h   the gate-up output (wdtype 0: bf16 [R][I], R = T*k + (I_shared ? T : 0))
 *   total  = moe_workspace_bytes(shape).
 * Inspection and testing aid; returns MOE_ERR_INVALID_ARG / UNSUPPORTED as
 * moe_workspace_bytes would return 0. */
typedef struct moe_workspace_map {
    size_t logits, ids, w, counts, offsets, perm, inv, xq, xs, h, total;
} moe_workspace_map;
moe_status moe_workspace_offsets(const moe_shape* shape, moe_workspace_map* map);

/* Workspace bytes moe_permute needs for T tokens, E experts, top-k. */
size_t moe_permute_workspace_bytes(int32_t T, int32_t E, int32_t k);

/* [RG] Offline split of n FP32 router weights: hi = RNE_bf16(W),
 * lo = RNE_bf16((W - hi) * 256); W ~= hi + lo / 256 within 2^-16 |W|. */
moe_status moe_router_split(const float* W, uint16_t* hi, uint16_t* lo, int64_t n,
                            void* stream);

/* [G8][HY] Offline FP8 quantisation of `batch` bf16 matrices [rows][cols]
 * (rows, cols multiples of 128): per 128x128 block s = fp32(amax)/448
 * (amax == 0 -> 1), q = e4m3_rne_satfinite(fp32(W / s)).
 * q [batch][rows][cols], scale [batch][rows/128][cols/128]. */
moe_status moe_quantize_weights_fp8(const uint16_t* W, int64_t batch, int32_t rows,
                                    int32_t cols, uint8_t* q, float* scale, void* stream);

/* [FM] Activation quantisation of a bf16 [rows][cols] matrix (cols % 128 ==
 * 0), per row per 1x128 group, same rule: q [rows][cols], scale
 * [rows][cols/128]. */
moe_status moe_quantize_act_fp8(const uint16_t* x, int64_t rows, int32_t cols,
                                uint8_t* q, float* scale, void* stream);

/* [MX] Offline MXFP8 quantisation ("PR #54160 完整报告", section 实现拆解 item 4:
 * the MXFP8 weight format; the format itself is OCP microscaling MXFP8 E4M3):
 * each row of `batch` bf16 matrices [rows][cols] (cols % 128 == 0; K = cols)
 * in blocks of 32: b = E8M0 byte of floor(log2 amax) - 8 (clamped to
 * [0, 254], 0 for an all-zero block), q = e4m3_rne_satfinite(W * 2^(127-b)).
 * rows % 128 == 0.  q [batch][rows][cols].  scale: batch*rows*cols/32 bytes in
 * the image the grouped GEMMs copy into TMEM: for matrix m, row r, block j
 * (K-block kb = j / 4 of 128 columns), at
 *   m*rows*cols/32 + (kb*(rows/128) + r/128)*512 + (r%32)*16 + ((r%128)/32)*4 + j%4
 * (each 512-byte piece is one k-block of 128 rows, fetched with one bulk copy). */
moe_status moe_quantize_weights_mxfp8(const uint16_t* W, int64_t batch, int32_t rows,
                                      int32_t cols, uint8_t* q, uint8_t* scale, void* stream);

/* [MX] The same quantisation of activation rows: x [rows][cols] bf16 ->
 * q [rows][cols] e4m3, scale E8M0 k-block-major [cols/128][rows][4] (byte j%4
 * of row r's record for K-block j/4), so a GEMM's gather of one k-block's
 * rows reads contiguous memory. */
moe_status moe_quantize_act_mxfp8(const uint16_t* x, int64_t rows, int32_t cols, uint8_t* q,
                                  uint8_t* scale, void* stream);

/* [MX] The same, in the permuted row order of the grouped GEMMs (as
 * moe_quantize_act_fp8_permuted): q [R][d], scale [d/128][R][4]. */
moe_status moe_quantize_act_mxfp8_permuted(const uint16_t* x, const int32_t* perm, int32_t T,
                                           int32_t k, int32_t with_shared, int32_t d,
                                           uint8_t* q, uint8_t* scale, void* stream);

/* [G8][HY] Offline per-tensor FP8 quantisation ("HPC-Ops ...", section
 * HPC-Ops的主要功能, GroupGEMM FP8: per-tensor FP8; "腾讯混元大模型：从多场景适配到
 * 高效部署的全栈技术解析", section 量化压缩技术实践 / FP8量化方案): each of `batch`
 * bf16 matrices [rows][cols] (cols % 8 == 0) gets one scale s = fp32(amax)/448
 * (amax == 0 -> 1), q = e4m3_rne_satfinite(fp32(W / s)).  q [batch][rows][cols],
 * scale float [batch] (also used as scratch while it runs). */
moe_status moe_quantize_weights_fp8_tensor(const uint16_t* W, int64_t batch, int32_t rows,
                                           int32_t cols, uint8_t* q, float* scale, void* stream);

/* [HY] Calibration of the static activation scales of a per-tensor FP8 layer
 * ("腾讯混元大模型：从多场景适配到高效部署的全栈技术解析", section 量化压缩技术实践 /
 * FP8量化方案: static FP8 scales precomputed from calibration data; the page
 * gives no recipe, so the plainest one is used).  On the shape->T tokens of
 * x [T][d] (bf16, 16-byte aligned), with the layer's BF16 weights (shape->wdtype
 * must be MOE_WDTYPE_BF16; `weights` the BF16 originals of the experts and the
 * router split), runs the router, top-k, permute and the BF16 gate-up, then
 * writes two device floats:
 *   scales[0] = fp32(max |x|) / 448,   scales[1] = fp32(max |h|) / 448
 * over every element of x and of the bf16 gate-up output h [R][I] (routed and
 * shared rows), divided in FP32 (IEEE), 1 where the maximum is 0.  These are
 * the act_scale_x and act_scale_h of moe_weights for wdtype 3.  ws:
 * moe_workspace_bytes(shape); T == 0 is MOE_ERR_INVALID_ARG (nothing to
 * calibrate on).  Asynchronous on `stream`. */
moe_status moe_calibrate_fp8_static(const moe_shape* shape, const moe_weights* weights,
                                    const uint16_t* x, float* scales, void* ws, size_t ws_bytes,
                                    void* stream);

/* [HY] Static activation quantisation with a calibrated scale (> 0):
 * q = e4m3_rne_satfinite(fp32(x / scale)); x [rows][cols] bf16, cols % 8 == 0. */
moe_status moe_quantize_act_fp8_static(const uint16_t* x, int64_t rows, int32_t cols, float scale,
                                       uint8_t* q, void* stream);

/* [HY] The same, in the permuted row order of the grouped GEMMs: q [R][d]. */
moe_status moe_quantize_act_fp8_static_permuted(const uint16_t* x, const int32_t* perm, int32_t T,
                                                int32_t k, int32_t with_shared, int32_t d,
                                                float scale, uint8_t* q, void* stream);

/* [FM] The same activation quantisation, written in the permuted row order
 * of the grouped GEMMs (the FP8 gate-up GEMM's A operand): row p < T*k holds
 * token perm[p] / k, rows T*k .. T*k+T-1 (with_shared != 0) hold tokens
 * 0 .. T-1.  x [T][d] bf16 -> q [R][d] e4m3, scale [R][d/128],
 * R = T*k + (with_shared ? T : 0). */
moe_status moe_quantize_act_fp8_permuted(const uint16_t* x, const int32_t* perm, int32_t T,
                                         int32_t k, int32_t with_shared, int32_t d, uint8_t* q,
                                         float* scale, void* stream);

/* [RG] Router logits on tensor cores:
 *   logits[t][e] = acc_hi + acc_lo / 256 (+ bias[e]),
 *   acc_* = sum_i x[t][i] * {hi,lo}[e][i] accumulated in FP32.
 * x [T][d] bf16, hi/lo [E][d] bf16, bias [E] or NULL, logits [T][E] f32. */
moe_status moe_router_logits(const uint16_t* x, const uint16_t* hi, const uint16_t* lo,
                             const float* bias, float* logits, int32_t T, int32_t d,
                             int32_t E, void* stream);

/* [FM][HY] Top-k routing of FP32 logits [T][E]: ids [T][k] in descending
 * logit order, ties to the lower expert id; w [T][k] = exp(l - l_max) /
 * sum over the selected k (renormalize = 1) or over all E (= 0). */
moe_status moe_route_topk(const float* logits, int32_t T, int32_t E, int32_t k,
                          int32_t renormalize, int32_t* ids, float* w, void* stream);

/* [FP] Per-expert counts [E], offsets [E+1] (exclusive scan, offsets[E] =
 * T*k), and the stable permutation of the flat assignments a = t*k + j:
 * rows of expert e are offsets[e] .. offsets[e+1]-1 in ascending a;
 * perm [T*k] maps row -> a, inv [T*k] maps a -> row.  Deterministic: the
 * result does not depend on scheduling.  An id outside [0, E) sets
 * MOE_ERR_DEVICE_BAD_INDEX in the workspace status word and is not placed.
 * ws: moe_permute_workspace_bytes(T, E, k) bytes. */
moe_status moe_permute(const int32_t* ids, int32_t T, int32_t E, int32_t k,
                       int32_t* counts, int32_t* offsets, int32_t* perm, int32_t* inv,
                       void* ws, size_t ws_bytes, void* stream);

/* moe_permute for callers that cannot allocate device memory (no counterpart
 * on the pages: an addition of this library).  Same inputs, outputs and
 * results as moe_permute, but no workspace argument: the scratch lives in a
 * fixed 256 KiB device array inside the library, which every GPU that loads
 * the library holds until the process exits.
 *  - Size limit: permute_segments * E <= 65536 with one segment per 1024
 *    assignments, i.e. ceil(T*k / 1024) * E <= 65536 (T*k <= 262144 at
 *    E = 256); larger calls return MOE_ERR_WORKSPACE_TOO_SMALL before any
 *    launch.
 *  - The first call on a device looks up the array's device address (once
 *    per device, with that device current); make that first call before any
 *    stream capture.
 *  - All calls share the one array: calls that overlap on the GPU (different
 *    streams without ordering, or concurrent host threads) race and must be
 *    serialised by the caller.
 *  - An expert id outside [0, E) is not placed and, with no workspace to hold
 *    a status word, not reported; use moe_permute to get the report. */
moe_status moe_permute_noalloc(const int32_t* ids, int32_t T, int32_t E, int32_t k,
                               int32_t* counts, int32_t* offsets, int32_t* perm,
                               int32_t* inv, void* stream);

/* [FM][FP][G8] Grouped Gate-Up GEMM with SiLU*mul epilogue.  Row p < T*k of
 * expert e (offsets[e] <= p < offsets[e+1]) reads token perm[p] / k straight
 * from x (no separate gather); rows T*k .. T*k+T-1 (when I_shared > 0) are
 * the shared expert on token p - T*k.
 *   h[p][n] = silu(x_t . Wg[e][n]) * (x_t . Wu[e][n]),  FP32 accumulation.
 * wdtype 0: x [T][d] bf16, x_scale NULL; h [R][I] bf16, h_scale NULL.
 * wdtype 1: x [R][d] e4m3 rows already in permuted order with x_scale float
 *           [R][d/128] (moe_quantize_act_fp8_permuted; perm is then not read
 *           and may be NULL); h [R][I] e4m3 with h_scale float [R][I/128]
 *           (1x128 quantisation of the FP32 h in the epilogue).
 * wdtype 3: x [R][d] e4m3 (moe_quantize_act_fp8_static_permuted with
 *           weights->act_scale_x), h [R][I] e4m3 quantised with act_scale_h;
 *           x_scale and h_scale are not read (may be NULL).
 * wdtype 2: the same with MXFP8: x_scale uint8 E8M0 [d/128][R][4]
 *           (moe_quantize_act_mxfp8_permuted), h_scale uint8 [I/128][R][4] (each
 *           1x32 block of the FP32 h quantised in the epilogue).
 * R = T*k + (I_shared ? T : 0).  ws: at least 256 bytes (the status word and
 * the tile counter). */
moe_status moe_gemm_gateup(const moe_shape* shape, const moe_weights* weights,
                           const void* x, const void* x_scale, const int32_t* perm,
                           const int32_t* offsets, void* h, void* h_scale,
                           void* ws, size_t ws_bytes, void* stream);

/* [FM][G8] Grouped Down GEMM: o[p] = h[p] . Wd[e]^T with FP32 accumulation,
 * same row grouping as moe_gemm_gateup, stored as IEEE FP16 (binary16 bit
 * patterns): o [R][d] f16, rounded to nearest even and saturating (finite
 * sums beyond +-65504 are stored as +-65504).  FP16 keeps 11 significant
 * bits, so this rounding (at most 2^-11 relative) adds little to the bf16
 * rounding of the layer output; bf16 rows would add a second rounding of
 * the output's own size.  ws: at least 256 bytes (the status word). */
moe_status moe_gemm_down(const moe_shape* shape, const moe_weights* weights,
                         const void* h, const void* h_scale, const int32_t* offsets,
                         void* o, void* ws, size_t ws_bytes, void* stream);

/* [FM] Top-K weighted aggregation plus the shared expert:
 *   y[t] = sum_j w[t][j] * o[inv[t*k+j]] + o[T*k+t]
 * o widened exactly to FP32, FP32 sum in the order j = 0..k-1 then the
 * shared term (only when I_shared > 0), one bf16 rounding.
 * o [R][d] f16 (as moe_gemm_down writes it), y [T][d] bf16. */
moe_status moe_combine(const moe_shape* shape, const void* o, const int32_t* inv,
                       const float* w, uint16_t* y, void* stream);

/* The whole layer in one call: router logits -> top-k -> permute ->
 * (FP8: quantise x) -> gate-up -> down -> combine, all on `stream`.
 * x [T][d] bf16, y [T][d] bf16.  ws: moe_workspace_bytes(shape). */
moe_status moe_forward(const moe_shape* shape, const moe_weights* weights,
                       const uint16_t* x, uint16_t* y, void* ws, size_t ws_bytes,
                       void* stream);

/* moe_forward that also records the caller's CUDA events (cudaEvent_t as
 * void*, created by the caller) on `stream` at the stage boundaries, so the
 * caller can time each kernel on the stream it runs on:
 *   events[0] start, [1] after router logits, [2] top-k, [3] permute,
 *   [4] activation quantisation (FP8; same point as [3] for BF16),
 *   [5] gate-up GEMM, [6] down GEMM, [7] combine.
 * n_events must be MOE_PROFILE_EVENTS. */
#define MOE_PROFILE_EVENTS 8
moe_status moe_forward_profiled(const moe_shape* shape, const moe_weights* weights,
                                const uint16_t* x, uint16_t* y, void* ws, size_t ws_bytes,
                                void* stream, void* const* events, int32_t n_events);

/* moe_forward on HOST buffers: copies x_host [T][d] in, runs the layer,
 * copies y_host [T][d] out and synchronises `stream` before returning.
 * Pinned host memory gives asynchronous copies.  Staging lives in the
 * workspace: ws_bytes >= moe_workspace_bytes(shape). */
moe_status moe_forward_host(const moe_shape* shape, const moe_weights* weights,
                            const uint16_t* x_host, uint16_t* y_host, void* ws,
                            size_t ws_bytes, void* stream);

/* The same without the final synchronisation: enqueues the copy of x_host in,
 * the forward and the copy of y out on `stream` and returns.  For pipelining
 * consecutive batches over several streams (the copies of one batch overlap
 * the kernels of another; H2D and D2H run on separate copy engines): use one
 * workspace per stream with work in flight, keep x_host unmodified and read
 * y_host only after `stream` has been synchronised (both pinned, or the copies
 * are not asynchronous).  Errors found on the device go to ws's status word
 * as for moe_forward. */
moe_status moe_forward_host_async(const moe_shape* shape, const moe_weights* weights,
                                  const uint16_t* x_host, uint16_t* y_host, void* ws,
                                  size_t ws_bytes, void* stream);

/* [FM][FP] The routing part of moe_forward alone: router logits with the
 * top-k fused into the router kernel, then the permute, into the workspace
 * regions moe_workspace_offsets reports (logits, ids, w, counts, offsets,
 * perm, inv).  Needs only the router weights of `weights`.  ws:
 * moe_workspace_bytes(shape).  Used by expert parallelism, which routes
 * locally and runs the experts where they live. */
moe_status moe_route(const moe_shape* shape, const moe_weights* weights, const uint16_t* x,
                     void* ws, size_t ws_bytes, void* stream);

/* Expert parallelism ("HPC-Ops ...", HPC-Ops的主要功能, "GroupGEMM FP8": the
 * grouped GEMM suits expert parallelism; "PR #54160 完整报告", 实现拆解: the
 * layer deployed over 8 GPUs).  Experts are split into contiguous ranges of
 * E_local per rank (rank r owns r*E_local .. (r+1)*E_local-1).  With the
 * routing of moe_route (ids [T][k], perm [T*k]), the permuted row order is
 * grouped by expert and therefore by owning rank:
 *   send_rows[p] = x[perm[p] / k]   (bf16 [T*k][d], d % 8 == 0)
 *   send_ids[p]  = ids[perm[p]] % E_local  (the expert's id at its owner)
 * Rows offsets[r*E_local] .. offsets[(r+1)*E_local]-1 go to rank r.  x and
 * send_rows 16-byte aligned. */
moe_status moe_ep_dispatch(const uint16_t* x, const int32_t* ids, const int32_t* perm, int32_t T,
                           int32_t d, int32_t k, int32_t E_local, uint16_t* send_rows,
                           int32_t* send_ids, void* stream);

/* Row gather: dst[i] = src[index[i]] for i < n, rows of row_bytes bytes (a
 * multiple of 16; src and dst 16-byte aligned).  Expert parallelism uses it
 * to put the expert outputs of received rows back in arrival order (index =
 * the inverse permutation of their local grouping) before returning them. */
moe_status moe_gather_rows(const void* src, const int32_t* index, int64_t n, int32_t row_bytes,
                           void* dst, void* stream);

/* [AN] Tensor-parallel all-reduce fused with the residual add and RMSNorm,
 * low-latency P2P form ("HPC-Ops - 騰訊混元開源的工業級高性能大模型推理算子庫",
 * HPC-Ops的技術原理, "Fused AllReduce+Norm": RMSNorm(AllReduce(x) + residual,
 * weight) as one NVLink operation; the decode version exchanges data by
 * Lamport P2P stores and overlaps the previous kernel through PDL).  Per token
 * t of each of the G ranks' x_r [T][d] bf16:
 *   s = sum_{r<G} x_r[t] + residual[t]   (FP32, ranks summed in order 0..G-1,
 *                                        then the residual: every rank gets the
 *                                        same bits)
 *   residual_out[t] = RNE_bf16(s),  out[t] = RNE_bf16(s * rsqrt(mean(s^2) + eps) * gamma)
 * Transport: every rank owns a Lamport buffer of moe_lamport_buffer_bytes(G,
 * T_max, d) bytes, filled once with moe_lamport_init; every rank maps every
 * other rank's buffer (CUDA IPC: moe_peer_buffer_alloc / _open).  Call number
 * `call` must be the same on all ranks and advance by one per call.  No
 * multicast and no TMA: plain 16-byte stores to peer memory and polling loads
 * of local memory.  Limits: 1 <= G <= 8, d % 8 == 0, d <= 8192, T <= T_max,
 * every pointer 16-byte aligned.  Each wait for a peer's data is bounded (2 s):
 * it then records MOE_ERR_DEVICE_TIMEOUT in ws's status word (not cleared by
 * this call, so that nothing separates it from the previous kernel; the
 * buffers must be re-initialised after a timeout).  Launched with
 * programmatic dependent launch: it may start while the previous kernel in
 * `stream` finishes and waits for it before reading x or the residual.
 *   bufs: HOST array of G device pointers, the buffers of ranks 0..G-1 as
 *         mapped in this process (bufs[rank] its own);
 *   residual, residual_out: may be NULL (no residual / not written);
 *   gamma [d] bf16; ws >= 256 bytes. */
size_t moe_lamport_buffer_bytes(int32_t G, int32_t T_max, int32_t d);
moe_status moe_lamport_init(void* buf, size_t bytes, void* stream);
moe_status moe_allreduce_rmsnorm(void* const* bufs, int32_t G, int32_t rank, uint32_t call,
                                 int32_t T_max, const uint16_t* x, const uint16_t* residual,
                                 const uint16_t* gamma, float eps, int32_t T, int32_t d,
                                 uint16_t* out, uint16_t* residual_out, void* ws, size_t ws_bytes,
                                 void* stream);

/* The same kernel for `ranks` ranks of a G-rank group emulated on ONE GPU, in
 * one cooperative launch (every rank's blocks resident at once, so the ranks
 * can wait on one another): bufs, x, residual, out, residual_out are HOST
 * arrays of device pointers indexed by rank (residual / residual_out arrays may
 * be NULL).  ranks < G leaves the missing ranks' data unsent, so the others'
 * waits run out after timeout_us and report MOE_ERR_DEVICE_TIMEOUT (the
 * failure path, without a GPU fault).  Clears ws's status word first.  For
 * tests of the protocol on one GPU. */
moe_status moe_allreduce_rmsnorm_emulated(void* const* bufs, int32_t G, int32_t ranks,
                                          uint32_t call, int32_t T_max, const uint16_t* const* x,
                                          const uint16_t* const* residual, const uint16_t* gamma,
                                          float eps, int32_t T, int32_t d, uint16_t* const* out,
                                          uint16_t* const* residual_out, int32_t timeout_us,
                                          void* ws, size_t ws_bytes, void* stream);

/* Peer-memory set-up for moe_allreduce_rmsnorm (set-up time only; the one
 * place this library allocates): moe_peer_buffer_alloc cudaMallocs `bytes`
 * on the current device and writes the 64-byte CUDA IPC handle of it;
 * another process opens it with moe_peer_buffer_open (mapped with peer access)
 * and unmaps it with moe_peer_buffer_close; the owner frees it with
 * moe_peer_buffer_free after every mapping is closed. */
moe_status moe_peer_buffer_alloc(size_t bytes, void** ptr, void* ipc_handle);
moe_status moe_peer_buffer_open(const void* ipc_handle, void** ptr);
moe_status moe_peer_buffer_close(void* ptr);
moe_status moe_peer_buffer_free(void* ptr);

/* Synchronises `stream` and returns the device status word of `ws`
 * (MOE_OK, MOE_ERR_DEVICE_TIMEOUT or MOE_ERR_DEVICE_BAD_INDEX). */
moe_status moe_read_device_status(const void* ws, void* stream);

/* Failure-path check of the bounded device waits: launches one block that
 * waits on a barrier nothing completes, gives up after `limit_us`
 * microseconds, records MOE_ERR_DEVICE_TIMEOUT in the status word of ws
 * (>= 256 bytes) and returns; read it with moe_read_device_status. */
moe_status moe_selftest_timeout(void* ws, int32_t limit_us, void* stream);

#ifdef __cplusplus
}
#endif
#endif /* MOE_B200_H */
