/* moe_oracle.h -- plain FP64 CPU oracle of the fused MoE layer forward.
 *
 * TEST INFRASTRUCTURE, NOT PART OF THE PRODUCT.  Only the test suite, the
 * package smoke check and the benchmark's CPU-baseline / reference leg may
 * load this library.  It shares no code, header, table or helper with the
 * CUDA library; the two only ever see the same seeded synthetic inputs.
 *
 * What it computes, and where the pages define it (page title -- section):
 *
 *  [RG]  "HPC-Ops - 騰訊混元開源的工業級高性能大模型推理算子庫", section
 *        "HPC-Ops的技術原理", paragraph "Router GEMM 雙 BF16 模擬 FP32":
 *        the FP32 router weight is split offline into a high BF16 part and a
 *        low BF16 residual with scale factor 1/256; inference runs two BF16
 *        GEMMs and combines them linearly (one FMA in the epilogue).
 *  [FM]  same page, section "HPC-Ops的主要功能", item "FusedMoE": five stages
 *        -- routing index, Gate-Up GEMM, activation quantisation, Down GEMM,
 *        Top-K weighted aggregation.
 *  [FP]  same page, section "HPC-Ops的技術原理", paragraph "FusedMoE 流水線重構":
 *        shared-memory blocked per-expert counting that reserves one
 *        contiguous output interval per expert; Gate-Up reads the original
 *        input through the routing index.
 *  [G8]  same page, section "HPC-Ops的主要功能", item "GroupGEMM FP8":
 *        grouped expert GEMM with block-wise FP8 quantisation.
 *  [HY]  "PR #54160 完整报告" ([Hy4] support Hy4-preview model), section
 *        "功能与动机": 256 routed experts, top-8, plus 1 shared expert per MoE
 *        layer; section "实现拆解" item 4: FP8 block-wise 128x128 scales.
 *
 * Readings where the pages are silent (each also listed in the design notes):
 *  - both roundings of the router split are round-to-nearest-even, and the
 *    low part is stored multiplied by 256 (W ~= hi + lo/256);
 *  - routing is a softmax over the selected top-k logits (renormalised), slot
 *    order is descending logit with ties to the lower expert id, and the
 *    selection is taken on FP32 logits (the precision the kernel decides in);
 *  - the expert FFN is SiLU-gated: h = silu(x Wg^T) * (x Wu^T), o = h Wd^T,
 *    with gate rows first in the fused [2I, d] gate-up matrix;
 *  - the shared expert is always on with weight 1;
 *  - FP8 scales: s = fp32(amax)/448 in FP32 (amax == 0 -> s = 1) and
 *    q = e4m3_rne_satfinite(fp32(v / s)), per 128x128 weight block and per
 *    1x128 activation group; the code decision is taken in FP32 on both sides.
 *
 * All arithmetic that is not a quantisation decision is FP64.  Pointers are
 * host memory owned by the caller; row-major; BF16 passed as uint16_t bits.
 */
#ifndef MOE_ORACLE_H
#define MOE_ORACLE_H
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* scalar format codecs, written from the format definitions */
double   orc_bf16_decode(uint16_t b);
uint16_t orc_bf16_round(double v);          /* nearest bf16, ties to even   */
double   orc_e4m3_decode(uint8_t b);
uint8_t  orc_e4m3_round(double v);          /* nearest e4m3, ties to even,
                                               |v| > 448 saturates to 448   */
void orc_bf16_round_array(const double* v, int64_t n, uint16_t* out);

/* [RG] offline split: hi = bf16(W), lo = bf16((W - hi) * 256) */
void orc_router_split(const float* W, int64_t n, uint16_t* hi, uint16_t* lo);

/* [RG] logits[t][e] = sum_i x[t][i] * (hi[e][i] + lo[e][i] / 256) (+ bias[e]) */
void orc_router_logits(const uint16_t* x, const uint16_t* hi, const uint16_t* lo,
                       const float* bias, int T, int d, int E, double* logits);

/* [FM][HY] top-k of FP32 logits, descending, ties to the lower id; weights are
 * the softmax over the selected k (renorm != 0) or over all E (renorm == 0). */
void orc_route_topk(const float* logits, int T, int E, int k, int renorm,
                    int32_t* ids, double* w);

/* [FP] counts[e], offsets[0..E] (exclusive scan), stable placement of the
 * flat assignment index a = t*k + j: perm[p] = a, inv[a] = p. */
void orc_permute(const int32_t* ids, int T, int E, int k, int32_t* counts,
                 int32_t* offsets, int32_t* perm, int32_t* inv);

/* [G8][HY] 128x128 block quantisation of `batch` row-major [rows][cols] bf16
 * matrices: q [batch][rows][cols], s [batch][rows/128][cols/128]. */
void orc_quant_fp8_blocks(const uint16_t* W, int64_t batch, int rows, int cols,
                          uint8_t* q, float* s);

/* [FM][G8] 1x128 group quantisation of each row of an FP32 matrix:
 * q [rows][cols], s [rows][cols/128]. */
void orc_quant_fp8_rows(const float* v, int64_t rows, int cols, uint8_t* q, float* s);

/* [MX] MXFP8 (OCP Microscaling formats v1.0, "MXFP8 E4M3"): blocks of 32
 * consecutive elements along K share one E8M0 scale X = 2^(b - 127) (byte b;
 * 255 is NaN).  For a block with amax = max |v| (taken in FP32):
 * shared_exp = floor(log2(amax)) - 8 (8 = exponent of the largest e4m3
 * normal, 448 = 1.75 * 2^8), clamped to [-127, 127]; amax == 0 -> -127.
 * q_i = e4m3_rne_satfinite(v_i / X) (exact power-of-two scaling, so FP32 and
 * FP64 take the same decision).  The pages name the format ("PR #54160 完整报告",
 * section 实现拆解 item 4: FP8 blockwise 128x128 and MXFP8 scale parameters);
 * its definition is the OCP one. */
double  orc_e8m0_decode(uint8_t b);
uint8_t orc_mx_scale_byte(float amax);
/* Rows of an FP32 matrix: q [rows][cols], s [rows][cols/32] (E8M0 bytes). */
void orc_quant_mx_rows(const float* v, int64_t rows, int cols, uint8_t* q, uint8_t* s);
/* Rows of `batch` bf16 matrices [rows][cols] (weights; K = cols):
 * q [batch][rows][cols], s [batch][rows][cols/32]. */
void orc_quant_mx_bf16(const uint16_t* W, int64_t batch, int rows, int cols, uint8_t* q,
                       uint8_t* s);

/* [G8][HY] Per-tensor FP8 ("HPC-Ops ...", section HPC-Ops的主要功能, GroupGEMM FP8:
 * per-tensor and block-wise FP8; "腾讯混元大模型：从多场景适配到高效部署的全栈技术解析",
 * section 量化压缩技术实践 / FP8量化方案: static FP8 quantisation of weights and
 * activations with scales precomputed from calibration data).  Weights: one
 * scale per matrix, s = fp32(amax) / 448 (amax == 0 -> 1), q = e4m3(fp32(W/s));
 * activations: a given static scale s, q = e4m3_rne_satfinite(fp32(v / s)). */
void orc_quant_fp8_tensor(const uint16_t* W, int64_t batch, int rows, int cols, uint8_t* q,
                          float* s);
void orc_quant_fp8_static(const float* v, int64_t n, float s, uint8_t* q);

typedef struct {
    int T, d, E, k, I, Is;     /* Is = 0: no shared expert                     */
    int wdtype;                /* 0: BF16 weights; 1: FP8 e4m3, 128x128 blocks;
                                  2: MXFP8 (e4m3, E8M0 scale per 1x32 along K);
                                  3: FP8 per tensor (one scale per weight matrix,
                                  static activation scales act_sx, act_sh)
                                  (the oracle quantises the BF16 weights itself) */
    int renorm;
    const uint16_t* w_gu;      /* bf16 [E][2I][d]: gate rows 0..I-1, up I..2I-1 */
    const uint16_t* w_d;       /* bf16 [E][d][I]                                */
    const uint16_t* ws_gu;     /* bf16 [2Is][d] or NULL                         */
    const uint16_t* ws_d;      /* bf16 [d][Is] or NULL                          */
    const float* router_w;     /* f32 [E][d]; the oracle splits it itself       */
    const float* router_bias;  /* f32 [E] or NULL                               */
    float act_sx, act_sh;      /* wdtype 3: static scales of x and of h         */
} orc_layer;

/* [FM][FP] Gate-Up stage over the permuted rows.  Rows p < T*k belong to the
 * expert whose offsets interval holds p and read token perm[p] / k; rows
 * T*k .. T*k+T-1 are the shared expert and read token p - T*k.
 * h: [T*k + (Is ? T : 0)][max(I, Is)] FP64, row stride hs = max(I, Is).
 * FP8 (wdtype 1): each input row is quantised per 1x128 group first;
 * MXFP8 (wdtype 2): per 1x32 block (MX).                                     */
void orc_gateup(const orc_layer* L, const uint16_t* x, const int32_t* perm,
                const int32_t* offsets, double* h);

/* [FM] Down stage: o[p] = h[p] Wd[e]^T, same row grouping as orc_gateup.
 * FP8: each h row is quantised per 1x128 group (FP32 decision) first;
 * MXFP8: per 1x32 block of the FP32-rounded h row.                           */
void orc_down(const orc_layer* L, const double* h, const int32_t* offsets, double* o);

/* [FM] Top-K weighted aggregation: y[t] = sum_j w[t][j] o[inv[t*k+j]] + o[T*k+t]. */
void orc_combine(const orc_layer* L, const double* o, const int32_t* inv,
                 const double* w, double* y);

/* The whole layer.  Every output pointer may be NULL except y. */
typedef struct {
    double* logits;   /* [T][E] */
    int32_t* ids;     /* [T][k] */
    double* w;        /* [T][k] */
    int32_t* counts;  /* [E]    */
    int32_t* offsets; /* [E+1]  */
    int32_t* perm;    /* [T*k]  */
    int32_t* inv;     /* [T*k]  */
    double* y;        /* [T][d] */
} orc_out;

int orc_forward(const orc_layer* L, const uint16_t* x, orc_out* out);

int orc_num_threads(void);

/* [AN] "HPC-Ops - 騰訊混元開源的工業級高性能大模型推理算子庫", section
 * HPC-Ops的技術原理, "Fused AllReduce+Norm": the tensor-parallel all-reduce of the
 * G ranks' partial outputs fused with the residual add and RMSNorm,
 * out = RMSNorm(AllReduce(x) + residual, weight).  In FP64, per token t:
 *   s[t][i]   = sum_{r < G} x[r][t][i] + residual[t][i]   (residual may be NULL)
 *   res[t][i] = s[t][i]                 (the new residual stream)
 *   out[t][i] = s[t][i] / sqrt(mean_i s[t][i]^2 + eps) * gamma[i]
 * x bf16 [G][T][d], residual bf16 [T][d], gamma bf16 [d]. */
void orc_allreduce_rmsnorm(const uint16_t* x, int G, int T, int d, const uint16_t* residual,
                           const uint16_t* gamma, double eps, double* res, double* out);

#ifdef __cplusplus
}
#endif
#endif
