/*
 * oracle.h - plain, slow CPU restatement of the int4 routed-expert MoE layer.
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing in the product path may include, link or
 * call this code; only the tests, the smoke check and the CPU-baseline leg of
 * the benchmark use it.  It shares no code with the CUDA library.
 *
 * Every floating-point reduction is carried out in double; values that the
 * method stores (scales, dequantised weights, routing weights, outputs) are
 * rounded to float where the container or the interface says they are f32.
 *
 * Sources (web pages, cited by title and section):
 *  [card]  "jlnsrk/GLM-5.2-colibri-int4 - Hugging Face" (model-card translation):
 *          the container paragraph (U8 packed int4 nibbles + F32 per-row scales,
 *          bit-identical to the engine's C kernels), the contents table (router and
 *          norms stay F32) and the conversion note (np.rint == the engine's lrintf).
 *  [int8]  "解密GLM-5.2-colibri-int4-with-int8-mtp", sections 模型架构深度解析
 *          (256 routed + 1 shared expert, num_experts_per_tok 8, scoring_func
 *          sigmoid, norm_topk_prob true) and 量化策略细节 (hidden_size 6144).
 *  [gh11k] "github一周涨11k⭐️！25GB 内存跑 744B GLM-5.2 模型！", section 三.1
 *          (DeepSeek-V3-style sigmoid router, 8 of 256 per token), 三.4
 *          (batch-union MoE) and 四.3 (bias-corrected selection; routing, selection
 *          and scaling semantics must be reproduced exactly).
 *  [guide] "colibrì 實戰指南", section 二 (per-token path: route -> union ->
 *          placement -> execution; three matrices of an expert stored adjacently)
 *          and 三 (gs64 group-scaled container preferred over per-row).
 */
#ifndef COLI_ORACLE_H
#define COLI_ORACLE_H

#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* Quantise a row-major [rows, cols] f32 matrix into the container layout:
 * packed[r, c/2] holds column c (even c in the low nibble, odd c in the high
 * nibble) as a signed two's-complement nibble; scales[r, g] is one f32 per
 * row (group == 0) or per 64-column group (group == 64).  Returns 0, or -1 on
 * bad arguments. */
int orc_quantize(const float* w, int64_t rows, int64_t cols, int32_t group,
                 uint8_t* packed, float* scales);

/* Inverse of the container encoding: out[r, c] = (float)q[r, c] * s[r, g]. */
int orc_dequantize(const uint8_t* packed, const float* scales, int64_t rows,
                   int64_t cols, int32_t group, float* out);

/* Sigmoid router with bias-corrected top-k.  x [T, H], wr [E, H], bias [E].
 * idx [T, k] is ordered by (selection score desc, expert index asc); w [T, k]
 * are the (renormalised when norm_topk != 0) sigmoid scores times
 * routed_scale.  gap [T] (may be NULL) receives sel_(k) - sel_(k+1) per token
 * (+inf when k == E). */
int orc_route(const float* x, int64_t T, int64_t H, const float* wr,
              const float* bias, int64_t E, int64_t k, double routed_scale,
              int norm_topk, int32_t* idx, float* w, double* gap);

/* Batch union by brute force: pairs (t, j) grouped by expert, experts
 * ascending, tokens ascending inside an expert.  offsets [E+1], pair_tok and
 * pair_slot [T*k], uniq [E] (ascending list of experts with >= 1 pair),
 * n_uniq [1]. */
int orc_union(const int32_t* idx, int64_t T, int64_t k, int64_t E,
              int32_t* offsets, int32_t* pair_tok, int32_t* pair_slot,
              int32_t* uniq, int32_t* n_uniq);

/* One SwiGLU expert on one token with dequantised f32 weights:
 * wg, wu [I, H], wd [H, I].  o[n] = (W_d h)[rows[n]] for the n_rows requested
 * output rows (rows == NULL means all H rows, in order), computed in double. */
int orc_expert(const float* x, int64_t H, int64_t I, const float* wg,
               const float* wu, const float* wd, const int32_t* rows,
               int64_t n_rows, double* o);

/* One token through the layer given its routing decision: y[n] =
 * sum_j w[j] * o_j[n] (j ascending) + sum_s o_shared_s[n], stored as float.
 * experts: k routed then n_shared shared experts, each as three dequantised
 * matrices (gate, up, down). */
int orc_token_forward(const float* x, int64_t H, int64_t I, int64_t k,
                      const float* w, const float* const* wg,
                      const float* const* wu, const float* const* wd,
                      int64_t n_shared, const int32_t* rows, int64_t n_rows,
                      float* y);

/* Whole layer for configurations small enough to hold every expert: masters
 * are f32 [n_exp, I, H] (gate, up) and [n_exp, H, I] (down) with the routed
 * experts first and the n_shared shared experts last.  The oracle quantises
 * and dequantises them itself, routes every token and applies the experts.
 * idx/w (may be NULL) receive the routing decision. */
int orc_layer_forward(const float* x, int64_t T, int64_t H, int64_t I,
                      int64_t E, int64_t k, int64_t n_shared, int32_t group,
                      double routed_scale, int norm_topk, const float* wr,
                      const float* bias, const float* gate_m, const float* up_m,
                      const float* down_m, float* y, int32_t* idx, float* w);

/* RMSNorm with unit gain: out = v / sqrt(mean(v^2) + eps), per row of [T, H]. */
int orc_rmsnorm(const float* x, int64_t T, int64_t H, double eps, float* out);

/* 8-bit variant of the container: codes[r, c] one signed byte in [-127, 127],
 * scales[r, g] = max|w| / 127 per row (group 0) or per 64 columns; q = rint(w/s).
 * dequantize8 writes (float)q * s.  Return 0, or -1 on bad arguments. */
int orc_quantize8(const float* w, int64_t rows, int64_t cols, int32_t group, int8_t* codes,
                  float* scales);
int orc_dequantize8(const int8_t* codes, const float* scales, int64_t rows, int64_t cols,
                    int32_t group, float* out);

/* Adaptive expert top-p of one token: of its k picks (weights w, experts idx,
 * pick order), keep the shortest run of the largest renormalised weights
 * (w_j / sum w; equal weights to the lower expert index) whose total reaches p.
 * keep[j] = 1 for kept picks.  Returns the number kept, or -1 on bad arguments. */
int64_t orc_topp_keep(const float* w, const int32_t* idx, int64_t k, double p, int32_t* keep);

/* FP8 (E4M3) matrix with one f32 scale per 128 x 128 block -> f32:
 * out[r, c] = e4m3(q[r, c]) * bs[r / 128, c / 128] (bs row-major
 * [ceil(rows/128), ceil(cols/128)]).  Returns 0, or -1 on bad arguments. */
int orc_fp8_block_dequant(const uint8_t* q, const float* bs, int64_t rows, int64_t cols,
                          float* out);

#ifdef __cplusplus
}
#endif
#endif
