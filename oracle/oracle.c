/*
 * oracle.c - plain, slow CPU restatement of the int4 routed-expert MoE layer.
 *
 * TEST INFRASTRUCTURE ONLY (tests, smoke check, CPU-baseline leg of the
 * benchmark).  It is written from the method's definitions, step by step, with
 * no blocking, fusion or reordering; every sum runs in double in index order.
 * See oracle.h for the sources.  Built with -O2 -fopenmp -ffp-contract=off so
 * that float expressions are evaluated exactly as written; OpenMP only splits
 * independent tokens / output rows, so results do not depend on thread count.
 */
#include "oracle.h"

#include <math.h>
#include <stdlib.h>
#include <string.h>

/* ------------------------------------------------------------------------- */
/* Container: quantise / dequantise                                           */
/* [card] container paragraph and conversion note; [guide] 三 (gs64).         */
/* ------------------------------------------------------------------------- */

static int64_t n_groups(int64_t cols, int32_t group) {
    return group == 0 ? 1 : cols / group;
}

static int bad_shape(int64_t rows, int64_t cols, int32_t group) {
    if (rows < 0 || cols <= 0 || (cols % 2) != 0) return 1;
    if (group != 0 && group != 64) return 1;
    if (group != 0 && (cols % group) != 0) return 1;
    return 0;
}

int orc_quantize(const float* w, int64_t rows, int64_t cols, int32_t group,
                 uint8_t* packed, float* scales) {
    if (!w || !packed || !scales || bad_shape(rows, cols, group)) return -1;
    const int64_t gsz = group == 0 ? cols : group;
    const int64_t ng = n_groups(cols, group);
    for (int64_t r = 0; r < rows; ++r) {
        const float* row = w + r * cols;
        uint8_t* prow = packed + r * (cols / 2);
        memset(prow, 0, (size_t)(cols / 2));
        for (int64_t g = 0; g < ng; ++g) {
            /* scale = max|w| over the group / 7, an f32 division */
            float m = 0.0f;
            for (int64_t c = g * gsz; c < (g + 1) * gsz; ++c) {
                float a = fabsf(row[c]);
                if (a > m) m = a;
            }
            float s = m / 7.0f;
            scales[r * ng + g] = s;
            for (int64_t c = g * gsz; c < (g + 1) * gsz; ++c) {
                int q = 0;
                if (s != 0.0f) {
                    float t = row[c] / s;           /* f32 division   */
                    float qf = rintf(t);            /* half to even   */
                    if (qf > 7.0f) qf = 7.0f;       /* guard only     */
                    if (qf < -7.0f) qf = -7.0f;
                    q = (int)qf;
                }
                uint8_t nib = (uint8_t)(q & 0xF);   /* two's complement */
                if (c & 1) prow[c / 2] |= (uint8_t)(nib << 4);
                else       prow[c / 2] |= nib;
            }
        }
    }
    return 0;
}

/* 8-bit variant of the container (the int8 MTP head: "解密GLM-5.2-colibri-int4-
 * with-int8-mtp", whose MTP head keeps 8-bit precision; the converter's
 * --io-bits 8, "GLM-5.2-colibri-int4专家流技术详解" project-source section).
 * The pages give no further rule; this follows the int4 container's: per row
 * or per 64 columns s = max|w| / 127 (f32 division), q = rint(w / s) (f32
 * division, half to even) in [-127, 127], one signed byte per weight. */
int orc_quantize8(const float* w, int64_t rows, int64_t cols, int32_t group, int8_t* codes,
                  float* scales) {
    if (!w || !codes || !scales || rows < 0 || cols <= 0 || (group != 0 && group != 64) ||
        (group && cols % group))
        return -1;
    const int64_t gsz = group == 0 ? cols : group;
    const int64_t ng = cols / gsz;
    for (int64_t r = 0; r < rows; ++r) {
        const float* row = w + r * cols;
        for (int64_t g = 0; g < ng; ++g) {
            float m = 0.0f;
            for (int64_t c = g * gsz; c < (g + 1) * gsz; ++c) {
                const float a = fabsf(row[c]);
                if (a > m) m = a;
            }
            const float s = m / 127.0f;
            scales[r * ng + g] = s;
            for (int64_t c = g * gsz; c < (g + 1) * gsz; ++c) {
                int q = 0;
                if (s != 0.0f) {
                    float qf = rintf(row[c] / s);
                    if (qf > 127.0f) qf = 127.0f;       /* guard only */
                    if (qf < -127.0f) qf = -127.0f;
                    q = (int)qf;
                }
                codes[r * cols + c] = (int8_t)q;
            }
        }
    }
    return 0;
}

int orc_dequantize8(const int8_t* codes, const float* scales, int64_t rows, int64_t cols,
                    int32_t group, float* out) {
    if (!codes || !scales || !out || rows < 0 || cols <= 0 || (group != 0 && group != 64) ||
        (group && cols % group))
        return -1;
    const int64_t gsz = group == 0 ? cols : group, ng = cols / gsz;
    for (int64_t r = 0; r < rows; ++r)
        for (int64_t c = 0; c < cols; ++c)
            out[r * cols + c] = (float)codes[r * cols + c] * scales[r * ng + c / gsz];
    return 0;
}

/* Adaptive expert top-p of one token ("colibrì 實戰指南" 三 and 五: --topp p reads
 * 30-40% fewer expert bytes per token; the rule itself is not given): order the
 * token's k picks by renormalised weight w_j / sum(w), largest first, equal
 * weights to the lower expert index, and keep the shortest prefix of that order
 * whose weights add up to at least p (in double).  Kept picks keep their
 * weights; the others contribute nothing.  keep[j] = 1 for a kept pick j (pick
 * order), else 0; returns the number kept (k when p >= the total). */
int64_t orc_topp_keep(const float* w, const int32_t* idx, int64_t k, double p, int32_t* keep) {
    if (!w || !idx || !keep || k < 1) return -1;
    double tot = 0.0;
    for (int64_t j = 0; j < k; ++j) {
        tot += (double)w[j];
        keep[j] = 0;
    }
    int64_t kept = 0;
    double mass = 0.0;
    while (kept < k && (kept == 0 || mass < p)) {
        int64_t best = -1;   /* largest weight not yet kept, then lower expert index */
        for (int64_t j = 0; j < k; ++j) {
            if (keep[j]) continue;
            if (best < 0 || w[j] > w[best] || (w[j] == w[best] && idx[j] < idx[best])) best = j;
        }
        keep[best] = 1;
        mass += tot > 0.0 ? (double)w[best] / tot : 0.0;
        ++kept;
    }
    return kept;
}

/* FP8 E4M3 code as a float, from the format's definition: sign bit, four
 * exponent bits with bias 7, three mantissa bits; exponent 0 holds the
 * subnormals m/8 * 2^-6; S.1111.111 is NaN and there are no infinities.
 * Every value is exact in f32. */
static float e4m3_value(uint8_t b) {
    const int sign = b >> 7, e = (b >> 3) & 0xF, m = b & 7;
    float v;
    if (e == 0) v = ldexpf((float)m / 8.0f, -6);
    else if (e == 15 && m == 7) v = NAN;
    else v = ldexpf(1.0f + (float)m / 8.0f, e - 7);
    return sign ? -v : v;
}

/* Block-scaled FP8 matrix -> f32: out[r, c] = e4m3(q[r, c]) * bs[r/128, c/128],
 * one f32 multiply (the checkpoint's 128 x 128 weight blocks, one scale each;
 * bs is [ceil(rows/128), ceil(cols/128)] row-major).  ["解密GLM-5.2-colibri-int4-
 * with-int8-mtp", quantisation-config paragraph: fmt e4m3, weight_block_size
 * [128, 128]; the int4 container is converted from that checkpoint: "GLM-5.2-
 * colibri-int4专家流技术详解", project-source section.] */
int orc_fp8_block_dequant(const uint8_t* q, const float* bs, int64_t rows, int64_t cols,
                          float* out) {
    if (!q || !bs || !out || rows < 1 || cols < 1) return -1;
    const int64_t kb = (cols + 127) / 128;
    for (int64_t r = 0; r < rows; ++r)
        for (int64_t c = 0; c < cols; ++c) {
            const float v = e4m3_value(q[r * cols + c]);
            const float s = bs[(r / 128) * kb + c / 128];
            out[r * cols + c] = v * s;             /* f32 multiply, round to nearest */
        }
    return 0;
}

static int decode_nibble(uint8_t byte, int high) {
    int n = high ? (byte >> 4) & 0xF : byte & 0xF;
    return n >= 8 ? n - 16 : n;                     /* sign-extend 4 bits */
}

int orc_dequantize(const uint8_t* packed, const float* scales, int64_t rows,
                   int64_t cols, int32_t group, float* out) {
    if (!packed || !scales || !out || bad_shape(rows, cols, group)) return -1;
    const int64_t gsz = group == 0 ? cols : group;
    const int64_t ng = n_groups(cols, group);
    for (int64_t r = 0; r < rows; ++r) {
        for (int64_t c = 0; c < cols; ++c) {
            int q = decode_nibble(packed[r * (cols / 2) + c / 2], (int)(c & 1));
            float s = scales[r * ng + c / gsz];
            out[r * cols + c] = (float)q * s;       /* one f32 multiply */
        }
    }
    return 0;
}

/* ------------------------------------------------------------------------- */
/* Router: [int8] 模型架构深度解析, [gh11k] 三.1 and 四.3, [card] contents     */
/* table (router kept F32).                                                   */
/* ------------------------------------------------------------------------- */

static double sigmoid(double z) { return 1.0 / (1.0 + exp(-z)); }

/* true when expert a ranks before expert b: higher score, then lower index */
static int ranks_before(double sa, int64_t a, double sb, int64_t b) {
    if (sa != sb) return sa > sb;
    return a < b;
}

int orc_route(const float* x, int64_t T, int64_t H, const float* wr,
              const float* bias, int64_t E, int64_t k, double routed_scale,
              int norm_topk, int32_t* idx, float* w, double* gap) {
    if (!x || !wr || !bias || !idx || !w || T < 0 || H <= 0 || E <= 0 ||
        k <= 0 || k > E)
        return -1;
    int bad = 0;
#pragma omp parallel for schedule(static)
    for (int64_t t = 0; t < T; ++t) {
        double* s = (double*)malloc(sizeof(double) * (size_t)E);
        double* sel = (double*)malloc(sizeof(double) * (size_t)E);
        int64_t* order = (int64_t*)malloc(sizeof(int64_t) * (size_t)E);
        if (!s || !sel || !order) {
            bad = 1;
            free(s); free(sel); free(order);
            continue;
        }
        for (int64_t e = 0; e < E; ++e) {
            double z = 0.0;
            for (int64_t h = 0; h < H; ++h)
                z += (double)wr[e * H + h] * (double)x[t * H + h];
            s[e] = sigmoid(z);
            sel[e] = s[e] + (double)bias[e];        /* bias: selection only */
            order[e] = e;
        }
        /* selection sort of the first k+1 places: plain and obviously right */
        int64_t places = k < E ? k + 1 : k;
        for (int64_t i = 0; i < places; ++i) {
            int64_t best = i;
            for (int64_t j = i + 1; j < E; ++j)
                if (ranks_before(sel[order[j]], order[j], sel[order[best]],
                                 order[best]))
                    best = j;
            int64_t tmp = order[i]; order[i] = order[best]; order[best] = tmp;
        }
        double denom = 0.0;
        for (int64_t j = 0; j < k; ++j) denom += s[order[j]];
        for (int64_t j = 0; j < k; ++j) {
            int64_t e = order[j];
            double wj = norm_topk ? s[e] / denom : s[e];
            idx[t * k + j] = (int32_t)e;
            w[t * k + j] = (float)(wj * routed_scale);
        }
        if (gap) gap[t] = k < E ? sel[order[k - 1]] - sel[order[k]] : INFINITY;
        free(s); free(sel); free(order);
    }
    return bad ? -2 : 0;
}

/* ------------------------------------------------------------------------- */
/* Batch union: [gh11k] 三.4, [guide] 二 (联集).  Brute force scan.           */
/* ------------------------------------------------------------------------- */

int orc_union(const int32_t* idx, int64_t T, int64_t k, int64_t E,
              int32_t* offsets, int32_t* pair_tok, int32_t* pair_slot,
              int32_t* uniq, int32_t* n_uniq) {
    if (!idx || !offsets || !pair_tok || !pair_slot || !uniq || !n_uniq ||
        T < 0 || k <= 0 || E <= 0)
        return -1;
    for (int64_t i = 0; i < T * k; ++i)
        if (idx[i] < 0 || idx[i] >= E) return -1;
    int32_t p = 0, u = 0;
    for (int64_t e = 0; e < E; ++e) {
        offsets[e] = p;
        for (int64_t t = 0; t < T; ++t)
            for (int64_t j = 0; j < k; ++j)
                if (idx[t * k + j] == e) {
                    pair_tok[p] = (int32_t)t;
                    pair_slot[p] = (int32_t)j;
                    ++p;
                }
        if (p > offsets[e]) uniq[u++] = (int32_t)e;
    }
    offsets[E] = p;
    *n_uniq = u;
    return 0;
}

/* ------------------------------------------------------------------------- */
/* Expert FFN (SwiGLU) and the weighted combine with the shared expert.       */
/* [int8] 模型架构深度解析 (1 shared expert); [guide] 二 (gate/up/down).       */
/* ------------------------------------------------------------------------- */

int orc_expert(const float* x, int64_t H, int64_t I, const float* wg,
               const float* wu, const float* wd, const int32_t* rows,
               int64_t n_rows, double* o) {
    if (!x || !wg || !wu || !wd || !o || H <= 0 || I <= 0) return -1;
    if (!rows) n_rows = H;
    double* h = (double*)malloc(sizeof(double) * (size_t)I);
    if (!h) return -2;
    for (int64_t i = 0; i < I; ++i) {
        double a = 0.0, u = 0.0;
        for (int64_t c = 0; c < H; ++c) {
            a += (double)wg[i * H + c] * (double)x[c];
            u += (double)wu[i * H + c] * (double)x[c];
        }
        double silu = a / (1.0 + exp(-a));
        h[i] = silu * u;
    }
    for (int64_t n = 0; n < n_rows; ++n) {
        int64_t r = rows ? rows[n] : n;
        if (r < 0 || r >= H) { free(h); return -1; }
        double acc = 0.0;
        for (int64_t i = 0; i < I; ++i) acc += (double)wd[r * I + i] * h[i];
        o[n] = acc;
    }
    free(h);
    return 0;
}

int orc_token_forward(const float* x, int64_t H, int64_t I, int64_t k,
                      const float* w, const float* const* wg,
                      const float* const* wu, const float* const* wd,
                      int64_t n_shared, const int32_t* rows, int64_t n_rows,
                      float* y) {
    if (!x || !w || !wg || !wu || !wd || !y || k < 0 || n_shared < 0) return -1;
    if (!rows) n_rows = H;
    double* acc = (double*)calloc((size_t)n_rows, sizeof(double));
    double* o = (double*)malloc(sizeof(double) * (size_t)n_rows);
    if (!acc || !o) { free(acc); free(o); return -2; }
    int rc = 0;
    for (int64_t j = 0; j < k + n_shared && rc == 0; ++j) {
        rc = orc_expert(x, H, I, wg[j], wu[j], wd[j], rows, n_rows, o);
        double wj = j < k ? (double)w[j] : 1.0;   /* shared: weight 1 */
        for (int64_t n = 0; n < n_rows; ++n) acc[n] += wj * o[n];
    }
    for (int64_t n = 0; n < n_rows; ++n) y[n] = (float)acc[n];
    free(acc); free(o);
    return rc;
}

int orc_layer_forward(const float* x, int64_t T, int64_t H, int64_t I,
                      int64_t E, int64_t k, int64_t n_shared, int32_t group,
                      double routed_scale, int norm_topk, const float* wr,
                      const float* bias, const float* gate_m, const float* up_m,
                      const float* down_m, float* y, int32_t* idx_out,
                      float* w_out) {
    if (!x || !wr || !bias || !gate_m || !up_m || !down_m || !y || T < 0 ||
        k <= 0 || k > E || n_shared < 0)
        return -1;
    const int64_t nx = E + n_shared;
    const int64_t gu = I * H, dn = H * I;
    float* deq_g = (float*)malloc(sizeof(float) * (size_t)(nx * gu));
    float* deq_u = (float*)malloc(sizeof(float) * (size_t)(nx * gu));
    float* deq_d = (float*)malloc(sizeof(float) * (size_t)(nx * dn));
    uint8_t* pk = (uint8_t*)malloc((size_t)(gu / 2 > dn / 2 ? gu / 2 : dn / 2));
    float* sc = (float*)malloc(sizeof(float) * (size_t)(gu > dn ? gu : dn));
    int32_t* idx = (int32_t*)malloc(sizeof(int32_t) * (size_t)(T * k + 1));
    float* w = (float*)malloc(sizeof(float) * (size_t)(T * k + 1));
    int rc = 0;
    if (!deq_g || !deq_u || !deq_d || !pk || !sc || !idx || !w) rc = -2;
    /* every expert matrix goes through the container and back */
    for (int64_t e = 0; e < nx && rc == 0; ++e) {
        rc |= orc_quantize(gate_m + e * gu, I, H, group, pk, sc);
        rc |= orc_dequantize(pk, sc, I, H, group, deq_g + e * gu);
        rc |= orc_quantize(up_m + e * gu, I, H, group, pk, sc);
        rc |= orc_dequantize(pk, sc, I, H, group, deq_u + e * gu);
        rc |= orc_quantize(down_m + e * dn, H, I, group, pk, sc);
        rc |= orc_dequantize(pk, sc, H, I, group, deq_d + e * dn);
    }
    if (rc == 0)
        rc = orc_route(x, T, H, wr, bias, E, k, routed_scale, norm_topk, idx, w,
                       NULL);
    if (rc == 0) {
        int bad = 0;
#pragma omp parallel for schedule(dynamic)
        for (int64_t t = 0; t < T; ++t) {
            const float* pg[1024];
            const float* pu[1024];
            const float* pd[1024];
            if (k + n_shared > 1024) { bad = 1; continue; }
            for (int64_t j = 0; j < k; ++j) {
                int64_t e = idx[t * k + j];
                pg[j] = deq_g + e * gu; pu[j] = deq_u + e * gu; pd[j] = deq_d + e * dn;
            }
            for (int64_t s = 0; s < n_shared; ++s) {
                int64_t e = E + s;
                pg[k + s] = deq_g + e * gu; pu[k + s] = deq_u + e * gu;
                pd[k + s] = deq_d + e * dn;
            }
            if (orc_token_forward(x + t * H, H, I, k, w + t * k, pg, pu, pd,
                                  n_shared, NULL, H, y + t * H) != 0)
                bad = 1;
        }
        if (bad) rc = -2;
    }
    if (rc == 0 && idx_out) memcpy(idx_out, idx, sizeof(int32_t) * (size_t)(T * k));
    if (rc == 0 && w_out) memcpy(w_out, w, sizeof(float) * (size_t)(T * k));
    free(deq_g); free(deq_u); free(deq_d); free(pk); free(sc); free(idx); free(w);
    return rc;
}

/* RMSNorm with unit gain between stacked layers (eps 1e-5 in the stack). */
int orc_rmsnorm(const float* x, int64_t T, int64_t H, double eps, float* out) {
    if (!x || !out || T < 0 || H <= 0) return -1;
    for (int64_t t = 0; t < T; ++t) {
        double ss = 0.0;
        for (int64_t h = 0; h < H; ++h) ss += (double)x[t * H + h] * (double)x[t * H + h];
        double inv = 1.0 / sqrt(ss / (double)H + eps);
        for (int64_t h = 0; h < H; ++h) out[t * H + h] = (float)((double)x[t * H + h] * inv);
    }
    return 0;
}
