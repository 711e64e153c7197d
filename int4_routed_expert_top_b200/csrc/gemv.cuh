// gemv.cuh - int4 expert kernels for small batches (decode, MTP verify).
//
// A CTA owns one unit (a routed expert picked by the batch, or a shared expert)
// and 64 output rows, and every token routed to that unit, so each weight byte
// is read from HBM once per launch however many of the unit's tokens use it
// (batch union, "github一周涨11k⭐️！25GB 内存跑 744B GLM-5.2 模型！" 三.4).  Warp w
// takes 16-row block w % 4 and half w / 4 of the reduction.  Every step a lane
// loads one 16-byte unit of a fragment tile (a whole warp: one coalesced 512-byte
// block), decodes its 32 nibbles to exact fp16 in registers and feeds them to
// the tensor cores as mma.sync A fragments.  The activations are the B operand,
// split into fp16 hi + lo parts scaled by a power of two per 64-column group,
// so the products carry ~22 significant bits into the f32 accumulators.  After
// each 64-column group the partial product is multiplied by the weight scale
// (per row, or per group for gs64) and by the activation group's inverse power
// of two, in f32.
//
//   gate/up: h[p, i] = silu(sum_c Wg'[i, c] x[c]) * (sum_c Wu'[i, c] x[c])
//            written as fp16 hi/lo per 64-row group with its power-of-two scale
//   down:    o[p, r] = sum_i Wd'[r, i] h[p, i]  (f32), and the last CTA to finish
//            a 64-row block forms y = residual + sum_j w_j o_j + sum_s o_shared
#pragma once

#include "common.cuh"

namespace coli {

constexpr int kGemvWarps = 8;
constexpr int kGemvMaxNT = 2;     // up to 2 column groups of 8: 8 tokens per pass

struct GemvArgs {
    const uint8_t* experts;
    int64_t blob_bytes;
    BlobLayout L;
    const int32_t* n_units;
    const int32_t* unit_expert;
    const int32_t* unit_begin;
    const int32_t* unit_end;
    const int32_t* pair_tok;
    const __half* xq;     // [T][H/64][128]  hi (64) then lo (64), scaled
    const float* xinv;    // [T][H/64]       inverse power-of-two scales
    __half* hq;           // [P][I/64][128]
    float* hinv;          // [P][I/64]
    float* o;             // [P][H]
    // combine (down pass)
    int32_t* counters;    // [H/64], zero on entry
    const int32_t* inv;   // [T*k] pair of (t, j)
    const float* w;       // [T*k]
    const float* residual;
    float* y;
    int T, k, n_shared;
    int H, I, group;
};

// One warp: 16 rows (block b16 of this CTA's 64), reduction steps [kb0, kb1)
// of 64 columns, NT column groups of 8.  Column n of group c carries token
// 4c + (n & 3), hi part for n < 4 and lo part for n >= 4.
//
// CHAIN (per-row weight scales and one activation scale per token): the MMAs
// accumulate straight through K and the caller applies both scales at the end.
// Otherwise every 64-column step ends with acc += (s_row * inv_act) * D_step.
// A register ring keeps the loads of the next D steps in flight: weight units,
// activation fragments and (per-step mode) the scales they need.
template <bool GATEUP, int NT, bool CHAIN>
__device__ __forceinline__ void gemv_warp(const GemvArgs& a, const uint8_t* __restrict__ codesA,
                                          const uint8_t* __restrict__ codesB,
                                          const float* __restrict__ sA,
                                          const float* __restrict__ sB, int K, int row0,
                                          int kb0, int kb1, int pc, int p1,
                                          float accA[NT][4], float accB[NT][4]) {
    const int lane = threadIdx.x & 31;
    const int g = lane >> 2, t = lane & 3;
    const int KB = K / 64;
    const int rt = row0 / kTileRows, b8 = (row0 % kTileRows) / 16;
    const int ng = a.group ? KB : 1;
    const int n = kb1 - kb0;
    constexpr int UNIT_STEP = 8 * 32;  // uint4 units between consecutive 64-column steps
    const uint4* pA = reinterpret_cast<const uint4*>(codesA + frag_unit_offset(rt, kb0, b8, lane, K));
    const uint4* pB = reinterpret_cast<const uint4*>(codesB + frag_unit_offset(rt, kb0, b8, lane, K));
    // activation fragments of this lane's B column: 4 fp16 per 16-column sub-block
    const uint2* pX[NT];
    bool bval[NT];
    // inverse activation scales of this lane's D columns 2t, 2t+1
    const float* pI[NT][2];
#pragma unroll
    for (int c = 0; c < NT; ++c) {
        const int pb = pc + 4 * c + (g & 3);
        bval[c] = pb < p1;
        const int sb = bval[c] ? (GATEUP ? a.pair_tok[pb] : pb) : 0;
        const __half* base = (GATEUP ? a.xq : a.hq) + ((int64_t)sb * KB + kb0) * 128 + (g >> 2) * 64;
        pX[c] = reinterpret_cast<const uint2*>(base) + t;
#pragma unroll
        for (int i = 0; i < 2; ++i) {
            const int pd = pc + 4 * c + ((2 * t) & 3) + i;
            const int sd = pd < p1 ? (GATEUP ? a.pair_tok[pd] : pd) : 0;
            pI[c][i] = (GATEUP ? a.xinv : a.hinv) + (int64_t)sd * KB + kb0;
        }
    }
    const float* pS[2] = {sA + scale_offset(row0 + g, 0, ng), sB + scale_offset(row0 + g, 0, ng)};
#pragma unroll
    for (int c = 0; c < NT; ++c)
#pragma unroll
        for (int i = 0; i < 4; ++i) { accA[c][i] = 0.0f; accB[c][i] = 0.0f; }
    float rowA0 = 0.f, rowA1 = 0.f, rowB0 = 0.f, rowB1 = 0.f;  // per-row scales
    if (!CHAIN && !a.group) {
        rowA0 = __ldg(pS[0]); rowA1 = __ldg(pS[0] + 8);
        if (GATEUP) { rowB0 = __ldg(pS[1]); rowB1 = __ldg(pS[1] + 8); }
    }

    constexpr int D = NT == 1 ? 4 : 2;
    uint4 rA[D], rB[D];
    uint2 rX[D][NT][4];
    float rI[D][NT][2], rS[D][4];
    auto fetch = [&](int slot, int rel) {
        rA[slot] = ldg_stream(pA + rel * UNIT_STEP);
        if (GATEUP) rB[slot] = ldg_stream(pB + rel * UNIT_STEP);
#pragma unroll
        for (int c = 0; c < NT; ++c)
#pragma unroll
            for (int j = 0; j < 4; ++j)
                rX[slot][c][j] = bval[c] ? __ldg(pX[c] + rel * 32 + 4 * j) : make_uint2(0u, 0u);
        if (!CHAIN) {
#pragma unroll
            for (int c = 0; c < NT; ++c) {
                rI[slot][c][0] = __ldg(pI[c][0] + rel);
                rI[slot][c][1] = __ldg(pI[c][1] + rel);
            }
            if (a.group) {
                rS[slot][0] = __ldg(pS[0] + (int64_t)(kb0 + rel) * kTileRows);
                rS[slot][1] = __ldg(pS[0] + (int64_t)(kb0 + rel) * kTileRows + 8);
                if (GATEUP) {
                    rS[slot][2] = __ldg(pS[1] + (int64_t)(kb0 + rel) * kTileRows);
                    rS[slot][3] = __ldg(pS[1] + (int64_t)(kb0 + rel) * kTileRows + 8);
                }
            }
        }
    };
#pragma unroll
    for (int sl = 0; sl < D; ++sl)
        if (sl < n) fetch(sl, sl);

    for (int base = 0; base < n; base += D) {
#pragma unroll
        for (int sl = 0; sl < D; ++sl) {
            const int rel = base + sl;
            if (rel < n) {
                const uint4 ua = rA[sl];
                const uint4 ub = GATEUP ? rB[sl] : ua;
                uint2 bx[NT][4];
                float iv[NT][2], sc[4];
#pragma unroll
                for (int c = 0; c < NT; ++c) {
#pragma unroll
                    for (int j = 0; j < 4; ++j) bx[c][j] = rX[sl][c][j];
                    if (!CHAIN) { iv[c][0] = rI[sl][c][0]; iv[c][1] = rI[sl][c][1]; }
                }
                if (!CHAIN) {
                    if (a.group) {
                        sc[0] = rS[sl][0]; sc[1] = rS[sl][1];
                        sc[2] = GATEUP ? rS[sl][2] : 0.f; sc[3] = GATEUP ? rS[sl][3] : 0.f;
                    } else {
                        sc[0] = rowA0; sc[1] = rowA1; sc[2] = rowB0; sc[3] = rowB1;
                    }
                }
                if (rel + D < n) fetch(sl, rel + D);
                const uint32_t wa[4] = {ua.x, ua.y, ua.z, ua.w};
                const uint32_t wb[4] = {ub.x, ub.y, ub.z, ub.w};
                if (CHAIN) {
#pragma unroll
                    for (int j = 0; j < 4; ++j) {
                        uint32_t fa[4];
                        decode_frag_word(wa[j], fa);
#pragma unroll
                        for (int c = 0; c < NT; ++c) mma_f16_16816(accA[c], fa, bx[c][j].x, bx[c][j].y);
                        if (GATEUP) {
                            uint32_t fb[4];
                            decode_frag_word(wb[j], fb);
#pragma unroll
                            for (int c = 0; c < NT; ++c) mma_f16_16816(accB[c], fb, bx[c][j].x, bx[c][j].y);
                        }
                    }
                } else {
                    float dA[NT][4], dB[NT][4];
#pragma unroll
                    for (int j = 0; j < 4; ++j) {
                        uint32_t fa[4];
                        decode_frag_word(wa[j], fa);
#pragma unroll
                        for (int c = 0; c < NT; ++c) {
                            if (j == 0) mma_f16_16816_zc(dA[c], fa, bx[c][j].x, bx[c][j].y);
                            else        mma_f16_16816(dA[c], fa, bx[c][j].x, bx[c][j].y);
                        }
                        if (GATEUP) {
                            uint32_t fb[4];
                            decode_frag_word(wb[j], fb);
#pragma unroll
                            for (int c = 0; c < NT; ++c) {
                                if (j == 0) mma_f16_16816_zc(dB[c], fb, bx[c][j].x, bx[c][j].y);
                                else        mma_f16_16816(dB[c], fb, bx[c][j].x, bx[c][j].y);
                            }
                        }
                    }
#pragma unroll
                    for (int c = 0; c < NT; ++c) {
                        accA[c][0] = fmaf(sc[0] * iv[c][0], dA[c][0], accA[c][0]);
                        accA[c][1] = fmaf(sc[0] * iv[c][1], dA[c][1], accA[c][1]);
                        accA[c][2] = fmaf(sc[1] * iv[c][0], dA[c][2], accA[c][2]);
                        accA[c][3] = fmaf(sc[1] * iv[c][1], dA[c][3], accA[c][3]);
                        if (GATEUP) {
                            accB[c][0] = fmaf(sc[2] * iv[c][0], dB[c][0], accB[c][0]);
                            accB[c][1] = fmaf(sc[2] * iv[c][1], dB[c][1], accB[c][1]);
                            accB[c][2] = fmaf(sc[3] * iv[c][0], dB[c][2], accB[c][2]);
                            accB[c][3] = fmaf(sc[3] * iv[c][1], dB[c][3], accB[c][3]);
                        }
                    }
                }
            }
        }
    }
}

template <bool GATEUP, int NT, bool CHAIN>
__device__ __forceinline__ void gemv_pass(const GemvArgs& a, float* red, const uint8_t* codesA,
                                          const uint8_t* codesB, const float* sA,
                                          const float* sB, int K, int rb64, int pc, int p1) {
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int g = lane >> 2, t = lane & 3;
    const int b16 = warp & 3, half = warp >> 2;
    const int KB = K / 64;
    const int row0 = rb64 * 64 + b16 * 16;
    float accA[NT][4], accB[NT][4];
    gemv_warp<GATEUP, NT, CHAIN>(a, codesA, codesB, sA, sB, K, row0, half * (KB / 2),
                                 (half + 1) * (KB / 2), pc, p1, accA, accB);
    // red layout: [mat 2][half 2][64 rows][8*NT cols]
    const int C = 8 * NT;
#pragma unroll
    for (int c = 0; c < NT; ++c)
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            const int r = b16 * 16 + g + (i >> 1) * 8, nn = 8 * c + 2 * t + (i & 1);
            red[((0 * 2 + half) * 64 + r) * C + nn] = accA[c][i];
            if (GATEUP) red[((1 * 2 + half) * 64 + r) * C + nn] = accB[c][i];
        }
    __syncthreads();
}

template <bool GATEUP, int NT, bool CHAIN>
__global__ void __launch_bounds__(kGemvWarps * 32)
expert_gemv_kernel(GemvArgs a) {
    __shared__ float red[2 * 2 * 64 * 8 * kGemvMaxNT];
    __shared__ float gmax[8 * kGemvMaxNT][2];
    __shared__ int last_flag;
    const int K = GATEUP ? a.H : a.I;
    const int R = GATEUP ? a.I : a.H;
    const int nrb = R / 64;
    const int u = blockIdx.x / nrb, rb64 = blockIdx.x % nrb;
    if (u >= *a.n_units) return;
    const int e = a.unit_expert[u], p0 = a.unit_begin[u], p1 = a.unit_end[u];
    const uint8_t* blob = a.experts + (int64_t)e * a.blob_bytes;
    const int mA = GATEUP ? 0 : 2;
    const uint8_t* codesA = blob + a.L.codes[mA];
    const uint8_t* codesB = blob + a.L.codes[1];
    const float* sA = reinterpret_cast<const float*>(blob + a.L.scales[mA]);
    const float* sB = reinterpret_cast<const float*>(blob + a.L.scales[1]);
    const int C = 8 * NT;
    const int tid = threadIdx.x;
    const int KB = K / 64;

    for (int pc = p0; pc < p1; pc += 4 * NT) {
        const int tc = min(4 * NT, p1 - pc);
        __syncthreads();  // previous pass finished with red
        gemv_pass<GATEUP, NT, CHAIN>(a, red, codesA, codesB, sA, sB, K, rb64, pc, p1);
        // combine halves and hi/lo: thread -> (token tt, row r)
        if (GATEUP) {
            // h for 64 rows x tc tokens, then one power-of-two scale per token
            for (int q = tid; q < tc * 64; q += kGemvWarps * 32) {
                const int tt = q / 64, r = q % 64;
                const int c = tt / 4, nn = 8 * c + (tt & 3);
                float ga = red[((0 * 2 + 0) * 64 + r) * C + nn] + red[((0 * 2 + 1) * 64 + r) * C + nn] +
                           red[((0 * 2 + 0) * 64 + r) * C + nn + 4] + red[((0 * 2 + 1) * 64 + r) * C + nn + 4];
                float ua = red[((1 * 2 + 0) * 64 + r) * C + nn] + red[((1 * 2 + 1) * 64 + r) * C + nn] +
                           red[((1 * 2 + 0) * 64 + r) * C + nn + 4] + red[((1 * 2 + 1) * 64 + r) * C + nn + 4];
                if (CHAIN) {  // per-row weight scale and the token's activation scale
                    const float inv = __ldg(a.xinv + (int64_t)a.pair_tok[pc + tt] * KB);
                    const int row = rb64 * 64 + r;
                    ga *= __ldg(sA + scale_offset(row, 0, 1)) * inv;
                    ua *= __ldg(sB + scale_offset(row, 0, 1)) * inv;
                }
                const float hv = silu_f(ga) * ua;
                red[((0 * 2 + 0) * 64 + r) * C + nn] = hv;  // reuse: h in slot (0, 0, r, nn)
                float m = fabsf(hv);
#pragma unroll
                for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
                if ((q & 31) == 0) gmax[tt][(q >> 5) & 1] = m;
            }
            __syncthreads();
            for (int q = tid; q < tc * 64; q += kGemvWarps * 32) {
                const int tt = q / 64, r = q % 64;
                const int c = tt / 4, nn = 8 * c + (tt & 3);
                const float hv = red[((0 * 2 + 0) * 64 + r) * C + nn];
                float inv;
                const float sc = act_group_scale(fmaxf(gmax[tt][0], gmax[tt][1]), &inv);
                __half hi, lo;
                split_f16(hv * sc, hi, lo);
                const int64_t p = pc + tt;
                __half* dst = a.hq + (p * (a.I / 64) + rb64) * 128;
                dst[r] = hi;
                dst[64 + r] = lo;
                if (r == 0) a.hinv[p * (a.I / 64) + rb64] = inv;
            }
        } else {
            for (int q = tid; q < tc * 64; q += kGemvWarps * 32) {
                const int tt = q / 64, r = q % 64;
                const int c = tt / 4, nn = 8 * c + (tt & 3);
                float v = red[((0 * 2 + 0) * 64 + r) * C + nn] + red[((0 * 2 + 1) * 64 + r) * C + nn] +
                          red[((0 * 2 + 0) * 64 + r) * C + nn + 4] + red[((0 * 2 + 1) * 64 + r) * C + nn + 4];
                a.o[(int64_t)(pc + tt) * a.H + rb64 * 64 + r] = v;
            }
        }
    }
    if (GATEUP) return;

    // ---- combine: the last unit to finish this 64-row block writes y ----
    __threadfence();
    __syncthreads();
    if (tid == 0) {
        const int done = atomicAdd(&a.counters[rb64], 1) + 1;
        last_flag = done == *a.n_units;
    }
    __syncthreads();
    if (!last_flag) return;
    __threadfence();
    for (int q = tid; q < a.T * 64; q += kGemvWarps * 32) {
        const int tt = q / 64, r = rb64 * 64 + q % 64;
        float acc = 0.0f;
        for (int j = 0; j < a.k; ++j) {
            const int p = __ldcg(a.inv + (int64_t)tt * a.k + j);
            acc = fmaf(__ldcg(a.w + (int64_t)tt * a.k + j), __ldcg(a.o + (int64_t)p * a.H + r), acc);
        }
        for (int s = 0; s < a.n_shared; ++s)
            acc += __ldcg(a.o + ((int64_t)a.T * a.k + (int64_t)s * a.T + tt) * a.H + r);
        if (a.residual) acc = a.residual[(int64_t)tt * a.H + r] + acc;
        a.y[(int64_t)tt * a.H + r] = acc;
    }
    if (tid == 0) a.counters[rb64] = 0;  // ready for the next call on this workspace
}

}  // namespace coli
