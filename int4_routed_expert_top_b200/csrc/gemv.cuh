// gemv.cuh - int4 expert kernels for small batches (decode, MTP verify).
//
// A CTA of 4 warps owns one unit (a routed expert picked by the batch, or a
// shared expert), 64 output rows, and every token routed to that unit, so each
// weight byte is read from HBM once per launch however many of the unit's
// tokens use it (batch union, "github一周涨11k⭐️！25GB 内存跑 744B GLM-5.2 模型！" 三.4).
// Warp w streams 16 rows over the whole reduction (gate/up) or half of it (down).
// Every step a lane loads one 16-byte unit of a fragment tile (a whole warp: one
// coalesced 512-byte block), decodes its 32 nibbles to exact fp16 in registers
// and feeds them to the tensor cores as mma.sync A fragments.  The activations
// are the B operand, split into fp16 hi + lo parts under a power-of-two scale,
// so the products carry ~22 significant bits into the f32 accumulators.  The
// weight scale (per row, or per 64-column group for gs64) and the activation's
// inverse scale are applied in f32: once at the end when both are constant along
// the reduction (CHAIN), else after every 64-column step.
//
//   gate/up: h[p, i] = silu(sum_c Wg'[i, c] x[c]) * (sum_c Wu'[i, c] x[c]),
//            stored as fp16 hi/lo with one power of two per 64 rows
//   down:    o[p, r] = sum_i Wd'[r, i] h[p, i] (f32; the two halves of the sum are
//            added into o, which the gate/up pass zeroed), and the last CTA to
//            finish a 64-row block forms y = residual + sum_j w_j o_j + sum_s o_s
#pragma once

#include "common.cuh"

namespace coli {

constexpr int kGemvWarps = 4;      // 64 rows per CTA
constexpr int kGemvMaxNT = 2;      // up to 2 column groups of 8: 8 tokens per pass
constexpr int kDownSplit = 2;      // the down reduction is split in halves

// fp16 magic constants of the nibble decode, passed as kernel parameters so
// they are read from the parameter bank instead of being rebuilt per use
struct DecodeK {
    uint32_t xlo = 0x64086408u;   // sign flip of a nibble at bits 0-3 + fp16 exponent of 1024
    uint32_t xhi = 0x64806480u;   // same for a nibble at bits 4-7
    uint32_t sub = 0x64086408u;   // 1032 = 1024 + 8
    uint32_t mul = 0x2C002C00u;   // 1/16
    uint32_t add = 0xD480D480u;   // -72 = -(1024 + 8*16)/16
};

__device__ __forceinline__ void decode_word(uint32_t w, uint32_t a[4], const DecodeK& k) {
    const uint32_t w8 = w >> 8;
    uint32_t t0, t1, t2, t3;
    asm("lop3.b32 %0, %1, 0x000F000F, %2, 0x6a;" : "=r"(t0) : "r"(w), "r"(k.xlo));
    asm("lop3.b32 %0, %1, 0x000F000F, %2, 0x6a;" : "=r"(t1) : "r"(w8), "r"(k.xlo));
    asm("lop3.b32 %0, %1, 0x00F000F0, %2, 0x6a;" : "=r"(t2) : "r"(w), "r"(k.xhi));
    asm("lop3.b32 %0, %1, 0x00F000F0, %2, 0x6a;" : "=r"(t3) : "r"(w8), "r"(k.xhi));
    asm("sub.rn.f16x2 %0, %1, %2;" : "=r"(a[0]) : "r"(t0), "r"(k.sub));
    asm("sub.rn.f16x2 %0, %1, %2;" : "=r"(a[1]) : "r"(t1), "r"(k.sub));
    asm("fma.rn.f16x2 %0, %1, %2, %3;" : "=r"(a[2]) : "r"(t2), "r"(k.mul), "r"(k.add));
    asm("fma.rn.f16x2 %0, %1, %2, %3;" : "=r"(a[3]) : "r"(t3), "r"(k.mul), "r"(k.add));
}

struct GemvArgs {
    const uint8_t* experts;
    int64_t blob_bytes;
    BlobLayout L;
    DecodeK dk;
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

// One warp: 16 rows starting at row0, reduction steps [kb0, kb1) of 64 columns,
// NT column groups of 8.  Column n of group c carries token 4c + (n & 3), hi
// part for n < 4 and lo part for n >= 4.  A register ring keeps the loads of
// the next D steps of weight units (and gs64 scales) in flight; the pass's
// activation rows and inverse scales are staged in shared memory by stage()
// (called by every thread of the CTA while the ring fills) as
// xs[token][K/64][128] fp16 and xi[token][K/64] f32.
template <bool GATEUP, int NT, bool CHAIN, typename Stage>
__device__ __forceinline__ void gemv_warp(const GemvArgs& a, const uint8_t* __restrict__ codesA,
                                          const uint8_t* __restrict__ codesB,
                                          const float* __restrict__ sA,
                                          const float* __restrict__ sB, int K, int row0,
                                          int kb0, int kb1, int tc, const __half* xs,
                                          const float* xi, Stage&& stage,
                                          float accA[NT][4], float accB[NT][4]) {
    const int lane = threadIdx.x & 31;
    const int g = lane >> 2, t = lane & 3;
    const int KB = K / 64;
    const int rt = row0 / kTileRows, b8 = (row0 % kTileRows) / 16;
    const int ng = a.group ? KB : 1;
    const int n = kb1 - kb0;
    const DecodeK dk = a.dk;
    constexpr int UNIT_STEP = 8 * 32;  // uint4 units between consecutive 64-column steps
    const uint4* pA = reinterpret_cast<const uint4*>(codesA + frag_unit_offset(rt, kb0, b8, lane, K));
    const uint4* pB = reinterpret_cast<const uint4*>(codesB + frag_unit_offset(rt, kb0, b8, lane, K));
    const uint2* pX[NT];
    bool bval[NT];
    const float* pI[NT][2];
#pragma unroll
    for (int c = 0; c < NT; ++c) {
        const int tb = 4 * c + (g & 3);
        bval[c] = tb < tc;
        pX[c] = reinterpret_cast<const uint2*>(xs + ((int64_t)(bval[c] ? tb : 0) * KB + kb0) * 128 +
                                               (g >> 2) * 64) + t;
#pragma unroll
        for (int i = 0; i < 2; ++i) {
            const int td = 4 * c + ((2 * t) & 3) + i;
            pI[c][i] = xi + (td < tc ? td : 0) * KB + kb0;
        }
    }
    const float* pS[2] = {sA + scale_offset(row0 + g, 0, ng), sB + scale_offset(row0 + g, 0, ng)};
    float cA[CHAIN ? NT : 1][4][4], cB[CHAIN ? NT : 1][4][4];  // CHAIN accumulators per sub-block
#pragma unroll
    for (int c = 0; c < NT; ++c)
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            accA[c][i] = 0.0f; accB[c][i] = 0.0f;
            if (CHAIN)
#pragma unroll
                for (int j = 0; j < 4; ++j) { cA[c][j][i] = 0.0f; cB[c][j][i] = 0.0f; }
        }
    float rowA0 = 0.f, rowA1 = 0.f, rowB0 = 0.f, rowB1 = 0.f;  // per-row scales
    if (!CHAIN && !a.group) {
        rowA0 = __ldg(pS[0]); rowA1 = __ldg(pS[0] + 8);
        if (GATEUP) { rowB0 = __ldg(pS[1]); rowB1 = __ldg(pS[1] + 8); }
    }

    // the ring holds what streams from HBM: weight units and (gs64) their scales;
    // activation fragments and their inverse scales are L1 hits shared by the
    // CTA's warps and are loaded when used
    constexpr int D = 8;
    uint4 rA[D], rB[D];
    float rS[D][4];
    auto fetch = [&](int slot, int rel) {
        rA[slot] = ldg_stream(pA + rel * UNIT_STEP);
        if (GATEUP) rB[slot] = ldg_stream(pB + rel * UNIT_STEP);
        if (!CHAIN && a.group) {
            rS[slot][0] = __ldg(pS[0] + (int64_t)(kb0 + rel) * kTileRows);
            rS[slot][1] = __ldg(pS[0] + (int64_t)(kb0 + rel) * kTileRows + 8);
            if (GATEUP) {
                rS[slot][2] = __ldg(pS[1] + (int64_t)(kb0 + rel) * kTileRows);
                rS[slot][3] = __ldg(pS[1] + (int64_t)(kb0 + rel) * kTileRows + 8);
            }
        }
    };
#pragma unroll
    for (int sl = 0; sl < D; ++sl)
        if (sl < n) fetch(sl, sl);
    stage();
    __syncthreads();

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
                    for (int j = 0; j < 4; ++j)
                        bx[c][j] = bval[c] ? pX[c][rel * 32 + 4 * j] : make_uint2(0u, 0u);
                    if (!CHAIN) { iv[c][0] = pI[c][0][rel]; iv[c][1] = pI[c][1][rel]; }
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
                    // one accumulator per 16-column sub-block: four independent MMA chains
#pragma unroll
                    for (int j = 0; j < 4; ++j) {
                        uint32_t fa[4];
                        decode_word(wa[j], fa, dk);
#pragma unroll
                        for (int c = 0; c < NT; ++c) mma_f16_16816(cA[c][j], fa, bx[c][j].x, bx[c][j].y);
                        if (GATEUP) {
                            uint32_t fb[4];
                            decode_word(wb[j], fb, dk);
#pragma unroll
                            for (int c = 0; c < NT; ++c) mma_f16_16816(cB[c][j], fb, bx[c][j].x, bx[c][j].y);
                        }
                    }
                } else {
                    // two fresh chains per step (sub-blocks 0,2 and 1,3), summed in the epilogue
                    float dA[NT][2][4], dB[NT][2][4];
#pragma unroll
                    for (int j = 0; j < 4; ++j) {
                        uint32_t fa[4];
                        decode_word(wa[j], fa, dk);
#pragma unroll
                        for (int c = 0; c < NT; ++c) {
                            if (j < 2) mma_f16_16816_zc(dA[c][j & 1], fa, bx[c][j].x, bx[c][j].y);
                            else       mma_f16_16816(dA[c][j & 1], fa, bx[c][j].x, bx[c][j].y);
                        }
                        if (GATEUP) {
                            uint32_t fb[4];
                            decode_word(wb[j], fb, dk);
#pragma unroll
                            for (int c = 0; c < NT; ++c) {
                                if (j < 2) mma_f16_16816_zc(dB[c][j & 1], fb, bx[c][j].x, bx[c][j].y);
                                else       mma_f16_16816(dB[c][j & 1], fb, bx[c][j].x, bx[c][j].y);
                            }
                        }
                    }
#pragma unroll
                    for (int c = 0; c < NT; ++c) {
                        float qa[4], qb[4];
#pragma unroll
                        for (int i = 0; i < 4; ++i) {
                            qa[i] = dA[c][0][i] + dA[c][1][i];
                            qb[i] = GATEUP ? dB[c][0][i] + dB[c][1][i] : 0.0f;
                        }
                        accA[c][0] = fmaf(sc[0] * iv[c][0], qa[0], accA[c][0]);
                        accA[c][1] = fmaf(sc[0] * iv[c][1], qa[1], accA[c][1]);
                        accA[c][2] = fmaf(sc[1] * iv[c][0], qa[2], accA[c][2]);
                        accA[c][3] = fmaf(sc[1] * iv[c][1], qa[3], accA[c][3]);
                        if (GATEUP) {
                            accB[c][0] = fmaf(sc[2] * iv[c][0], qb[0], accB[c][0]);
                            accB[c][1] = fmaf(sc[2] * iv[c][1], qb[1], accB[c][1]);
                            accB[c][2] = fmaf(sc[3] * iv[c][0], qb[2], accB[c][2]);
                            accB[c][3] = fmaf(sc[3] * iv[c][1], qb[3], accB[c][3]);
                        }
                    }
                }
            }
        }
    }
    if (CHAIN) {
#pragma unroll
        for (int c = 0; c < NT; ++c)
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                accA[c][i] = (cA[c][0][i] + cA[c][1][i]) + (cA[c][2][i] + cA[c][3][i]);
                if (GATEUP) accB[c][i] = (cB[c][0][i] + cB[c][1][i]) + (cB[c][2][i] + cB[c][3][i]);
            }
    }
    // hi + lo: lanes t and t ^ 2 hold the two parts of the same tokens
#pragma unroll
    for (int c = 0; c < NT; ++c)
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            accA[c][i] += __shfl_xor_sync(0xffffffffu, accA[c][i], 2);
            if (GATEUP) accB[c][i] += __shfl_xor_sync(0xffffffffu, accB[c][i], 2);
        }
}

// ---------------------------------------------------------------------------
// gate/up + SwiGLU.  After the shuffle, lane (g, t < 2) holds rows g, g + 8 of
// the warp's 16 and tokens 4c + 2t + {0, 1}.
// ---------------------------------------------------------------------------
// stage activation rows src[i] (i < tc) of one pass: [tc][KB][128] fp16 plus
// [tc][KB] inverse scales, 16-byte copies by every thread of the CTA
__device__ __forceinline__ void stage_rows(const __half* __restrict__ q, const float* __restrict__ inv,
                                           const int* src, int tc, int KB, __half* xs, float* xi) {
    const int per = KB * 16;  // uint4 per row
    for (int i = threadIdx.x; i < tc * per; i += kGemvWarps * 32) {
        const int r = i / per, c = i - r * per;
        reinterpret_cast<uint4*>(xs)[i] =
            __ldg(reinterpret_cast<const uint4*>(q + (int64_t)src[r] * KB * 128) + c);
    }
    for (int i = threadIdx.x; i < tc * KB; i += kGemvWarps * 32) {
        const int r = i / KB, c = i - r * KB;
        xi[i] = __ldg(inv + (int64_t)src[r] * KB + c);
    }
}

template <int NT, bool CHAIN>
__global__ void __launch_bounds__(kGemvWarps * 32)
gateup_gemv_kernel(GemvArgs a) {
    extern __shared__ uint4 gv_smem[];
    __shared__ float wmax[kGemvWarps][8 * kGemvMaxNT];
    __shared__ int src[8 * kGemvMaxNT];
    const int nrb = a.I / 64;
    const int u = blockIdx.x / nrb, rb64 = blockIdx.x % nrb;
    if (u >= *a.n_units) return;
    const int e = a.unit_expert[u], p0 = a.unit_begin[u], p1 = a.unit_end[u];
    const uint8_t* blob = a.experts + (int64_t)e * a.blob_bytes;
    const uint8_t* codesA = blob + a.L.codes[0];
    const uint8_t* codesB = blob + a.L.codes[1];
    const float* sA = reinterpret_cast<const float*>(blob + a.L.scales[0]);
    const float* sB = reinterpret_cast<const float*>(blob + a.L.scales[1]);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int g = lane >> 2, t = lane & 3;
    const int KB = a.H / 64;
    const int row0 = rb64 * 64 + warp * 16;
    __half* xs = reinterpret_cast<__half*>(gv_smem);
    float* xi = reinterpret_cast<float*>(xs + (size_t)4 * NT * KB * 128);

    // zero this CTA's share of the unit's down-projection outputs o[p0:p1, :]
    {
        float4* o4 = reinterpret_cast<float4*>(a.o + (int64_t)p0 * a.H);
        const int64_t n4 = (int64_t)(p1 - p0) * a.H / 4;
        const int64_t beg = n4 * rb64 / nrb, end = n4 * (rb64 + 1) / nrb;
        for (int64_t i = beg + threadIdx.x; i < end; i += kGemvWarps * 32)
            o4[i] = make_float4(0.f, 0.f, 0.f, 0.f);
    }

    for (int pc = p0; pc < p1; pc += 4 * NT) {
        const int tc = min(4 * NT, p1 - pc);
        __syncthreads();  // the previous pass is done with xs, xi, src and wmax
        if (threadIdx.x < tc) src[threadIdx.x] = a.pair_tok[pc + threadIdx.x];
        __syncthreads();
        float accA[NT][4], accB[NT][4];
        gemv_warp<true, NT, CHAIN>(a, codesA, codesB, sA, sB, a.H, row0, 0, KB, tc, xs, xi,
                                   [&] { stage_rows(a.xq, a.xinv, src, tc, KB, xs, xi); },
                                   accA, accB);
        // SwiGLU on rows g, g+8 for tokens 4c + 2t + {0, 1} (lanes t < 2)
        float hv[NT][4];
        float mx[NT][2];
#pragma unroll
        for (int c = 0; c < NT; ++c) {
            mx[c][0] = 0.0f; mx[c][1] = 0.0f;
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                const int tt = 4 * c + 2 * (t & 1) + (i & 1);
                const int row = row0 + g + 8 * (i >> 1);
                float ga = accA[c][i], ua = accB[c][i];
                if (CHAIN && pc + tt < p1) {
                    const float inv = xi[tt * KB];
                    ga *= __ldg(sA + scale_offset(row, 0, 1)) * inv;
                    ua *= __ldg(sB + scale_offset(row, 0, 1)) * inv;
                }
                hv[c][i] = (t < 2 && pc + tt < p1) ? silu_f(ga) * ua : 0.0f;
                mx[c][i & 1] = fmaxf(mx[c][i & 1], fabsf(hv[c][i]));
            }
        }
        // max over the warp's 16 rows per token, then over the CTA's 64 rows
#pragma unroll
        for (int c = 0; c < NT; ++c)
#pragma unroll
            for (int q = 0; q < 2; ++q) {
                float m = mx[c][q];
                m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, 4));
                m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, 8));
                m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, 16));
                if (g == 0 && t < 2) wmax[warp][4 * c + 2 * t + q] = m;
            }
        __syncthreads();
        if (t < 2) {
#pragma unroll
            for (int c = 0; c < NT; ++c)
#pragma unroll
                for (int q = 0; q < 2; ++q) {
                    const int tt = 4 * c + 2 * t + q;
                    if (pc + tt >= p1) continue;
                    float m = wmax[0][tt];
#pragma unroll
                    for (int ww = 1; ww < kGemvWarps; ++ww) m = fmaxf(m, wmax[ww][tt]);
                    float inv;
                    const float sc = act_group_scale(m, &inv);
                    const int64_t p = pc + tt;
                    __half* dst = a.hq + (p * (a.I / 64) + rb64) * 128;
#pragma unroll
                    for (int hr = 0; hr < 2; ++hr) {
                        __half hi, lo;
                        split_f16(hv[c][2 * hr + q] * sc, hi, lo);
                        const int r = warp * 16 + g + 8 * hr;
                        dst[r] = hi;
                        dst[64 + r] = lo;
                    }
                    if (warp == 0 && g == 0) a.hinv[p * (a.I / 64) + rb64] = inv;
                }
        }
    }
}

// ---------------------------------------------------------------------------
// down projection + combine.  CTA = (unit, 64-row block, half of the reduction).
// ---------------------------------------------------------------------------
template <int NT>
__global__ void __launch_bounds__(kGemvWarps * 32)
down_gemv_kernel(GemvArgs a) {
    extern __shared__ uint4 gv_smem[];
    __shared__ int last_flag;
    __shared__ int src[8 * kGemvMaxNT];
    const int nrb = a.H / 64;
    const int u = blockIdx.x / (nrb * kDownSplit);
    const int rem = blockIdx.x % (nrb * kDownSplit);
    const int rb64 = rem / kDownSplit, half = rem % kDownSplit;
    const int n_units = *a.n_units;
    if (u >= n_units) return;
    const int e = a.unit_expert[u], p0 = a.unit_begin[u], p1 = a.unit_end[u];
    const uint8_t* blob = a.experts + (int64_t)e * a.blob_bytes;
    const uint8_t* codesA = blob + a.L.codes[2];
    const float* sA = reinterpret_cast<const float*>(blob + a.L.scales[2]);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int g = lane >> 2, t = lane & 3;
    const int KB = a.I / 64;
    const int kb0 = half * KB / kDownSplit, kb1 = (half + 1) * KB / kDownSplit;
    const int row0 = rb64 * 64 + warp * 16;
    __half* xs = reinterpret_cast<__half*>(gv_smem);
    float* xi = reinterpret_cast<float*>(xs + (size_t)4 * NT * KB * 128);

    for (int pc = p0; pc < p1; pc += 4 * NT) {
        const int tc = min(4 * NT, p1 - pc);
        __syncthreads();
        if (threadIdx.x < tc) src[threadIdx.x] = pc + threadIdx.x;
        __syncthreads();
        float accA[NT][4], accB[NT][4];
        gemv_warp<false, NT, false>(a, codesA, codesA, sA, sA, a.I, row0, kb0, kb1, tc, xs, xi,
                                    [&] { stage_rows(a.hq, a.hinv, src, tc, KB, xs, xi); },
                                    accA, accB);
        if (t < 2) {
#pragma unroll
            for (int c = 0; c < NT; ++c)
#pragma unroll
                for (int i = 0; i < 4; ++i) {
                    const int tt = 4 * c + 2 * t + (i & 1);
                    // two addends per element (the halves) into a zeroed o: the sum
                    // does not depend on which half lands first
                    if (pc + tt < p1)
                        atomicAdd(a.o + (int64_t)(pc + tt) * a.H + row0 + g + 8 * (i >> 1), accA[c][i]);
                }
        }
    }

    // ---- combine: the last CTA to finish this 64-row block writes y ----
    __threadfence();
    __syncthreads();
    if (threadIdx.x == 0) {
        const int done = atomicAdd(&a.counters[rb64], 1) + 1;
        last_flag = done == n_units * kDownSplit;
    }
    __syncthreads();
    if (!last_flag) return;
    __threadfence();
    for (int q = threadIdx.x; q < a.T * 64; q += kGemvWarps * 32) {
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
    if (threadIdx.x == 0) a.counters[rb64] = 0;  // ready for the next call on this workspace
}

}  // namespace coli
