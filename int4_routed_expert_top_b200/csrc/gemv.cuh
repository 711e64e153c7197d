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
constexpr int kGemvMaxNT = 4;     // up to 4 column groups of 8: 16 tokens per pass

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

// One warp: 16 rows (block b16 of this CTA's 64), reduction groups
// [kb0, kb1), NT column groups of 8.  Column n of group c carries token
// 4c + (n & 3), hi part for n < 4 and lo part for n >= 4.
template <bool GATEUP, int NT>
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
    // this lane's B column: token pc + 4c + (g & 3), part g >> 2
    const __half* bsrc[NT];
    const float* bsig[NT];
    bool bvalid[NT];
    // this lane's D columns 2t, 2t+1: tokens pc + 4c + (2t & 3) + {0, 1}
    const float* dsig[NT][2];
#pragma unroll
    for (int c = 0; c < NT; ++c) {
        const int pb = pc + 4 * c + (g & 3);
        bvalid[c] = pb < p1;
        const int sb = bvalid[c] ? (GATEUP ? a.pair_tok[pb] : pb) : 0;
        bsrc[c] = (GATEUP ? a.xq : a.hq) + (int64_t)sb * KB * 128 + (g >> 2) * 64 + 4 * t;
        bsig[c] = (GATEUP ? a.xinv : a.hinv) + (int64_t)sb * KB;
#pragma unroll
        for (int i = 0; i < 2; ++i) {
            const int pd = pc + 4 * c + ((2 * t) & 3) + i;
            const int sd = pd < p1 ? (GATEUP ? a.pair_tok[pd] : pd) : 0;
            dsig[c][i] = (GATEUP ? a.xinv : a.hinv) + (int64_t)sd * KB;
        }
    }
    const float* rowsA0 = sA + scale_offset(row0 + g, 0, ng);
    const float* rowsB0 = sB + scale_offset(row0 + g, 0, ng);
#pragma unroll
    for (int c = 0; c < NT; ++c)
#pragma unroll
        for (int i = 0; i < 4; ++i) { accA[c][i] = 0.0f; accB[c][i] = 0.0f; }

    // weight-scale rows (hoisted for per-row scales)
    float sa0 = __ldg(rowsA0), sa1 = __ldg(rowsA0 + 8), sb0 = 0.f, sb1 = 0.f;
    if (GATEUP) { sb0 = __ldg(rowsB0); sb1 = __ldg(rowsB0 + 8); }

    // register ring: the unit loads of the next D steps are always in flight
    constexpr int D = NT == 1 ? 8 : NT == 2 ? 4 : 2;
    uint4 ringA[D], ringB[D];
#pragma unroll
    for (int i = 0; i < D; ++i) {
        if (kb0 + i < kb1) {
            const int64_t uoff = frag_unit_offset(rt, kb0 + i, b8, lane, K);
            ringA[i] = ldg_stream(codesA + uoff);
            if (GATEUP) ringB[i] = ldg_stream(codesB + uoff);
        }
    }
    for (int kb_base = kb0; kb_base < kb1; kb_base += D) {
#pragma unroll
        for (int i = 0; i < D; ++i) {
            const int kb = kb_base + i;
            if (kb >= kb1) break;
            const uint4 ua = ringA[i];
            const uint4 ub = GATEUP ? ringB[i] : make_uint4(0, 0, 0, 0);
            if (kb + D < kb1) {
                const int64_t uoff = frag_unit_offset(rt, kb + D, b8, lane, K);
                ringA[i] = ldg_stream(codesA + uoff);
                if (GATEUP) ringB[i] = ldg_stream(codesB + uoff);
            }
            // B fragments: 4 fp16 of this lane's column for each 16-column sub-block
            uint2 bf[NT][4];
#pragma unroll
            for (int c = 0; c < NT; ++c)
#pragma unroll
                for (int j = 0; j < 4; ++j)
                    bf[c][j] = bvalid[c] ? *reinterpret_cast<const uint2*>(bsrc[c] + (int64_t)kb * 128 + 16 * j)
                                         : make_uint2(0u, 0u);
            float dA[NT][4], dB[NT][4];
#pragma unroll
            for (int c = 0; c < NT; ++c)
#pragma unroll
                for (int q = 0; q < 4; ++q) { dA[c][q] = 0.0f; dB[c][q] = 0.0f; }
            const uint32_t wa[4] = {ua.x, ua.y, ua.z, ua.w};
            const uint32_t wb[4] = {ub.x, ub.y, ub.z, ub.w};
#pragma unroll
            for (int j = 0; j < 4; ++j) {
                uint32_t r0, r1, r2, r3;
                decode_frag_word(wa[j], r0, r1, r2, r3);
                // A fragment: a0 = row g (k 2t,2t+1) <- r0, a1 = row g+8 <- r2,
                // a2 = row g (k 2t+8, 2t+9) <- r1, a3 = row g+8 <- r3; the column
                // permutation is matched by the B layout (4 consecutive columns)
#pragma unroll
                for (int c = 0; c < NT; ++c) mma_f16_16816(dA[c], r0, r2, r1, r3, bf[c][j].x, bf[c][j].y);
                if (GATEUP) {
                    decode_frag_word(wb[j], r0, r1, r2, r3);
#pragma unroll
                    for (int c = 0; c < NT; ++c) mma_f16_16816(dB[c], r0, r2, r1, r3, bf[c][j].x, bf[c][j].y);
                }
            }
            // group epilogue: weight scale of rows g, g+8 times the activation
            // group's inverse scale of columns 2t, 2t+1
            if (a.group) {
                sa0 = __ldg(rowsA0 + (int64_t)kb * kTileRows);
                sa1 = __ldg(rowsA0 + (int64_t)kb * kTileRows + 8);
                if (GATEUP) {
                    sb0 = __ldg(rowsB0 + (int64_t)kb * kTileRows);
                    sb1 = __ldg(rowsB0 + (int64_t)kb * kTileRows + 8);
                }
            }
#pragma unroll
            for (int c = 0; c < NT; ++c) {
                const float i0 = __ldg(dsig[c][0] + kb), i1 = __ldg(dsig[c][1] + kb);
                accA[c][0] = fmaf(sa0 * i0, dA[c][0], accA[c][0]);
                accA[c][1] = fmaf(sa0 * i1, dA[c][1], accA[c][1]);
                accA[c][2] = fmaf(sa1 * i0, dA[c][2], accA[c][2]);
                accA[c][3] = fmaf(sa1 * i1, dA[c][3], accA[c][3]);
                if (GATEUP) {
                    accB[c][0] = fmaf(sb0 * i0, dB[c][0], accB[c][0]);
                    accB[c][1] = fmaf(sb0 * i1, dB[c][1], accB[c][1]);
                    accB[c][2] = fmaf(sb1 * i0, dB[c][2], accB[c][2]);
                    accB[c][3] = fmaf(sb1 * i1, dB[c][3], accB[c][3]);
                }
            }
        }
    }
}

template <bool GATEUP, int NT>
__device__ __forceinline__ void gemv_pass(const GemvArgs& a, float* red, const uint8_t* codesA,
                                          const uint8_t* codesB, const float* sA,
                                          const float* sB, int K, int rb64, int pc, int p1) {
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int g = lane >> 2, t = lane & 3;
    const int b16 = warp & 3, half = warp >> 2;
    const int KB = K / 64;
    const int row0 = rb64 * 64 + b16 * 16;
    float accA[NT][4], accB[NT][4];
    gemv_warp<GATEUP, NT>(a, codesA, codesB, sA, sB, K, row0, half * (KB / 2),
                          (half + 1) * (KB / 2), pc, p1, accA, accB);
    // red layout: [mat 2][half 2][64 rows][8*NT cols]
    const int C = 8 * NT;
#pragma unroll
    for (int c = 0; c < NT; ++c)
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            const int r = b16 * 16 + g + (i >> 1) * 8, n = 8 * c + 2 * t + (i & 1);
            red[((0 * 2 + half) * 64 + r) * C + n] = accA[c][i];
            if (GATEUP) red[((1 * 2 + half) * 64 + r) * C + n] = accB[c][i];
        }
    __syncthreads();
}

template <bool GATEUP, int NT>
__global__ void __launch_bounds__(kGemvWarps * 32)
expert_gemv_kernel(GemvArgs a) {
    __shared__ float red[2 * 2 * 64 * 8 * kGemvMaxNT];
    __shared__ float gmax[16][2];
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

    for (int pc = p0; pc < p1; pc += 4 * NT) {
        const int tc = min(4 * NT, p1 - pc);
        __syncthreads();  // previous pass finished with red
        gemv_pass<GATEUP, NT>(a, red, codesA, codesB, sA, sB, K, rb64, pc, p1);
        // combine halves and hi/lo: thread -> (token tt, row r)
        if (GATEUP) {
            // h for 64 rows x tc tokens, then one power-of-two scale per token
            for (int q = tid; q < tc * 64; q += kGemvWarps * 32) {
                const int tt = q / 64, r = q % 64;
                const int c = tt / 4, n = 8 * c + (tt & 3);
                const float ga = red[((0 * 2 + 0) * 64 + r) * C + n] + red[((0 * 2 + 1) * 64 + r) * C + n] +
                                 red[((0 * 2 + 0) * 64 + r) * C + n + 4] + red[((0 * 2 + 1) * 64 + r) * C + n + 4];
                const float ua = red[((1 * 2 + 0) * 64 + r) * C + n] + red[((1 * 2 + 1) * 64 + r) * C + n] +
                                 red[((1 * 2 + 0) * 64 + r) * C + n + 4] + red[((1 * 2 + 1) * 64 + r) * C + n + 4];
                const float hv = silu_f(ga) * ua;
                red[((0 * 2 + 0) * 64 + r) * C + n] = hv;  // reuse: h in slot (0, 0, r, n)
                float m = fabsf(hv);
#pragma unroll
                for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
                if ((q & 31) == 0) gmax[tt][(q >> 5) & 1] = m;
            }
            __syncthreads();
            for (int q = tid; q < tc * 64; q += kGemvWarps * 32) {
                const int tt = q / 64, r = q % 64;
                const int c = tt / 4, n = 8 * c + (tt & 3);
                const float hv = red[((0 * 2 + 0) * 64 + r) * C + n];
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
                const int c = tt / 4, n = 8 * c + (tt & 3);
                const float v = red[((0 * 2 + 0) * 64 + r) * C + n] + red[((0 * 2 + 1) * 64 + r) * C + n] +
                                red[((0 * 2 + 0) * 64 + r) * C + n + 4] + red[((0 * 2 + 1) * 64 + r) * C + n + 4];
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
