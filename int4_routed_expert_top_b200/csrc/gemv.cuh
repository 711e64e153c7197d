// gemv.cuh - CUDA-core int4 expert kernels for small batches (decode, MTP
// verify) and the weighted combine.
//
// One CTA owns 32 output rows of one unit (a routed expert picked by the batch,
// or a shared expert) and every token routed to that unit: the weights are read
// from HBM once per launch no matter how many of the unit's tokens use them
// (batch union, "github一周涨11k⭐️！25GB 内存跑 744B GLM-5.2 模型！" 三.4).  Lane l of
// every warp owns row 32*rb + l; the 8 warps split the reduction dimension in
// 64-column steps.  A lane's 16-byte loads of consecutive rows are adjacent in
// the device layout, so each warp load is one coalesced 512-byte transaction.
// Nibbles are decoded in registers exactly (see decode8) and multiplied in f32
// with packed f32x2 FMAs; partial sums of the 8 warps meet in shared memory.
//
// gate/up pass:  h[p, i] = silu(sum_c Wg'[i, c] x[c]) * (sum_c Wu'[i, c] x[c])
// down pass:     o[p, r] = sum_i Wd'[r, i] h[p, i]
// combine:       y[t]    = residual[t] + sum_j w[t, j] o[pair(t, j)] + sum_s o_shared
// with W' = q * s, the scale applied per 64-column step (gs64) or per row.
#pragma once

#include "common.cuh"

namespace coli {

constexpr int kGemvWarps = 8;
constexpr int kGemvTC = 4;  // tokens per pass over a unit's weights

struct GemvArgs {
    const uint8_t* experts;
    int64_t blob_bytes;
    BlobLayout L;
    const int32_t* n_units;
    const int32_t* unit_expert;
    const int32_t* unit_begin;
    const int32_t* unit_end;
    const int32_t* pair_tok;
    const void* x;   // [T, H] f32 or bf16 (gate/up input)
    float* h;        // [P, I] f32: gate/up output, down input
    float* o;        // [P, H] f32: down output
    int H, I, group;
};

template <bool GATEUP, int TC>
__device__ __forceinline__ void gemv_pass(const GemvArgs& a, const float4* __restrict__ xs4,
                                          float (*red)[kGemvTC][2][32], int K, int rb,
                                          const uint8_t* __restrict__ baseA,
                                          const uint8_t* __restrict__ baseB,
                                          const float* __restrict__ sA,
                                          const float* __restrict__ sB, int pc) {
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int NG64 = K / kGroupCols;
    const int K4 = K / 4;
    const bool grouped = a.group != 0;
    float accA[TC], accB[TC];
#pragma unroll
    for (int t = 0; t < TC; ++t) { accA[t] = 0.0f; accB[t] = 0.0f; }

#pragma unroll 2
    for (int g = warp; g < NG64; g += kGemvWarps) {
        // two 16-byte units (64 columns) per matrix; a unit step is 128*16 bytes
        const uint4 a0 = ldg_stream(baseA + (int64_t)(2 * g) * (kTileRows * 16));
        const uint4 a1 = ldg_stream(baseA + (int64_t)(2 * g + 1) * (kTileRows * 16));
        uint4 b0 = make_uint4(0, 0, 0, 0), b1 = b0;
        if (GATEUP) {
            b0 = ldg_stream(baseB + (int64_t)(2 * g) * (kTileRows * 16));
            b1 = ldg_stream(baseB + (int64_t)(2 * g + 1) * (kTileRows * 16));
        }
        const float scA = grouped ? __ldg(sA + (int64_t)g * kTileRows) : 1.0f;
        const float scB = (GATEUP && grouped) ? __ldg(sB + (int64_t)g * kTileRows) : 1.0f;
        const uint32_t wa[8] = {a0.x, a0.y, a0.z, a0.w, a1.x, a1.y, a1.z, a1.w};
        const uint32_t wb[8] = {b0.x, b0.y, b0.z, b0.w, b1.x, b1.y, b1.z, b1.w};
        f2_t pa[TC], pb[TC];
#pragma unroll
        for (int t = 0; t < TC; ++t) { pa[t] = 0ull; pb[t] = 0ull; }
#pragma unroll
        for (int i = 0; i < 8; ++i) {
            f2_t da[4], db[4];
            decode8(wa[i], da);
            if (GATEUP) decode8(wb[i], db);
#pragma unroll
            for (int t = 0; t < TC; ++t) {
                const float4* xp = xs4 + t * K4 + (g * kGroupCols + 8 * i) / 4;
                const float4 x0 = xp[0], x1 = xp[1];
                const f2_t x01 = f2pack(x0.x, x0.y), x23 = f2pack(x0.z, x0.w);
                const f2_t x45 = f2pack(x1.x, x1.y), x67 = f2pack(x1.z, x1.w);
                pa[t] = f2fma(da[0], x01, pa[t]);
                pa[t] = f2fma(da[1], x23, pa[t]);
                pa[t] = f2fma(da[2], x45, pa[t]);
                pa[t] = f2fma(da[3], x67, pa[t]);
                if (GATEUP) {
                    pb[t] = f2fma(db[0], x01, pb[t]);
                    pb[t] = f2fma(db[1], x23, pb[t]);
                    pb[t] = f2fma(db[2], x45, pb[t]);
                    pb[t] = f2fma(db[3], x67, pb[t]);
                }
            }
        }
#pragma unroll
        for (int t = 0; t < TC; ++t) {
            const float2 va = f2unpack(pa[t]);
            accA[t] = fmaf(scA, va.x + va.y, accA[t]);
            if (GATEUP) {
                const float2 vb = f2unpack(pb[t]);
                accB[t] = fmaf(scB, vb.x + vb.y, accB[t]);
            }
        }
    }
#pragma unroll
    for (int t = 0; t < TC; ++t) {
        red[warp][t][0][lane] = accA[t];
        red[warp][t][1][lane] = accB[t];
    }
    __syncthreads();
    if (threadIdx.x < TC * 32) {
        const int t = threadIdx.x >> 5, r = threadIdx.x & 31;
        float A = 0.0f, B = 0.0f;
#pragma unroll
        for (int w = 0; w < kGemvWarps; ++w) { A += red[w][t][0][r]; B += red[w][t][1][r]; }
        if (!grouped) {  // per-row scale, applied once after the full sum
            A *= __ldg(sA);
            if (GATEUP) B *= __ldg(sB);
        }
        const int row = rb * 32 + r;
        if (GATEUP) a.h[(int64_t)(pc + t) * a.I + row] = silu_f(A) * B;
        else        a.o[(int64_t)(pc + t) * a.H + row] = A;
    }
}

template <bool GATEUP, typename XT>
__global__ void __launch_bounds__(kGemvWarps * 32)
expert_gemv_kernel(GemvArgs a) {
    extern __shared__ float4 gemv_xs4[];  // [TC][K/4] pre-scaled input rows
    __shared__ float red[kGemvWarps][kGemvTC][2][32];
    const int K = GATEUP ? a.H : a.I;
    const int R = GATEUP ? a.I : a.H;
    const int nb = R / 32;
    const int u = blockIdx.x / nb, rb = blockIdx.x % nb;
    if (u >= *a.n_units) return;
    const int e = a.unit_expert[u], p0 = a.unit_begin[u], p1 = a.unit_end[u];
    const uint8_t* blob = a.experts + (int64_t)e * a.blob_bytes;
    const int lane = threadIdx.x & 31;
    const int row = rb * 32 + lane;
    const int mA = GATEUP ? 0 : 2;
    const int ng = a.L.ngroups[mA];
    const uint8_t* baseA = blob + a.L.codes[mA] + code_unit_offset(row, 0, K);
    const uint8_t* baseB = blob + a.L.codes[1] + code_unit_offset(row, 0, K);
    const float* sA = reinterpret_cast<const float*>(blob + a.L.scales[mA]) + scale_offset(row, 0, ng);
    const float* sB = reinterpret_cast<const float*>(blob + a.L.scales[1]) + scale_offset(row, 0, ng);
    const int K4 = K / 4;

    for (int pc = p0; pc < p1; pc += kGemvTC) {
        const int tc = min(kGemvTC, p1 - pc);
        __syncthreads();  // previous pass done with xs and red
        for (int i = threadIdx.x; i < tc * K4; i += kGemvWarps * 32) {
            const int t = i / K4, c4 = i - t * K4;
            float4 v;
            if (GATEUP) {
                const XT* src = reinterpret_cast<const XT*>(a.x) +
                                (int64_t)a.pair_tok[pc + t] * a.H + 4 * c4;
                v = make_float4(to_f32(src[0]), to_f32(src[1]), to_f32(src[2]), to_f32(src[3]));
            } else {
                v = *reinterpret_cast<const float4*>(a.h + (int64_t)(pc + t) * a.I + 4 * c4);
            }
            const int j = (4 * c4) & 7;  // column position inside its 8-nibble word
            v.x *= kPosScale(j); v.y *= kPosScale(j + 1);
            v.z *= kPosScale(j + 2); v.w *= kPosScale(j + 3);
            gemv_xs4[t * K4 + c4] = v;
        }
        __syncthreads();
        switch (tc) {
            case 4: gemv_pass<GATEUP, 4>(a, gemv_xs4, red, K, rb, baseA, baseB, sA, sB, pc); break;
            case 3: gemv_pass<GATEUP, 3>(a, gemv_xs4, red, K, rb, baseA, baseB, sA, sB, pc); break;
            case 2: gemv_pass<GATEUP, 2>(a, gemv_xs4, red, K, rb, baseA, baseB, sA, sB, pc); break;
            default: gemv_pass<GATEUP, 1>(a, gemv_xs4, red, K, rb, baseA, baseB, sA, sB, pc); break;
        }
    }
}

// y[t] = residual[t] + sum_j w[t, j] * o[inv[t, j]] + sum_s o[T*k + s*T + t]
__global__ void __launch_bounds__(256)
combine_kernel(const float* __restrict__ o, const int32_t* __restrict__ inv,
               const float* __restrict__ w, int T, int k, int n_shared, int H,
               const float* residual, float* y) {
    const int64_t i = (int64_t)blockIdx.x * 256 + threadIdx.x;
    const int H4 = H / 4;
    if (i >= (int64_t)T * H4) return;
    const int t = (int)(i / H4), c = (int)(i % H4) * 4;
    float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
    for (int j = 0; j < k; ++j) {
        const int p = inv[(int64_t)t * k + j];
        const float wj = w[(int64_t)t * k + j];
        const float4 v = *reinterpret_cast<const float4*>(o + (int64_t)p * H + c);
        acc.x = fmaf(wj, v.x, acc.x); acc.y = fmaf(wj, v.y, acc.y);
        acc.z = fmaf(wj, v.z, acc.z); acc.w = fmaf(wj, v.w, acc.w);
    }
    for (int s = 0; s < n_shared; ++s) {
        const int64_t p = (int64_t)T * k + (int64_t)s * T + t;
        const float4 v = *reinterpret_cast<const float4*>(o + p * H + c);
        acc.x += v.x; acc.y += v.y; acc.z += v.z; acc.w += v.w;
    }
    if (residual) {
        const float4 r = *reinterpret_cast<const float4*>(residual + (int64_t)t * H + c);
        acc.x = r.x + acc.x; acc.y = r.y + acc.y; acc.z = r.z + acc.z; acc.w = r.w + acc.w;
    }
    *reinterpret_cast<float4*>(y + (int64_t)t * H + c) = acc;
}

}  // namespace coli
