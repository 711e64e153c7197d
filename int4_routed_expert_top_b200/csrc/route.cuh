// route.cuh - router logits (one kernel per batch-size range), sigmoid +
// bias-corrected top-k, the batch union, and the activation operands of the
// expert kernels (fp16 hi/lo digits; s8 digits for the fused kernel).
//
// Router ("解密GLM-5.2-colibri-int4-with-int8-mtp" 模型架构深度解析; "github一周涨11k
// ⭐️！25GB 内存跑 744B GLM-5.2 模型！" 三.1 and 四.3): z = W_r x in f32 (plain FMA on
// CUDA cores, no TF32), s = sigmoid(z), the k largest s + b win (ties to the
// lower index), weights come from s alone.
// Union (same article 三.4; "colibrì 實戰指南" 二): (token, slot) pairs grouped by
// expert, experts ascending, tokens ascending inside an expert.
#pragma once

#include "common.cuh"
#include "pipeline.cuh"

namespace coli {

constexpr int kMaxKS = 8;

// Four consecutive activations as f32 (16-byte f32 or 8-byte bf16 load).
__device__ __forceinline__ float4 load4_f32(const float* p) {
    return *reinterpret_cast<const float4*>(p);
}
__device__ __forceinline__ float4 load4_f32(const __nv_bfloat16* p) {
    const uint2 u = *reinterpret_cast<const uint2*>(p);
    return make_float4(__uint_as_float(u.x << 16), __uint_as_float(u.x & 0xFFFF0000u),
                       __uint_as_float(u.y << 16), __uint_as_float(u.y & 0xFFFF0000u));
}

// ---------------------------------------------------------------------------
// fp16 hi/lo activation operand, one CTA (256 threads) per token: one power of
// two per token from the row's largest magnitude, xq[t][g][0..64) = hi and
// [64..128) = lo of x * 2^sh for 64-column group g, xinv[t][g] = 2^-sh.
// ---------------------------------------------------------------------------
template <typename XT>
__device__ __forceinline__ void act_quant_token(const XT* __restrict__ x, int H, int t,
                                                __half* __restrict__ xq, float* __restrict__ xinv) {
    __shared__ float part[8];
    const XT* row = x + (int64_t)t * H;
    float m = 0.0f;
    for (int c = threadIdx.x; c < H; c += 256) m = fmaxf(m, fabsf(to_f32(row[c])));
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
    if ((threadIdx.x & 31) == 0) part[threadIdx.x >> 5] = m;
    __syncthreads();
    m = part[0];
#pragma unroll
    for (int i = 1; i < 8; ++i) m = fmaxf(m, part[i]);
    float inv;
    const float sc = act_group_scale(m, &inv);
    const int KB = H / 64;
    for (int c = 2 * threadIdx.x; c < H; c += 512) {
        __half h0, l0, h1, l1;
        split_f16(to_f32(row[c]) * sc, h0, l0);
        split_f16(to_f32(row[c + 1]) * sc, h1, l1);
        __half* dst = xq + ((int64_t)t * KB + c / 64) * 128 + (c % 64);
        *reinterpret_cast<__half2*>(dst) = __halves2half2(h0, h1);
        *reinterpret_cast<__half2*>(dst + 64) = __halves2half2(l0, l1);
    }
    for (int kb = threadIdx.x; kb < KB; kb += 256) xinv[(int64_t)t * KB + kb] = inv;
}

template <typename XT>
__global__ void __launch_bounds__(256)
act_quant_kernel(const XT* __restrict__ x, int T, int H, __half* __restrict__ xq,
                 float* __restrict__ xinv) {
    act_quant_token(x, H, blockIdx.x, xq, xinv);
}

// ---------------------------------------------------------------------------
// Router logits, small batches: one warp per (expert row, K slice).  The warp
// issues all of its 16-byte loads of W_r before the first FMA.  Partial sums go
// to zpart[ks][t][e]; top-k adds the slices in order.  Blocks past the router's
// share build the fp16 activation operand (xq) when xq != nullptr.
// ---------------------------------------------------------------------------
constexpr int kRouterMaxSlice = 1024;  // columns per warp slice (<= 8 loads per lane)
constexpr int kRouterMaxT = 64;        // tokens per call of the small-batch router

// ---------------------------------------------------------------------------
// s8 activation operand of the fused small-batch kernel (fused.cuh): each value
// becomes two signed 8-bit digits of a 15-bit fixed-point number under one
// power-of-two scale per 256 columns (one gate/up stage of that kernel), so a
// few outlier channels coarsen only the 256-column group they sit in.
// ---------------------------------------------------------------------------
// Byte position of column c (0..63) of a 64-column step in the activation
// operand: lane t's 16 bytes hold columns 4t..4t+3, 16+4t.., 32+4t.., 48+4t..,
// i.e. its B registers of the two k32 halves of the step.
__host__ __device__ inline int fz_act_pos(int c) {
    return 16 * ((c % 16) / 4) + 4 * (c / 16) + (c % 4);
}

// Record of one token's 256-column group: 4 steps x (64 hi + 64 lo bytes), the
// f32 inverse scale 2^-sh at byte 512, at byte 516 the ratio of the previous
// group's inverse scale to this one's (a power of two; 1 for the first group),
// zero padding to 576 bytes (a multiple of 16 for bulk copies; 64 mod 128 so
// that records of consecutive tokens in shared memory start in other banks).
// A consumer summing over the groups keeps its running sum in the current
// group's units and multiplies it by the ratio on entering the next group,
// which is exact.
constexpr int kActRec = 576;
constexpr int kActRecScale = 512;
constexpr int kActRecRatio = 516;
constexpr int kActMaxGroups = 64;  // H <= 16384 on the fused path

// Power-of-two scale for a block whose largest magnitude is m: returns sh with
// m * 2^sh in [2^13, 2^14) and *inv = 2^-sh (1 for an all-zero block).
__device__ __forceinline__ float fz_scale(float m, float* inv) {
    if (!(m > 0.0f) || !isfinite(m)) { *inv = 1.0f; return 1.0f; }
    int e;
    frexpf(m, &e);
    const int sh = max(-100, min(100, 14 - e));
    *inv = ldexpf(1.0f, -sh);
    return ldexpf(1.0f, sh);
}

// x16 = rint(v * sc) split into hi (high digit) and lo (low digit)
__device__ __forceinline__ void fz_split(float v, float sc, int& hi, int& lo) {
    const int x = __float2int_rn(v * sc);
    hi = (x + 128) >> 8;
    lo = x - 256 * hi;
}

// s8 activation operand of one token, one CTA of 256 threads: records
// xq8[t][H/256][kActRec] as above (H a multiple of 256, at most 16384).
// Thread tid owns columns 4 tid + 1024 j; the 64 threads of two consecutive
// warps cover one 256-column group.  First every group's largest magnitude
// (the row read once, up to 8 blocks of 1024 columns in flight together), then
// the digits, scales and ratios.
template <typename XT>
__device__ __forceinline__ void act_quant8_token(const XT* __restrict__ x, int H, int t,
                                                 int8_t* __restrict__ xq8) {
    constexpr int kJ = 8;
    __shared__ float part8[kJ][8];
    __shared__ float ginv[kActMaxGroups];
    const XT* row = x + (int64_t)t * H;
    const bool vec = (reinterpret_cast<uintptr_t>(row) & (4 * sizeof(XT) - 1)) == 0;
    const int warp = threadIdx.x >> 5;
    const int G = H / 256;
    int8_t* trec = xq8 + (int64_t)t * G * kActRec;
    auto load = [&](int c) {
        return vec ? load4_f32(row + c)
                   : make_float4(to_f32(row[c]), to_f32(row[c + 1]), to_f32(row[c + 2]),
                                 to_f32(row[c + 3]));
    };
    // pass 1: the inverse scale of every group
    for (int j0 = 0; j0 * 1024 < H; j0 += kJ) {
        float4 v[kJ];
#pragma unroll
        for (int jj = 0; jj < kJ; ++jj) {
            const int c = 4 * threadIdx.x + 1024 * (j0 + jj);
            v[jj] = c < H ? load(c) : make_float4(0.0f, 0.0f, 0.0f, 0.0f);
        }
#pragma unroll
        for (int jj = 0; jj < kJ; ++jj) {
            float m = fmaxf(fmaxf(fabsf(v[jj].x), fabsf(v[jj].y)),
                            fmaxf(fabsf(v[jj].z), fabsf(v[jj].w)));
#pragma unroll
            for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
            if ((threadIdx.x & 31) == 0) part8[jj][warp] = m;
        }
        __syncthreads();
        if (threadIdx.x < kJ * 4) {  // group 4 (j0 + jj) + w2 of this block of columns
            const int jj = threadIdx.x >> 2, w2 = threadIdx.x & 3;
            const int g = 4 * (j0 + jj) + w2;
            if (g < G) {
                float inv;
                fz_scale(fmaxf(part8[jj][2 * w2], part8[jj][2 * w2 + 1]), &inv);
                ginv[g] = inv;
            }
        }
        __syncthreads();
    }
    // pass 2: digits (the row again, now from L1/L2), scales, ratios
    for (int c = 4 * threadIdx.x; c < H; c += 1024) {
        const float4 v = load(c);
        const int g = c / 256;
        const float inv = ginv[g];
        const float sc = 1.0f / inv;  // a power of two: exact
        const float f[4] = {v.x, v.y, v.z, v.w};
        uint32_t wh = 0, wl = 0;
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            int hi, lo;
            fz_split(f[i], sc, hi, lo);
            wh |= (uint32_t)(hi & 0xFF) << (8 * i);
            wl |= (uint32_t)(lo & 0xFF) << (8 * i);
        }
        int8_t* rec = trec + (int64_t)g * kActRec;
        int8_t* step = rec + ((c % 256) / 64) * 128;
        const int pos = fz_act_pos(c % 64);
        *reinterpret_cast<uint32_t*>(step + pos) = wh;
        *reinterpret_cast<uint32_t*>(step + 64 + pos) = wl;
        const int lt = (c % 256) / 4;  // thread within the group
        if (lt < (kActRec - kActRecScale) / 16) {  // scale, ratio, then zero padding
            const float ratio = g == 0 ? 1.0f : ginv[g - 1] / inv;
            const uint4 z = lt == 0 ? make_uint4(__float_as_uint(inv), __float_as_uint(ratio), 0u, 0u)
                                    : make_uint4(0u, 0u, 0u, 0u);
            *reinterpret_cast<uint4*>(rec + kActRecScale + 16 * lt) = z;
        }
    }
}

// Extra blocks after the router's: one per token for the activation operand
// (fp16 hi/lo into xq, or s8 digits into xq8 for the fused kernel), then one
// that clears `zero_n` ints at `zero` (the fused kernel's counters).
struct RouterExtras {
    __half* xq = nullptr;
    float* xinv = nullptr;
    int8_t* xq8 = nullptr;
    int32_t* zero = nullptr;
    int zero_n = 0;
    int32_t* err = nullptr;  // device error flags, cleared by the same block
    // scores for the fused kernel: when set, zpart receives s = sigmoid(z) and
    // sel receives s + bias instead of the logits
    float* sel = nullptr;
    const float* bias = nullptr;
};


template <typename XT>
__global__ void __launch_bounds__(256)
router_gemv_kernel(const XT* __restrict__ x, int T, int H, const float* __restrict__ wr,
                   int E, int KS, float* __restrict__ zpart, int router_blocks,
                   RouterExtras ex) {
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    // the dependent fused kernel may start its prologue (it waits for this
    // grid's completion before reading anything written here)
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
    // launched as a programmatic dependent: x may come from the previous grid
    asm volatile("griddepcontrol.wait;" ::: "memory");
    if ((int)blockIdx.x >= router_blocks) {
        const int b = blockIdx.x - router_blocks;
        if (b < T) {  // one CTA per token: activation operand
            if (ex.xq) act_quant_token(x, H, b, ex.xq, ex.xinv);
            if (ex.xq8) act_quant8_token(x, H, b, ex.xq8);
        } else {
            for (int i = threadIdx.x; i < ex.zero_n; i += 256) ex.zero[i] = 0;
            if (threadIdx.x == 0 && ex.err) *ex.err = 0;
        }
        return;
    }
    // The CTA's 8 warps are the KS slices of 8 / KS experts (KS divides 8): the
    // slices are summed here, in slice order, and z[t][e] is written.
    __shared__ float part[8][kRouterMaxT];
    const int gw = blockIdx.x * 8 + warp;
    const int e = gw / KS, ks = gw % KS;
    const bool valid = e < E;
    const int SL = H / KS;  // multiple of 128, at most kRouterMaxSlice
    const int per = 8 / KS;  // experts of this CTA
    // this thread's first output's bias, loaded beside the weights
    float bias0 = 0.0f;
    if (ex.sel && (int)threadIdx.x < per * T) {
        const int ee = blockIdx.x * per + (int)threadIdx.x / T;
        if (ee < E) bias0 = __ldg(ex.bias + ee);
    }
    if (valid) {
        const float* wrow = wr + (int64_t)e * H + (int64_t)ks * SL;
        float4 wv[kRouterMaxSlice / 128];
#pragma unroll
        for (int i = 0; i < kRouterMaxSlice / 128; ++i)
            if (i * 128 < SL) wv[i] = __ldg(reinterpret_cast<const float4*>(wrow + i * 128 + lane * 4));
        // vector loads when the rows are aligned for them (H is a multiple of 128)
        const bool vec = (reinterpret_cast<uintptr_t>(x) & (4 * sizeof(XT) - 1)) == 0;
        for (int t = 0; t < T; ++t) {
            const XT* xr = x + (int64_t)t * H + (int64_t)ks * SL + lane * 4;
            float acc = 0.0f;
#pragma unroll
            for (int i = 0; i < kRouterMaxSlice / 128; ++i) {
                if (i * 128 < SL) {
                    const XT* xp = xr + i * 128;
                    const float4 xv = vec ? load4_f32(xp)
                                          : make_float4(to_f32(xp[0]), to_f32(xp[1]),
                                                        to_f32(xp[2]), to_f32(xp[3]));
                    acc = fmaf(wv[i].x, xv.x, acc);
                    acc = fmaf(wv[i].y, xv.y, acc);
                    acc = fmaf(wv[i].z, xv.z, acc);
                    acc = fmaf(wv[i].w, xv.w, acc);
                }
            }
            acc = warp_sum(acc);
            if (lane == 0) part[warp][t] = acc;
        }
    }
    __syncthreads();
    for (int j = threadIdx.x; j < per * T; j += 256) {
        const int el = j / T, t = j % T, ee = blockIdx.x * per + el;
        if (ee >= E) continue;
        float z = 0.0f;
        for (int k2 = 0; k2 < KS; ++k2) z += part[el * KS + k2][t];
        if (ex.sel) {
            const float sc = 1.0f / (1.0f + expf(-z));
            zpart[(int64_t)t * E + ee] = sc;
            ex.sel[(int64_t)t * E + ee] = sc + (j == (int)threadIdx.x ? bias0 : __ldg(ex.bias + ee));
        } else {
            zpart[(int64_t)t * E + ee] = z;
        }
    }
}

// ---------------------------------------------------------------------------
// Router for a few tokens (T <= kRouterRowMaxT, H <= kRouterRowMaxH), one CTA
// per expert e: the expert's router row (H f32, contiguous) arrives in shared
// memory by one bulk copy while every thread loads its activation columns
// c = 4 tid + 1024 j of the first token, so that the CTA waits for about one
// trip to memory.  Each thread sums its columns in j order, the warp by
// warp_sum, then the 8 warps in warp order.  The CTAs after the E routers
// build the activation operands and clear the work queue and error flag, as
// in router_gemv_kernel; the flag is cleared within microseconds of the launch
// and a bounded wait here gives up only after about a second, so a timeout it
// reports is not lost to the clearing.
// ---------------------------------------------------------------------------
constexpr int kRouterRowMaxT = 4;
constexpr int kRouterRowMaxH = 8192;

template <typename XT>
__global__ void __launch_bounds__(256)
router_row_kernel(const XT* __restrict__ x, int T, int H, const float* __restrict__ wr, int E,
                  float* __restrict__ zout, RouterExtras ex) {
    constexpr int kJ = kRouterRowMaxH / 1024;
    __shared__ __align__(128) float wrow[kRouterRowMaxH];
    __shared__ float part[8][kRouterRowMaxT];
    __shared__ __align__(8) uint64_t bar;
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
    // launched as a programmatic dependent: x may come from the previous grid
    asm volatile("griddepcontrol.wait;" ::: "memory");
    const int e = blockIdx.x;
    if (e >= E) {
        const int b = e - E;
        if (b < T) {
            if (ex.xq) act_quant_token(x, H, b, ex.xq, ex.xinv);
            if (ex.xq8) act_quant8_token(x, H, b, ex.xq8);
        } else {
            for (int i = threadIdx.x; i < ex.zero_n; i += 256) ex.zero[i] = 0;
            if (threadIdx.x == 0 && ex.err) *ex.err = 0;
        }
        return;
    }
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    if (threadIdx.x == 0) {
        mbar_init(&bar, 1);
        fence_mbar_init();
        mbar_expect_tx(&bar, (uint32_t)H * 4u);
        bulk_g2s(wrow, wr + (int64_t)e * H, (uint32_t)H * 4u, &bar);
    }
    const float bias = (ex.sel && (int)threadIdx.x < T) ? __ldg(ex.bias + e) : 0.0f;
    const bool vec = (reinterpret_cast<uintptr_t>(x) & (4 * sizeof(XT) - 1)) == 0;
    auto load_token = [&](int t, float4 (&xv)[kJ]) {
        const XT* xr = x + (int64_t)t * H;
#pragma unroll
        for (int j = 0; j < kJ; ++j) {
            const int c = 4 * threadIdx.x + 1024 * j;
            if (c < H)
                xv[j] = vec ? load4_f32(xr + c)
                            : make_float4(to_f32(xr[c]), to_f32(xr[c + 1]), to_f32(xr[c + 2]),
                                          to_f32(xr[c + 3]));
        }
    };
    float4 cur[kJ], nxt[kJ];
    load_token(0, cur);
    __syncthreads();  // the barrier's initialisation, before anyone waits on it
    const bool ok = mbar_wait_warp(&bar, 0, ex.err);
    for (int t = 0; t < T; ++t) {
        if (t + 1 < T) load_token(t + 1, nxt);
        float acc = 0.0f;
#pragma unroll
        for (int j = 0; j < kJ; ++j) {
            const int c = 4 * threadIdx.x + 1024 * j;
            if (c < H) {
                const float4 w = *reinterpret_cast<const float4*>(wrow + c);
                acc = fmaf(w.x, cur[j].x, acc);
                acc = fmaf(w.y, cur[j].y, acc);
                acc = fmaf(w.z, cur[j].z, acc);
                acc = fmaf(w.w, cur[j].w, acc);
            }
        }
        acc = warp_sum(acc);
        if (lane == 0) part[warp][t] = acc;
#pragma unroll
        for (int j = 0; j < kJ; ++j) cur[j] = nxt[j];
    }
    __syncthreads();
    if (!ok || (int)threadIdx.x >= T) return;
    const int t = threadIdx.x;
    float z = 0.0f;
#pragma unroll
    for (int w = 0; w < 8; ++w) z += part[w][t];
    if (ex.sel) {
        const float sc = 1.0f / (1.0f + expf(-z));
        zout[(int64_t)t * E + e] = sc;
        ex.sel[(int64_t)t * E + e] = sc + bias;
    } else {
        zout[(int64_t)t * E + e] = z;
    }
}

// ---------------------------------------------------------------------------
// Router logits, large batches: 64x64 register-tiled f32 GEMM z = x W_r^T with
// a K split (grid.z) so that the grid fills the GPU.  Every thread owns a 4x4
// block of (token, expert) outputs.
// ---------------------------------------------------------------------------
template <typename XT>
__global__ void __launch_bounds__(256)
router_tiled_kernel(const XT* __restrict__ x, int T, int H, const float* __restrict__ wr,
                    int E, int KS, float* __restrict__ zpart) {
    constexpr int BT = 64, BE = 64, BK = 16;
    __shared__ float xs[BK][BT + 4];
    __shared__ float ws[BK][BE + 4];
    const int t0 = blockIdx.x * BT, e0 = blockIdx.y * BE, ks = blockIdx.z;
    const int SL = H / KS;
    const int kbeg = ks * SL, kend = kbeg + SL;
    const int tid = threadIdx.x;
    const int tr = (tid / 16) * 4, er = (tid % 16) * 4;
    float acc[4][4] = {};
    for (int k0 = kbeg; k0 < kend; k0 += BK) {
        for (int i = tid; i < BT * BK; i += 256) {
            const int r = i / BK, c = i % BK;
            const int t = t0 + r, e = e0 + r;
            xs[c][r] = t < T ? to_f32(x[(int64_t)t * H + k0 + c]) : 0.0f;
            ws[c][r] = e < E ? wr[(int64_t)e * H + k0 + c] : 0.0f;
        }
        __syncthreads();
#pragma unroll
        for (int c = 0; c < BK; ++c) {
            float av[4], bv[4];
#pragma unroll
            for (int i = 0; i < 4; ++i) { av[i] = xs[c][tr + i]; bv[i] = ws[c][er + i]; }
#pragma unroll
            for (int i = 0; i < 4; ++i)
#pragma unroll
                for (int j = 0; j < 4; ++j) acc[i][j] = fmaf(av[i], bv[j], acc[i][j]);
        }
        __syncthreads();
    }
#pragma unroll
    for (int i = 0; i < 4; ++i)
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            const int t = t0 + tr + i, e = e0 + er + j;
            if (t < T && e < E) zpart[((int64_t)ks * T + t) * E + e] = acc[i][j];
        }
}

// ---------------------------------------------------------------------------
// Sigmoid, bias-corrected top-k and weights for one token, by one warp, with
// sel / s in shared memory (2E floats).  Writes idx[t, :], w[t, :].
// ---------------------------------------------------------------------------
__device__ __forceinline__ void topk_token(const float* __restrict__ zpart, int KS, int T, int E,
                                           const float* __restrict__ bias, int k,
                                           float routed_scale, int norm_topk,
                                           const PickFilter& filter, int t, float* sel,
                                           float* sc, int32_t* __restrict__ idx,
                                           float* __restrict__ w) {
    const int lane = threadIdx.x & 31;
#pragma unroll 4
    for (int e = lane; e < E; e += 32) {
        float zp[kMaxKS];
#pragma unroll
        for (int ks = 0; ks < kMaxKS; ++ks)
            zp[ks] = ks < KS ? __ldcg(zpart + ((int64_t)ks * T + t) * E + e) : 0.0f;
        float z = 0.0f;
#pragma unroll
        for (int ks = 0; ks < kMaxKS; ++ks) z += zp[ks];
        const float s = 1.0f / (1.0f + expf(-z));
        sc[e] = s;
        sel[e] = s + __ldg(bias + e);
    }
    __syncwarp();
    float mine = 0.0f;  // lane j keeps the score of the j-th pick
    int mine_e = 0;
    for (int j = 0; j < k; ++j) {
        float bv = -INFINITY;
        int be = 0x7fffffff;
        for (int e = lane; e < E; e += 32) {
            const float v = sel[e];
            if (v > bv || (v == bv && e < be)) { bv = v; be = e; }
        }
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) {
            const float ov = __shfl_xor_sync(0xffffffffu, bv, o);
            const int oe = __shfl_xor_sync(0xffffffffu, be, o);
            if (ov > bv || (ov == bv && oe < be)) { bv = ov; be = oe; }
        }
        if (lane == j) { mine = sc[be]; mine_e = be; }
        __syncwarp();
        if (lane == 0) sel[be] = -INFINITY;
        __syncwarp();
    }
    float denom = 0.0f;  // renormalise over the k picks in pick order
    for (int j = 0; j < k; ++j) denom += __shfl_sync(0xffffffffu, mine, j);
    const float wgt = (norm_topk ? mine / denom : mine) * routed_scale;
    const bool kept = pick_kept(filter, k, wgt, mine_e);  // weight 0: not computed
    if (lane < k) {
        idx[(int64_t)t * k + lane] = mine_e;
        w[(int64_t)t * k + lane] = kept ? wgt : 0.0f;
    }
}

constexpr int kTopkWarps = 4;

__global__ void __launch_bounds__(32 * kTopkWarps)
topk_kernel(const float* __restrict__ zpart, int KS, int T, int E,
            const float* __restrict__ bias, int k, float routed_scale, int norm_topk,
            PickFilter filter, int32_t* __restrict__ idx, float* __restrict__ w) {
    extern __shared__ float tk_smem[];
    const int warp = threadIdx.x >> 5;
    const int t = blockIdx.x * kTopkWarps + warp;
    if (t >= T) return;
    float* sel = tk_smem + (int64_t)warp * 2 * E;
    topk_token(zpart, KS, T, E, bias, k, routed_scale, norm_topk, filter, t, sel, sel + E, idx, w);
}

// ---------------------------------------------------------------------------
// Batch union in one CTA of 1024 threads: per-expert counts, an exclusive scan
// and a stable scatter.  A pair's rank inside its expert is the number of
// earlier tokens that chose the same expert, read from a per-expert token
// bitmap (a token picks an expert at most once), so the order never depends on
// timing.  Optionally also emits the expert kernels' work list and clears the
// combine counters.
// ---------------------------------------------------------------------------
struct UnionOut {
    int32_t* offsets;      // [E+1]
    int32_t* pair_tok;     // [T*k] (+ T*n_shared shared pairs when unit_expert)
    int32_t* pair_slot;    // [T*k]
    int32_t* uniq;         // [E]
    int32_t* n_uniq;       // [1]
    int32_t* inv;          // [T*k] pair index of (t, j), or nullptr
    int32_t* unit_expert;  // [E + n_shared] or nullptr
    int32_t* unit_begin;
    int32_t* unit_end;
    int32_t* n_units;      // [1]
    int32_t* counters;     // combine counters to clear, or nullptr
    int32_t n_counters;
    int32_t* err;          // device error flags to clear, or nullptr
    int32_t n_shared;
    const float* w = nullptr;  // [T*k] pick weights: a pick of weight 0 is left out
                               //   (inv = -1), or nullptr: every pick
};

constexpr int kUnionThreads = 1024;

__device__ __forceinline__ void union_body(const int32_t* idx, int T, int k, int E,
                                           const UnionOut& o, uint32_t* un_smem) {
    const int W = (T + 31) / 32;
    uint32_t* bits = un_smem;                                           // [E][W]
    int32_t* cnt = reinterpret_cast<int32_t*>(bits + (int64_t)E * W);   // [E]
    int32_t* excl = cnt + E;                                            // [E]
    int32_t* uexcl = excl + E;                                          // [E]
    __shared__ int32_t warp_tot[2][32];
    const int tid = threadIdx.x;
    for (int i = tid; i < E * W; i += kUnionThreads) bits[i] = 0u;
    for (int i = tid; i < E; i += kUnionThreads) cnt[i] = 0;
    if (o.counters)
        for (int i = tid; i < o.n_counters; i += kUnionThreads) o.counters[i] = 0;
    if (o.err && tid == 0) *o.err = 0;
    __syncthreads();
    const int P = T * k;
    for (int i = tid; i < P; i += kUnionThreads) {
        const int e = idx[i];
        if (e < 0 || e >= E || (o.w && o.w[i] == 0.0f)) continue;
        const int t = i / k;
        atomicAdd(&cnt[e], 1);
        atomicOr(&bits[(int64_t)e * W + t / 32], 1u << (t % 32));
    }
    __syncthreads();
    // block-wide exclusive scans of counts and of (count > 0), E <= 1024
    const int lane = tid & 31, warp = tid >> 5;
    const int c = tid < E ? cnt[tid] : 0;
    const int f = c > 0 ? 1 : 0;
    int sc = c, sf = f;
#pragma unroll
    for (int d = 1; d < 32; d <<= 1) {
        const int a = __shfl_up_sync(0xffffffffu, sc, d);
        const int b = __shfl_up_sync(0xffffffffu, sf, d);
        if (lane >= d) { sc += a; sf += b; }
    }
    if (lane == 31) { warp_tot[0][warp] = sc; warp_tot[1][warp] = sf; }
    __syncthreads();
    if (warp == 0) {
        const int a = warp_tot[0][lane], b = warp_tot[1][lane];
        int pa = a, pb = b;
#pragma unroll
        for (int d = 1; d < 32; d <<= 1) {
            const int x = __shfl_up_sync(0xffffffffu, pa, d);
            const int y = __shfl_up_sync(0xffffffffu, pb, d);
            if (lane >= d) { pa += x; pb += y; }
        }
        warp_tot[0][lane] = pa - a;
        warp_tot[1][lane] = pb - b;
    }
    __syncthreads();
    if (tid < E) {
        const int ex = sc - c + warp_tot[0][warp];
        const int ux = sf - f + warp_tot[1][warp];
        excl[tid] = ex;
        uexcl[tid] = ux;
        o.offsets[tid] = ex;
        if (f) o.uniq[ux] = tid;
        if (tid == E - 1) {
            o.offsets[E] = ex + c;
            *o.n_uniq = ux + f;
            if (o.n_units) *o.n_units = ux + f + o.n_shared;
        }
    }
    __syncthreads();
    for (int i = tid; i < P; i += kUnionThreads) {
        const int e = idx[i];
        if (e < 0 || e >= E || (o.w && o.w[i] == 0.0f)) {
            if (o.inv) o.inv[i] = -1;
            continue;
        }
        const int t = i / k, j = i % k;
        const uint32_t* row = bits + (int64_t)e * W;
        int rank = __popc(row[t / 32] & ((1u << (t % 32)) - 1u));
        for (int q = 0; q < t / 32; ++q) rank += __popc(row[q]);
        const int p = excl[e] + rank;
        o.pair_tok[p] = t;
        o.pair_slot[p] = j;
        if (o.inv) o.inv[i] = p;
    }
    if (o.w) {  // pairs left free by picks not computed: token 0, so that
                // kernels sweeping every pair index read valid rows
        const int used = excl[E - 1] + cnt[E - 1];
        for (int p = used + tid; p < P; p += kUnionThreads) {
            o.pair_tok[p] = 0;
            o.pair_slot[p] = 0;
        }
    }
    if (o.unit_expert) {
        for (int e = tid; e < E; e += kUnionThreads) {
            if (cnt[e] > 0) {
                const int u = uexcl[e];
                o.unit_expert[u] = e;
                o.unit_begin[u] = excl[e];
                o.unit_end[u] = excl[e] + cnt[e];
            }
        }
        const int n_uniq = uexcl[E - 1] + (cnt[E - 1] > 0 ? 1 : 0);
        for (int s = tid; s < o.n_shared; s += kUnionThreads) {
            o.unit_expert[n_uniq + s] = E + s;
            o.unit_begin[n_uniq + s] = P + s * T;
            o.unit_end[n_uniq + s] = P + (s + 1) * T;
        }
        for (int i = tid; i < o.n_shared * T; i += kUnionThreads) o.pair_tok[P + i] = i % T;
    }
}

__global__ void __launch_bounds__(kUnionThreads)
union_kernel(const int32_t* __restrict__ idx, int T, int k, int E, UnionOut o) {
    extern __shared__ uint32_t un_smem[];
    union_body(idx, T, k, E, o, un_smem);
}

// Small batches (T * E <= 4096): top-k of every token and the union in one CTA.
// Every (token, expert) pair gets a thread that sums the router slices and
// applies the sigmoid and the bias, then counts the experts that rank before
// it (higher selection score, or equal score and lower index); the k with rank
// < k are the picks, in rank order.  Short loops over shared memory, no
// long single-warp path.
constexpr int kSmallSelect = 4096;

__global__ void __launch_bounds__(kUnionThreads)
topk_union_kernel(const float* __restrict__ zpart, int KS, int T, int E,
                  const float* __restrict__ bias, int k, float routed_scale, int norm_topk,
                  PickFilter filter, int32_t* idx, float* w, UnionOut o) {
    extern __shared__ uint32_t un_smem[];
    float* sc = reinterpret_cast<float*>(un_smem);  // [T][E] sigmoid scores
    float* sel = sc + T * E;                         // [T][E] selection scores
    __shared__ float pick_s[kSmallSelect / 32][32];
    __shared__ int pick_e[kSmallSelect / 32][32];
    const int n = T * E;
    for (int i = threadIdx.x; i < n; i += kUnionThreads) {
        const int t = i / E, e = i - t * E;
        float z = 0.0f;
        for (int ks = 0; ks < KS; ++ks) z += __ldcg(zpart + ((int64_t)ks * T + t) * E + e);
        const float s = 1.0f / (1.0f + expf(-z));
        sc[i] = s;
        sel[i] = s + __ldg(bias + e);
    }
    __syncthreads();
    for (int i = threadIdx.x; i < n; i += kUnionThreads) {
        const int t = i / E, e = i - t * E;
        const float v = sel[i];
        const float* row = sel + t * E;
        int r = 0;
        for (int e2 = 0; e2 < E; ++e2) {
            const float v2 = row[e2];
            r += (v2 > v) | ((v2 == v) & (e2 < e));
        }
        if (r < k) { pick_e[t][r] = e; pick_s[t][r] = sc[i]; }
    }
    __syncthreads();
    // one warp per token: weights (denominator in pick order), then the pick filter
    for (int t = threadIdx.x >> 5; t < T; t += kUnionThreads / 32) {
        const int j = threadIdx.x & 31;
        float denom = 0.0f;
        for (int q = 0; q < k; ++q) denom += pick_s[t][q];
        const float sj = j < k ? pick_s[t][j] : 0.0f;
        const int ej = j < k ? pick_e[t][j] : 0;
        const float wgt = (norm_topk ? sj / denom : sj) * routed_scale;
        const bool kept = pick_kept(filter, k, wgt, ej);
        if (j < k) {
            idx[t * k + j] = ej;
            w[t * k + j] = kept ? wgt : 0.0f;
        }
    }
    __threadfence_block();
    __syncthreads();
    union_body(idx, T, k, E, o, un_smem);
}

}  // namespace coli
