// route.cuh - router logits, sigmoid + bias-corrected top-k, and the batch union.
//
// Router ("解密GLM-5.2-colibri-int4-with-int8-mtp" 模型架构深度解析; "github一周涨11k
// ⭐️！25GB 内存跑 744B GLM-5.2 模型！" 三.1 and 四.3): z = W_r x in f32 (plain FMA on
// CUDA cores, no TF32), s = sigmoid(z), the k largest s + b win (ties to the
// lower index), weights come from s alone.
// Union (same article 三.4; "colibrì 實戰指南" 二): (token, slot) pairs grouped by
// expert, experts ascending, tokens ascending inside an expert.
#pragma once

#include "common.cuh"

namespace coli {

// ---------------------------------------------------------------------------
// Router logits, small batches: one warp per (expert row, K slice).  The warp
// streams its slice of W_r once with 16-byte loads and dots it with every
// token.  Partial sums go to zpart[ks][t][e]; top-k adds the slices in order.
// ---------------------------------------------------------------------------
template <typename XT>
__global__ void __launch_bounds__(256)
router_gemv_kernel(const XT* __restrict__ x, int T, int H, const float* __restrict__ wr,
                   int E, int KS, float* __restrict__ zpart) {
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int gw = blockIdx.x * 8 + warp;
    const int e = gw / KS, ks = gw % KS;
    if (e >= E) return;
    const int SL = H / KS;  // multiple of 128
    const float* wrow = wr + (int64_t)e * H + (int64_t)ks * SL;
    for (int t0 = 0; t0 < T; t0 += 8) {
        const int tn = min(8, T - t0);
        float acc[8];
#pragma unroll
        for (int i = 0; i < 8; ++i) acc[i] = 0.0f;
        for (int c = lane * 4; c < SL; c += 128) {
            const float4 wv = *reinterpret_cast<const float4*>(wrow + c);
#pragma unroll
            for (int i = 0; i < 8; ++i) {
                if (i < tn) {
                    const XT* xp = x + (int64_t)(t0 + i) * H + (int64_t)ks * SL + c;
                    acc[i] = fmaf(wv.x, to_f32(xp[0]), acc[i]);
                    acc[i] = fmaf(wv.y, to_f32(xp[1]), acc[i]);
                    acc[i] = fmaf(wv.z, to_f32(xp[2]), acc[i]);
                    acc[i] = fmaf(wv.w, to_f32(xp[3]), acc[i]);
                }
            }
        }
#pragma unroll
        for (int i = 0; i < 8; ++i) {
            if (i < tn) {
                const float v = warp_sum(acc[i]);
                if (lane == 0) zpart[((int64_t)ks * T + t0 + i) * E + e] = v;
            }
        }
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
        // 64 rows x 16 columns of x and of W_r: 1024 values each, 4 per thread
        for (int i = tid; i < BT * BK; i += 256) {
            const int r = i / BK, c = i % BK;
            const int t = t0 + r, e = e0 + r;
            xs[c][r] = t < T ? to_f32(x[(int64_t)t * H + k0 + c]) : 0.0f;
            ws[c][r] = e < E ? wr[(int64_t)e * H + k0 + c] : 0.0f;
        }
        __syncthreads();
#pragma unroll
        for (int c = 0; c < BK; ++c) {
            float a[4], b[4];
#pragma unroll
            for (int i = 0; i < 4; ++i) { a[i] = xs[c][tr + i]; b[i] = ws[c][er + i]; }
#pragma unroll
            for (int i = 0; i < 4; ++i)
#pragma unroll
                for (int j = 0; j < 4; ++j) acc[i][j] = fmaf(a[i], b[j], acc[i][j]);
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
// Sigmoid, bias-corrected top-k and weights: one warp per token.  The warp
// keeps the token's E scores in shared memory and runs k rounds of a warp
// arg-max over (sel desc, index asc).
// ---------------------------------------------------------------------------
constexpr int kTopkWarps = 4;

__global__ void __launch_bounds__(32 * kTopkWarps)
topk_kernel(const float* __restrict__ zpart, int KS, int T, int E,
            const float* __restrict__ bias, int k, float routed_scale, int norm_topk,
            int32_t* __restrict__ idx, float* __restrict__ w) {
    extern __shared__ float tk_smem[];
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int t = blockIdx.x * kTopkWarps + warp;
    if (t >= T) return;
    float* sel = tk_smem + (int64_t)warp * 2 * E;
    float* sc = sel + E;
    for (int e = lane; e < E; e += 32) {
        float z = 0.0f;
        for (int ks = 0; ks < KS; ++ks) z += zpart[((int64_t)ks * T + t) * E + e];
        const float s = 1.0f / (1.0f + expf(-z));
        sc[e] = s;
        sel[e] = s + bias[e];
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
    // renormalise over the k picks in pick order
    float denom = 0.0f;
    for (int j = 0; j < k; ++j) denom += __shfl_sync(0xffffffffu, mine, j);
    if (lane < k) {
        idx[(int64_t)t * k + lane] = mine_e;
        w[(int64_t)t * k + lane] = (norm_topk ? mine / denom : mine) * routed_scale;
    }
}

// ---------------------------------------------------------------------------
// Batch union in one CTA: per-expert counts, an exclusive scan, and a stable
// scatter.  A pair's rank inside its expert is the number of earlier tokens
// that chose the same expert, read from a per-expert token bitmap (a token
// picks an expert at most once), so the order never depends on timing.
// Optionally also emits the work list the expert kernels consume.
// ---------------------------------------------------------------------------
struct UnionOut {
    int32_t* offsets;      // [E+1]
    int32_t* pair_tok;     // [T*k] (+ T*n_shared shared pairs when units != 0)
    int32_t* pair_slot;    // [T*k]
    int32_t* uniq;         // [E]
    int32_t* n_uniq;       // [1]
    int32_t* inv;          // [T*k] pair index of (t, j), or nullptr
    int32_t* unit_expert;  // [E + n_shared] or nullptr
    int32_t* unit_begin;
    int32_t* unit_end;
    int32_t* n_units;      // [1]
    int32_t n_shared;
};

constexpr int kUnionThreads = 1024;

__global__ void __launch_bounds__(kUnionThreads)
union_kernel(const int32_t* __restrict__ idx, int T, int k, int E, UnionOut o) {
    extern __shared__ uint32_t un_smem[];
    const int W = (T + 31) / 32;
    uint32_t* bits = un_smem;                       // [E][W]
    int32_t* cnt = reinterpret_cast<int32_t*>(bits + (int64_t)E * W);  // [E]
    int32_t* excl = cnt + E;                        // [E]
    int32_t* uexcl = excl + E;                      // [E]
    __shared__ int32_t warp_tot[2][32];
    const int tid = threadIdx.x;
    for (int i = tid; i < E * W; i += kUnionThreads) bits[i] = 0u;
    for (int i = tid; i < E; i += kUnionThreads) cnt[i] = 0;
    __syncthreads();
    const int P = T * k;
    for (int i = tid; i < P; i += kUnionThreads) {
        const int e = idx[i];
        if (e < 0 || e >= E) continue;
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
        int a = warp_tot[0][lane], b = warp_tot[1][lane];
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
        if (e < 0 || e >= E) continue;
        const int t = i / k, j = i % k;
        const uint32_t* row = bits + (int64_t)e * W;
        int rank = __popc(row[t / 32] & ((1u << (t % 32)) - 1u));
        for (int q = 0; q < t / 32; ++q) rank += __popc(row[q]);
        const int p = excl[e] + rank;
        o.pair_tok[p] = t;
        o.pair_slot[p] = j;
        if (o.inv) o.inv[i] = p;
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
        __syncthreads();
        const int n_uniq = uexcl[E - 1] + (cnt[E - 1] > 0 ? 1 : 0);
        for (int s = tid; s < o.n_shared; s += kUnionThreads) {
            o.unit_expert[n_uniq + s] = E + s;
            o.unit_begin[n_uniq + s] = P + s * T;
            o.unit_end[n_uniq + s] = P + (s + 1) * T;
        }
        for (int i = tid; i < o.n_shared * T; i += kUnionThreads) o.pair_tok[P + i] = i % T;
    }
}

}  // namespace coli
