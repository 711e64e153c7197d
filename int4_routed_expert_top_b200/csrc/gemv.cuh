// gemv.cuh - int4 expert kernels for small batches (decode, MTP verify).
//
// A CTA owns one unit (a routed expert picked by the batch, or a shared expert),
// 64 output rows, and every token routed to that unit, so each weight byte is
// read from HBM once per launch however many of the unit's tokens use it (batch
// union, "github一周涨11k⭐️！25GB 内存跑 744B GLM-5.2 模型！" 三.4).
//
// Data movement: a producer warp (one elected lane issuing) streams the unit's fragment tiles with bulk
// copies (the TMA engine, no tensor map) into an 8-stage shared-memory ring.
// One stage is one 64-column step of the CTA's 64 rows: 2 KB of codes per matrix
// (four contiguous 512-byte blocks), plus the step's 64 scales for gs64.  Stages
// complete on mbarriers; consumers release them through a second set.
//
// Math: consumer warp w owns 16 rows.  Each lane reads its 16-byte unit of the
// stage, decodes the 32 nibbles to exact fp16 mma.sync A fragments in registers
// and multiplies them on the tensor cores with the activations (B operand),
// which are split into fp16 hi + lo parts under a power-of-two scale and staged
// in shared memory, so the products carry ~22 significant bits into the f32
// accumulators.  The weight scale (per row, or per 64 columns for gs64) and the
// activation's inverse scale are applied in f32: once at the end when both are
// constant along the reduction (per-row scales on gate/up), else after every
// 64-column step.
//
//   gate/up: h[p, i] = silu(sum_c Wg'[i, c] x[c]) * (sum_c Wu'[i, c] x[c]),
//            stored as fp16 hi/lo with one power of two per 64 rows
//   down:    o[p, r] = sum_i Wd'[r, i] h[p, i] (f32; the two halves of the sum are
//            added into o, which the gate/up pass zeroed), and the last CTA to
//            finish a 64-row block forms y = residual + sum_j w_j o_j + sum_s o_s
#pragma once

#include "common.cuh"
#include "pipeline.cuh"

namespace coli {

constexpr int kConsumers = 4;                       // consumer warps: 64 rows per CTA
constexpr int kGemvThreads = 32 * (kConsumers + 1);  // + one producer warp
constexpr int kStages = 8;
constexpr int kGemvMaxNT = 2;   // up to 2 column groups of 8: 8 tokens per pass
constexpr int kDownSplit = 2;   // the down reduction is split in halves

struct GemvArgs {
    ExpertStore store;
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
    int32_t* err;         // device error flags
    int tok_cap;          // activation rows staged per pass (shared memory is sized for it)
    int T, k, n_shared;
    int H, I, group;
};

// ring stage: [A codes 2 KB][B codes 2 KB][A scales 256 B][B scales 256 B]
template <bool TWO, bool GS>
struct Stage {
    static constexpr int kB = 2048;
    static constexpr int kSA = TWO ? 4096 : 2048;
    static constexpr int kSB = kSA + 256;
    static constexpr int kBytes = (TWO ? 4096 : 2048) + (GS ? (TWO ? 512 : 256) : 0);
};

// Producer (whole warp, elected lane issues): `passes` sweeps over steps kb0 .. kb0+n-1 of the 64 rows
// starting at 16-row block b8_0 of tile rt.
template <bool TWO, bool GS>
__device__ __forceinline__ void gemv_produce(const uint8_t* cA, const uint8_t* cB,
                                             const float* sA, const float* sB, int K, int rt,
                                             int b8_0, int kb0, int n, int passes,
                                             uint8_t* ring, uint64_t* full, uint64_t* empty,
                                             int32_t* err) {
    using S = Stage<TWO, GS>;
    const int ng = K / 64;
    const int total = passes * n;
    int it = 0;
    for (; it < total; ++it) {
        const int s = it % kStages;
        if (it >= kStages && !mbar_wait_warp(&empty[s], ((it / kStages) - 1) & 1, err)) break;
        const int kb = kb0 + it % n;
        uint8_t* st = ring + s * S::kBytes;
        mbar_expect_tx_elect(&full[s], S::kBytes);
        const int64_t uoff = frag_unit_offset(rt, kb, b8_0, 0, K);
        bulk_g2s_elect(st, cA + uoff, 2048, &full[s]);
        if (TWO) bulk_g2s_elect(st + S::kB, cB + uoff, 2048, &full[s]);
        if (GS) {
            const int64_t soff = ((int64_t)rt * ng + kb) * kTileRows + b8_0 * 16;
            bulk_g2s_elect(st + S::kSA, sA + soff, 256, &full[s]);
            if (TWO) bulk_g2s_elect(st + S::kSB, sB + soff, 256, &full[s]);
        }
    }
    if (it < total) {  // abandoned: let the copies already issued land before leaving
        for (int j = it > kStages ? it - kStages : 0; j < it; ++j)
            mbar_wait_warp(&full[j % kStages], (j / kStages) & 1, nullptr);
    }
}

// Consumer warp: 16 rows (block w of the CTA's 64) starting at row0 over the
// steps the producer streams for one pass, NT column groups of 8.  Column n of
// group c carries token 4c + (n & 3) of the pass, hi part for n < 4, lo for
// n >= 4.  Activations: xs[tc][K/64][128] fp16, xi[tc][K/64] f32 in shared
// memory.  `it0` is the pipeline step index of the pass's first step.
// Returns false if a wait timed out (the flag is in a.err; the results are then
// meaningless, but every barrier of the CTA is still reached).
template <bool GATEUP, int NT, bool GS>
__device__ __forceinline__ bool gemv_consume(const GemvArgs& a, int K, int row0, int kb0, int n,
                                             int tc, const __half* xs, const float* xi,
                                             const float* sA, const float* sB, uint8_t* ring,
                                             uint64_t* full, uint64_t* empty, int it0,
                                             float accA[NT][4], float accB[NT][4]) {
    using S = Stage<GATEUP, GS>;
    constexpr bool CHAIN = GATEUP && !GS;  // scales constant along K: apply at the end
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int g = lane >> 2, t = lane & 3;
    const int KB = K / 64;
    const DecodeK dk = a.dk;
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
    float rowA0 = 0.f, rowA1 = 0.f, rowB0 = 0.f, rowB1 = 0.f;  // per-row scales
    if (!GS && !CHAIN) {
        rowA0 = __ldg(sA + scale_offset(row0 + g, 0, 1));
        rowA1 = __ldg(sA + scale_offset(row0 + g + 8, 0, 1));
    }
    float cA[NT][4][4], cB[NT][4][4];  // CHAIN: one accumulator per 16-column sub-block
#pragma unroll
    for (int c = 0; c < NT; ++c)
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            accA[c][i] = 0.0f; accB[c][i] = 0.0f;
#pragma unroll
            for (int j = 0; j < 4; ++j) { cA[c][j][i] = 0.0f; cB[c][j][i] = 0.0f; }
        }

    bool ok = true;  // after a timed-out wait: keep every barrier, skip further waits
    for (int rel = 0; rel < n; ++rel) {
        const int it = it0 + rel;
        const int s = it % kStages;
        if (ok && !mbar_wait_warp(&full[s], (it / kStages) & 1, a.err)) ok = false;
        const uint8_t* st = ring + s * S::kBytes;
        const uint4 ua = reinterpret_cast<const uint4*>(st)[warp * 32 + lane];
        const uint4 ub = GATEUP ? reinterpret_cast<const uint4*>(st + S::kB)[warp * 32 + lane] : ua;
        float sc[4] = {rowA0, rowA1, rowB0, rowB1};
        if (GS) {
            const float* ssa = reinterpret_cast<const float*>(st + S::kSA) + warp * 16 + g;
            sc[0] = ssa[0]; sc[1] = ssa[8];
            if (GATEUP) {
                const float* ssb = reinterpret_cast<const float*>(st + S::kSB) + warp * 16 + g;
                sc[2] = ssb[0]; sc[3] = ssb[8];
            }
        }
        // decode the whole step before releasing the stage
        uint32_t fa[4][4], fb[4][4];
        decode_word(ua.x, fa[0], dk); decode_word(ua.y, fa[1], dk);
        decode_word(ua.z, fa[2], dk); decode_word(ua.w, fa[3], dk);
        if (GATEUP) {
            decode_word(ub.x, fb[0], dk); decode_word(ub.y, fb[1], dk);
            decode_word(ub.z, fb[2], dk); decode_word(ub.w, fb[3], dk);
        }
        asm volatile("" ::"f"(sc[0]), "f"(sc[1]), "f"(sc[2]), "f"(sc[3]));
        __syncwarp();
        if (lane == 0) mbar_arrive(&empty[s]);

        uint2 bx[NT][4];
        float iv[NT][2];
#pragma unroll
        for (int c = 0; c < NT; ++c) {
#pragma unroll
            for (int j = 0; j < 4; ++j)
                bx[c][j] = bval[c] ? pX[c][rel * 32 + 4 * j] : make_uint2(0u, 0u);
            iv[c][0] = pI[c][0][rel];
            iv[c][1] = pI[c][1][rel];
        }
        if (CHAIN) {
#pragma unroll
            for (int j = 0; j < 4; ++j)
#pragma unroll
                for (int c = 0; c < NT; ++c) {
                    mma_f16_16816(cA[c][j], fa[j], bx[c][j].x, bx[c][j].y);
                    mma_f16_16816(cB[c][j], fb[j], bx[c][j].x, bx[c][j].y);
                }
        } else {
            float dA[NT][2][4], dB[NT][2][4];
#pragma unroll
            for (int j = 0; j < 4; ++j)
#pragma unroll
                for (int c = 0; c < NT; ++c) {
                    if (j < 2) mma_f16_16816_zc(dA[c][j & 1], fa[j], bx[c][j].x, bx[c][j].y);
                    else       mma_f16_16816(dA[c][j & 1], fa[j], bx[c][j].x, bx[c][j].y);
                    if (GATEUP) {
                        if (j < 2) mma_f16_16816_zc(dB[c][j & 1], fb[j], bx[c][j].x, bx[c][j].y);
                        else       mma_f16_16816(dB[c][j & 1], fb[j], bx[c][j].x, bx[c][j].y);
                    }
                }
#pragma unroll
            for (int c = 0; c < NT; ++c)
#pragma unroll
                for (int i = 0; i < 4; ++i) {
                    const float f = sc[i >> 1] * iv[c][i & 1];
                    accA[c][i] = fmaf(f, dA[c][0][i] + dA[c][1][i], accA[c][i]);
                    if (GATEUP) {
                        const float fu = sc[2 + (i >> 1)] * iv[c][i & 1];
                        accB[c][i] = fmaf(fu, dB[c][0][i] + dB[c][1][i], accB[c][i]);
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
                accB[c][i] = (cB[c][0][i] + cB[c][1][i]) + (cB[c][2][i] + cB[c][3][i]);
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
    return ok;
}

// stage activation rows src[i] (i < tc) of one pass: [tc][KB][128] fp16 plus
// [tc][KB] inverse scales, 16-byte copies by the consumer threads
__device__ __forceinline__ void stage_rows(const __half* __restrict__ q, const float* __restrict__ inv,
                                           const int* src, int tc, int KB, __half* xs, float* xi) {
    const int per = KB * 16;  // uint4 per row
    for (int i = threadIdx.x; i < tc * per; i += 32 * kConsumers) {
        const int r = i / per, c = i - r * per;
        reinterpret_cast<uint4*>(xs)[i] =
            __ldg(reinterpret_cast<const uint4*>(q + (int64_t)src[r] * KB * 128) + c);
    }
    for (int i = threadIdx.x; i < tc * KB; i += 32 * kConsumers) {
        const int r = i / KB, c = i - r * KB;
        xi[i] = __ldg(inv + (int64_t)src[r] * KB + c);
    }
}

// dynamic shared memory: ring + staged activations of one pass
template <bool TWO, bool GS>
__host__ __device__ constexpr int gemv_ring_bytes() { return kStages * Stage<TWO, GS>::kBytes; }
__host__ __device__ inline int gemv_act_bytes(int tok_cap, int K) { return tok_cap * (K / 64) * (128 * 2 + 4); }
// dynamic shared memory a GEMV CTA may ask for (the opt-in limit less the static part)
constexpr int kGemvSmemMax = 227 * 1024 - 2048;

// ---------------------------------------------------------------------------
// gate/up + SwiGLU.  After the shuffle, lane (g, t < 2) holds rows g, g + 8 of
// the warp's 16 and tokens 4c + 2t + {0, 1}.
// ---------------------------------------------------------------------------
template <int NT, bool GS>
__global__ void __launch_bounds__(kGemvThreads)
gateup_gemv_kernel(GemvArgs a) {
    extern __shared__ __align__(128) uint8_t gv_smem[];
    __shared__ __align__(8) uint64_t full[kStages], empty[kStages];
    __shared__ float wmax[kConsumers][8 * kGemvMaxNT];
    __shared__ int src[8 * kGemvMaxNT];
    const int nrb = a.I / 64;
    const int u = blockIdx.x / nrb, rb64 = blockIdx.x % nrb;
    if (u >= *a.n_units) return;
    const int e = a.unit_expert[u], p0 = a.unit_begin[u], p1 = a.unit_end[u];
    const uint8_t* blob = a.store.blob(e);
    const uint8_t* codesA = blob + a.L.codes[0];
    const uint8_t* codesB = blob + a.L.codes[1];
    const float* sA = reinterpret_cast<const float*>(blob + a.L.scales[0]);
    const float* sB = reinterpret_cast<const float*>(blob + a.L.scales[1]);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int KB = a.H / 64;
    const int passes = (p1 - p0 + a.tok_cap - 1) / a.tok_cap;
    uint8_t* ring = gv_smem;
    __half* xs = reinterpret_cast<__half*>(gv_smem + gemv_ring_bytes<true, GS>());
    float* xi = reinterpret_cast<float*>(xs + (size_t)a.tok_cap * KB * 128);
    const int rt = (rb64 * 64) / kTileRows, b8_0 = ((rb64 * 64) % kTileRows) / 16;

    if (threadIdx.x == 0) {
        for (int s = 0; s < kStages; ++s) { mbar_init(&full[s], 1); mbar_init(&empty[s], kConsumers); }
        fence_mbar_init();
    }
    __syncthreads();
    if (warp == kConsumers) {  // producer warp
        gemv_produce<true, GS>(codesA, codesB, sA, sB, a.H, rt, b8_0, 0, KB, passes, ring,
                                   full, empty, a.err);
        return;
    }

    const int g = lane >> 2, t = lane & 3;
    const int row0 = rb64 * 64 + warp * 16;
    // zero this CTA's share of the unit's down-projection outputs o[p0:p1, :]
    {
        float4* o4 = reinterpret_cast<float4*>(a.o + (int64_t)p0 * a.H);
        const int64_t n4 = (int64_t)(p1 - p0) * a.H / 4;
        const int64_t beg = n4 * rb64 / nrb, end = n4 * (rb64 + 1) / nrb;
        for (int64_t i = beg + threadIdx.x; i < end; i += 32 * kConsumers)
            o4[i] = make_float4(0.f, 0.f, 0.f, 0.f);
    }

    int pass = 0;
    for (int pc = p0; pc < p1; pc += a.tok_cap, ++pass) {
        const int tc = min(a.tok_cap, p1 - pc);
        named_sync(32 * kConsumers);  // the previous pass is done with xs, xi, src, wmax
        if (threadIdx.x < tc) src[threadIdx.x] = a.pair_tok[pc + threadIdx.x];
        named_sync(32 * kConsumers);
        stage_rows(a.xq, a.xinv, src, tc, KB, xs, xi);
        named_sync(32 * kConsumers);
        float accA[NT][4], accB[NT][4];
        gemv_consume<true, NT, GS>(a, a.H, row0, 0, KB, tc, xs, xi, sA, sB, ring, full, empty,
                                   pass * KB, accA, accB);
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
                if (!GS && tt < tc) {  // per-row weight scales and the token's activation scale
                    const float inv = xi[tt * KB];
                    ga *= __ldg(sA + scale_offset(row, 0, 1)) * inv;
                    ua *= __ldg(sB + scale_offset(row, 0, 1)) * inv;
                }
                hv[c][i] = (t < 2 && tt < tc) ? silu_f(ga) * ua : 0.0f;
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
        named_sync(32 * kConsumers);
        if (t < 2) {
#pragma unroll
            for (int c = 0; c < NT; ++c)
#pragma unroll
                for (int q = 0; q < 2; ++q) {
                    const int tt = 4 * c + 2 * t + q;
                    if (tt >= tc) continue;
                    float m = wmax[0][tt];
#pragma unroll
                    for (int ww = 1; ww < kConsumers; ++ww) m = fmaxf(m, wmax[ww][tt]);
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
template <int NT, bool GS>
__global__ void __launch_bounds__(kGemvThreads)
down_gemv_kernel(GemvArgs a) {
    extern __shared__ __align__(128) uint8_t gv_smem[];
    __shared__ __align__(8) uint64_t full[kStages], empty[kStages];
    __shared__ int last_flag;
    __shared__ int src[8 * kGemvMaxNT];
    const int nrb = a.H / 64;
    const int u = blockIdx.x / (nrb * kDownSplit);
    const int rem = blockIdx.x % (nrb * kDownSplit);
    const int rb64 = rem / kDownSplit, half = rem % kDownSplit;
    const int n_units = *a.n_units;
    if (u >= n_units) {
        if (n_units == 0 && u == 0 && half == 0) {
            // nothing to compute for this call (every pick elsewhere, no shared
            // expert): y of this 64-row block is the residual, or zero
            for (int q = threadIdx.x; q < a.T * 64; q += blockDim.x) {
                const int64_t o = (int64_t)(q / 64) * a.H + rb64 * 64 + q % 64;
                a.y[o] = a.residual ? a.residual[o] : 0.0f;
            }
        }
        return;
    }
    const int e = a.unit_expert[u], p0 = a.unit_begin[u], p1 = a.unit_end[u];
    const uint8_t* blob = a.store.blob(e);
    const uint8_t* codesA = blob + a.L.codes[2];
    const float* sA = reinterpret_cast<const float*>(blob + a.L.scales[2]);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int KB = a.I / 64;
    const int kb0 = half * KB / kDownSplit, kb1 = (half + 1) * KB / kDownSplit;
    const int n = kb1 - kb0;
    const int passes = (p1 - p0 + a.tok_cap - 1) / a.tok_cap;
    uint8_t* ring = gv_smem;
    __half* xs = reinterpret_cast<__half*>(gv_smem + gemv_ring_bytes<false, GS>());
    float* xi = reinterpret_cast<float*>(xs + (size_t)a.tok_cap * KB * 128);
    const int rt = (rb64 * 64) / kTileRows, b8_0 = ((rb64 * 64) % kTileRows) / 16;

    if (threadIdx.x == 0) {
        for (int s = 0; s < kStages; ++s) { mbar_init(&full[s], 1); mbar_init(&empty[s], kConsumers); }
        fence_mbar_init();
    }
    __syncthreads();
    if (warp == kConsumers) {
        gemv_produce<false, GS>(codesA, codesA, sA, sA, a.I, rt, b8_0, kb0, n, passes, ring,
                                    full, empty, a.err);
        return;
    }

    const int g = lane >> 2, t = lane & 3;
    const int row0 = rb64 * 64 + warp * 16;
    int pass = 0;
    for (int pc = p0; pc < p1; pc += a.tok_cap, ++pass) {
        const int tc = min(a.tok_cap, p1 - pc);
        named_sync(32 * kConsumers);
        if (threadIdx.x < tc) src[threadIdx.x] = pc + threadIdx.x;
        named_sync(32 * kConsumers);
        stage_rows(a.hq, a.hinv, src, tc, KB, xs, xi);
        named_sync(32 * kConsumers);
        float accA[NT][4], accB[NT][4];
        gemv_consume<false, NT, GS>(a, a.I, row0, kb0, n, tc, xs, xi, sA, sA, ring, full, empty,
                                    pass * n, accA, accB);
        if (t < 2) {
#pragma unroll
            for (int c = 0; c < NT; ++c)
#pragma unroll
                for (int i = 0; i < 4; ++i) {
                    const int tt = 4 * c + 2 * t + (i & 1);
                    // two addends per element (the halves) into a zeroed o: the sum
                    // does not depend on which half lands first
                    if (tt < tc)
                        atomicAdd(a.o + (int64_t)(pc + tt) * a.H + row0 + g + 8 * (i >> 1), accA[c][i]);
                }
        }
    }

    // ---- combine: the last CTA to finish this 64-row block writes y ----
    __threadfence();
    named_sync(32 * kConsumers);
    if (threadIdx.x == 0) {
        const int done = atomicAdd(&a.counters[rb64], 1) + 1;
        last_flag = done == n_units * kDownSplit;
    }
    named_sync(32 * kConsumers);
    if (!last_flag) return;
    __threadfence();
    for (int q = threadIdx.x; q < a.T * 64; q += 32 * kConsumers) {
        const int tt = q / 64, r = rb64 * 64 + q % 64;
        float acc = 0.0f;
        for (int j = 0; j < a.k; ++j) {
            const int p = __ldcg(a.inv + (int64_t)tt * a.k + j);
            if (p < 0) continue;  // a pick this call does not compute
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
