// gemm.cuh - tcgen05 grouped GEMM of the int4 experts for large batches
// (prefill and big verify batches), where each expert sees enough tokens for the
// work to be a dense contraction.
//
// Orientation ("swap AB"): D[r, n] = sum_k W[r, k] * X[n, k] with the weight
// rows as the MMA M dimension (a 128-row tile) and the unit's tokens as N, so a
// unit with few tokens does not waste a 128-token tile.  Per CTA (persistent,
// one per SM, all 512 TMEM columns):
//   warp 0      producer: 1-D bulk copies of the int4 fragment tiles of a
//               128-row tile and one 64-column step (4 KB per matrix, plus the
//               step's scales for gs64) and 2-D TMA loads of the B tile (the
//               unit's tokens as fp16, 128-byte swizzle) into a 4-stage ring;
//   warp 1      one lane issues tcgen05.mma (kind::f16, f32 accumulators in
//               TMEM) with A read from TMEM and B from shared memory;
//   warps 4-7   decode matrix 0 (gate, or down): each lane turns its 16-byte
//               unit into exact fp16 (q, or q*s for gs64) and writes it to TMEM
//               with tcgen05.st.16x256b, whose lane/column layout is that of the
//               fragment tiles; these warps also run the epilogue;
//   warps 8-11  decode matrix 1 (up) for the gate/up pass.
// TMEM columns: D0 [0, 128), D1 [128, 256), A stage s at 256 + 64 s (matrix 0)
// and 256 + 64 s + 32 (matrix 1).
//
// Epilogues: gate/up writes h = silu(a) * u in f32 and the per-pair max |h|;
// down writes o in f32.  Weight scales (per row) and the activations' powers of
// two are applied there in f32.
#pragma once

#include <cuda.h>

#include "coli_moe.h"
#include "common.cuh"
#include "pipeline.cuh"

namespace coli {

constexpr int kGemmThreads = 384;
constexpr int kGemmStages = 4;
constexpr int kGemmMaxN = 128;
constexpr int kStageB = 16384;                       // B tile: up to 128 rows x 128 B
constexpr int kStageCodes = 4096;                    // one matrix, 128 rows x 64 columns
constexpr int kStageBytes = kStageB + 2 * kStageCodes + 2 * 512;   // 25600, 1 KB multiple
// + alignment slack; the request is kept above half of the SM's shared memory so
// that exactly one CTA (which takes all 512 TMEM columns) is resident per SM
constexpr int kGemmSmem = 120 * 1024;
static_assert(kGemmStages * kStageBytes + 1024 <= kGemmSmem, "gemm ring does not fit");
constexpr uint32_t kTmemCols = 512;

struct GemmArgs {
    const uint8_t* experts;
    int64_t blob_bytes;
    BlobLayout L;
    DecodeK dk;
    const int32_t* n_units;
    const int32_t* unit_expert;
    const int32_t* unit_begin;
    const int32_t* unit_end;
    const int32_t* pair_tok;
    int two;             // 1: gate/up (matrices 0 and 1), 0: down (matrix 2)
    int K, R;            // reduction length and output rows of the matrices
    int group;
    const float* act_inv;   // gate/up: xinv [T][H/64]; down: per-pair inverse scale [P]
    float* hf;              // gate/up out: h [P][I] f32
    uint32_t* hmax;         // gate/up out: per-pair max |h| (f32 bits, atomicMax)
    float* o;               // down out: [P][H] f32
    int32_t* err;
    int I, H;
};

__device__ __forceinline__ void tmem_alloc(uint32_t* slot, uint32_t cols) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(slot)),
                 "r"(cols));
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;");
}
__device__ __forceinline__ void tmem_dealloc(uint32_t base, uint32_t cols) {
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(base), "r"(cols));
}
__device__ __forceinline__ void tc_fence_before() { asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory"); }
__device__ __forceinline__ void tc_fence_after() { asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory"); }
__device__ __forceinline__ void tc_commit(uint64_t* bar) {
    asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(smem_u32(bar))
                 : "memory");
}
// D[tmem] (+)= A[tmem] * B[smem desc], M = 128, N from idesc, K = 16
__device__ __forceinline__ void tc_mma_ts(uint32_t d, uint32_t a, uint64_t bdesc, uint32_t idesc,
                                          uint32_t accumulate) {
    asm volatile(
        "{\n .reg .pred p;\n setp.ne.b32 p, %4, 0;\n"
        " tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, p;\n}"
        ::"r"(d), "r"(a), "l"(bdesc), "r"(idesc), "r"(accumulate));
}
__device__ __forceinline__ void tmem_st_16x256b_x4(uint32_t taddr, const uint32_t r[16]) {
    asm volatile(
        "tcgen05.st.sync.aligned.16x256b.x4.b32 [%0], {%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16};"
        ::"r"(taddr), "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]),
        "r"(r[7]), "r"(r[8]), "r"(r[9]), "r"(r[10]), "r"(r[11]), "r"(r[12]), "r"(r[13]), "r"(r[14]),
        "r"(r[15]));
}
__device__ __forceinline__ void tmem_ld_32x32b_x16(uint32_t taddr, uint32_t r[16]) {
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x16.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15}, [%16];"
        : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
          "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15])
        : "r"(taddr));
}
__device__ __forceinline__ void tmem_wait_st() { asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory"); }
__device__ __forceinline__ void tmem_wait_ld() { asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory"); }

__device__ __forceinline__ void tma_load_2d(void* dst, const CUtensorMap* map, int x, int y,
                                            uint64_t* bar) {
    asm volatile(
        "cp.async.bulk.tensor.2d.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1, {%3, %4}], [%2];"
        ::"r"(smem_u32(dst)), "l"(map), "r"(smem_u32(bar)), "r"(x), "r"(y)
        : "memory");
}

// shared-memory descriptor of a K-major operand in the 128-byte swizzle layout:
// rows of 64 fp16 (128 B), 8-row groups 1024 B apart
__device__ __forceinline__ uint64_t smem_desc_sw128(const void* p) {
    const uint64_t addr = smem_u32(p);
    uint64_t d = 0;
    d |= (addr >> 4) & 0x3FFFull;            // start address
    d |= (uint64_t)1 << 16;                  // leading byte offset (unused for this layout)
    d |= (uint64_t)(1024 >> 4) << 32;        // stride byte offset: 8 rows x 128 B
    d |= (uint64_t)1 << 46;                  // descriptor version (sm_100)
    d |= (uint64_t)2 << 61;                  // swizzle 128 B
    return d;
}

// instruction descriptor: f16 x f16 -> f32, both K-major, M = 128, N = n
__host__ __device__ constexpr uint32_t idesc_f16_f32(int n) {
    return (1u << 4) | (0u << 7) | (0u << 10) | ((uint32_t)(n >> 3) << 17) | ((uint32_t)(128 >> 4) << 24);
}

// tile index -> (unit, first token of the n-tile, n, row tile); tiles are
// ordered unit by unit, n-tile by n-tile, row tile fastest
__device__ __forceinline__ bool gemm_tile(const GemmArgs& a, int n_units, int idx, int& u, int& p0,
                                          int& n, int& rt) {
    const int RT = a.R / kTileRows;
    for (u = 0; u < n_units; ++u) {
        const int b = a.unit_begin[u], e = a.unit_end[u];
        const int nt = (e - b + kGemmMaxN - 1) / kGemmMaxN;
        if (idx < nt * RT) {
            const int j = idx / RT;
            rt = idx % RT;
            p0 = b + j * kGemmMaxN;
            n = min(kGemmMaxN, e - p0);
            return true;
        }
        idx -= nt * RT;
    }
    return false;
}

__global__ void __launch_bounds__(kGemmThreads, 1)
moe_gemm_kernel(const __grid_constant__ CUtensorMap bmap, GemmArgs a) {
    extern __shared__ uint8_t gm_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(gm_raw) + 1023) & ~uintptr_t(1023));
    __shared__ __align__(8) uint64_t full[kGemmStages], empty[kGemmStages];
    __shared__ __align__(8) uint64_t afull[kGemmStages], aempty[kGemmStages];
    __shared__ __align__(8) uint64_t accfull, accempty;
    __shared__ uint32_t tmem_slot;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int n_units = *a.n_units;
    const int KB = a.K / 64;
    const int ng = a.group ? KB : 1;
    const int ndec = a.two ? 8 : 4;  // decode warps
    const int mA = a.two ? 0 : 2;

    if (warp == 0) tmem_alloc(&tmem_slot, kTmemCols);
    if (threadIdx.x == 32) {
        for (int s = 0; s < kGemmStages; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&empty[s], ndec + 1);
            mbar_init(&afull[s], ndec);
            mbar_init(&aempty[s], 1);
        }
        mbar_init(&accfull, 1);
        mbar_init(&accempty, 4);
        fence_mbar_init();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = tmem_slot;
    bool ok = true;  // cleared by a timed-out wait: then no further waits, every barrier kept

    if (warp == 0) {
      if (lane == 0) {
        // ---------------- producer ----------------
        int it = 0;
        for (int tile = blockIdx.x;; tile += gridDim.x) {
            int u, p0, n, rt;
            if (!gemm_tile(a, n_units, tile, u, p0, n, rt)) break;
            const uint8_t* blob = a.experts + (int64_t)a.unit_expert[u] * a.blob_bytes;
            const uint8_t* c0 = blob + a.L.codes[mA];
            const uint8_t* c1 = blob + a.L.codes[1];
            const float* s0 = reinterpret_cast<const float*>(blob + a.L.scales[mA]);
            const float* s1 = reinterpret_cast<const float*>(blob + a.L.scales[1]);
            const int nb = (n + 15) / 16;
            const uint32_t bytes = (uint32_t)(nb * 2048 + kStageCodes * (a.two ? 2 : 1) +
                                              (a.group ? 512 * (a.two ? 2 : 1) : 0));
            for (int kb = 0; kb < KB; ++kb, ++it) {
                const int s = it % kGemmStages;
                if (it >= kGemmStages && ok && !mbar_wait(&empty[s], ((it / kGemmStages) - 1) & 1, a.err)) ok = false;
                uint8_t* st = smem + s * kStageBytes;
                mbar_expect_tx(&full[s], bytes);
                const int64_t uoff = frag_unit_offset(rt, kb, 0, 0, a.K);
                bulk_g2s(st + kStageB, c0 + uoff, kStageCodes, &full[s]);
                if (a.two) bulk_g2s(st + kStageB + kStageCodes, c1 + uoff, kStageCodes, &full[s]);
                if (a.group) {
                    const int64_t soff = ((int64_t)rt * ng + kb) * kTileRows;
                    bulk_g2s(st + kStageB + 2 * kStageCodes, s0 + soff, 512, &full[s]);
                    if (a.two) bulk_g2s(st + kStageB + 2 * kStageCodes + 512, s1 + soff, 512, &full[s]);
                }
                for (int i = 0; i < nb; ++i) tma_load_2d(st + i * 2048, &bmap, kb * 64, p0 + 16 * i, &full[s]);
            }
        }
      }
      __syncwarp();
    } else if (warp == 1) {
      if (lane == 0) {
        // ---------------- MMA issuer ----------------
        int it = 0, tcount = 0;
        for (int tile = blockIdx.x;; tile += gridDim.x, ++tcount) {
            int u, p0, n, rt;
            if (!gemm_tile(a, n_units, tile, u, p0, n, rt)) break;
            const int np = (n + 15) / 16 * 16;  // N: multiple of 16 for M = 128
            const uint32_t idesc = idesc_f16_f32(np);
            if (tcount > 0 && ok && !mbar_wait(&accempty, (tcount - 1) & 1, a.err)) ok = false;
            tc_fence_after();
            for (int kb = 0; kb < KB; ++kb, ++it) {
                const int s = it % kGemmStages;
                if (ok && !mbar_wait(&afull[s], (it / kGemmStages) & 1, a.err)) ok = false;
                if (ok && !mbar_wait(&full[s], (it / kGemmStages) & 1, a.err)) ok = false;
                tc_fence_after();
                const uint64_t bdesc = smem_desc_sw128(smem + s * kStageBytes);
                const uint32_t a0 = tmem + 256 + 64 * s;
#pragma unroll
                for (int j = 0; j < 4; ++j) {
                    const uint32_t acc = (kb > 0 || j > 0) ? 1u : 0u;
                    tc_mma_ts(tmem + 0, a0 + 8 * j, bdesc + 2 * j, idesc, acc);
                    if (a.two) tc_mma_ts(tmem + 128, a0 + 32 + 8 * j, bdesc + 2 * j, idesc, acc);
                }
                tc_commit(&aempty[s]);
                tc_commit(&empty[s]);
            }
            tc_commit(&accfull);
        }
      }
      __syncwarp();
    } else if (warp >= 4 && warp < 4 + ndec) {
        // ---------------- decode (+ epilogue on warps 4-7) ----------------
        const int grp = (warp - 4) / 4;           // 0: matrix 0, 1: matrix 1
        const int q = warp & 3;                   // TMEM lane quarter of this warp
        const int g = lane >> 2;
        const DecodeK dk = a.dk;
        int it = 0, tcount = 0;
        for (int tile = blockIdx.x;; tile += gridDim.x, ++tcount) {
            int u, p0, n, rt;
            if (!gemm_tile(a, n_units, tile, u, p0, n, rt)) break;
            for (int kb = 0; kb < KB; ++kb, ++it) {
                const int s = it % kGemmStages;
                if (ok && !mbar_wait(&full[s], (it / kGemmStages) & 1, a.err)) ok = false;
                if (it >= kGemmStages && ok && !mbar_wait(&aempty[s], ((it / kGemmStages) - 1) & 1, a.err)) ok = false;
                tc_fence_after();
                const uint8_t* st = smem + s * kStageBytes + kStageB + grp * kStageCodes;
                const float* ss = reinterpret_cast<const float*>(smem + s * kStageBytes + kStageB + 2 * kStageCodes + grp * 512);
#pragma unroll
                for (int hb = 0; hb < 2; ++hb) {
                    const int b8 = 2 * q + hb;
                    const uint4 un = reinterpret_cast<const uint4*>(st)[b8 * 32 + lane];
                    const uint32_t wd[4] = {un.x, un.y, un.z, un.w};
                    uint32_t r[16];
#pragma unroll
                    for (int j = 0; j < 4; ++j) {
                        uint32_t f[4];
                        decode_word(wd[j], f, dk);
                        // 16x256b register order: (row g, c0..c0+1), (row g, c0+2..),
                        // (row g+8, c0..), (row g+8, c0+2..)
                        r[4 * j + 0] = f[0]; r[4 * j + 1] = f[2];
                        r[4 * j + 2] = f[1]; r[4 * j + 3] = f[3];
                    }
                    if (a.group) {  // gs64: A = fp16(q * s)
                        const __half2 s0 = __float2half2_rn(ss[b8 * 16 + g]);
                        const __half2 s1 = __float2half2_rn(ss[b8 * 16 + g + 8]);
#pragma unroll
                        for (int j = 0; j < 4; ++j) {
                            __half2* h = reinterpret_cast<__half2*>(r + 4 * j);
                            h[0] = __hmul2(h[0], s0); h[1] = __hmul2(h[1], s0);
                            h[2] = __hmul2(h[2], s1); h[3] = __hmul2(h[3], s1);
                        }
                    }
                    const uint32_t taddr = tmem + ((uint32_t)(32 * q + 16 * hb) << 16) + 256 + 64 * s + 32 * grp;
                    tmem_st_16x256b_x4(taddr, r);
                }
                tmem_wait_st();
                tc_fence_before();
                __syncwarp();
                if (lane == 0) { mbar_arrive(&afull[s]); mbar_arrive(&empty[s]); }
            }
            if (grp != 0) continue;
            // ---------------- epilogue: rows 32q + lane of the tile ----------------
            if (ok && !mbar_wait(&accfull, tcount & 1, a.err)) ok = false;
            tc_fence_after();
            const int row = rt * kTileRows + 32 * q + lane;
            const uint8_t* blob = a.experts + (int64_t)a.unit_expert[u] * a.blob_bytes;
            const float srow0 = a.group ? 1.0f
                : __ldg(reinterpret_cast<const float*>(blob + a.L.scales[mA]) + scale_offset(row, 0, 1));
            const float srow1 = (a.group || !a.two) ? 1.0f
                : __ldg(reinterpret_cast<const float*>(blob + a.L.scales[1]) + scale_offset(row, 0, 1));
            const uint32_t lane_off = (uint32_t)(32 * q) << 16;
            for (int c0 = 0; c0 < n; c0 += 16) {
                uint32_t d0[16], d1[16];
                tmem_ld_32x32b_x16(tmem + lane_off + c0, d0);
                if (a.two) tmem_ld_32x32b_x16(tmem + lane_off + 128 + c0, d1);
                tmem_wait_ld();
#pragma unroll
                for (int i = 0; i < 16; ++i) {
                    const int nn = c0 + i;
                    const bool valid = nn < n;
                    const int p = p0 + (valid ? nn : 0);
                    if (a.two) {
                        const float inv = valid ? __ldg(a.act_inv + (int64_t)a.pair_tok[p] * (a.H / 64)) : 0.f;
                        const float ga = __uint_as_float(d0[i]) * srow0 * inv;
                        const float ua = __uint_as_float(d1[i]) * srow1 * inv;
                        const float h = silu_f(ga) * ua;
                        if (valid) a.hf[(int64_t)p * a.I + row] = h;
                        float m = valid ? fabsf(h) : 0.0f;
#pragma unroll
                        for (int o2 = 16; o2 > 0; o2 >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o2));
                        if (lane == 0 && valid) atomicMax(a.hmax + p, __float_as_uint(m));
                    } else if (valid) {
                        a.o[(int64_t)p * a.H + row] = __uint_as_float(d0[i]) * srow0 * __ldg(a.act_inv + p);
                    }
                }
            }
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&accempty);
        }
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (warp == 0) tmem_dealloc(tmem, kTmemCols);
}

// ---------------------------------------------------------------------------
// Glue of the tensor-core path
// ---------------------------------------------------------------------------

// xg[p][:] = hi fp16 part of token pair_tok[p] (scaled by its power of two);
// also clears the per-pair max |h| used by the h conversion
__global__ void __launch_bounds__(256)
gather_x_kernel(const __half* __restrict__ xq, const int32_t* __restrict__ pair_tok, int P, int H,
                __half* __restrict__ xg, uint32_t* __restrict__ hmax) {
    const int64_t i = (int64_t)blockIdx.x * 256 + threadIdx.x;   // one 16-byte chunk (8 fp16)
    const int per = H / 8;
    if (i < (int64_t)P * per) {
        const int p = (int)(i / per), c = (int)(i % per);
        const int kb = c / 8, within = c % 8;   // 8 chunks of hi per 64-column group
        const uint4 v = __ldg(reinterpret_cast<const uint4*>(xq + ((int64_t)pair_tok[p] * (H / 64) + kb) * 128) + within);
        reinterpret_cast<uint4*>(xg)[i] = v;
    }
    if (i < P) hmax[i] = 0u;
}

// hg[p][:] = fp16(h[p][:] * 2^sh(p)), hinv[p] = 2^-sh(p), from the per-pair max
__global__ void __launch_bounds__(256)
convert_h_kernel(const float* __restrict__ hf, const uint32_t* __restrict__ hmax, int P, int I,
                 __half* __restrict__ hg, float* __restrict__ hinv) {
    const int64_t i = (int64_t)blockIdx.x * 256 + threadIdx.x;  // pairs of values
    if (i >= (int64_t)P * I / 2) return;
    const int p = (int)(i / (I / 2));
    float inv;
    const float sc = act_group_scale(__uint_as_float(hmax[p]), &inv);
    const float2 v = reinterpret_cast<const float2*>(hf)[i];
    reinterpret_cast<__half2*>(hg)[i] = __floats2half2_rn(v.x * sc, v.y * sc);
    if (i % (I / 2) == 0) hinv[p] = inv;
}

// y[t] = residual[t] + sum_j w[t, j] * o[inv(t, j)] + sum_s o[shared pair of t]
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
        const float4 v = *reinterpret_cast<const float4*>(o + ((int64_t)T * k + (int64_t)s * T + t) * H + c);
        acc.x += v.x; acc.y += v.y; acc.z += v.z; acc.w += v.w;
    }
    if (residual) {
        const float4 r = *reinterpret_cast<const float4*>(residual + (int64_t)t * H + c);
        acc.x = r.x + acc.x; acc.y = r.y + acc.y; acc.z = r.z + acc.z; acc.w = r.w + acc.w;
    }
    *reinterpret_cast<float4*>(y + (int64_t)t * H + c) = acc;
}

}  // namespace coli
