// gemm.cuh - tcgen05 grouped GEMM of the int4 experts for large batches
// (prefill and big verify batches), where each expert sees enough tokens for the
// work to be a dense contraction.
//
// Orientation ("swap AB"): D[r, n] = sum_k W[r, k] * X[n, k] with the weight
// rows as the MMA M dimension (a 128-row tile) and up to 64 of a unit's tokens
// as N.  At these batch sizes the layer streams every expert once and does
// little arithmetic per weight byte, so the kernel is built to keep HBM busy and
// the int4 decode off the critical path.  Per CTA (persistent, one per SM, all
// 512 TMEM columns, 24 warps):
//   warp 0       producer: 1-D bulk copies of the int4 fragment tiles (32 KB
//                a stage: gate and up of four 64-column steps, or eight steps of
//                down) with their gs64 scales, and one 2-D TMA load of the
//                tokens (fp16, 128-byte swizzle, a 64 x 64 box) per step into a
//                3-stage ring of 68 KB stages;
//   warp 1       one lane issues tcgen05.mma (kind::f16, f32 accumulators in
//                TMEM), A from TMEM and B from shared memory;
//   warps 4-7    epilogue: TMEM accumulators -> registers -> global;
//   warps 8-23   decode: each warp turns one 16-row x 64-column block of an A
//                unit (512 B of nibbles) into exact fp16 (q, or q*s for gs64)
//                and writes it to TMEM with tcgen05.st.16x256b, whose lane and
//                column layout is that of the fragment tiles.
// TMEM columns: accumulators [0, 256) as two buffers of 128 (gate at +0, up at
// +64; down at +0), so the epilogue of one tile overlaps the next tile's main
// loop; A stages at 256 + 64 a (a = 0..3), 32 columns per slot.
//
// Epilogues: gate/up writes h = silu(a) * u in f32 and the per-pair max |h|;
// down writes o in f32.  Per-row weight scales and the activations' powers of
// two are applied there in f32.
#pragma once

#include <cuda.h>

#include "coli_moe.h"
#include "common.cuh"
#include "pipeline.cuh"

namespace coli {

constexpr int kGemmThreads = 768;
constexpr int kGemmStages = 3;                        // shared-memory ring (68 KB stages)
constexpr int kGemmAStages = 4;                       // TMEM A ring
constexpr int kGemmAccBufs = 2;                       // TMEM accumulator buffers (128 columns each)
constexpr int kGemmABase = 128 * kGemmAccBufs;        // first TMEM column of the A ring
static_assert(kGemmABase + 64 * kGemmAStages <= 512, "TMEM holds 512 columns");
constexpr int kGemmMaxN = 64;                         // tokens per tile
constexpr int kGemmDecodeWarp0 = 8;
constexpr int kGemmDecodeWarps = 16;
constexpr int kGemmEpiWarp0 = 4;
// A ring stage holds four 64-column steps of the tokens (B atoms) and the int4
// codes that meet them: for gate/up four A units (one step of gate and of up,
// 8 KB of codes each), for down two A units (two steps of down each).
constexpr int kAtomBytes = kGemmMaxN * 128;           // one 64-column B atom, 64 rows
constexpr int kStageAtoms = 4;
constexpr int kStageB = kStageAtoms * kAtomBytes;     // 32 KB
constexpr int kStageCodes = 8 * 4096;                 // 32 KB: eight 128 x 64 nibble blocks
constexpr int kStageScales = 8 * 512;
constexpr int kStageBytes = kStageB + kStageCodes + kStageScales;   // 68 KB, 1 KB multiple
constexpr int kGemmSmem = kGemmStages * kStageBytes + 1024;        // + alignment slack
static_assert(kStageBytes % 1024 == 0, "stages must stay 1 KB aligned for the swizzle");
constexpr uint32_t kTmemCols = 512;

struct GemmArgs {
    ExpertStore store;
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
// elected-lane forms (see pipeline.cuh): the whole warp executes them
__device__ __forceinline__ void tc_commit_elect(uint64_t* bar) {
    asm volatile(
        "{\n .reg .pred e;\n elect.sync _|e, 0xffffffff;\n"
        " @e tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];\n}"
        ::"r"(smem_u32(bar))
        : "memory");
}
__device__ __forceinline__ void tc_mma_ts_elect(uint32_t d, uint32_t a, uint64_t bdesc, uint32_t idesc,
                                                uint32_t accumulate) {
    asm volatile(
        "{\n .reg .pred p, e;\n elect.sync _|e, 0xffffffff;\n setp.ne.b32 p, %4, 0;\n"
        " @e tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, p;\n}"
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

// Walks the tiles of one CTA in increasing order: unit by unit, N tile by N
// tile, row tile fastest (so CTAs running at the same time share a unit's
// tokens in L2).  The cursor only moves forward, so a CTA scans the unit list
// once.
struct TileCursor {
    int u = 0, base = 0;
    __device__ __forceinline__ bool next(const GemmArgs& a, int n_units, int RT, int tile, int& p0,
                                         int& n, int& rt) {
        for (; u < n_units; ++u) {
            const int b = a.unit_begin[u], e = a.unit_end[u];
            const int cnt = (e - b + kGemmMaxN - 1) / kGemmMaxN * RT;
            if (tile < base + cnt) {
                const int idx = tile - base, j = idx / RT;
                rt = idx - j * RT;
                p0 = b + j * kGemmMaxN;
                n = min(kGemmMaxN, e - p0);
                return true;
            }
            base += cnt;
        }
        return false;
    }
};

__device__ __forceinline__ uint4 lds128(uint32_t addr) {
    uint4 v;
    asm volatile("ld.shared.v4.b32 {%0, %1, %2, %3}, [%4];"
                 : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w) : "r"(addr));
    return v;
}
__device__ __forceinline__ float lds32f(uint32_t addr) {
    float v;
    asm volatile("ld.shared.f32 %0, [%1];" : "=f"(v) : "r"(addr));
    return v;
}

__global__ void __launch_bounds__(kGemmThreads, 1)
moe_gemm_kernel(const __grid_constant__ CUtensorMap bmap, GemmArgs a) {
    extern __shared__ uint8_t gm_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(gm_raw) + 1023) & ~uintptr_t(1023));
    __shared__ __align__(8) uint64_t full[kGemmStages], empty[kGemmStages];
    __shared__ __align__(8) uint64_t afull[kGemmAStages], aempty[kGemmAStages];
    __shared__ __align__(8) uint64_t accfull[kGemmAccBufs], accempty[kGemmAccBufs];
    __shared__ uint32_t tmem_slot;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int n_units = *a.n_units;
    const int KB = a.K / 64;
    const int ng = a.group ? KB : 1;
    const int SPS = KB % 4 == 0 ? 4 : 2;         // 64-column steps per ring stage (KB is even)
    const int KS = KB / SPS;                     // ring stages per tile
    const int APS = a.two ? SPS : SPS / 2;       // A units per ring stage
    const int KA = KS * APS;                     // A units per tile
    const int RT = a.R / kTileRows;
    const int mA = a.two ? 0 : 2;

    if (warp == 0) tmem_alloc(&tmem_slot, kTmemCols);
    if (threadIdx.x == 32) {
        for (int s = 0; s < kGemmStages; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&empty[s], kGemmDecodeWarps + 1);
        }
        for (int s = 0; s < kGemmAStages; ++s) {
            mbar_init(&afull[s], kGemmDecodeWarps);
            mbar_init(&aempty[s], 1);
        }
        for (int b = 0; b < kGemmAccBufs; ++b) {
            mbar_init(&accfull[b], 1);
            mbar_init(&accempty[b], 4);
        }
        fence_mbar_init();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = tmem_slot;
    bool ok = true;  // cleared by a timed-out wait: then no further waits, every barrier kept
    TileCursor cur;

    if (warp == 0) {
        // ---------------- producer (whole warp, elected lane issues) ----------------
        const uint64_t pol = l2_evict_first_policy();
        int u = 0;
        int p0, n, rt;
        for (int tile = blockIdx.x; cur.next(a, n_units, RT, tile, p0, n, rt); tile += gridDim.x) {
            const uint8_t* blob = a.store.blob(a.unit_expert[cur.u]);
            const uint8_t* c0 = blob + a.L.codes[mA];
            const uint8_t* c1 = blob + a.L.codes[1];
            const float* s0 = reinterpret_cast<const float*>(blob + a.L.scales[mA]);
            const float* s1 = reinterpret_cast<const float*>(blob + a.L.scales[1]);
            // a stage: APS A units; gate/up: steps kb0 .. kb0 + SPS - 1 of gate and of
            // up, down: the same steps of down; B: those steps of the tile's tokens
            const uint32_t cbytes = (uint32_t)SPS * 4096;            // per matrix
            const uint32_t sbytes = a.group ? (uint32_t)SPS * 512 : 0u;
            const uint32_t bytes = (cbytes + sbytes) * (a.two ? 2u : 1u) + (uint32_t)SPS * kAtomBytes;
            for (int ks = 0; ks < KS; ++ks, ++u) {
                const int s = u % kGemmStages;
                if (u >= kGemmStages && ok && !mbar_wait_warp_sleep(&empty[s], ((u / kGemmStages) - 1) & 1, a.err)) ok = false;
                uint8_t* st = smem + s * kStageBytes;
                uint8_t* sc = st + kStageB;
                mbar_expect_tx_elect(&full[s], bytes);
                const int kb0 = SPS * ks;
                const int64_t uoff = frag_unit_offset(rt, kb0, 0, 0, a.K);
                bulk_g2s_hint_elect(sc, c0 + uoff, cbytes, &full[s], pol);
                if (a.two) bulk_g2s_hint_elect(sc + cbytes, c1 + uoff, cbytes, &full[s], pol);
                if (a.group) {
                    const int64_t soff = ((int64_t)rt * ng + kb0) * kTileRows;
                    bulk_g2s_elect(sc + kStageCodes, s0 + soff, sbytes, &full[s]);
                    if (a.two) bulk_g2s_elect(sc + kStageCodes + sbytes, s1 + soff, sbytes, &full[s]);
                }
                for (int i = 0; i < SPS; ++i)
                    tma_load_2d_elect(st + i * kAtomBytes, &bmap, (kb0 + i) * 64, p0, &full[s]);
            }
        }
    } else if (warp == 1) {
        // ---------------- MMA issuer (whole warp, elected lane issues) ----------------
        int u = 0, tcount = 0;
        int p0, n, rt;
        for (int tile = blockIdx.x; cur.next(a, n_units, RT, tile, p0, n, rt); tile += gridDim.x, ++tcount) {
            const int np = (n + 15) / 16 * 16;  // N: multiple of 16 for M = 128
            const uint32_t idesc = idesc_f16_f32(np);
            const int buf = tcount % kGemmAccBufs;
            if (tcount >= kGemmAccBufs && ok &&
                !mbar_wait_warp_sleep(&accempty[buf], ((tcount / kGemmAccBufs) - 1) & 1, a.err))
                ok = false;
            tc_fence_after();
            const uint32_t dacc = tmem + 128 * buf;
            for (int ka = 0; ka < KA; ++ka, ++u) {
                const int su = u / APS, w = u - su * APS;  // ring stage, A unit inside it
                const int s = su % kGemmStages, as = u % kGemmAStages;
                if (ok && !mbar_wait_warp_sleep(&afull[as], (u / kGemmAStages) & 1, a.err)) ok = false;
                if (ok && !mbar_wait_warp_sleep(&full[s], (su / kGemmStages) & 1, a.err)) ok = false;
                tc_fence_after();
                uint8_t* st = smem + s * kStageBytes;
                const uint32_t a0 = tmem + kGemmABase + 64 * as;
                if (a.two) {
                    const uint64_t bdesc = smem_desc_sw128(st + w * kAtomBytes);
#pragma unroll
                    for (int slot = 0; slot < 2; ++slot)
#pragma unroll
                        for (int j = 0; j < 4; ++j)
                            tc_mma_ts_elect(dacc + 64 * slot, a0 + 32 * slot + 8 * j, bdesc + 2 * j, idesc,
                                            (ka > 0 || j > 0) ? 1u : 0u);
                } else {
#pragma unroll
                    for (int slot = 0; slot < 2; ++slot) {
                        const uint64_t bdesc = smem_desc_sw128(st + (2 * w + slot) * kAtomBytes);
#pragma unroll
                        for (int j = 0; j < 4; ++j)
                            tc_mma_ts_elect(dacc, a0 + 32 * slot + 8 * j, bdesc + 2 * j, idesc,
                                            (ka > 0 || slot > 0 || j > 0) ? 1u : 0u);
                    }
                }
                tc_commit_elect(&aempty[as]);
                if (w == APS - 1) tc_commit_elect(&empty[s]);
            }
            tc_commit_elect(&accfull[buf]);
        }
    } else if (warp >= kGemmEpiWarp0 && warp < kGemmEpiWarp0 + 4) {
        // ---------------- epilogue: rows 32q + lane of the tile ----------------
        const int q = warp & 3;
        const uint32_t lane_off = (uint32_t)(32 * q) << 16;
        int tcount = 0;
        int p0, n, rt;
        for (int tile = blockIdx.x; cur.next(a, n_units, RT, tile, p0, n, rt); tile += gridDim.x, ++tcount) {
            const int buf = tcount % kGemmAccBufs;
            const int row = rt * kTileRows + 32 * q + lane;
            const uint8_t* blob = a.store.blob(a.unit_expert[cur.u]);
            const float srow0 = a.group ? 1.0f
                : __ldg(reinterpret_cast<const float*>(blob + a.L.scales[mA]) + scale_offset(row, 0, 1));
            const float srow1 = (a.group || !a.two) ? 1.0f
                : __ldg(reinterpret_cast<const float*>(blob + a.L.scales[1]) + scale_offset(row, 0, 1));
            // the activation scale of columns lane and 32 + lane, broadcast below
            float cinv[2];
#pragma unroll
            for (int h = 0; h < 2; ++h) {
                const int c = 32 * h + lane;
                cinv[h] = 0.0f;
                if (c < n) {
                    const int p = p0 + c;
                    cinv[h] = a.two ? __ldg(a.act_inv + (int64_t)a.pair_tok[p] * (a.H / 64))
                                    : __ldg(a.act_inv + p);
                }
            }
            if (ok && !mbar_wait_warp_sleep(&accfull[buf], (tcount / kGemmAccBufs) & 1, a.err)) ok = false;
            tc_fence_after();
            const uint32_t dacc = tmem + lane_off + 128 * buf;
            for (int c0 = 0; c0 < n; c0 += 16) {
                uint32_t d0[16], d1[16];
                tmem_ld_32x32b_x16(dacc + c0, d0);
                if (a.two) tmem_ld_32x32b_x16(dacc + 64 + c0, d1);
                tmem_wait_ld();
                const float ci = c0 < 32 ? cinv[0] : cinv[1];
#pragma unroll
                for (int i = 0; i < 16; ++i) {
                    const int nn = c0 + i;
                    const float inv = __shfl_sync(0xffffffffu, ci, (c0 + i) & 31);
                    if (nn >= n) continue;               // uniform across the warp
                    const int64_t p = p0 + nn;
                    if (a.two) {
                        const float ga = __uint_as_float(d0[i]) * srow0 * inv;
                        const float ua = __uint_as_float(d1[i]) * srow1 * inv;
                        const float h = silu_f(ga) * ua;
                        a.hf[p * a.I + row] = h;
                        float m = fabsf(h);
#pragma unroll
                        for (int o2 = 16; o2 > 0; o2 >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o2));
                        if (lane == 0) atomicMax(a.hmax + p, __float_as_uint(m));
                    } else {
                        a.o[p * a.H + row] = __uint_as_float(d0[i]) * srow0 * inv;
                    }
                }
            }
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&accempty[buf]);
        }
    } else if (warp >= kGemmDecodeWarp0) {
        // ---------------- decode: one 16-row unit block per stage ----------------
        const int dw = warp - kGemmDecodeWarp0;
        const int q = warp & 3;                   // TMEM lane quarter of this warp
        const int hb = (dw >> 2) & 1, slot = dw >> 3;
        const int b8 = 2 * q + hb;
        const int g = lane >> 2;
        const DecodeK dk = a.dk;
        const uint32_t sbase = smem_u32(smem);
        const uint32_t tlane = tmem + ((uint32_t)(32 * q + 16 * hb) << 16) + kGemmABase + 32 * slot;
        int u = 0;
        int p0, n, rt;
        for (int tile = blockIdx.x; cur.next(a, n_units, RT, tile, p0, n, rt); tile += gridDim.x) {
            for (int ka = 0; ka < KA; ++ka, ++u) {
                const int su = u / APS, w = u - su * APS;  // ring stage, A unit inside it
                const int s = su % kGemmStages, as = u % kGemmAStages;
                if (ok && !mbar_wait_warp_sleep(&full[s], (su / kGemmStages) & 1, a.err)) ok = false;
                if (u >= kGemmAStages && ok && !mbar_wait_warp_sleep(&aempty[as], ((u / kGemmAStages) - 1) & 1, a.err)) ok = false;
                tc_fence_after();
                const uint32_t sc = sbase + s * kStageBytes + kStageB;
                // gate/up: matrix `slot`, step w; down: step 2w + slot
                const int blk = a.two ? slot * SPS + w : 2 * w + slot;
                const uint4 un = lds128(sc + blk * 4096 + (b8 * 32 + lane) * 16);
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
                    const uint32_t sa = sc + kStageCodes + blk * 512 + (b8 * 16 + g) * 4;
                    const __half2 s0 = __float2half2_rn(lds32f(sa));
                    const __half2 s1 = __float2half2_rn(lds32f(sa + 32));
#pragma unroll
                    for (int j = 0; j < 4; ++j) {
                        __half2* h = reinterpret_cast<__half2*>(r + 4 * j);
                        h[0] = __hmul2(h[0], s0); h[1] = __hmul2(h[1], s0);
                        h[2] = __hmul2(h[2], s1); h[3] = __hmul2(h[3], s1);
                    }
                }
                tmem_st_16x256b_x4(tlane + 64 * as, r);
                tmem_wait_st();
                tc_fence_before();
                __syncwarp();
                if (lane == 0) {
                    mbar_arrive(&afull[as]);
                    if (w == APS - 1) mbar_arrive(&empty[s]);
                }
            }
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
        if (p < 0) continue;  // a pick this call does not compute
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
