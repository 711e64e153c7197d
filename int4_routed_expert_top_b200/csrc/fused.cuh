// fused.cuh - the whole routed MoE layer after the router logits in ONE
// persistent kernel, for small batches (decode, MTP verify: T <= 16 tokens).
//
// Steps (sources are web pages, cited by title and section):
//   top-k   sigmoid scores, bias-corrected selection of k experts (ties to the
//           lower index), weights renormalised over the picks
//           ["解密GLM-5.2-colibri-int4-with-int8-mtp" 模型架构深度解析;
//            "github一周涨11k⭐️！25GB 内存跑 744B GLM-5.2 模型！" 三.1, 四.3]
//   union   (token, slot) pairs grouped by expert, every distinct expert read
//           once for all of its tokens [same article 三.4; "colibrì 實戰指南" 二]
//   gate/up h = silu(Wg' x) * (Wu' x), W' = q * s dequantised int4
//   down    o = Wd' h, then y = sum_j w_j o_j + shared experts (+ residual)
//
// Every CTA (one per SM) first repeats the top-k and the union for the whole
// batch in its own shared memory; the result is deterministic, so all CTAs
// agree without exchanging it.  Then the CTA's producer warp claims work items
// from a global counter: first every (unit, 128-row tile) of gate/up, then every
// (unit, 128-row tile) of down, where a unit is a distinct routed expert of the
// batch or a shared expert.  It streams each item's fragment tiles with 1-D bulk
// copies (the TMA engine) into a ring of 32 KB stages, together with the gs64
// scales and the stage's activation slices of the unit's tokens.  Sixteen
// consumer warps decode the int4 codes in registers and multiply on the tensor
// cores (mma.sync s8 x s8 -> s32), so every sum over a 64-column step is exact.
//
// Activations enter the tensor cores as two signed 8-bit digits of a 15-bit
// fixed-point value: x16 = rint(x * 2^sh) = 256 * hi + lo with hi in [-64, 64]
// and lo in [-128, 127], sh a power of two per token (gate/up input) or per
// (pair, 128 rows of h) (down input) that puts the largest magnitude in
// [2^13, 2^14).  A weight nibble q enters as the s8 value 16 q (the nibble
// placed in the high half of a byte), so the int32 sums are exact; the factor
// 1/16, the weight scales and the activation scales are applied in f32.
//
// A down item of unit u needs h of all of u's gate/up tiles: the producer waits
// (bounded) on the unit's completion counter before copying h.  Gate/up items
// are all claimed before the first down item, so the wait always ends.  The
// CTA that finishes the last down item of a 128-row block of y forms y for the
// block: the same fixed-order sum as the oracle's combine.
#pragma once

#include "common.cuh"
#include "pipeline.cuh"
#include "route.cuh"

namespace coli {

constexpr int kFzWarps = 16;                     // consumer warps
constexpr int kFzProducer = kFzWarps;            // warp that streams the ring
constexpr int kFzService = kFzWarps + 1;         // warp that publishes finished items
constexpr int kFzThreads = 32 * (kFzWarps + 2);
constexpr int kFzHand = 4;                       // finished-item records in flight
constexpr int kFzMaxT = 16;                      // tokens per call on this path
constexpr int kFzMaxE = 256;                     // routed experts on this path
constexpr int kFzMaxUnits = kFzMaxE + 4;
constexpr int kFzMaxK = 32;
constexpr int kFzMaxSlots = 6;
constexpr int kFzCodeBytes = 32768;              // int4 codes per stage
constexpr int kFzScaleOff = kFzCodeBytes;        // gs64 scales, up to 4 KB
constexpr int kFzActOff = kFzCodeBytes + 4096;   // activation records

// Activation slices of one pair in a stage of ns 64-column steps: ns x (64 hi
// bytes + 64 lo bytes), then up to 4 f32 scales, padded so that consecutive
// records are 64 bytes apart modulo 128 (conflict-free 16-byte shared loads).
__host__ __device__ constexpr int fz_rec_bytes(int ns) { return ns * 128 + 64; }

// Steps (64 columns) per stage: gate/up holds two matrices, down one.
__host__ __device__ inline int fz_ns_gateup(int H) { return (H / 64) % 4 == 0 ? 4 : 2; }
__host__ __device__ inline int fz_ns_down(int I) {
    return (I / 64) % 8 == 0 ? 8 : ((I / 64) % 4 == 0 ? 4 : 2);
}

struct FusedArgs {
    const uint8_t* experts;
    int64_t blob_bytes;
    BlobLayout L;
    const float* zpart;     // [KS][T][E] router logit slices
    int KS;
    const float* bias;      // [E]
    float routed_scale;
    int norm_topk;
    const int8_t* xq8;      // [T][H/64][128]  hi (64 B) + lo (64 B) per step, permuted
    const float* xinv8;     // [T] inverse activation scale
    int8_t* hq8;            // [I/64/ns_dn][P][rec_dn]
    float* o;               // [P][H]
    int32_t* sync;          // queue [1] | gu_done [kFzMaxUnits] | dn_done [H/128], zeroed per call
    int32_t* idx;           // [T*k] picks (written by CTA 0)
    float* w;               // [T*k]
    const float* residual;  // [T][H] or nullptr
    float* y;               // [T][H]
    int32_t* err;
    int T, E, k, n_shared, H, I, group;
    int slots;              // ring stages
    int slot_bytes;
};

__host__ __device__ inline int fz_sync_ints(int H) { return 1 + kFzMaxUnits + H / 128; }

// D (16x8 s32) += A (16x32 s8, row) * B (32x8 s8, col)
__device__ __forceinline__ void mma_s8_16832(int d[4], const uint32_t a[4], uint32_t b0,
                                             uint32_t b1) {
    asm volatile(
        "mma.sync.aligned.m16n8k32.row.col.s32.s8.s8.s32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, "
        "{%8,%9}, {%0,%1,%2,%3};"
        : "+r"(d[0]), "+r"(d[1]), "+r"(d[2]), "+r"(d[3])
        : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

// One fragment-tile word (rows r0, r1 = r0 + 8; columns c0..c0+3, nibble order
// documented in common.cuh) into two s8x4 registers: row r0 then row r1, each
// holding 16 q for columns c0, c0+1, c0+2, c0+3 in byte order.
__device__ __forceinline__ void decode_word_s8(uint32_t w, uint32_t& r0, uint32_t& r1) {
    const uint32_t lo = (w << 4) & 0xF0F0F0F0u;  // (r0,c0) (r1,c0) (r0,c0+1) (r1,c0+1)
    const uint32_t hi = w & 0xF0F0F0F0u;         // (r0,c0+2) (r1,c0+2) (r0,c0+3) (r1,c0+3)
    r0 = __byte_perm(lo, hi, 0x6420);
    r1 = __byte_perm(lo, hi, 0x7531);
}

__device__ __forceinline__ int ld_acquire_gpu(const int32_t* p) {
    int v;
    asm volatile("ld.acquire.gpu.global.b32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
    return v;
}

// order this thread's generic-proxy view before its later async-proxy (bulk
// copy) reads of global memory
__device__ __forceinline__ void fence_proxy_async_global() {
    asm volatile("fence.proxy.async.global;" ::: "memory");
}

}  // namespace coli

namespace coli {


// ---------------------------------------------------------------------------
// Shared memory of a fused CTA besides the ring (static).
// ---------------------------------------------------------------------------
struct FusedShared {
    uint64_t full[kFzMaxSlots], empty[kFzMaxSlots];
    uint64_t hand_full[kFzHand], hand_empty[kFzHand];
    uint64_t cbar;
    int meta_item[kFzMaxSlots], meta_st[kFzMaxSlots];
    int hand_item[kFzHand];
    int u_exp[kFzMaxUnits], u_p0[kFzMaxUnits], u_p1[kFzMaxUnits];
    int pair_tok[kFzMaxT * (kFzMaxK + 4)];
    int inv[kFzMaxT * kFzMaxK];
    int pick_e[kFzMaxT * kFzMaxK];
    float pick_w[kFzMaxT * kFzMaxK];
    float xinv[kFzMaxT];
    float xch[8][16][kFzMaxT];   // epilogue exchange between warp pairs
    float wmax[8][kFzMaxT];
    int n_uniq;
};

// Top-k of token t by one warp (E <= 256: up to 8 candidates per lane).
// Order: selection score descending, expert index ascending.
__device__ __forceinline__ void fz_topk_token(const FusedArgs& a, int t, FusedShared& sh) {
    const int lane = threadIdx.x & 31;
    float z[8], sc[8], sel[8];
#pragma unroll
    for (int i = 0; i < 8; ++i) {
        const int e = lane + 32 * i;
        z[i] = e < a.E ? __ldcg(a.zpart + (int64_t)t * a.E + e) : 0.0f;
    }
    for (int ks = 1; ks < a.KS; ++ks)  // further K slices, in slice order
#pragma unroll
        for (int i = 0; i < 8; ++i) {
            const int e = lane + 32 * i;
            if (e < a.E) z[i] += __ldcg(a.zpart + ((int64_t)ks * a.T + t) * a.E + e);
        }
#pragma unroll
    for (int i = 0; i < 8; ++i) {
        const int e = lane + 32 * i;
        sc[i] = 0.0f;
        sel[i] = -INFINITY;
        if (e < a.E) {
            const float s = 1.0f / (1.0f + expf(-z[i]));
            sc[i] = s;
            sel[i] = s + __ldg(a.bias + e);
        }
    }
    float mine = 0.0f;
    int mine_e = 0;
    for (int j = 0; j < a.k; ++j) {
        float bv = -INFINITY, bs = 0.0f;
        int be = 0x7fffffff;
#pragma unroll
        for (int i = 0; i < 8; ++i) {
            const int e = lane + 32 * i;
            if (sel[i] > bv || (sel[i] == bv && e < be)) { bv = sel[i]; be = e; bs = sc[i]; }
        }
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) {
            const float ov = __shfl_xor_sync(0xffffffffu, bv, o);
            const int oe = __shfl_xor_sync(0xffffffffu, be, o);
            const float os = __shfl_xor_sync(0xffffffffu, bs, o);
            if (ov > bv || (ov == bv && oe < be)) { bv = ov; be = oe; bs = os; }
        }
        if (lane == j) { mine = bs; mine_e = be; }
#pragma unroll
        for (int i = 0; i < 8; ++i)
            if (lane + 32 * i == be) sel[i] = -INFINITY;
    }
    float denom = 0.0f;  // over the picks in pick order
    for (int j = 0; j < a.k; ++j) denom += __shfl_sync(0xffffffffu, mine, j);
    if (lane < a.k) {
        sh.pick_e[t * a.k + lane] = mine_e;
        sh.pick_w[t * a.k + lane] = (a.norm_topk ? mine / denom : mine) * a.routed_scale;
    }
}

// Top-k of every token and the batch union, in this CTA's shared memory.
// scratch: 3 * E ints (any shared memory not yet in use).  Returns the units.
__device__ __forceinline__ int fz_route_union(const FusedArgs& a, FusedShared& sh,
                                              int* scratch) {
    constexpr int kAllWarps = kFzThreads / 32;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    int* cnt = scratch;
    uint32_t* bits = reinterpret_cast<uint32_t*>(scratch + a.E);
    int* excl = scratch + 2 * a.E;
    for (int e = threadIdx.x; e < a.E; e += kFzThreads) { cnt[e] = 0; bits[e] = 0u; }
    for (int t = threadIdx.x; t < a.T; t += kFzThreads) sh.xinv[t] = __ldcg(a.xinv8 + t);
    for (int t = warp; t < a.T; t += kAllWarps) fz_topk_token(a, t, sh);
    __syncthreads();
    const int Tk = a.T * a.k;
    for (int i = threadIdx.x; i < Tk; i += kFzThreads) {
        const int e = sh.pick_e[i];
        atomicAdd(&cnt[e], 1);
        atomicOr(&bits[e], 1u << (i / a.k));
    }
    __syncthreads();
    if (warp == 0) {  // exclusive scans of counts and of (count > 0): 8 experts per lane
        int c[8], f[8], sc = 0, sf = 0;
#pragma unroll
        for (int i = 0; i < 8; ++i) {
            const int e = 8 * lane + i;
            c[i] = e < a.E ? cnt[e] : 0;
            f[i] = c[i] > 0;
            sc += c[i]; sf += f[i];
        }
        int ic = sc, jf = sf;
#pragma unroll
        for (int d = 1; d < 32; d <<= 1) {
            const int x = __shfl_up_sync(0xffffffffu, ic, d);
            const int y = __shfl_up_sync(0xffffffffu, jf, d);
            if (lane >= d) { ic += x; jf += y; }
        }
        int ec = ic - sc, ef = jf - sf;
#pragma unroll
        for (int i = 0; i < 8; ++i) {
            const int e = 8 * lane + i;
            if (e < a.E) {
                excl[e] = ec;
                if (f[i]) { sh.u_exp[ef] = e; sh.u_p0[ef] = ec; sh.u_p1[ef] = ec + c[i]; }
            }
            ec += c[i]; ef += f[i];
        }
        if (lane == 31) sh.n_uniq = ef;
    }
    __syncthreads();
    const int nu = sh.n_uniq;
    for (int i = threadIdx.x; i < Tk; i += kFzThreads) {
        const int t = i / a.k, e = sh.pick_e[i];
        const int p = excl[e] + __popc(bits[e] & ((1u << t) - 1u));
        sh.pair_tok[p] = t;
        sh.inv[i] = p;
    }
    for (int s = threadIdx.x; s < a.n_shared; s += kFzThreads) {
        sh.u_exp[nu + s] = a.E + s;
        sh.u_p0[nu + s] = Tk + s * a.T;
        sh.u_p1[nu + s] = Tk + (s + 1) * a.T;
    }
    for (int i = threadIdx.x; i < a.n_shared * a.T; i += kFzThreads) sh.pair_tok[Tk + i] = i % a.T;
    if (blockIdx.x == 0)
        for (int i = threadIdx.x; i < Tk; i += kFzThreads) {
            a.idx[i] = sh.pick_e[i];
            a.w[i] = sh.pick_w[i];
        }
    __syncthreads();
    return nu + a.n_shared;
}

// D = A * B with C = 0 (a fresh 64-column partial sum)
__device__ __forceinline__ void mma_s8_16832_zc(int d[4], const uint32_t a[4], uint32_t b0,
                                                uint32_t b1) {
    const int z = 0;
    asm volatile(
        "mma.sync.aligned.m16n8k32.row.col.s32.s8.s8.s32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, "
        "{%8,%9}, {%10,%10,%10,%10};"
        : "=r"(d[0]), "=r"(d[1]), "=r"(d[2]), "=r"(d[3])
        : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1), "r"(z));
}

// Warp-wide bounded wait on an mbarrier phase; every lane returns the result
// and is ordered after lane 0's acquire.
__device__ __forceinline__ bool fz_wait(uint64_t* bar, uint32_t parity, int32_t* err) {
    int ok = 1;
    if ((threadIdx.x & 31) == 0) ok = mbar_wait(bar, parity, err) ? 1 : 0;
    ok = __shfl_sync(0xffffffffu, ok, 0);
    __syncwarp();
    return ok != 0;
}

// Barrier of the consumer warps on an mbarrier (count kFzWarps) with a bounded
// wait, so that a failed warp cannot leave the others blocked for good.
__device__ __forceinline__ bool fz_cbar(uint64_t* bar, uint32_t& phase, int32_t* err) {
    __syncwarp();
    if ((threadIdx.x & 31) == 0) mbar_arrive(bar);
    const bool ok = fz_wait(bar, phase, err);
    phase ^= 1u;
    return ok;
}

// decode the 16-byte unit of one 64-column step into the A fragments of its
// two k32 halves
__device__ __forceinline__ void fz_decode_step(const uint8_t* p, uint32_t A0[4], uint32_t A1[4]) {
    const uint4 u = *reinterpret_cast<const uint4*>(p);
    decode_word_s8(u.x, A0[0], A0[1]);
    decode_word_s8(u.y, A0[2], A0[3]);
    decode_word_s8(u.z, A1[0], A1[1]);
    decode_word_s8(u.w, A1[2], A1[3]);
}

// Work item -> (gate/up?, unit, 128-row tile).  Items: all gate/up tiles of all
// units first (unit-major), then all down tiles.
struct FzItem {
    int gu, u, rt;
};
__device__ __forceinline__ FzItem fz_item(int item, int n_units, int TG, int TD) {
    FzItem r;
    r.gu = item < n_units * TG;
    const int rel = r.gu ? item : item - n_units * TG;
    const int per = r.gu ? TG : TD;
    r.u = rel / per;
    r.rt = rel - r.u * per;
    return r;
}

}  // namespace coli

namespace coli {

// ---------------------------------------------------------------------------
// Producer warp: claim items, stream their stages, then the end marker.
// Ring position: slot s, lap parity lap (flips whenever s wraps to 0).  An
// item's last stage also carries its tile's per-row weight scales.
// ---------------------------------------------------------------------------
template <bool GS>
__device__ __forceinline__ void fz_produce(const FusedArgs& a, FusedShared& sh, uint8_t* ring,
                                           int n_units) {
    const int lane = threadIdx.x & 31;
    const int TG = a.I / 128, TD = a.H / 128;
    const int n_items = n_units * (TG + TD);
    const int P = a.T * (a.k + a.n_shared);
    const int ns_gu = fz_ns_gateup(a.H), ns_dn = fz_ns_down(a.I);
    const int rec_gu = fz_rec_bytes(ns_gu), rec_dn = fz_rec_bytes(ns_dn);
    int32_t* queue = a.sync;
    const int32_t* gu_done = a.sync + 1;
    int s = 0, issued = 0;
    uint32_t lap = 0;
    bool ok = true;
    while (ok) {
        int item = 0;
        if (lane == 0) item = atomicAdd(queue, 1);
        item = __shfl_sync(0xffffffffu, item, 0);
        if (item >= n_items) break;
        const FzItem w = fz_item(item, n_units, TG, TD);
        const int e = sh.u_exp[w.u], p0 = sh.u_p0[w.u], np = sh.u_p1[w.u] - p0;
        const uint8_t* blob = a.experts + (int64_t)e * a.blob_bytes;
        const int ns = w.gu ? ns_gu : ns_dn;
        const int K = w.gu ? a.H : a.I;
        const int nst = K / 64 / ns, ng = GS ? K / 64 : 1;
        const uint8_t* cA = blob + a.L.codes[w.gu ? 0 : 2];
        const uint8_t* cB = blob + a.L.codes[1];
        const float* sA = reinterpret_cast<const float*>(blob + a.L.scales[w.gu ? 0 : 2]);
        const float* sB = reinterpret_cast<const float*>(blob + a.L.scales[1]);
        const int mats = w.gu ? 2 : 1;
        const uint32_t cbytes = (uint32_t)ns * 4096, sbytes = GS ? (uint32_t)ns * 512 : 0u;
        const uint32_t abytes = w.gu ? (uint32_t)(np * ns * 128) : (uint32_t)(np * rec_dn);
        const uint32_t tx = mats * (cbytes + sbytes) + abytes;
        for (int st = 0; st < nst; ++st) {
            if (issued >= a.slots && !fz_wait(&sh.empty[s], lap ^ 1u, a.err)) { ok = false; break; }
            if (lane == 0) { sh.meta_item[s] = item; sh.meta_st[s] = st; }
            __syncwarp();
            uint8_t* sl = ring + (int64_t)s * a.slot_bytes;
            const int kb0 = st * ns;
            const bool rowsc = !GS && st == nst - 1;
            mbar_expect_tx_elect(&sh.full[s], tx + (rowsc ? mats * 512u : 0u));
            const int64_t coff = frag_unit_offset(w.rt, kb0, 0, 0, K);
            bulk_g2s_elect(sl, cA + coff, cbytes, &sh.full[s]);
            if (w.gu) bulk_g2s_elect(sl + cbytes, cB + coff, cbytes, &sh.full[s]);
            if (GS) {
                const int64_t soff = ((int64_t)w.rt * ng + kb0) * kTileRows;
                bulk_g2s_elect(sl + kFzScaleOff, sA + soff, sbytes, &sh.full[s]);
                if (w.gu) bulk_g2s_elect(sl + kFzScaleOff + sbytes, sB + soff, sbytes, &sh.full[s]);
            }
            if (rowsc) {  // per-row scales of the tile, for the epilogue
                bulk_g2s_elect(sl + kFzScaleOff, sA + (int64_t)w.rt * kTileRows, 512u, &sh.full[s]);
                if (w.gu) bulk_g2s_elect(sl + kFzScaleOff + 512, sB + (int64_t)w.rt * kTileRows, 512u,
                                         &sh.full[s]);
            }
            if (w.gu) {
                for (int pp = 0; pp < np; ++pp) {
                    const int tok = sh.pair_tok[p0 + pp];
                    bulk_g2s_elect(sl + kFzActOff + pp * rec_gu,
                                   a.xq8 + ((int64_t)tok * (a.H / 64) + kb0) * 128,
                                   (uint32_t)ns * 128, &sh.full[s]);
                }
            } else {
                if (st == 0) {  // h of this unit: every gate/up tile must be published
                    int done = 1;
                    if (lane == 0) {
                        done = 0;
                        for (uint32_t i = 0; i < kWaitTries; ++i) {
                            if (ld_acquire_gpu(gu_done + w.u) >= TG) { done = 1; break; }
                            __nanosleep(64);
                        }
                        if (!done) atomicOr(a.err, kErrWaitTimeout);
                    }
                    __syncwarp();
                    fence_proxy_async_global();
                }
                bulk_g2s_elect(sl + kFzActOff, a.hq8 + ((int64_t)st * P + p0) * rec_dn, abytes,
                               &sh.full[s]);
            }
            ++issued;
            if (++s == a.slots) { s = 0; lap ^= 1u; }
        }
    }
    if (ok && (issued < a.slots || fz_wait(&sh.empty[s], lap ^ 1u, a.err))) {  // end marker
        if (lane == 0) sh.meta_item[s] = -1;
        __syncwarp();
        if (lane == 0) mbar_arrive(&sh.full[s]);
        ++issued;
    }
    // leave only once every copy issued into the ring has landed
    for (int j = issued > a.slots ? issued - a.slots : 0; j < issued; ++j)
        fz_wait(&sh.full[j % a.slots], (j / a.slots) & 1, nullptr);
}

// ---------------------------------------------------------------------------
// Per-stage tensor-core work of a consumer warp.  Warp w: gate/up -> matrix
// w / 8 (gate, up), 16-row block w % 8, every step of the stage; down -> 16-row
// block w % 8, half w / 8 of the stage's steps.  After an MMA, lane (g, t)
// holds rows g, g + 8 and columns 2t, 2t + 1 of an 8-column group c: column n
// carries pair 4c + (n & 3), high digit for n < 4, low digit for n >= 4, so
// lanes t and t ^ 2 hold the two digits of the same pairs.
// ---------------------------------------------------------------------------
template <int NT, bool GS>
__device__ __forceinline__ void fz_stage_gateup(const uint8_t* sl, int ns, int m, int rb, int lane,
                                                int rec_gu, int acc_i[NT][4], float acc_f[NT][4]) {
    const int g = lane >> 2, t = lane & 3;
    const float lanefac = t < 2 ? 256.0f : 1.0f;
    const uint8_t* cp = sl + m * ns * 4096 + rb * 512 + lane * 16;
    const uint8_t* ap = sl + kFzActOff + (g >> 2) * 64 + t * 16 + (g & 3) * rec_gu;
    const float* scl = reinterpret_cast<const float*>(sl + kFzScaleOff + m * ns * 512) + 16 * rb + g;
#pragma unroll
    for (int j = 0; j < 4; ++j) {
        if (j < ns) {
            uint32_t A0[4], A1[4];
            fz_decode_step(cp + j * 4096, A0, A1);
            if (GS) {
                const float s0 = scl[j * 128] * lanefac, s1 = scl[j * 128 + 8] * lanefac;
#pragma unroll
                for (int c = 0; c < NT; ++c) {
                    const uint4 b = *reinterpret_cast<const uint4*>(ap + 4 * c * rec_gu + j * 128);
                    int d[4];
                    mma_s8_16832_zc(d, A0, b.x, b.y);
                    mma_s8_16832(d, A1, b.z, b.w);
                    acc_f[c][0] = fmaf((float)d[0], s0, acc_f[c][0]);
                    acc_f[c][1] = fmaf((float)d[1], s0, acc_f[c][1]);
                    acc_f[c][2] = fmaf((float)d[2], s1, acc_f[c][2]);
                    acc_f[c][3] = fmaf((float)d[3], s1, acc_f[c][3]);
                }
            } else {
#pragma unroll
                for (int c = 0; c < NT; ++c) {
                    const uint4 b = *reinterpret_cast<const uint4*>(ap + 4 * c * rec_gu + j * 128);
                    mma_s8_16832(acc_i[c], A0, b.x, b.y);
                    mma_s8_16832(acc_i[c], A1, b.z, b.w);
                }
            }
        }
    }
}

template <int NT, bool GS>
__device__ __forceinline__ void fz_stage_down(const uint8_t* sl, int ns, int half, int rb, int lane,
                                              int rec_dn, float acc_f[NT][4]) {
    const int g = lane >> 2, t = lane & 3;
    const float lanefac = t < 2 ? 256.0f : 1.0f;
    const int nsh = ns / 2, j0 = half * nsh;
    const uint8_t* cp = sl + (j0 * 8 + rb) * 512 + lane * 16;
    const uint8_t* ap = sl + kFzActOff + (g >> 2) * 64 + t * 16 + (g & 3) * rec_dn + j0 * 128;
    // inverse scales of h for the two pairs of this lane's columns
    const float* hsc = reinterpret_cast<const float*>(sl + kFzActOff + ns * 128 + 2 * (t & 1) * rec_dn) + j0 / 2;
    const float* scl = reinterpret_cast<const float*>(sl + kFzScaleOff) + j0 * 128 + 16 * rb + g;
#pragma unroll
    for (int jj = 0; jj < 4; ++jj) {
        if (jj < nsh) {
            uint32_t A0[4], A1[4];
            fz_decode_step(cp + jj * 4096, A0, A1);
            const float s0 = GS ? scl[jj * 128] * lanefac : lanefac;
            const float s1 = GS ? scl[jj * 128 + 8] * lanefac : lanefac;
#pragma unroll
            for (int c = 0; c < NT; ++c) {
                const uint4 b = *reinterpret_cast<const uint4*>(ap + 4 * c * rec_dn + jj * 128);
                int d[4];
                mma_s8_16832_zc(d, A0, b.x, b.y);
                mma_s8_16832(d, A1, b.z, b.w);
                const float* hs = reinterpret_cast<const float*>(
                    reinterpret_cast<const uint8_t*>(hsc) + 4 * c * rec_dn) + jj / 2;
                const float h0 = hs[0];
                const float h1 = *reinterpret_cast<const float*>(reinterpret_cast<const uint8_t*>(hs) + rec_dn);
                acc_f[c][0] = fmaf((float)d[0], s0 * h0, acc_f[c][0]);
                acc_f[c][1] = fmaf((float)d[1], s0 * h1, acc_f[c][1]);
                acc_f[c][2] = fmaf((float)d[2], s1 * h0, acc_f[c][2]);
                acc_f[c][3] = fmaf((float)d[3], s1 * h1, acc_f[c][3]);
            }
        }
    }
}

}  // namespace coli

namespace coli {

// Hand a finished item to the service warp: every consumer warp arrives on
// the record's barrier after its own global writes (warp 0 writes the record).
struct FzHand {
    int slot = 0, pushed = 0;
    uint32_t lap = 0;
};
__device__ __forceinline__ bool fz_hand_push(FusedShared& sh, FzHand& h, int item, int32_t* err) {
    const int lane = threadIdx.x & 31;
    if (h.pushed >= kFzHand && !fz_wait(&sh.hand_empty[h.slot], h.lap ^ 1u, err)) return false;
    if (threadIdx.x == 0) sh.hand_item[h.slot] = item;
    __syncwarp();
    if (lane == 0) mbar_arrive(&sh.hand_full[h.slot]);
    ++h.pushed;
    if (++h.slot == kFzHand) { h.slot = 0; h.lap ^= 1u; }
    return true;
}

// ---------------------------------------------------------------------------
// Consumer warps: stages, then per item an epilogue that exchanges partial
// results through shared memory, writes h (gate/up) or o (down) to global
// memory and hands the item to the service warp.
// ---------------------------------------------------------------------------
template <int NT, bool GS>
__device__ __forceinline__ void fz_consume(const FusedArgs& a, FusedShared& sh, uint8_t* ring,
                                           int n_units) {
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int g = lane >> 2, t = lane & 3;
    const int rb = warp & 7, half = warp >> 3;
    const int TG = a.I / 128, TD = a.H / 128;
    const int P = a.T * (a.k + a.n_shared);
    const int ns_gu = fz_ns_gateup(a.H), ns_dn = fz_ns_down(a.I);
    const int rec_gu = fz_rec_bytes(ns_gu), rec_dn = fz_rec_bytes(ns_dn);
    const float lanefac = t < 2 ? 256.0f : 1.0f;
    const bool wr = t < 2;  // after the digit combine: lanes holding results
    uint32_t cphase = 0, lap = 0;
    int s = 0;
    FzHand hand;
    FzItem w{0, 0, 0};
    int p0 = 0, np = 0, nst = 0;
    float sw0 = 1.0f, sw1 = 1.0f;  // per-row weight scales of rows g, g + 8
    int acc_i[NT][4];
    float acc_f[NT][4];
    for (;;) {
        if (!fz_wait(&sh.full[s], lap, a.err)) return;
        const int item = sh.meta_item[s], st = sh.meta_st[s];
        if (item < 0) {
            fz_hand_push(sh, hand, -1, a.err);
            return;
        }
        if (st == 0) {  // a new item
            w = fz_item(item, n_units, TG, TD);
            p0 = sh.u_p0[w.u];
            np = sh.u_p1[w.u] - p0;
            nst = w.gu ? a.H / 64 / ns_gu : a.I / 64 / ns_dn;
#pragma unroll
            for (int c = 0; c < NT; ++c)
#pragma unroll
                for (int i = 0; i < 4; ++i) { acc_i[c][i] = 0; acc_f[c][i] = 0.0f; }
        }
        const uint8_t* sl = ring + (int64_t)s * a.slot_bytes;
        if (w.gu) fz_stage_gateup<NT, GS>(sl, ns_gu, half, rb, lane, rec_gu, acc_i, acc_f);
        else      fz_stage_down<NT, GS>(sl, ns_dn, half, rb, lane, rec_dn, acc_f);
        const bool last = st == nst - 1;
        if (!GS && last) {
            const float* rs = reinterpret_cast<const float*>(sl + kFzScaleOff + (w.gu ? half * 512 : 0)) +
                              16 * rb + g;
            sw0 = rs[0];
            sw1 = rs[8];
        }
        __syncwarp();
        if (lane == 0) mbar_arrive(&sh.empty[s]);
        if (++s == a.slots) { s = 0; lap ^= 1u; }
        if (!last) continue;

        // ---------------- epilogue of the item ----------------
        float v[NT][4];
#pragma unroll
        for (int c = 0; c < NT; ++c)
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                float x = (w.gu && !GS) ? (float)acc_i[c][i] * lanefac : acc_f[c][i];
                x += __shfl_xor_sync(0xffffffffu, x, 2);  // high digit * 256 + low digit
                if (!GS) x *= (i >> 1) ? sw1 : sw0;
                v[c][i] = x;
            }
        // lanes t < 2 now hold rows g + 8 (i >> 1), pairs 4c + 2t + (i & 1)
        if (w.gu) {
            const int m = half;
#pragma unroll
            for (int c = 0; c < NT; ++c)
#pragma unroll
                for (int i = 0; i < 4; ++i) {
                    const int pp = 4 * c + 2 * t + (i & 1), rr = g + 8 * (i >> 1);
                    if (wr && pp < np) {
                        v[c][i] *= sh.xinv[sh.pair_tok[p0 + pp]] * 0.0625f;
                        if (m == 1) sh.xch[rb][rr][pp] = v[c][i];
                    }
                }
            if (!fz_cbar(&sh.cbar, cphase, a.err)) return;
            if (m == 0) {
#pragma unroll
                for (int c = 0; c < NT; ++c) {
                    float mx[2] = {0.0f, 0.0f};
#pragma unroll
                    for (int i = 0; i < 4; ++i) {
                        const int pp = 4 * c + 2 * t + (i & 1), rr = g + 8 * (i >> 1);
                        float h = 0.0f;
                        if (wr && pp < np) h = silu_f(v[c][i]) * sh.xch[rb][rr][pp];
                        v[c][i] = h;
                        mx[i & 1] = fmaxf(mx[i & 1], fabsf(h));
                    }
#pragma unroll
                    for (int q = 0; q < 2; ++q) {
                        float mm = mx[q];
                        mm = fmaxf(mm, __shfl_xor_sync(0xffffffffu, mm, 4));
                        mm = fmaxf(mm, __shfl_xor_sync(0xffffffffu, mm, 8));
                        mm = fmaxf(mm, __shfl_xor_sync(0xffffffffu, mm, 16));
                        const int pp = 4 * c + 2 * t + q;
                        if (g == 0 && wr && pp < np) sh.wmax[rb][pp] = mm;
                    }
                }
            }
            if (!fz_cbar(&sh.cbar, cphase, a.err)) return;
            if (m == 0 && wr) {
                const int dstep = 2 * w.rt + rb / 4;  // down step holding these rows of h
                const int sd = dstep / ns_dn, jj = dstep % ns_dn;
#pragma unroll
                for (int c = 0; c < NT; ++c)
#pragma unroll
                    for (int q = 0; q < 2; ++q) {
                        const int pp = 4 * c + 2 * t + q;
                        if (pp >= np) continue;
                        float M = sh.wmax[0][pp];
#pragma unroll
                        for (int r2 = 1; r2 < 8; ++r2) M = fmaxf(M, sh.wmax[r2][pp]);
                        float inv;
                        const float sc = fz_scale(M, &inv);
                        int8_t* rec = a.hq8 + ((int64_t)sd * P + p0 + pp) * rec_dn;
#pragma unroll
                        for (int hr = 0; hr < 2; ++hr) {
                            int hi, lo;
                            fz_split(v[c][2 * hr + q], sc, hi, lo);
                            const int pos = fz_act_pos(16 * (rb % 4) + g + 8 * hr);
                            rec[jj * 128 + pos] = (int8_t)hi;
                            rec[jj * 128 + 64 + pos] = (int8_t)lo;
                        }
                        if (rb == 0 && g == 0)
                            reinterpret_cast<float*>(rec + ns_dn * 128)[(2 * w.rt % ns_dn) / 2] = inv;
                    }
            }
        } else {
            if (half == 1 && wr) {
#pragma unroll
                for (int c = 0; c < NT; ++c)
#pragma unroll
                    for (int i = 0; i < 4; ++i) {
                        const int pp = 4 * c + 2 * t + (i & 1), rr = g + 8 * (i >> 1);
                        if (pp < np) sh.xch[rb][rr][pp] = v[c][i];
                    }
            }
            if (!fz_cbar(&sh.cbar, cphase, a.err)) return;
            if (half == 0 && wr) {
#pragma unroll
                for (int c = 0; c < NT; ++c)
#pragma unroll
                    for (int i = 0; i < 4; ++i) {
                        const int pp = 4 * c + 2 * t + (i & 1), rr = g + 8 * (i >> 1);
                        if (pp >= np) continue;
                        // the half-1 partial was scaled by its lanes too
                        const float x = (v[c][i] + sh.xch[rb][rr][pp]) * 0.0625f;
                        a.o[(int64_t)(p0 + pp) * a.H + w.rt * 128 + 16 * rb + rr] = x;
                    }
            }
        }
        if (!fz_hand_push(sh, hand, item, a.err)) return;
    }
}

// ---------------------------------------------------------------------------
// Service warp: for every finished item, make its global writes visible and
// count it (gate/up: per unit; down: per 128-row block of y).  The item that
// completes a block of y has this warp form y there: for each token, the sum
// over its picks in pick order of w_j * o_j, then the shared experts, then the
// residual.
// ---------------------------------------------------------------------------
__device__ __forceinline__ void fz_service(const FusedArgs& a, FusedShared& sh, int n_units) {
    const int lane = threadIdx.x & 31;
    const int TG = a.I / 128, TD = a.H / 128;
    int32_t* gu_done = a.sync + 1;
    int32_t* dn_done = a.sync + 1 + kFzMaxUnits;
    const int Tk = a.T * a.k;
    int hs = 0;
    uint32_t hlap = 0;
    for (;;) {
        if (!fz_wait(&sh.hand_full[hs], hlap, a.err)) return;
        const int item = sh.hand_item[hs];
        if (item < 0) return;
        const FzItem w = fz_item(item, n_units, TG, TD);
        int last = 0;
        if (lane == 0) {
            __threadfence();  // the consumers' writes of this item, before the count
            if (w.gu) atomicAdd(gu_done + w.u, 1);
            else last = atomicAdd(dn_done + w.rt, 1) == n_units - 1;
        }
        last = __shfl_sync(0xffffffffu, last, 0);
        if (last) {  // every unit's o of this 128-row block is written: form y
            __threadfence();
            for (int q = lane; q < a.T * 128; q += 32) {
                const int tt = q >> 7, r = w.rt * 128 + (q & 127);
                float acc = 0.0f;
                for (int j0 = 0; j0 < a.k; j0 += 8) {  // loads of 8 picks in flight
                    float ov[8];
#pragma unroll
                    for (int jj = 0; jj < 8; ++jj)
                        ov[jj] = j0 + jj < a.k
                                     ? __ldcg(a.o + (int64_t)sh.inv[tt * a.k + j0 + jj] * a.H + r)
                                     : 0.0f;
#pragma unroll
                    for (int jj = 0; jj < 8; ++jj)
                        if (j0 + jj < a.k) acc = fmaf(sh.pick_w[tt * a.k + j0 + jj], ov[jj], acc);
                }
                for (int s2 = 0; s2 < a.n_shared; ++s2)
                    acc += __ldcg(a.o + ((int64_t)Tk + (int64_t)s2 * a.T + tt) * a.H + r);
                if (a.residual) acc = a.residual[(int64_t)tt * a.H + r] + acc;
                a.y[(int64_t)tt * a.H + r] = acc;
            }
        }
        __syncwarp();
        if (lane == 0) mbar_arrive(&sh.hand_empty[hs]);
        if (++hs == kFzHand) { hs = 0; hlap ^= 1u; }
    }
}

template <int NT, bool GS>
__global__ void __launch_bounds__(kFzThreads, 1)
moe_fused_kernel(FusedArgs a) {
    extern __shared__ __align__(128) uint8_t fz_smem[];
    __shared__ FusedShared sh;
    const int n_units = fz_route_union(a, sh, reinterpret_cast<int*>(fz_smem));
    if (threadIdx.x == 0) {
        for (int s = 0; s < a.slots; ++s) { mbar_init(&sh.full[s], 1); mbar_init(&sh.empty[s], kFzWarps); }
        for (int h = 0; h < kFzHand; ++h) { mbar_init(&sh.hand_full[h], kFzWarps); mbar_init(&sh.hand_empty[h], 1); }
        mbar_init(&sh.cbar, kFzWarps);
        fence_mbar_init();
    }
    __syncthreads();
    const int warp = threadIdx.x >> 5;
    if (warp == kFzProducer) fz_produce<GS>(a, sh, fz_smem, n_units);
    else if (warp == kFzService) fz_service(a, sh, n_units);
    else fz_consume<NT, GS>(a, sh, fz_smem, n_units);
}

}  // namespace coli
