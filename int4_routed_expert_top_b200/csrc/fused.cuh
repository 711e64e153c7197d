// fused.cuh - the routed MoE layer after the router for small batches
// (decode, MTP verify and batches up to T = 64 tokens) in one persistent
// kernel, plus the kernel that forms y from its partial sums.
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
// agree without exchanging it.  A unit is a distinct routed expert of the batch
// or a shared expert.  A work item is (unit u, up to 16 of its pairs, 128-row
// tile tc of I): the CTA's producer warp streams the item's gate and up rows tc
// (all of H) and then the matching 128 columns of the down matrix (all H rows)
// through a ring of ~37 KB stages (32 KB of int4 codes, their scales and the
// activation digits) with 1-D bulk copies (the TMA engine; for 2 to 4 tokens a
// 2-D TMA box brings every token's activation slice).  With one token the
// units are the picks in slot order, so the producer starts streaming as soon
// as warp 0 has the picks, while warp 0 builds the tables the consumers need;
// with at most 32 picks the union is one warp's match/ballot/scan, in the
// order the picks first name their experts (a work order only).  Sixteen consumer warps
// decode the int4 codes in registers and multiply on the tensor cores
// (mma.sync s8 x s8 -> s32, exact int32 sums over each 64-column step).  h of
// the tile never leaves shared memory: the down part of the item multiplies it
// right away, so items depend on nothing but the routing, and each writes the
// partial down product of its 128 columns of I for every H row.  The second
// kernel adds the I/128 partials of every pair in a fixed order and forms y.
//
// Activations enter the tensor cores as two signed 8-bit digits of a 15-bit
// fixed-point value: x16 = rint(x * 2^sh) = 256 * hi + lo with hi in [-64, 64]
// and lo in [-128, 127], sh a power of two per (token, 256 columns) for the
// gate/up input and per (pair, tile) for the down input, putting the largest
// magnitude of its block in [2^13, 2^14).  A weight nibble q enters as the s8
// value 16 q (the nibble placed in the high half of a byte), so the int32 sums
// over a stage are exact; the factor 1/16, the weight scales and the
// activation scales are applied in f32 (once per stage).
#pragma once

#include "common.cuh"
#include "pipeline.cuh"
#include "route.cuh"

namespace coli {

constexpr int kFzWarps = 16;                     // consumer warps
constexpr int kFzProducer = kFzWarps;            // warp that streams the ring
constexpr int kFzThreads = 32 * (kFzWarps + 1);
constexpr int kFzMaxT = 64;                      // tokens per call on this path
constexpr int kFzChunk = 16;                     // pairs per work item (a unit's pairs in chunks)
constexpr int kFzMaxPairs = 640;                 // T * (k + n_shared) on this path
constexpr int kFzMaxE = 256;                     // routed experts on this path
constexpr int kFzMaxUnits = kFzMaxE + 4;
constexpr int kFzMaxK = 32;
constexpr int kFzMaxSlots = 6;
constexpr int kFzSlots = 5;                      // ring stages
constexpr int kFzCodeBytes = 32768;              // int4 codes per stage
constexpr int kFzScaleOff = kFzCodeBytes;        // gs64 scales, up to 4 KB
constexpr int kFzActOff = kFzCodeBytes + 4096;   // activation records
constexpr int kFzRecH = 320;                     // h record of a pair: 2 steps x 128 B + scale

// Activation slices of one pair in a stage of ns 64-column steps: ns x (64 hi
// bytes + 64 lo bytes), then up to 4 f32 scales, padded so that consecutive
// records are 64 bytes apart modulo 128 (conflict-free 16-byte shared loads).
__host__ __device__ constexpr int fz_rec_bytes(int ns) { return ns * 128 + 64; }

// Steps (64 columns) per gate/up stage (both matrices): 32 KB of codes, 4 steps
// of 4-bit codes or 2 of 8-bit ones; the fused path needs H to be a multiple of
// 256 (one activation record per 256 columns).
template <bool W8> __host__ __device__ constexpr int fz_ns_gateup() { return W8 ? 2 : 4; }
// code bytes of one 64-column step of a 128-row tile
template <bool W8> __host__ __device__ constexpr int fz_step_bytes() { return W8 ? 8192 : 4096; }

struct FusedArgs {
    ExpertStore store;
    BlobLayout L;
    PickFilter filter;      // picks this call computes (top-p, expert range)
    const float* score;     // [T][E] sigmoid scores s (router kernel)
    const float* sel;       // [T][E] selection scores s + bias (router kernel)
    float routed_scale;
    int norm_topk;
    const int8_t* xq8;      // [T][H/256][kActRec]: per 256 columns 4 steps of hi (64 B) +
                            //   lo (64 B), permuted, then the f32 inverse scale
    float* part;            // [T][k + n_shared][I/128][H] partial down products
    int32_t* queue;         // work-item counter, zeroed by the router kernel
    int32_t* idx;           // [T*k] picks (written by CTA 0)
    float* w;               // [T*k] weights as applied (0: pick not computed)
    int32_t* inv;           // [T*k] pair of (t, j), -1 for a pick not computed
    int32_t* err;
    int T, E, k, n_shared, H, I, group;
    int slots;              // ring stages
    int slot_bytes;
    // 1: a gate/up stage takes every token's activation record with one 2-D TMA
    // box of the kernel's tensor map over xq8 (T rows of H/256 records read as
    // 32-bit words, boxes of T x kActRec/4 words), stored [token][record];
    // used for 2 <= T <= 4 (one column group).  0: one bulk copy per pair,
    // stored per pair record.
    int act_tma;
    // test of the bounded waits (kernels instantiated with TW only): CTA 0's
    // producer withholds ring stage withhold (its copies are never issued, so
    // the consumers' wait on it runs out) and every wait takes a short limit
    int withhold;
};

// row tiles (of 128 H rows) per down stage: the largest of 4, 3, 2, 1 dividing
// H/128 (4-bit codes, 8 KB per tile) or of 2, 1 (8-bit codes, 16 KB per tile)
__host__ __device__ inline int fz_down_tiles(int H, bool w8) {
    const int n = H / 128;
    if (w8) return n % 2 == 0 ? 2 : 1;
    return n % 4 == 0 ? 4 : (n % 3 == 0 ? 3 : (n % 2 == 0 ? 2 : 1));
}

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
// holding 16 q for columns c0, c0+1, c0+2, c0+3 in byte order (the nibble in
// the high half of a byte reads as the signed byte 16 q).
__device__ __forceinline__ void decode_word_s8(uint32_t w, uint32_t& r0, uint32_t& r1) {
    r0 = w & 0xF0F0F0F0u;
    r1 = (w << 4) & 0xF0F0F0F0u;
}

}  // namespace coli

namespace coli {


// ---------------------------------------------------------------------------
// Shared memory of a fused CTA besides the ring (static).
// ---------------------------------------------------------------------------
struct FusedShared {
    uint64_t full[kFzMaxSlots], empty[kFzMaxSlots];
    uint64_t cbar;
    int meta_item[kFzMaxSlots], meta_st[kFzMaxSlots];
    int u_exp[kFzMaxUnits], u_p0[kFzMaxUnits], u_p1[kFzMaxUnits];
    int u_item0[kFzMaxUnits + 1];                 // first work item of each unit
    int pair_tok[kFzMaxPairs];
    int pair_pick[kFzMaxPairs];                   // t * (k + n_shared) + j of each pair
    float xch[8][16][kFzChunk];                   // up values for the gate warps
    float wmax[8][kFzChunk];                      // per-warp max |h| of each pair
    __align__(16) int8_t hbuf[kFzChunk * kFzRecH]; // h of the current item, s8 digits
    int pick1_e[kFzMaxK];                         // one token: its picks (outside the ring,
    float pick1_w[kFzMaxK];                       // which fills while they are read),
    int unit1_e[kFzMaxK];                         // the computed ones in slot order
    int n_kept1;                                  // and their number
    int n_uniq, n_items;
};

// Top-k and union scratch in the (not yet used) ring: per expert a count, a
// 64-bit token mask and an exclusive prefix; per pick its expert and weight.
struct FzScratch {
    int* cnt;
    unsigned long long* bits;
    int* excl;
    int* pick_e;
    float* pick_w;           // weight as applied: 0 for a pick this call does not compute
    int* unit_e = nullptr;   // one token: computed picks' experts, compacted (or nullptr)
    int* n_kept = nullptr;
};
__device__ __forceinline__ FzScratch fz_scratch(uint8_t* ring, int E) {
    FzScratch r;
    r.bits = reinterpret_cast<unsigned long long*>(ring);
    r.cnt = reinterpret_cast<int*>(ring + 8 * E);
    r.excl = r.cnt + E;
    r.pick_e = r.excl + E;
    r.pick_w = reinterpret_cast<float*>(r.pick_e + kFzMaxT * kFzMaxK);
    return r;
}

// Order-preserving key of a selection score: a larger float gives a larger
// key; -0 and +0 give the same key (they compare equal as floats).
__device__ __forceinline__ uint32_t fz_order_key(float f) {
    const uint32_t u = __float_as_uint(__fadd_rn(f, 0.0f));
    return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}

// Top-k of token t by one warp (E <= 256: up to 8 candidates per lane).
// Order: selection score descending, expert index ascending.  Each round takes
// every lane's best remaining candidate (largest key, then smallest expert),
// the warp's largest key by redux.sync and, among the lanes holding it, the
// smallest expert; that lane retires the candidate.
__device__ __forceinline__ void fz_topk_token(const FusedArgs& a, int t, const FzScratch& sc8) {
    const int lane = threadIdx.x & 31;
    float sc[8];
    uint32_t key[8];
#pragma unroll
    for (int i = 0; i < 8; ++i) {
        const int e = lane + 32 * i;
        const bool ok = e < a.E;
        sc[i] = ok ? __ldcg(a.score + (int64_t)t * a.E + e) : 0.0f;
        key[i] = ok ? fz_order_key(__ldcg(a.sel + (int64_t)t * a.E + e)) : 0u;  // 0: none
    }
    float mine = 0.0f;
    int mine_e = 0;
    for (int j = 0; j < a.k; ++j) {
        uint32_t bk = key[0];
        int bi = 0;
#pragma unroll
        for (int i = 1; i < 8; ++i)
            if (key[i] > bk) { bk = key[i]; bi = i; }
        const uint32_t wk = __reduce_max_sync(0xffffffffu, bk);
        const uint32_t we = __reduce_min_sync(0xffffffffu, bk == wk ? (uint32_t)(lane + 32 * bi) : 0xffffffffu);
        float bs = 0.0f;
#pragma unroll
        for (int i = 0; i < 8; ++i)
            if (i == bi) bs = sc[i];
        const float ws = __shfl_sync(0xffffffffu, bs, (int)(we & 31u));
        if (lane == (int)(we & 31u)) {
#pragma unroll
            for (int i = 0; i < 8; ++i)
                if (i == bi) key[i] = 0u;
        }
        if (lane == j) { mine = ws; mine_e = (int)we; }
    }
    float denom = 0.0f;  // over the picks in pick order
    for (int j = 0; j < a.k; ++j) denom += __shfl_sync(0xffffffffu, mine, j);
    const float wgt = (a.norm_topk ? mine / denom : mine) * a.routed_scale;
    // computed: kept by the pick filter and with a weight that can add something
    const bool kept = pick_kept(a.filter, a.k, wgt, mine_e) && wgt != 0.0f;
    if (lane < a.k) {
        sc8.pick_e[t * a.k + lane] = mine_e;
        sc8.pick_w[t * a.k + lane] = kept ? wgt : 0.0f;
    }
    if (sc8.unit_e) {
        const unsigned km = __ballot_sync(0xffffffffu, kept);
        if (kept) sc8.unit_e[__popc(km & ((1u << lane) - 1u))] = mine_e;
        if (lane == 0) *sc8.n_kept = __popc(km);
    }
}

// The batch union by one warp when there are at most 32 picks, in the order
// the picks first name their experts: units in order of first appearance in
// (token, slot) order, pairs inside a unit in token order.  The work order is
// a scheduling choice only: partial products are indexed by pick, so y does
// not depend on it.  Lane i holds pick i; __match_any_sync finds the picks of
// the same expert, a ballot the first ones, and one shuffle scan of packed
// (pairs, items) gives every unit's first pair and first item.
__device__ __forceinline__ void fz_union_warp(const FusedArgs& a, FusedShared& sh,
                                              const FzScratch& sc8) {
    const int lane = threadIdx.x & 31;
    const int Tk = a.T * a.k, TG = a.I / 128;
    const bool pick = lane < Tk;
    const bool valid = pick && sc8.pick_w[lane] != 0.0f;  // a pick this call computes
    const int e = pick ? sc8.pick_e[lane] : 0;
    const int t = pick ? lane / a.k : 0;
    const unsigned lt = (1u << lane) - 1u;
    const unsigned same = __match_any_sync(0xffffffffu, valid ? e : -1);  // idle lanes: one group
    const bool first = valid && (same & lt) == 0u;
    const unsigned firsts = __ballot_sync(0xffffffffu, first);
    const int nu = __popc(firsts);
    const int cnt = __popc(same);
    const int items = first ? (cnt + kFzChunk - 1) / kFzChunk * TG : 0;
    // inclusive scan of (pairs | items << 16) over the first lanes, lane order
    int incl = first ? (cnt | (items << 16)) : 0;
#pragma unroll
    for (int d = 1; d < 32; d <<= 1) {
        const int v = __shfl_up_sync(0xffffffffu, incl, d);
        if (lane >= d) incl += v;
    }
    const int excl_p = (incl & 0xffff) - (first ? cnt : 0);
    const int excl_i = (incl >> 16) - items;
    const int routed_items = __shfl_sync(0xffffffffu, incl, 31) >> 16;
    // every pick's pair: its unit's first pair plus the earlier picks of the unit
    const int p = __shfl_sync(0xffffffffu, excl_p, __ffs(same) - 1) + __popc(same & lt);
    if (first) {
        const int u = __popc(firsts & lt);
        sh.u_exp[u] = e;
        sh.u_p0[u] = excl_p;
        sh.u_p1[u] = excl_p + cnt;
        sh.u_item0[u] = excl_i;
    }
    if (valid) {
        sh.pair_tok[p] = t;
        sh.pair_pick[p] = t * (a.k + a.n_shared) + (lane - t * a.k);
    }
    if (pick && blockIdx.x == 0) {
        a.idx[lane] = e;
        a.w[lane] = sc8.pick_w[lane];
        a.inv[lane] = valid ? p : -1;
    }
    const int per_shared = (a.T + kFzChunk - 1) / kFzChunk * TG;
    if (lane < a.n_shared) {
        sh.u_exp[nu + lane] = a.E + lane;
        sh.u_p0[nu + lane] = Tk + lane * a.T;
        sh.u_p1[nu + lane] = Tk + (lane + 1) * a.T;
        sh.u_item0[nu + lane] = routed_items + lane * per_shared;
    }
    for (int i = lane; i < a.n_shared * a.T; i += 32) {
        const int tt = i % a.T;
        sh.pair_tok[Tk + i] = tt;
        sh.pair_pick[Tk + i] = tt * (a.k + a.n_shared) + a.k + i / a.T;
    }
    if (lane == 0) {
        sh.n_uniq = nu;
        sh.u_item0[nu + a.n_shared] = routed_items + a.n_shared * per_shared;
        sh.n_items = routed_items + a.n_shared * per_shared;
    }
}

// Top-k of every token and the batch union, in this CTA's shared memory, and
// the work items: unit u's pairs in chunks of kFzChunk, I/128 items per chunk.
// CTA 0 also publishes the picks, weights and pair indices.  Returns the units.
__device__ __forceinline__ int fz_route_union(const FusedArgs& a, FusedShared& sh, uint8_t* ring) {
    constexpr int kAllWarps = kFzThreads / 32;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const FzScratch sc8 = fz_scratch(ring, a.E);
    const int Tk = a.T * a.k;
    const bool small = Tk <= 32;
    if (!small)
        for (int e = threadIdx.x; e < a.E; e += kFzThreads) { sc8.cnt[e] = 0; sc8.bits[e] = 0ull; }
    for (int t = warp; t < a.T; t += kAllWarps) fz_topk_token(a, t, sc8);
    __syncthreads();
    if (small) {
        if (warp == 0) fz_union_warp(a, sh, sc8);
        __syncthreads();
        return sh.n_uniq + a.n_shared;
    }
    for (int i = threadIdx.x; i < Tk; i += kFzThreads) {
        if (sc8.pick_w[i] == 0.0f) continue;  // not computed by this call
        const int e = sc8.pick_e[i];
        atomicAdd(&sc8.cnt[e], 1);
        atomicOr(&sc8.bits[e], 1ull << (i / a.k));
    }
    __syncthreads();
    const int TG = a.I / 128;
    if (warp == 0) {  // exclusive scans of counts, of (count > 0) and of items: 8 experts per lane
        int c[8], f[8], sc = 0, sf = 0, si = 0;
#pragma unroll
        for (int i = 0; i < 8; ++i) {
            const int e = 8 * lane + i;
            c[i] = e < a.E ? sc8.cnt[e] : 0;
            f[i] = c[i] > 0;
            sc += c[i]; sf += f[i]; si += (c[i] + kFzChunk - 1) / kFzChunk;
        }
        int ic = sc, jf = sf, ki = si;
#pragma unroll
        for (int d = 1; d < 32; d <<= 1) {
            const int x = __shfl_up_sync(0xffffffffu, ic, d);
            const int y = __shfl_up_sync(0xffffffffu, jf, d);
            const int z = __shfl_up_sync(0xffffffffu, ki, d);
            if (lane >= d) { ic += x; jf += y; ki += z; }
        }
        int ec = ic - sc, ef = jf - sf, ei = ki - si;
#pragma unroll
        for (int i = 0; i < 8; ++i) {
            const int e = 8 * lane + i;
            if (e < a.E) {
                sc8.excl[e] = ec;
                if (f[i]) {
                    sh.u_exp[ef] = e; sh.u_p0[ef] = ec; sh.u_p1[ef] = ec + c[i];
                    sh.u_item0[ef] = ei * TG;
                }
            }
            ec += c[i]; ef += f[i]; ei += (c[i] + kFzChunk - 1) / kFzChunk;
        }
        if (lane == 31) {
            sh.n_uniq = ef;
            int item = ei * TG;  // the shared experts follow, T pairs each
            for (int s2 = 0; s2 < a.n_shared; ++s2) {
                sh.u_item0[ef + s2] = item;
                item += (a.T + kFzChunk - 1) / kFzChunk * TG;
            }
            sh.u_item0[ef + a.n_shared] = item;
            sh.n_items = item;
        }
    }
    __syncthreads();
    const int nu = sh.n_uniq;
    for (int i = threadIdx.x; i < Tk; i += kFzThreads) {
        const int t = i / a.k, e = sc8.pick_e[i];
        const bool valid = sc8.pick_w[i] != 0.0f;
        const int p = sc8.excl[e] + __popcll(sc8.bits[e] & ((1ull << t) - 1ull));
        if (valid) {
            sh.pair_tok[p] = t;
            sh.pair_pick[p] = t * (a.k + a.n_shared) + (i - t * a.k);
        }
        if (blockIdx.x == 0) {
            a.idx[i] = e;
            a.w[i] = sc8.pick_w[i];
            a.inv[i] = valid ? p : -1;
        }
    }
    for (int s = threadIdx.x; s < a.n_shared; s += kFzThreads) {
        sh.u_exp[nu + s] = a.E + s;
        sh.u_p0[nu + s] = Tk + s * a.T;
        sh.u_p1[nu + s] = Tk + (s + 1) * a.T;
    }
    for (int i = threadIdx.x; i < a.n_shared * a.T; i += kFzThreads) {
        const int t = i % a.T;
        sh.pair_tok[Tk + i] = t;
        sh.pair_pick[Tk + i] = t * (a.k + a.n_shared) + a.k + i / a.T;
    }
    __syncthreads();
    return nu + a.n_shared;
}

// Work item -> (unit, its pairs p0 .. p0 + np - 1, 128-row tile tc of I):
// the unit by binary search over the units' first items.
struct FzWork {
    int u, p0, np, tc;
};
__device__ __forceinline__ FzWork fz_work(const FusedShared& sh, int n_units, int TG, int item) {
    int lo = 0, hi = n_units - 1;  // last unit whose first item is <= item
    while (lo < hi) {
        const int mid = (lo + hi + 1) >> 1;
        if (sh.u_item0[mid] <= item) lo = mid; else hi = mid - 1;
    }
    FzWork w;
    w.u = lo;
    const int rel = item - sh.u_item0[lo];
    const int ch = rel / TG;
    w.tc = rel - ch * TG;
    w.p0 = sh.u_p0[lo] + ch * kFzChunk;
    w.np = min(kFzChunk, sh.u_p1[lo] - w.p0);
    return w;
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
// test: the wait test (a stage withheld): a short limit instead of the default
constexpr uint32_t kFzTestWaitTries = 1u << 12;
__device__ __forceinline__ bool fz_wait(uint64_t* bar, uint32_t parity, int32_t* err, bool test) {
    int ok = 1;
    if ((threadIdx.x & 31) == 0)
        ok = mbar_wait(bar, parity, err, test ? kFzTestWaitTries : kWaitTries) ? 1 : 0;
    ok = __shfl_sync(0xffffffffu, ok, 0);
    __syncwarp();
    return ok != 0;
}

// Barrier of the consumer warps on an mbarrier (count kFzWarps) with a bounded
// wait, so that a failed warp cannot leave the others blocked for good.
__device__ __forceinline__ bool fz_cbar(uint64_t* bar, uint32_t& phase, int32_t* err, bool test) {
    __syncwarp();
    if ((threadIdx.x & 31) == 0) mbar_arrive(bar);
    const bool ok = fz_wait(bar, phase, err, test);
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

}  // namespace coli

namespace coli {

// Stages of one item: the gate/up part, then the down part.
struct FzShape {
    int ns_gu, nst_gu;   // 64-column steps per gate/up stage; gate/up stages
    int rs, nst_dn;      // 128-row tiles per down stage; down stages
    int TG;              // 128-row tiles of I (items per unit)
};
template <bool W8>
__device__ __forceinline__ FzShape fz_shape(const FusedArgs& a) {
    FzShape z;
    z.ns_gu = fz_ns_gateup<W8>();
    z.nst_gu = a.H / 64 / z.ns_gu;
    z.rs = fz_down_tiles(a.H, W8);
    z.nst_dn = a.H / 128 / z.rs;
    z.TG = a.I / 128;
    return z;
}

// ---------------------------------------------------------------------------
// Producer warp: claim items (u, tc), stream their stages, then the end marker.
// Ring position: slot s, lap parity lap (flips whenever s wraps to 0).
//   gate/up stage st: rows tc of gate and of up, steps ns st .. ns st + ns - 1
//     [codes gate | codes up | gs64 scales gate, up | activation records of
//     the pairs (the 256-column record holding these steps)] and, on the last
//     one, the tile's per-row scales of gate and up;
//   down stage: rs tiles of 128 H rows, columns 128 tc .. 128 tc + 127
//     [codes, 8 or 16 KB per tile | scales (per row: 512 B per tile; gs64: 1 KB)].
// ---------------------------------------------------------------------------
template <bool GS, bool W8, bool TW>
__device__ __forceinline__ void fz_produce(const FusedArgs& a, const CUtensorMap* xmap,
                                           FusedShared& sh, uint8_t* ring, int n_units, bool one) {
    const int lane = threadIdx.x & 31;
    const FzShape z = fz_shape<W8>(a);
    constexpr uint32_t kStep = fz_step_bytes<W8>();
    // one token: unit u = item / TG is the u-th computed pick (slot order),
    // then the shared experts, one pair each (token 0); no tables needed
    const int n_items = one ? n_units * z.TG : sh.n_items;
    const int n_kept = n_units - a.n_shared;
    const int rec_gu = kActRec;
    const int ngH = GS ? a.H / 64 : 1, ngI = GS ? a.I / 64 : 1;
    const uint64_t pol = l2_evict_first_policy();
    int s = 0, issued = 0;
    uint32_t lap = 0;
    bool ok = true;
    int item = blockIdx.x;  // first item: by CTA index; later ones from the queue
    while (ok && item < n_items) {
        FzWork wk;
        int e;
        if (one) {
            wk.u = item / z.TG;
            wk.tc = item - wk.u * z.TG;
            wk.p0 = wk.u;
            wk.np = 1;
            e = wk.u < n_kept ? sh.unit1_e[wk.u] : a.E + (wk.u - n_kept);
        } else {
            wk = fz_work(sh, n_units, z.TG, item);
            e = sh.u_exp[wk.u];
        }
        const int tc = wk.tc, p0 = wk.p0, np = wk.np;
        const uint8_t* blob = a.store.blob(e);
        const uint8_t* cG = blob + a.L.codes[0];
        const uint8_t* cU = blob + a.L.codes[1];
        const uint8_t* cD = blob + a.L.codes[2];
        const float* sG = reinterpret_cast<const float*>(blob + a.L.scales[0]);
        const float* sU = reinterpret_cast<const float*>(blob + a.L.scales[1]);
        const float* sD = reinterpret_cast<const float*>(blob + a.L.scales[2]);
        const int nst = z.nst_gu + z.nst_dn;
        for (int st = 0; st < nst; ++st) {
            if (issued >= a.slots && !fz_wait(&sh.empty[s], lap ^ 1u, a.err, TW)) {
                ok = false;
                break;
            }
            if (lane == 0) { sh.meta_item[s] = item; sh.meta_st[s] = st; }
            __syncwarp();
            uint8_t* sl = ring + (int64_t)s * a.slot_bytes;
            if (TW && issued == a.withhold && blockIdx.x == 0) {
                // nothing is copied and the stage's barrier never completes
            } else if (st < z.nst_gu) {
                const int kb0 = st * z.ns_gu;
                const int rec = kb0 / 4;  // the activation record of these steps
                const bool rowsc = !GS && st == z.nst_gu - 1;
                const uint32_t cb = (uint32_t)z.ns_gu * kStep, sb = GS ? (uint32_t)z.ns_gu * 512 : 0u;
                const int nrec = a.act_tma ? a.T : np;  // activation records of the stage
                mbar_expect_tx_elect(&sh.full[s], 2 * (cb + sb) + (uint32_t)(nrec * kActRec) +
                                                      (rowsc ? 1024u : 0u));
                const int64_t coff = (int64_t)tc * (a.H / 64) * kStep + (int64_t)kb0 * kStep;
                bulk_g2s_hint_elect(sl, cG + coff, cb, &sh.full[s], pol);
                bulk_g2s_hint_elect(sl + cb, cU + coff, cb, &sh.full[s], pol);
                if (GS) {
                    const int64_t soff = ((int64_t)tc * ngH + kb0) * kTileRows;
                    bulk_g2s_elect(sl + kFzScaleOff, sG + soff, sb, &sh.full[s]);
                    bulk_g2s_elect(sl + kFzScaleOff + sb, sU + soff, sb, &sh.full[s]);
                }
                if (rowsc) {
                    bulk_g2s_elect(sl + kFzScaleOff, sG + (int64_t)tc * kTileRows, 512u, &sh.full[s]);
                    bulk_g2s_elect(sl + kFzScaleOff + 512, sU + (int64_t)tc * kTileRows, 512u, &sh.full[s]);
                }
                if (a.act_tma) {  // every token's record, [token][kActRec] (x in 4-byte units)
                    tma_load_2d_elect(sl + kFzActOff, xmap, rec * (kActRec / 4), 0, &sh.full[s]);
                } else {
                    for (int pp = 0; pp < np; ++pp) {
                        const int tok = one ? 0 : sh.pair_tok[p0 + pp];
                        bulk_g2s_elect(sl + kFzActOff + pp * rec_gu,
                                       a.xq8 + ((int64_t)tok * (a.H / 256) + rec) * kActRec,
                                       (uint32_t)kActRec, &sh.full[s]);
                    }
                }
            } else {
                const int rt0 = (st - z.nst_gu) * z.rs;
                const uint32_t sb = GS ? 1024u : 512u;
                mbar_expect_tx_elect(&sh.full[s], (uint32_t)z.rs * (2 * kStep + sb));
                for (int q = 0; q < z.rs; ++q) {
                    const int rt = rt0 + q;
                    bulk_g2s_hint_elect(sl + q * 2 * kStep,
                                        cD + (int64_t)rt * (a.I / 64) * kStep + (int64_t)2 * tc * kStep,
                                        2 * kStep, &sh.full[s], pol);
                    if (GS)
                        bulk_g2s_elect(sl + kFzScaleOff + q * 1024,
                                       sD + ((int64_t)rt * ngI + 2 * tc) * kTileRows, 1024u, &sh.full[s]);
                }
                if (!GS)
                    bulk_g2s_elect(sl + kFzScaleOff, sD + (int64_t)rt0 * kTileRows, (uint32_t)z.rs * 512u,
                                   &sh.full[s]);
            }
            ++issued;
            if (++s == a.slots) { s = 0; lap ^= 1u; }
        }
        if (lane == 0) item = (int)gridDim.x + atomicAdd(a.queue, 1);
        item = __shfl_sync(0xffffffffu, item, 0);
    }
    if (ok && (issued < a.slots || fz_wait(&sh.empty[s], lap ^ 1u, a.err, TW))) {  // end marker
        if (lane == 0) sh.meta_item[s] = -1;
        __syncwarp();
        if (lane == 0) mbar_arrive(&sh.full[s]);
        ++issued;
    }
    // leave only once every copy issued into the ring has landed
    for (int j = issued > a.slots ? issued - a.slots : 0; j < issued; ++j)
        fz_wait(&sh.full[j % a.slots], (j / a.slots) & 1, nullptr, TW);
}

}  // namespace coli

namespace coli {

// ---------------------------------------------------------------------------
// Gate/up stage of a consumer warp: matrix m = w / 8 (gate, up), 16-row block
// rb = w % 8 of the tile, every step of the stage.  After an MMA, lane (g, t)
// holds rows g, g + 8 and columns 2t, 2t + 1 of an 8-column group c: column n
// carries pair 4c + (n & 3), high digit for n < 4, low digit for n >= 4, so
// lanes t and t ^ 2 hold the two digits of the same pairs.  The stage's sum
// (exact int32 for per-row weight scales; with the weight scale of each step
// for 64-column groups) is added to acc_f times the activation scale of its
// pair's 256-column record, the lane's digit factor (256 for high digits) and,
// for 4-bit codes, 1/16 (the nibble sits in the high half of an s8 byte).
// xsoff0[q]: offset of the activation record of pair 2(t & 1) + q; jo:
// the first of the stage's steps within that record.
// ---------------------------------------------------------------------------
static_assert(fz_rec_bytes(4) == kActRec, "pair records of a stage are the global records");

// A registers of one 64-column step (both k32 halves) of one lane: 4-bit codes
// are expanded to s8 in registers, 8-bit codes are the registers already
template <bool W8>
__device__ __forceinline__ void fz_load_step(const uint8_t* p, uint32_t A0[4], uint32_t A1[4]) {
    if (W8) {
        const uint4 u0 = *reinterpret_cast<const uint4*>(p);
        const uint4 u1 = *reinterpret_cast<const uint4*>(p + 16);
        A0[0] = u0.x; A0[1] = u0.y; A0[2] = u0.z; A0[3] = u0.w;
        A1[0] = u1.x; A1[1] = u1.y; A1[2] = u1.z; A1[3] = u1.w;
    } else {
        fz_decode_step(p, A0, A1);
    }
}

template <int NT, bool GS, bool W8>
__device__ __forceinline__ void fz_stage_gateup(const uint8_t* sl, int m, int rb, int lane,
                                                int rec_gu, int aoff, const int* xsoff0, int np,
                                                int jo, int ntc, bool last, float acc_f[NT][4]) {
    constexpr int ns = fz_ns_gateup<W8>();
    constexpr int kStep = fz_step_bytes<W8>();
    const int g = lane >> 2, t = lane & 3;
    const uint8_t* cp = sl + m * ns * kStep + rb * (kStep / 8) + lane * (kStep / 256);
    // aoff: this lane's pair record (column group 0); groups c > 0 follow at 4 c rec_gu
    const uint8_t* ap = sl + kFzActOff + (g >> 2) * 64 + t * 16 + aoff + jo * 128;
    const float* scl = reinterpret_cast<const float*>(sl + kFzScaleOff + m * ns * 512) + 16 * rb + g;
    const uint8_t* xr = sl + kFzActOff;
    // the records of the lane's two accumulator pairs: column group 0 from the
    // item's table (records by token or by pair); later groups (several column
    // groups: records by pair) at fixed offsets from the lane's first pair.  A
    // pair past np reads a record the stage did not fill (inside the slot): it
    // only scales that pair's own columns, whose results are never used.
    const uint8_t* xr_lane = xr + 2 * (t & 1) * kActRec;
    auto rec_at = [&](int c, int q) -> const uint8_t* {
        if (c == 0) return xr + xsoff0[q];
        return xr_lane + (4 * c + q) * kActRec;
    };
    // entering a new record (a new 256-column group of activations): the
    // running sums move to its units, an exact power-of-two rescale
    if (jo == 0) {
#pragma unroll
        for (int c = 0; c < NT; ++c) {
            if (NT > 1 && c >= ntc) break;
            const float r0 = *reinterpret_cast<const float*>(rec_at(c, 0) + kActRecRatio);
            const float r1 = *reinterpret_cast<const float*>(rec_at(c, 1) + kActRecRatio);
            acc_f[c][0] *= r0; acc_f[c][1] *= r1; acc_f[c][2] *= r0; acc_f[c][3] *= r1;
        }
    }
    // per-row scales: exact int32 sums, two chains (even and odd steps) for one
    // column group, one chain when several groups give independent MMAs
    constexpr int CH = NT == 1 ? 2 : 1;
    int acc_i[CH][NT][4];
#pragma unroll
    for (int j = 0; j < ns; ++j) {
        uint32_t A0[4], A1[4];
        fz_load_step<W8>(cp + j * kStep, A0, A1);
        float s0 = 0.0f, s1 = 0.0f;
        if (GS) { s0 = scl[j * 128]; s1 = scl[j * 128 + 8]; }
#pragma unroll
        for (int c = 0; c < NT; ++c) {
            if (NT > 1 && c >= ntc) break;  // column groups with no pair of this item
            const uint4 b = *reinterpret_cast<const uint4*>(ap + 4 * c * rec_gu + j * 128);
            if (GS) {  // 64-column weight scales: each step into f32 at once
                int d[4];
                mma_s8_16832_zc(d, A0, b.x, b.y);
                mma_s8_16832(d, A1, b.z, b.w);
                acc_f[c][0] = fmaf((float)d[0], s0, acc_f[c][0]);
                acc_f[c][1] = fmaf((float)d[1], s0, acc_f[c][1]);
                acc_f[c][2] = fmaf((float)d[2], s1, acc_f[c][2]);
                acc_f[c][3] = fmaf((float)d[3], s1, acc_f[c][3]);
            } else {
                if (j < CH) mma_s8_16832_zc(acc_i[j % CH][c], A0, b.x, b.y);
                else mma_s8_16832(acc_i[j % CH][c], A0, b.x, b.y);
                mma_s8_16832(acc_i[j % CH][c], A1, b.z, b.w);
            }
        }
    }
    if (!GS) {
#pragma unroll
        for (int c = 0; c < NT; ++c) {
            if (NT > 1 && c >= ntc) break;
#pragma unroll
            for (int i = 0; i < 4; ++i)
                acc_f[c][i] += (float)(CH == 2 ? acc_i[0][c][i] + acc_i[CH - 1][c][i] : acc_i[0][c][i]);
        }
    }
    if (last) {  // out of record units: the last record's scale, the digit factor
                 // (and 1/16 for nibbles)
        const float f = (t < 2 ? 256.0f : 1.0f) * (W8 ? 1.0f : 0.0625f);
#pragma unroll
        for (int c = 0; c < NT; ++c) {
            if (NT > 1 && c >= ntc) break;
            const float x0 = *reinterpret_cast<const float*>(rec_at(c, 0) + kActRecScale) * f;
            const float x1 = *reinterpret_cast<const float*>(rec_at(c, 1) + kActRecScale) * f;
            acc_f[c][0] *= x0; acc_f[c][1] *= x1; acc_f[c][2] *= x0; acc_f[c][3] *= x1;
        }
    }
}

// ---------------------------------------------------------------------------
// Down stage of a consumer warp: 16-row blocks B = BPW w .. BPW w + BPW - 1 of
// the stage's rs tiles (block B: tile B / 8, block B % 8 of it; BPW = 2 for
// 4-bit codes, 1 for 8-bit ones), both steps (the tile's 128 columns of I)
// against h of the item in shared memory.  Writes the partial products of
// pairs p0 .. p0 + np - 1 for these rows.
// ---------------------------------------------------------------------------
template <int NT, bool W8>
// hf[c][q]: lanefac * (inverse scale of h) (/ 16 for 4-bit codes) of pair 4c + 2(t & 1) + q;
// dst[c][q]: element offset in part of that pair's row 0 (-1: not written by
// this lane).  Both are constant over the down stages of an item.
__device__ __forceinline__ void fz_stage_down_prep(const FusedArgs& a, const FusedShared& sh,
                                                   int tc, int p0, int np, int lane,
                                                   float (*hf)[2], int (*dst)[2]) {
    const int t = lane & 3;
    const float lanefac = t < 2 ? 256.0f : 1.0f;
    const int TG = a.I / 128;
    for (int c = 0; c < NT; ++c)
        for (int q = 0; q < 2; ++q) {
            const int ph = 4 * c + 2 * (t & 1) + q;  // pair of this lane's digit columns
            hf[c][q] = lanefac * *reinterpret_cast<const float*>(sh.hbuf + ph * kFzRecH + 256) *
                       (W8 ? 1.0f : 0.0625f);
            const int pw = 4 * c + 2 * t + q;         // pair this lane writes (t < 2)
            dst[c][q] = (t < 2 && pw < np) ? (sh.pair_pick[p0 + pw] * TG + tc) * a.H : -1;
        }
}

template <int NT, bool GS, bool W8>
__device__ __forceinline__ void fz_stage_down(const FusedArgs& a, const FusedShared& sh,
                                              const uint8_t* sl, int rs, int rt0, int ntc,
                                              const float (*hf)[2], const int (*dst)[2],
                                              int warp, int lane) {
    constexpr int BPW = W8 ? 1 : 2;
    constexpr int WPT = 8 / BPW;  // warps per tile
    constexpr int kStep = fz_step_bytes<W8>();
    const int q = warp / WPT;
    if (q >= rs) return;
    const int g = lane >> 2, t = lane & 3;
    const int8_t* hb = sh.hbuf + (g >> 2) * 64 + t * 16 + (g & 3) * kFzRecH;
#pragma unroll
    for (int bb = 0; bb < BPW; ++bb) {
        const int b8 = BPW * (warp % WPT) + bb;
        const uint8_t* cp = sl + q * 2 * kStep + b8 * (kStep / 8) + lane * (kStep / 256);
        const float* scl = reinterpret_cast<const float*>(sl + kFzScaleOff) +
                           (GS ? q * 256 : q * 128) + 16 * b8 + g;
        float v[NT][4];
        int acc[NT][4];
#pragma unroll
        for (int c = 0; c < NT; ++c)
#pragma unroll
            for (int i = 0; i < 4; ++i) { v[c][i] = 0.0f; acc[c][i] = 0; }
#pragma unroll
        for (int j = 0; j < 2; ++j) {
            uint32_t A0[4], A1[4];
            fz_load_step<W8>(cp + j * kStep, A0, A1);
#pragma unroll
            for (int c = 0; c < NT; ++c) {
                if (NT > 1 && c >= ntc) break;
                const uint4 b = *reinterpret_cast<const uint4*>(hb + 4 * c * kFzRecH + j * 128);
                if (GS) {
                    int d[4];
                    mma_s8_16832_zc(d, A0, b.x, b.y);
                    mma_s8_16832(d, A1, b.z, b.w);
                    const float s0 = scl[j * 128], s1 = scl[j * 128 + 8];
                    v[c][0] = fmaf((float)d[0], s0, v[c][0]);
                    v[c][1] = fmaf((float)d[1], s0, v[c][1]);
                    v[c][2] = fmaf((float)d[2], s1, v[c][2]);
                    v[c][3] = fmaf((float)d[3], s1, v[c][3]);
                } else {  // one chain per step, added below
                    int d[4];
                    mma_s8_16832_zc(d, A0, b.x, b.y);
                    mma_s8_16832(d, A1, b.z, b.w);
#pragma unroll
                    for (int i = 0; i < 4; ++i) acc[c][i] += d[i];
                }
            }
        }
        const float sw0 = GS ? 1.0f : scl[0], sw1 = GS ? 1.0f : scl[8];
        const int r0 = (rt0 + q) * 128 + 16 * b8 + g;
#pragma unroll
        for (int c = 0; c < NT; ++c) {
            if (NT > 1 && c >= ntc) break;
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                float x = GS ? v[c][i] : (float)acc[c][i] * ((i >> 1) ? sw1 : sw0);
                x *= hf[c][i & 1];
                x += __shfl_xor_sync(0xffffffffu, x, 2);  // high digit * 256 + low digit
                const int o = dst[c][i & 1];
                if (o >= 0) a.part[(int64_t)o + r0 + 8 * (i >> 1)] = x;
            }
        }
    }
}

}  // namespace coli

namespace coli {

// ---------------------------------------------------------------------------
// Consumer warps: the stages of each item; after its gate/up part, h of the
// tile (SwiGLU of the two accumulators) becomes s8 digits in shared memory
// with one power-of-two scale per pair.
// ---------------------------------------------------------------------------
template <int NT, bool GS, bool W8, bool TW>
__device__ __forceinline__ void fz_consume(const FusedArgs& a, FusedShared& sh, uint8_t* ring,
                                           int n_units) {
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int g = lane >> 2, t = lane & 3;
    const int rb = warp & 7, m = warp >> 3;
    const FzShape z = fz_shape<W8>(a);
    const int rec_gu = kActRec;
    const bool wr = t < 2;  // after the digit combine: lanes holding results
    uint32_t cphase = 0, lap = 0;
    int s = 0;
    int u = 0, tc = 0, p0 = 0, np = 0;
    int aoff = 0;  // this lane's activation record in a gate/up stage
    int xsoff0[2];                 // records of the lane's accumulator pairs (group 0)
    float sw0 = 1.0f, sw1 = 1.0f;  // per-row weight scales of rows g, g + 8
    float hf[NT][2];               // down part: digit and h scale factors
    int dst[NT][2];                //            partial-product offsets
    float acc_f[NT][4];            // running gate/up sums, in the current record's units
    for (;;) {
        if (!fz_wait(&sh.full[s], lap, a.err, TW)) return;
        const int item = sh.meta_item[s], st = sh.meta_st[s];
        if (item < 0) return;
        const uint8_t* sl = ring + (int64_t)s * a.slot_bytes;
        if (st == 0) {  // a new item
            const FzWork wk = fz_work(sh, n_units, z.TG, item);
            u = wk.u;
            tc = wk.tc;
            p0 = wk.p0;
            np = wk.np;
            // records by token (TMA box) or by pair of the item; pairs past np
            // read pair 0's record (their results are never used)
            auto rec_of = [&](int pp) {
                if (pp >= np) pp = 0;
                return a.act_tma ? sh.pair_tok[p0 + pp] * kActRec : pp * rec_gu;
            };
            aoff = rec_of(g & 3);
            xsoff0[0] = rec_of(2 * (t & 1));
            xsoff0[1] = rec_of(2 * (t & 1) + 1);
#pragma unroll
            for (int c = 0; c < NT; ++c)
#pragma unroll
                for (int i = 0; i < 4; ++i) acc_f[c][i] = 0.0f;
        }
        const bool gu = st < z.nst_gu;
        const int ntc = (np + 3) >> 2;  // column groups holding the item's pairs
        if (gu) {
            // the column-group count as a compile-time constant: no branch inside
            // the unrolled MMA loops
            const int jo = W8 ? (st & 1) * 2 : 0;
            const bool lst = st == z.nst_gu - 1;
#define FZ_GU(K) fz_stage_gateup<K, GS, W8>(sl, m, rb, lane, rec_gu, aoff, xsoff0, np, jo, K, lst, acc_f)
            if constexpr (NT == 1) {
                FZ_GU(1);
            } else if constexpr (NT == 2) {
                if (ntc == 1) FZ_GU(1); else FZ_GU(2);
            } else {
                switch (ntc) {
                    case 1: FZ_GU(1); break;
                    case 2: FZ_GU(2); break;
                    case 3: FZ_GU(3); break;
                    default: FZ_GU(4); break;
                }
            }
#undef FZ_GU
            if (!GS && st == z.nst_gu - 1) {
                const float* rsc = reinterpret_cast<const float*>(sl + kFzScaleOff + m * 512) + 16 * rb + g;
                sw0 = rsc[0];
                sw1 = rsc[8];
            }
        } else {
            const int rt0 = (st - z.nst_gu) * z.rs;
#define FZ_DN(K) fz_stage_down<K, GS, W8>(a, sh, sl, z.rs, rt0, K, hf, dst, warp, lane)
            if constexpr (NT == 1) {
                FZ_DN(1);
            } else if constexpr (NT == 2) {
                if (ntc == 1) FZ_DN(1); else FZ_DN(2);
            } else {
                switch (ntc) {
                    case 1: FZ_DN(1); break;
                    case 2: FZ_DN(2); break;
                    case 3: FZ_DN(3); break;
                    default: FZ_DN(4); break;
                }
            }
#undef FZ_DN
        }
        __syncwarp();
        if (lane == 0) mbar_arrive(&sh.empty[s]);
        if (++s == a.slots) { s = 0; lap ^= 1u; }
        if (!gu || st != z.nst_gu - 1) continue;

        // ---------------- h of the tile ----------------
        float v[NT][4];
#pragma unroll
        for (int c = 0; c < NT; ++c)
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                float x = acc_f[c][i];
                x += __shfl_xor_sync(0xffffffffu, x, 2);  // high digit * 256 + low digit
                if (!GS) x *= (i >> 1) ? sw1 : sw0;
                v[c][i] = x;
            }
        // lanes t < 2 hold rows g + 8 (i >> 1), pairs 4c + 2t + (i & 1)
#pragma unroll
        for (int c = 0; c < NT; ++c)
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                const int pp = 4 * c + 2 * t + (i & 1), rr = g + 8 * (i >> 1);
                if (wr && pp < np && m == 1) sh.xch[rb][rr][pp] = v[c][i];
            }
        if (!fz_cbar(&sh.cbar, cphase, a.err, TW)) return;
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
        if (!fz_cbar(&sh.cbar, cphase, a.err, TW)) return;
        if (m == 0 && wr) {
            const int j = rb / 4;  // 64-column step of the down part holding these rows of h
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
                    int8_t* rec = sh.hbuf + pp * kFzRecH;
#pragma unroll
                    for (int hr = 0; hr < 2; ++hr) {
                        int hi, lo;
                        fz_split(v[c][2 * hr + q], sc, hi, lo);
                        const int pos = fz_act_pos(16 * (rb % 4) + g + 8 * hr);
                        rec[j * 128 + pos] = (int8_t)hi;
                        rec[j * 128 + 64 + pos] = (int8_t)lo;
                    }
                    if (rb == 0 && g == 0) *reinterpret_cast<float*>(rec + 256) = inv;
                }
        }
        if (!fz_cbar(&sh.cbar, cphase, a.err, TW)) return;  // h complete before the down stages
        fz_stage_down_prep<NT, W8>(a, sh, tc, p0, np, lane, hf, dst);
    }
}

// TW: the wait test (coli_moe_layer_set_wait_test): CTA 0's producer withholds
// one ring stage and every wait takes a short limit.  A separate instantiation,
// so that the default launches keep compile-time limits (a limit chosen at run
// time made the consumer loop ~12% slower).
template <int NT, bool GS, bool W8, bool TW>
__global__ void __launch_bounds__(kFzThreads, 1)
moe_fused_kernel(const __grid_constant__ CUtensorMap xmap, FusedArgs a) {
    extern __shared__ __align__(128) uint8_t fz_smem[];
    __shared__ FusedShared sh;
    if (threadIdx.x == 0) {
        for (int s = 0; s < a.slots; ++s) { mbar_init(&sh.full[s], 1); mbar_init(&sh.empty[s], kFzWarps); }
        mbar_init(&sh.cbar, kFzWarps);
        fence_mbar_init();
    }
    // the combine kernel may be scheduled now; it waits for this grid to finish
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
    // everything below reads what the router kernel wrote
    asm volatile("griddepcontrol.wait;" ::: "memory");
    const int warp = threadIdx.x >> 5;
    if (a.T == 1) {
        // One token: the producer needs only the picks (named barrier 2: warp
        // 0 and the producer), so it starts streaming while warp 0 writes the
        // unit and pair tables for the consumer warps (named barrier 1).
        __syncthreads();  // barrier initialisation, before any wait on them
        if (warp == kFzProducer) {
            asm volatile("bar.sync 2, %0;" ::"n"(64) : "memory");
            // the computed picks are distinct experts: one unit each
            fz_produce<GS, W8, TW>(a, &xmap, sh, fz_smem, sh.n_kept1 + a.n_shared, true);
            return;
        }
        if (warp == 0) {
            FzScratch one;
            one.bits = nullptr; one.cnt = nullptr; one.excl = nullptr;
            one.pick_e = sh.pick1_e;
            one.pick_w = sh.pick1_w;
            one.unit_e = sh.unit1_e;
            one.n_kept = &sh.n_kept1;
            fz_topk_token(a, 0, one);
            __syncwarp();
            asm volatile("bar.arrive 2, %0;" ::"n"(64) : "memory");
            fz_union_warp(a, sh, one);
        }
        asm volatile("bar.sync 1, %0;" ::"n"(32 * kFzWarps) : "memory");
        fz_consume<NT, GS, W8, TW>(a, sh, fz_smem, sh.n_uniq + a.n_shared);
        return;
    }
    const int n_units = fz_route_union(a, sh, fz_smem);
    if (warp == kFzProducer) fz_produce<GS, W8, TW>(a, &xmap, sh, fz_smem, n_units, false);
    else fz_consume<NT, GS, W8, TW>(a, sh, fz_smem, n_units);
}

// ---------------------------------------------------------------------------
// y from the partial down products.  CTA (token t, 32 rows), one warp per pick
// j (k routed picks, then the shared experts): the warp sums pick j's I/128
// partials in tile order (all loads in flight at once); warp 0 then adds the
// picks up in pick order, weighted, then the shared experts, then the residual.
// ---------------------------------------------------------------------------
constexpr int kCombineMaxTiles = 32;  // I <= 4096

struct CombineArgs {
    const float* part;     // [T][k + n_shared][TG][H]
    const float* w;        // [T*k]
    const int32_t* inv;    // [T*k], < 0 for a pick the fused kernel did not compute
    const float* residual; // [T][H] or nullptr
    float* y;              // [T][H]
    int T, k, n_shared, H, TG;
};

__global__ void __launch_bounds__(1024)
moe_combine_kernel(CombineArgs c) {
    __shared__ float oj[kFzMaxK + 4][32];
    // the next kernel may be scheduled now (this library's kernels wait for
    // this grid before reading y); then wait for the fused kernel's partials
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
    asm volatile("griddepcontrol.wait;" ::: "memory");
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int nw = blockDim.x >> 5;
    const int nrg = c.H / 32;
    const int t = blockIdx.x / nrg, r = (blockIdx.x - t * nrg) * 32 + lane;
    const int J = c.k + c.n_shared;
    for (int j = warp; j < J; j += nw) {
        if (j < c.k && __ldcg(c.inv + t * c.k + j) < 0) continue;  // not computed: adds nothing
        const float* src = c.part + ((int64_t)t * J + j) * c.TG * c.H + r;
        float pv[kCombineMaxTiles];
#pragma unroll
        for (int i = 0; i < kCombineMaxTiles; ++i)
            pv[i] = i < c.TG ? __ldcg(src + (int64_t)i * c.H) : 0.0f;
        float o = 0.0f;
#pragma unroll
        for (int i = 0; i < kCombineMaxTiles; ++i)
            if (i < c.TG) o += pv[i];
        oj[j][lane] = j < c.k ? o * __ldcg(c.w + t * c.k + j) : o;
    }
    __syncthreads();
    if (warp == 0) {
        float acc = 0.0f;
        for (int j = 0; j < c.k; ++j)
            if (__ldcg(c.inv + t * c.k + j) >= 0) acc += oj[j][lane];
        for (int s = 0; s < c.n_shared; ++s) acc += oj[c.k + s][lane];
        if (c.residual) acc = c.residual[(int64_t)t * c.H + r] + acc;
        c.y[(int64_t)t * c.H + r] = acc;
    }
}

}  // namespace coli
