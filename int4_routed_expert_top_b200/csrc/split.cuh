// split.cuh - two-pass int4 expert kernels for batches past the fused path's
// limits (prefill and large verify batches).
//
// The batch union ("github一周涨11k⭐️！25GB 内存跑 744B GLM-5.2 模型！" 三.4) makes
// every unique expert one unit holding all of the batch's (token, slot) pairs
// that picked it; a unit's pairs are cut into chunks of kFzChunk.  Two
// launches of one persistent kernel (one CTA per SM, items from a counter):
//
//   gate/up pass: item = (unit, 128-row tile of I, chunk).  Stages stream the
//     tile's rows of gate and of up over H (four 64-column steps a stage) with
//     the chunk's pairs' activation records; h = silu(W_g x) * (W_u x) of those
//     rows goes to global memory in f32.
//   down pass:    item = (unit, two 128-row tiles of H, chunk), the same stages
//     over I with h's activation records (made from the f32 h between the
//     passes); o = W_d h of those rows goes to global memory in f32.
//
// The math of a stage is the fused kernel's gate/up stage (int4 codes expanded
// to s8 in registers, two-digit s8 activations, mma.sync m16n8k32 s8, exact
// int32 step sums scaled in f32), so both passes carry the same ~15 significant
// activation bits.  Inside a unit, the chunks of one tile are consecutive items:
// CTAs that take them run at about the same time and the repeated weight reads
// are served by L2 (those copies carry no evict-first hint).  The combine of
// the tensor-core path forms y from o.
#pragma once

#include "fused.cuh"

namespace coli {

constexpr int kSpSlots = 5;  // ring stages (as many as fit)

struct SplitArgs {
    ExpertStore store;
    BlobLayout L;
    const int32_t* n_units;      // union units: routed experts with pairs, then the shared ones
    const int32_t* unit_expert;
    const int32_t* unit_begin;   // first pair of each unit
    const int32_t* unit_end;
    const int32_t* pair_tok;     // token of each pair
    const int8_t* act;           // gate/up: x records [T][H/256]; down: h records [P][I/256]
    float* out;                  // gate/up: h [P][I]; down: o [P][H]
    int32_t* queue;              // work-item counter, zero on entry
    int32_t* err;
    int H, I;
    int down;                    // 0: gate/up pass, 1: down pass
    int slots, slot_bytes;
};

struct SplitShared {
    uint64_t full[kFzMaxSlots], empty[kFzMaxSlots];
    uint64_t cbar;
    int meta_item[kFzMaxSlots], meta_st[kFzMaxSlots];
    int u_exp[kFzMaxUnits], u_p0[kFzMaxUnits], u_p1[kFzMaxUnits];
    int u_item0[kFzMaxUnits + 1];
    int n_items;
    float xch[8][16][kFzChunk];  // gate/up pass: up values for the gate warps
};

// items per chunk: row tiles of the pass's output
__device__ __forceinline__ int sp_tiles(const SplitArgs& a) { return a.down ? a.H / 256 : a.I / 128; }

// Unit table and first item of every unit, by warp 0 (a shuffle scan over the
// units, 32 at a time); the other warps wait at the block barrier.
__device__ __forceinline__ void sp_tables(const SplitArgs& a, SplitShared& sh) {
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    if (warp == 0) {
        // the host launches only layers with E + n_shared <= kFzMaxUnits
        const int nu = min(__ldcg(a.n_units), kFzMaxUnits);
        const int TI = sp_tiles(a);
        int carry = 0;
        for (int base = 0; base < nu; base += 32) {
            const int u = base + lane;
            int items = 0, e = 0, b = 0, f = 0;
            if (u < nu) {
                e = __ldcg(a.unit_expert + u);
                b = __ldcg(a.unit_begin + u);
                f = __ldcg(a.unit_end + u);
                items = (f - b + kFzChunk - 1) / kFzChunk * TI;
            }
            int incl = items;
#pragma unroll
            for (int d = 1; d < 32; d <<= 1) {
                const int v = __shfl_up_sync(0xffffffffu, incl, d);
                if (lane >= d) incl += v;
            }
            if (u < nu) {
                sh.u_exp[u] = e;
                sh.u_p0[u] = b;
                sh.u_p1[u] = f;
                sh.u_item0[u] = carry + incl - items;
            }
            carry += __shfl_sync(0xffffffffu, incl, 31);
        }
        if (lane == 0) {
            sh.u_item0[nu] = carry;
            sh.n_items = carry;
        }
    }
    __syncthreads();
}

struct SpWork {
    int u, tc, p0, np;
};
// item -> unit (last unit whose first item is <= item), then tile-major,
// chunk-minor inside the unit
__device__ __forceinline__ SpWork sp_work(const SplitShared& sh, int n_units_hint, int item) {
    int lo = 0, hi = n_units_hint - 1;
    while (lo < hi) {
        const int mid = (lo + hi + 1) >> 1;
        if (sh.u_item0[mid] <= item) lo = mid; else hi = mid - 1;
    }
    SpWork w;
    w.u = lo;
    const int rel = item - sh.u_item0[lo];
    const int nch = (sh.u_p1[lo] - sh.u_p0[lo] + kFzChunk - 1) / kFzChunk;
    w.tc = rel / nch;
    const int ch = rel - w.tc * nch;
    w.p0 = sh.u_p0[lo] + ch * kFzChunk;
    w.np = min(kFzChunk, sh.u_p1[lo] - w.p0);
    return w;
}

// Producer warp.  Stage st of an item: steps 4 st .. 4 st + 3 of the item's two
// 128-row tiles (gate/up: row tile tc of gate and of up; down: row tiles 2 tc
// and 2 tc + 1 of down) [codes tile 0 | codes tile 1 | gs64 scales tile 0, 1 |
// the activation record st of each pair (by token for x, by pair for h)] and,
// on the last stage, the tiles' per-row scales.
template <bool GS>
__device__ __forceinline__ void sp_produce(const SplitArgs& a, SplitShared& sh, uint8_t* ring,
                                           int n_units) {
    const int lane = threadIdx.x & 31;
    constexpr uint32_t kStep = 4096;   // codes of one 64-column step of a 128-row tile
    const int K = a.down ? a.I : a.H;
    const int nst = K / 256;           // one activation record per stage
    const int ngK = GS ? K / 64 : 1;
    const uint64_t pol = l2_evict_first_policy();
    const int n_items = sh.n_items;
    int s = 0, issued = 0;
    uint32_t lap = 0;
    bool ok = true;
    int item = blockIdx.x;
    while (ok && item < n_items) {
        const SpWork wk = sp_work(sh, n_units, item);
        const uint8_t* blob = a.store.blob(sh.u_exp[wk.u]);
        const bool shared_reads = sh.u_p1[wk.u] - sh.u_p0[wk.u] > kFzChunk;  // other chunks follow
        const int mc = a.down ? 2 : 0;
        const int r0 = a.down ? 2 * wk.tc : wk.tc, r1 = a.down ? 2 * wk.tc + 1 : wk.tc;
        const uint8_t* c0 = blob + a.L.codes[mc] + (int64_t)r0 * (K / 64) * kStep;
        const uint8_t* c1 = blob + a.L.codes[a.down ? 2 : 1] + (int64_t)r1 * (K / 64) * kStep;
        const float* s0 = reinterpret_cast<const float*>(blob + a.L.scales[mc]) +
                          (int64_t)r0 * ngK * kTileRows;
        const float* s1 = reinterpret_cast<const float*>(blob + a.L.scales[a.down ? 2 : 1]) +
                          (int64_t)r1 * ngK * kTileRows;
        // lane pp < np copies pair pp's records: its activation row (the token
        // for x, the pair itself for h) loaded once per item
        int64_t arow = 0;
        if (lane < wk.np) arow = a.down ? (int64_t)(wk.p0 + lane) : (int64_t)__ldcg(a.pair_tok + wk.p0 + lane);
        for (int st = 0; st < nst; ++st) {
            if (issued >= a.slots && !fz_wait(&sh.empty[s], lap ^ 1u, a.err, false)) {
                ok = false;
                break;
            }
            if (lane == 0) { sh.meta_item[s] = item; sh.meta_st[s] = st; }
            __syncwarp();
            uint8_t* sl = ring + (int64_t)s * a.slot_bytes;
            const int kb0 = 4 * st;
            const bool rowsc = !GS && st == nst - 1;
            const uint32_t cb = 4 * kStep, sb = GS ? 4u * 512u : 0u;
            mbar_expect_tx_elect(&sh.full[s], 2 * (cb + sb) + (uint32_t)(wk.np * kActRec) +
                                                  (rowsc ? 1024u : 0u));
            if (shared_reads) {
                bulk_g2s_elect(sl, c0 + (int64_t)kb0 * kStep, cb, &sh.full[s]);
                bulk_g2s_elect(sl + cb, c1 + (int64_t)kb0 * kStep, cb, &sh.full[s]);
            } else {
                bulk_g2s_hint_elect(sl, c0 + (int64_t)kb0 * kStep, cb, &sh.full[s], pol);
                bulk_g2s_hint_elect(sl + cb, c1 + (int64_t)kb0 * kStep, cb, &sh.full[s], pol);
            }
            if (GS) {
                bulk_g2s_elect(sl + kFzScaleOff, s0 + (int64_t)kb0 * kTileRows, sb, &sh.full[s]);
                bulk_g2s_elect(sl + kFzScaleOff + sb, s1 + (int64_t)kb0 * kTileRows, sb, &sh.full[s]);
            }
            if (rowsc) {
                bulk_g2s_elect(sl + kFzScaleOff, s0, 512u, &sh.full[s]);
                bulk_g2s_elect(sl + kFzScaleOff + 512, s1, 512u, &sh.full[s]);
            }
            __syncwarp();  // the expected bytes are registered before any record copy
            if (lane < wk.np)
                bulk_g2s(sl + kFzActOff + lane * kActRec, a.act + (arow * nst + st) * kActRec,
                         (uint32_t)kActRec, &sh.full[s]);
            __syncwarp();
            ++issued;
            if (++s == a.slots) { s = 0; lap ^= 1u; }
        }
        if (lane == 0) item = (int)gridDim.x + atomicAdd(a.queue, 1);
        item = __shfl_sync(0xffffffffu, item, 0);
    }
    if (ok && (issued < a.slots || fz_wait(&sh.empty[s], lap ^ 1u, a.err, false))) {  // end marker
        if (lane == 0) sh.meta_item[s] = -1;
        __syncwarp();
        if (lane == 0) mbar_arrive(&sh.full[s]);
        ++issued;
    }
    // leave only once every copy issued into the ring has landed
    for (int j = issued > a.slots ? issued - a.slots : 0; j < issued; ++j)
        fz_wait(&sh.full[j % a.slots], (j / a.slots) & 1, nullptr, false);
}

// Consumer warps: warp w takes 16-row block w % 8 of tile w / 8 over every
// stage of an item; after the last stage lanes t < 2 hold rows g, g + 8 of
// pairs 4c + 2t, 4c + 2t + 1 (column group c).
template <bool GS>
__device__ __forceinline__ void sp_consume(const SplitArgs& a, SplitShared& sh, uint8_t* ring,
                                           int n_units) {
    constexpr int NT = kFzChunk / 4;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int g = lane >> 2, t = lane & 3;
    const int rb = warp & 7, m = warp >> 3;
    const int K = a.down ? a.I : a.H;
    const int nst = K / 256;
    const bool wr = t < 2;
    uint32_t cphase = 0, lap = 0;
    int s = 0;
    int tc = 0, p0 = 0, np = 0, aoff = 0;
    int xsoff0[2] = {0, 0};
    float sw0 = 1.0f, sw1 = 1.0f;
    float acc_f[NT][4];
    for (;;) {
        if (!fz_wait(&sh.full[s], lap, a.err, false)) return;
        const int item = sh.meta_item[s], st = sh.meta_st[s];
        if (item < 0) return;
        const uint8_t* sl = ring + (int64_t)s * a.slot_bytes;
        if (st == 0) {
            const SpWork wk = sp_work(sh, n_units, item);
            tc = wk.tc;
            p0 = wk.p0;
            np = wk.np;
            // records by pair of the item; pairs past np read pair 0's record
            // (their results are never stored)
            auto rec_of = [&](int pp) { return (pp >= np ? 0 : pp) * kActRec; };
            aoff = rec_of(g & 3);
            xsoff0[0] = rec_of(2 * (t & 1));
            xsoff0[1] = rec_of(2 * (t & 1) + 1);
#pragma unroll
            for (int c = 0; c < NT; ++c)
#pragma unroll
                for (int i = 0; i < 4; ++i) acc_f[c][i] = 0.0f;
        }
        const bool last = st == nst - 1;
        // the chunk's column groups as a compile-time count: no branch inside
        // the unrolled MMA loops
        switch ((np + 3) >> 2) {
            case 1: fz_stage_gateup<1, GS, false>(sl, m, rb, lane, kActRec, aoff, xsoff0, np, 0, 1, last, acc_f); break;
            case 2: fz_stage_gateup<2, GS, false>(sl, m, rb, lane, kActRec, aoff, xsoff0, np, 0, 2, last, acc_f); break;
            case 3: fz_stage_gateup<3, GS, false>(sl, m, rb, lane, kActRec, aoff, xsoff0, np, 0, 3, last, acc_f); break;
            default: fz_stage_gateup<4, GS, false>(sl, m, rb, lane, kActRec, aoff, xsoff0, np, 0, 4, last, acc_f); break;
        }
        if (!GS && last) {
            const float* rsc = reinterpret_cast<const float*>(sl + kFzScaleOff + m * 512) + 16 * rb + g;
            sw0 = rsc[0];
            sw1 = rsc[8];
        }
        __syncwarp();
        if (lane == 0) mbar_arrive(&sh.empty[s]);
        if (++s == a.slots) { s = 0; lap ^= 1u; }
        if (!last) continue;

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
        if (a.down) {  // o of rows (2 tc + m) * 128 + 16 rb + g (+ 8)
            const int64_t r = (int64_t)(2 * tc + m) * kTileRows + 16 * rb + g;
#pragma unroll
            for (int c = 0; c < NT; ++c)
#pragma unroll
                for (int i = 0; i < 4; ++i) {
                    const int pp = 4 * c + 2 * t + (i & 1);
                    if (wr && pp < np) a.out[(int64_t)(p0 + pp) * a.H + r + 8 * (i >> 1)] = v[c][i];
                }
            continue;
        }
        // gate/up: the up warps hand their values to the gate warps of the same rows
#pragma unroll
        for (int c = 0; c < NT; ++c)
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                const int pp = 4 * c + 2 * t + (i & 1);
                if (wr && pp < np && m == 1) sh.xch[rb][g + 8 * (i >> 1)][pp] = v[c][i];
            }
        if (!fz_cbar(&sh.cbar, cphase, a.err, false)) return;
        if (m == 0) {
            const int64_t r = (int64_t)tc * kTileRows + 16 * rb + g;
#pragma unroll
            for (int c = 0; c < NT; ++c)
#pragma unroll
                for (int i = 0; i < 4; ++i) {
                    const int pp = 4 * c + 2 * t + (i & 1), rr = g + 8 * (i >> 1);
                    if (wr && pp < np)
                        a.out[(int64_t)(p0 + pp) * a.I + r + 8 * (i >> 1)] =
                            silu_f(v[c][i]) * sh.xch[rb][rr][pp];
                }
        }
        if (!fz_cbar(&sh.cbar, cphase, a.err, false)) return;  // the exchange buffer is free again
    }
}

template <bool GS>
__global__ void __launch_bounds__(kFzThreads, 1)
moe_split_kernel(SplitArgs a) {
    extern __shared__ __align__(128) uint8_t sp_smem[];
    __shared__ SplitShared sh;
    if (threadIdx.x == 0) {
        for (int s = 0; s < a.slots; ++s) { mbar_init(&sh.full[s], 1); mbar_init(&sh.empty[s], kFzWarps); }
        mbar_init(&sh.cbar, kFzWarps);
        fence_mbar_init();
    }
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
    asm volatile("griddepcontrol.wait;" ::: "memory");  // the union and the records
    sp_tables(a, sh);
    const int nu = min(__ldcg(a.n_units), kFzMaxUnits);
    if ((threadIdx.x >> 5) == kFzProducer) sp_produce<GS>(a, sh, sp_smem, nu);
    else sp_consume<GS>(a, sh, sp_smem, nu);
}

// Activation records (the fused kernel's s8 operand) of `rows` rows of `cols`
// columns: one CTA of 256 threads per row.
template <typename XT>
__global__ void __launch_bounds__(256)
act_records_kernel(const XT* __restrict__ x, int cols, int8_t* __restrict__ rec) {
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
    asm volatile("griddepcontrol.wait;" ::: "memory");
    act_quant8_token(x, cols, blockIdx.x, rec);
}

}  // namespace coli
