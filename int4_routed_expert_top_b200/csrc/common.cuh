// common.cuh - shared device helpers for libcolimoe (sm_100a).
#pragma once

#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>
#include <stdint.h>

namespace coli {

constexpr int kTileRows = 128;  // rows per device tile of a weight matrix
constexpr int kUnitCols = 32;   // columns per 16-byte code unit
constexpr int kGroupCols = 64;  // columns per loop step of the GEMV kernels

// ---------------------------------------------------------------------------
// Device layout of one expert blob (see include/coli_moe.h for the contract).
// ---------------------------------------------------------------------------
struct BlobLayout {
    int64_t codes[3];   // byte offsets of gate, up, down codes
    int64_t scales[3];  // byte offsets of gate, up, down scales
    int64_t bytes;      // total blob size (multiple of 256)
    int32_t rows[3];    // R of gate, up, down
    int32_t cols[3];    // K of gate, up, down
    int32_t ngroups[3]; // K / G (1 for per-row scales)
};

__host__ __device__ inline int64_t align256(int64_t v) { return (v + 255) & ~int64_t(255); }

__host__ __device__ inline BlobLayout make_blob_layout(int H, int I, int group) {
    BlobLayout L;
    L.rows[0] = I; L.cols[0] = H;
    L.rows[1] = I; L.cols[1] = H;
    L.rows[2] = H; L.cols[2] = I;
    int64_t off = 0;
    for (int m = 0; m < 3; ++m) {
        L.codes[m] = off;
        off = align256(off + (int64_t)L.rows[m] * L.cols[m] / 2);
    }
    for (int m = 0; m < 3; ++m) {
        L.ngroups[m] = group == 0 ? 1 : L.cols[m] / group;
        L.scales[m] = off;
        off = align256(off + (int64_t)L.rows[m] * L.ngroups[m] * 4);
    }
    L.bytes = off;
    return L;
}

// Blob of an expert with 8-bit codes (one signed byte per weight): the same
// three matrices and scale sections as make_blob_layout, codes R * K bytes.
__host__ __device__ inline BlobLayout make_blob_layout8(int H, int I, int group) {
    BlobLayout L;
    L.rows[0] = I; L.cols[0] = H;
    L.rows[1] = I; L.cols[1] = H;
    L.rows[2] = H; L.cols[2] = I;
    int64_t off = 0;
    for (int m = 0; m < 3; ++m) {
        L.codes[m] = off;
        off = align256(off + (int64_t)L.rows[m] * L.cols[m]);
    }
    for (int m = 0; m < 3; ++m) {
        L.ngroups[m] = group == 0 ? 1 : L.cols[m] / group;
        L.scales[m] = off;
        off = align256(off + (int64_t)L.rows[m] * L.ngroups[m] * 4);
    }
    L.bytes = off;
    return L;
}

// Where the blobs of a layer's experts sit in device memory: routed expert e
// (e_lo <= e < E) at routed + (e - e_lo) * bytes, shared expert s at shared +
// s * bytes.  A whole layer has e_lo = 0 and shared = routed + E * bytes; a
// handle restricted to an expert range (expert parallelism) holds only that
// range's blobs, then its shared experts, if any.
struct ExpertStore {
    const uint8_t* routed;
    const uint8_t* shared;
    int64_t bytes;
    int e_lo, E;
    __host__ __device__ __forceinline__ const uint8_t* blob(int e) const {
        return e < E ? routed + (int64_t)(e - e_lo) * bytes : shared + (int64_t)(e - E) * bytes;
    }
};

// Which routed picks a call computes.  Adaptive top-p ("colibrì 實戰指南" 三 and
// 五, `--topp`; the pages give no rule, so: keep the shortest run of the
// largest renormalised weights w_j / sum(w), equal weights to the lower expert
// index, whose total reaches p, at least one pick) when 0 < topp <= 1; then
// only experts e_lo <= e < e_hi (expert parallelism).  A pick not computed gets
// weight 0 and adds nothing to y.
struct PickFilter {
    float topp = 0.0f;  // outside (0, 1]: every pick
    int e_lo = 0, e_hi = 1 << 30;
};

// Lane j < k holds pick j (weight w, expert e) of one token; every lane of the
// warp takes part.  Returns whether lane j's pick is computed (false for lanes
// >= k).  The top-p rule runs in double, with the weights in the order of the
// rule and the same divisions as its plain statement, so that the decision
// equals a double-precision evaluation of the rule on the same f32 weights.
__device__ __forceinline__ bool pick_kept(const PickFilter& f, int k, float w, int e) {
    const int lane = threadIdx.x & 31;
    const bool mine = lane < k;
    bool keep = mine;
    if (f.topp > 0.0f && f.topp <= 1.0f) {
        double tot = 0.0;  // in pick order
        for (int j = 0; j < k; ++j) tot += (double)__shfl_sync(0xffffffffu, w, j);
        int rank = 0;      // position in (w descending, expert ascending)
        for (int j = 0; j < k; ++j) {
            const float wj = __shfl_sync(0xffffffffu, w, j);
            const int ej = __shfl_sync(0xffffffffu, e, j);
            rank += (wj > w || (wj == w && ej < e)) ? 1 : 0;
        }
        const double p = (double)f.topp;
        double mass = 0.0;
        bool kept = false;
        for (int r = 0; r < k; ++r) {
            const unsigned who = __ballot_sync(0xffffffffu, mine && rank == r);
            const float wr = __shfl_sync(0xffffffffu, w, __ffs(who) - 1);
            const bool take = r == 0 || mass < p;  // decided before adding pick r
            if (mine && rank == r) kept = take;
            mass += tot > 0.0 ? (double)wr / tot : 0.0;
        }
        keep = mine && kept;
    }
    return keep && e >= f.e_lo && e < f.e_hi;
}

// 8-bit fragment tiles: 16-row x 64-column blocks ordered [R/128][K/64][8][32
// lanes] as for 4-bit codes, 32 bytes per lane: for each 32-column half h of
// the step, four words i = 0..3 that are the lane's mma.sync m16n8k32 s8 A
// registers: i = 0 row r0 = 16 b + g, columns 32 h + 4 t .. + 3; i = 1 row
// r0 + 8, same columns; i = 2 row r0, columns 32 h + 16 + 4 t .. + 3; i = 3 row
// r0 + 8, those columns; byte j of a word is its first column + j.
__host__ __device__ inline int64_t frag8_byte_offset(int r, int c, int K) {
    const int rt = r / 128, b8 = (r % 128) / 16, g = r % 8, upper = (r % 16) / 8;
    const int kb = c / 64, h = (c % 64) / 32, c32 = c % 32;
    const int hi16 = c32 / 16, t = (c32 % 16) / 4, j = c32 % 4;
    const int lane = 4 * g + t, word = 4 * h + 2 * hi16 + upper;
    return ((((int64_t)rt * (K / 64) + kb) * 8 + b8) * 32 + lane) * 32 + 4 * word + j;
}

// Fragment tiles.  A matrix [R, K] is cut into 16-row x 64-column blocks; the
// block is 32 units of 16 bytes, one per lane l = 4*g + t of a warp, so one warp
// load of 512 bytes fetches a whole block.  Unit l holds rows r0 = 16*b + g and
// r1 = r0 + 8 of the block, and for each 16-column sub-block j the 4 columns
// c0 = 16*j + 4*t .. c0 + 3 of both rows: 8 nibbles in word j, byte i of the
// word holding column c0 + i, row r0 in its high nibble and row r1 in its low
// nibble.  These are the elements that lane owns in a 16x16 tensor-core operand
// tile (mma.sync A fragment up to a column permutation, and the tcgen05
// 16x256b TMEM access).  Blocks are ordered [R/128][K/64][8][32 lanes], so the
// eight blocks of a 128-row tile and one 64-column step are 4 KB of contiguous
// bytes.  With row r0 in the high nibbles, w & 0xF0F0F0F0 is row r0's four
// values times 16 as signed bytes, and (w << 4) & 0xF0F0F0F0 row r1's.
//
// nibble position of (row r, column c) inside its 32-bit word
__host__ __device__ inline int frag_nibble_shift(int r, int c) {
    const int upper = (r % 16) / 8, cc = c % 4;
    return 8 * cc + (upper ? 0 : 4);
}

// byte offset of the 16-byte unit of lane l, 16-row block b8 (0..7) of tile rt,
// 64-column step kb, in a matrix with K columns
__host__ __device__ inline int64_t frag_unit_offset(int rt, int kb, int b8, int lane, int K) {
    return ((((int64_t)rt * (K / 64) + kb) * 8 + b8) * 32 + lane) * 16;
}

// byte offset of the word holding (row r, column c)
__host__ __device__ inline int64_t frag_word_offset(int r, int c, int K) {
    const int rt = r / kTileRows, b8 = (r % kTileRows) / 16, g = r % 8;
    const int kb = c / 64, j = (c % 64) / 16, t = (c % 16) / 4;
    return frag_unit_offset(rt, kb, b8, 4 * g + t, K) + 4 * j;
}

// element offset of the scale of (row r, group g) with ng groups per row
__host__ __device__ inline int64_t scale_offset(int r, int g, int ng) {
    const int t = r / kTileRows, m = r % kTileRows;
    return ((int64_t)t * ng + g) * kTileRows + m;
}

// ---------------------------------------------------------------------------
// Packed f32x2 arithmetic (sm_100: add/fma on two f32 lanes per instruction).
// ---------------------------------------------------------------------------
typedef unsigned long long f2_t;

__device__ __forceinline__ f2_t f2pack(float a, float b) {
    f2_t r;
    asm("mov.b64 %0, {%1, %2};" : "=l"(r) : "f"(a), "f"(b));
    return r;
}
__device__ __forceinline__ float2 f2unpack(f2_t v) {
    float2 r;
    asm("mov.b64 {%0, %1}, %2;" : "=f"(r.x), "=f"(r.y) : "l"(v));
    return r;
}
__device__ __forceinline__ f2_t f2add(f2_t a, f2_t b) {
    f2_t r;
    asm("add.rn.f32x2 %0, %1, %2;" : "=l"(r) : "l"(a), "l"(b));
    return r;
}
__device__ __forceinline__ f2_t f2fma(f2_t a, f2_t b, f2_t c) {
    f2_t r;
    asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(r) : "l"(a), "l"(b), "l"(c));
    return r;
}

// ---------------------------------------------------------------------------
// Exact int4 -> fp16 decode of one word of a fragment tile (see above) into the
// four f16x2 registers (row r0: c0,c0+1 | row r0: c0+2,c0+3 | row r1: c0,c0+1 |
// row r1: c0+2,c0+3).  The nibble is masked in place, its sign bit flipped and
// the fp16 exponent of 1024 OR-ed in: a nibble at bits 0-3 of a half reads as
// 1024 + (q + 8), one at bits 4-7 as 1024 + 16 (q + 8); one packed subtract or
// fused multiply-add per two values then leaves q exactly.
// ---------------------------------------------------------------------------
__device__ __forceinline__ uint32_t h2sub_1032(uint32_t v) {
    uint32_t r;
    asm("sub.rn.f16x2 %0, %1, %2;" : "=r"(r) : "r"(v), "r"(0x64086408u));
    return r;
}
__device__ __forceinline__ uint32_t h2fma_16th_m72(uint32_t v) {
    uint32_t r;  // v * 1/16 - 72
    asm("fma.rn.f16x2 %0, %1, %2, %3;" : "=r"(r) : "r"(v), "r"(0x2C002C00u), "r"(0xD480D480u));
    return r;
}
// D[16x8] (f32) (+)= A[16x16] (f16) * B[16x8] (f16), warp-wide
__device__ __forceinline__ void mma_f16_16816(float d[4], const uint32_t a[4], uint32_t b0,
                                              uint32_t b1) {
    asm volatile(
        "mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, "
        "{%8,%9}, {%0,%1,%2,%3};"
        : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
        : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}
__device__ __forceinline__ void mma_f16_16816_zc(float d[4], const uint32_t a[4], uint32_t b0,
                                                 uint32_t b1) {
    const float z = 0.0f;  // C = 0: starts a fresh partial product
    asm volatile(
        "mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, "
        "{%8,%9}, {%10,%10,%10,%10};"
        : "=f"(d[0]), "=f"(d[1]), "=f"(d[2]), "=f"(d[3])
        : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1), "f"(z));
}

// fp16 magic constants of the nibble decode, passed as kernel parameters so
// they are read from the parameter bank instead of being rebuilt per use
struct DecodeK {
    uint32_t xlo = 0x64086408u;   // sign flip of a nibble at bits 0-3 + fp16 exponent of 1024
    uint32_t xhi = 0x64806480u;   // same for a nibble at bits 4-7
    uint32_t sub = 0x64086408u;   // 1032 = 1024 + 8
    uint32_t mul = 0x2C002C00u;   // 1/16
    uint32_t add = 0xD480D480u;   // -72 = -(1024 + 8*16)/16
};

// Decode one fragment-tile word straight into an mma.sync m16n8k16 A fragment:
// a[0] = row r0 (c0, c0+1), a[1] = row r1 (c0, c0+1), a[2] = row r0 (c0+2, c0+3),
// a[3] = row r1 (c0+2, c0+3).  Swapping the word's middle bytes puts columns
// c0, c0+1 in the two 16-bit halves (row r0 at bits 4-7, row r1 at bits 0-3);
// shifted right by 8, columns c0+2, c0+3 sit the same way.
__device__ __forceinline__ void decode_word(uint32_t w, uint32_t a[4], const DecodeK& k) {
    const uint32_t p = __byte_perm(w, 0u, 0x3120);
    const uint32_t p8 = p >> 8;
    uint32_t t0, t1, t2, t3;
    asm("lop3.b32 %0, %1, 0x00F000F0, %2, 0x6a;" : "=r"(t0) : "r"(p), "r"(k.xhi));
    asm("lop3.b32 %0, %1, 0x000F000F, %2, 0x6a;" : "=r"(t1) : "r"(p), "r"(k.xlo));
    asm("lop3.b32 %0, %1, 0x00F000F0, %2, 0x6a;" : "=r"(t2) : "r"(p8), "r"(k.xhi));
    asm("lop3.b32 %0, %1, 0x000F000F, %2, 0x6a;" : "=r"(t3) : "r"(p8), "r"(k.xlo));
    asm("fma.rn.f16x2 %0, %1, %2, %3;" : "=r"(a[0]) : "r"(t0), "r"(k.mul), "r"(k.add));
    asm("sub.rn.f16x2 %0, %1, %2;" : "=r"(a[1]) : "r"(t1), "r"(k.sub));
    asm("fma.rn.f16x2 %0, %1, %2, %3;" : "=r"(a[2]) : "r"(t2), "r"(k.mul), "r"(k.add));
    asm("sub.rn.f16x2 %0, %1, %2;" : "=r"(a[3]) : "r"(t3), "r"(k.sub));
}

// Activation operand: power-of-two scale 2^(14 - e) for a group whose largest
// magnitude is m = 2^e * f (f in [1, 2)), so the scaled values stay below 2^15
// in fp16; returns the inverse scale.  All-zero groups use 1.
__device__ __forceinline__ float act_group_scale(float m, float* inv) {
    if (!(m > 0.0f) || !isfinite(m)) { *inv = 1.0f; return 1.0f; }
    int e;
    frexpf(m, &e);                 // m = f * 2^e, f in [0.5, 1)
    int sh = 15 - e;               // m * 2^sh in [2^14, 2^15)
    sh = max(-100, min(100, sh));
    *inv = ldexpf(1.0f, -sh);
    return ldexpf(1.0f, sh);
}

// split v (already scaled) into fp16 hi + lo with v ~= hi + lo to ~22 bits
__device__ __forceinline__ void split_f16(float v, __half& hi, __half& lo) {
    hi = __float2half_rn(v);
    lo = __float2half_rn(v - __half2float(hi));
}

// Read-only 16-byte global load that bypasses L1 allocation (weights are
// streamed exactly once per launch).
__device__ __forceinline__ uint4 ldg_stream(const void* p) {
    uint4 r;
    asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0, %1, %2, %3}, [%4];"
                 : "=r"(r.x), "=r"(r.y), "=r"(r.z), "=r"(r.w) : "l"(p));
    return r;
}

template <typename T> __device__ __forceinline__ float to_f32(T v);
template <> __device__ __forceinline__ float to_f32<float>(float v) { return v; }
template <> __device__ __forceinline__ float to_f32<__nv_bfloat16>(__nv_bfloat16 v) {
    return __bfloat162float(v);
}

__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
    return v;
}

__device__ __forceinline__ float silu_f(float a) { return a / (1.0f + expf(-a)); }

}  // namespace coli
