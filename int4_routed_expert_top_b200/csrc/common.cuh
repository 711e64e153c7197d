// common.cuh - shared device helpers for libcolimoe (sm_100a).
#pragma once

#include <cuda_bf16.h>
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

// byte offset of code unit (row r, unit c) inside a matrix with K columns
__host__ __device__ inline int64_t code_unit_offset(int r, int c, int K) {
    const int t = r / kTileRows, m = r % kTileRows;
    return (((int64_t)t * (K / kUnitCols) + c) * kTileRows + m) * 16;
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
// Exact int4 -> f32 decode without integer-to-float conversions.
//
// A nibble n sitting at bit position 4p (p <= 4) of a word is masked in place
// and its sign bit flipped, and the f32 exponent of 2^23 is OR-ed in:
//   bits = (w & (0xF << 4p)) ^ (0x4B000000 | 0x8 << 4p)
//   value = 2^23 + 16^p * (n ^ 8) = 2^23 + 16^p * (q + 8)   (q = signed code)
// Subtracting the constant 2^23 + 8 * 16^p leaves 16^p * q exactly.  The
// factor 16^p is undone by pre-scaling the activation of that column by
// 16^-p (exact powers of two), so (16^p q) * (16^-p x) rounds like q * x.
// Nibbles 5..7 are first moved down by 12 bits to positions 2..4.
// Column j of a word (j = 0..7) therefore uses position
//   pos(j) = {0, 1, 2, 3, 4, 2, 3, 4}[j]
// ---------------------------------------------------------------------------
__host__ __device__ constexpr float kPosScale(int j) {
    return j == 0 ? 1.0f : j == 1 ? 0.0625f : (j == 2 || j == 5) ? 0.00390625f
         : (j == 3 || j == 6) ? 0.000244140625f : 0.0000152587890625f;
}

// decode the 8 nibbles of w into 4 f32 pairs: (c0,c1), (c2,c3), (c4,c5), (c6,c7)
__device__ __forceinline__ void decode8(uint32_t w, f2_t out[4]) {
    const uint32_t u = w >> 12;
    const float a0 = __uint_as_float((w & 0x0000000Fu) ^ 0x4B000008u);
    const float a1 = __uint_as_float((w & 0x000000F0u) ^ 0x4B000080u);
    const float a2 = __uint_as_float((w & 0x00000F00u) ^ 0x4B000800u);
    const float a3 = __uint_as_float((w & 0x0000F000u) ^ 0x4B008000u);
    const float a4 = __uint_as_float((w & 0x000F0000u) ^ 0x4B080000u);
    const float a5 = __uint_as_float((u & 0x00000F00u) ^ 0x4B000800u);
    const float a6 = __uint_as_float((u & 0x0000F000u) ^ 0x4B008000u);
    const float a7 = __uint_as_float((u & 0x000F0000u) ^ 0x4B080000u);
    out[0] = f2add(f2pack(a0, a1), f2pack(-8388616.0f, -8388736.0f));
    out[1] = f2add(f2pack(a2, a3), f2pack(-8390656.0f, -8421376.0f));
    out[2] = f2add(f2pack(a4, a5), f2pack(-8912896.0f, -8390656.0f));
    out[3] = f2add(f2pack(a6, a7), f2pack(-8421376.0f, -8912896.0f));
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
