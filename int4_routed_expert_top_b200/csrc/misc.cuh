// misc.cuh - device quantiser/packer, dequantiser (test helper), RMSNorm and the
// staging copies of the host-buffer entry points.
//
// Quantiser ("jlnsrk/GLM-5.2-colibri-int4 - Hugging Face": container paragraph
// and conversion note): per row or per 64 columns s = max|w| / 7, q =
// rint(w / s) in [-7, 7] (IEEE f32 division, round half to even), written
// straight into the tiled device layout.
#pragma once

#include <cuda_fp8.h>

#include "common.cuh"

namespace coli {

__device__ __forceinline__ int quant_one(float v, float s) {
    if (s == 0.0f) return 0;
    float q = rintf(__fdiv_rn(v, s));
    q = fminf(fmaxf(q, -7.0f), 7.0f);
    return (int)q;
}

// Row sources of the device quantiser: f32 masters, or FP8 E4M3 codes with one
// f32 scale per 128 x 128 block (the checkpoint the container is converted
// from: "解密GLM-5.2-colibri-int4-with-int8-mtp", quantisation-config
// paragraph, fmt e4m3 with weight_block_size [128, 128]).  The E4M3 value is
// exact in half and f32; the block scale is applied by one f32 multiply.
struct QzF32 {
    const float* w;
    __device__ __forceinline__ float at(int64_t r, int c, int K) const { return w[r * K + c]; }
};
struct QzFp8Block {
    const uint8_t* q;   // [R, K] E4M3 codes
    const float* bs;    // [ceil(R/128), ceil(K/128)] block scales
    int kb;             // ceil(K / 128)
    __device__ __forceinline__ float at(int64_t r, int c, int K) const {
        const __half_raw h = __nv_cvt_fp8_to_halfraw((__nv_fp8_storage_t)q[r * K + c], __NV_E4M3);
        return __fmul_rn(__half2float(__half(h)), bs[(r / 128) * kb + c / 128]);
    }
};

// One CTA per 16-row block of a 128-row tile.  Each warp quantises two rows
// into shared memory in container byte order, then every thread assembles
// 16-byte fragment-tile units (see common.cuh) and stores them.
template <typename Src>
__global__ void __launch_bounds__(256)
quantize_rows_kernel(Src src, int R, int K, int group,
                     uint8_t* __restrict__ codes, float* __restrict__ scales) {
    extern __shared__ uint4 qz_smem[];
    uint8_t* rows = reinterpret_cast<uint8_t*>(qz_smem);  // [16][K/2]
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int blk = blockIdx.x;                            // 16-row block index
    const int rt = blk / 8, b8 = blk % 8;
    const int gs = group ? group : K;
    const int ng = K / gs;
    for (int lr = warp; lr < 16; lr += 8) {
        const int r = blk * 16 + lr;
        uint8_t* buf = rows + (int64_t)lr * (K / 2);
        for (int g = 0; g < ng; ++g) {
            float m = 0.0f;
            for (int c = g * gs + lane; c < (g + 1) * gs; c += 32) m = fmaxf(m, fabsf(src.at(r, c, K)));
#pragma unroll
            for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
            const float s = __fdiv_rn(m, 7.0f);
            if (lane == 0) scales[scale_offset(r, g, ng)] = s;
            for (int cp = g * gs / 2 + lane; cp < (g + 1) * gs / 2; cp += 32) {
                const int q0 = quant_one(src.at(r, 2 * cp, K), s), q1 = quant_one(src.at(r, 2 * cp + 1, K), s);
                buf[cp] = (uint8_t)((q0 & 15) | ((q1 & 15) << 4));
            }
        }
    }
    __syncthreads();
    for (int i = threadIdx.x; i < (K / 64) * 32; i += 256) {
        const int kb = i / 32, l = i % 32, g = l >> 2, t = l & 3;
        uint32_t wd[4];
        for (int j = 0; j < 4; ++j) {
            uint32_t word = 0;
            for (int upper = 0; upper < 2; ++upper)
                for (int cc = 0; cc < 4; ++cc) {
                    const int lr = g + 8 * upper, c = kb * 64 + 16 * j + 4 * t + cc;
                    const uint8_t byte = rows[(int64_t)lr * (K / 2) + c / 2];
                    const uint32_t nib = (c & 1) ? (byte >> 4) : (byte & 15);
                    word |= nib << frag_nibble_shift(lr, c);
                }
            wd[j] = word;
        }
        *reinterpret_cast<uint4*>(codes + frag_unit_offset(rt, kb, b8, l, K)) =
            make_uint4(wd[0], wd[1], wd[2], wd[3]);
    }
}

// 8-bit codes (the engine keeps its MTP head at 8 bits: "解密GLM-5.2-colibri-
// int4-with-int8-mtp"): the container's rule with 127 in place of 7, one signed
// byte per weight, written into 8-bit fragment tiles (common.cuh).
__device__ __forceinline__ int quant_one8(float v, float s) {
    if (s == 0.0f) return 0;
    float q = rintf(__fdiv_rn(v, s));
    q = fminf(fmaxf(q, -127.0f), 127.0f);
    return (int)q;
}

template <typename Src>
__global__ void __launch_bounds__(256)
quantize_rows8_kernel(Src src, int R, int K, int group,
                      uint8_t* __restrict__ codes, float* __restrict__ scales) {
    extern __shared__ uint4 qz_smem[];
    int8_t* rows = reinterpret_cast<int8_t*>(qz_smem);  // [16][K]
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int blk = blockIdx.x;                           // 16-row block index
    const int rt = blk / 8, b8 = blk % 8;
    const int gs = group ? group : K;
    const int ng = K / gs;
    for (int lr = warp; lr < 16; lr += 8) {
        const int r = blk * 16 + lr;
        int8_t* buf = rows + (int64_t)lr * K;
        for (int g = 0; g < ng; ++g) {
            float m = 0.0f;
            for (int c = g * gs + lane; c < (g + 1) * gs; c += 32) m = fmaxf(m, fabsf(src.at(r, c, K)));
#pragma unroll
            for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
            const float s = __fdiv_rn(m, 127.0f);
            if (lane == 0) scales[scale_offset(r, g, ng)] = s;
            for (int c = g * gs + lane; c < (g + 1) * gs; c += 32)
                buf[c] = (int8_t)quant_one8(src.at(r, c, K), s);
        }
    }
    __syncthreads();
    // lane l's 32 bytes of each 64-column step: words i = 4h + 2 hi16 + upper
    for (int i = threadIdx.x; i < (K / 64) * 32; i += 256) {
        const int kb = i / 32, l = i % 32, g = l >> 2, t = l & 3;
        uint32_t wd[8];
        for (int w = 0; w < 8; ++w) {
            const int h = w >> 2, hi16 = (w >> 1) & 1, upper = w & 1;
            const int lr = g + 8 * upper, c0 = kb * 64 + 32 * h + 16 * hi16 + 4 * t;
            wd[w] = *reinterpret_cast<const uint32_t*>(rows + (int64_t)lr * K + c0);
        }
        uint8_t* dst = codes + ((((int64_t)rt * (K / 64) + kb) * 8 + b8) * 32 + l) * 32;
        *reinterpret_cast<uint4*>(dst) = make_uint4(wd[0], wd[1], wd[2], wd[3]);
        *reinterpret_cast<uint4*>(dst + 16) = make_uint4(wd[4], wd[5], wd[6], wd[7]);
    }
}

// one thread per element of an 8-bit matrix: out[r, c] = (float)q * s
__global__ void __launch_bounds__(256)
dequant8_kernel(const uint8_t* __restrict__ codes, const float* __restrict__ scales,
                int R, int K, int group, float* __restrict__ out) {
    const int64_t i = (int64_t)blockIdx.x * 256 + threadIdx.x;
    if (i >= (int64_t)R * K) return;
    const int r = (int)(i / K), c = (int)(i % K);
    const int ng = group ? K / group : 1;
    const int q = (int8_t)codes[frag8_byte_offset(r, c, K)];
    const float s = scales[scale_offset(r, group ? c / group : 0, ng)];
    out[i] = __fmul_rn((float)q, s);
}

// one thread per element: out[r, c] = (float)q * s
__global__ void __launch_bounds__(256)
dequant_kernel(const uint8_t* __restrict__ codes, const float* __restrict__ scales,
               int R, int K, int group, float* __restrict__ out) {
    const int64_t i = (int64_t)blockIdx.x * 256 + threadIdx.x;
    if (i >= (int64_t)R * K) return;
    const int r = (int)(i / K), c = (int)(i % K);
    const int ng = group ? K / group : 1;
    const uint32_t word = *reinterpret_cast<const uint32_t*>(codes + frag_word_offset(r, c, K));
    int n = (word >> frag_nibble_shift(r, c)) & 15;
    n = n >= 8 ? n - 16 : n;
    const float s = scales[scale_offset(r, group ? c / group : 0, ng)];
    out[i] = __fmul_rn((float)n, s);
}

// RMSNorm with unit gain: one CTA per row, f32 sum of squares
__global__ void __launch_bounds__(256)
rmsnorm_kernel(const float* x, int H, float eps, float* out) {
    __shared__ float part[8];
    // a programmatic dependent: the next kernel (the router) may be scheduled
    // now, and x may come from the previous grid
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
    asm volatile("griddepcontrol.wait;" ::: "memory");
    const int64_t t = blockIdx.x;
    const float* xr = x + t * H;
    float ss = 0.0f;
    for (int c = threadIdx.x * 4; c < H; c += 1024) {
        const float4 v = *reinterpret_cast<const float4*>(xr + c);
        ss = fmaf(v.x, v.x, ss); ss = fmaf(v.y, v.y, ss);
        ss = fmaf(v.z, v.z, ss); ss = fmaf(v.w, v.w, ss);
    }
    ss = warp_sum(ss);
    if ((threadIdx.x & 31) == 0) part[threadIdx.x >> 5] = ss;
    __syncthreads();
    float tot = 0.0f;
#pragma unroll
    for (int i = 0; i < 8; ++i) tot += part[i];
    const float inv = 1.0f / sqrtf(tot / (float)H + eps);
    __syncthreads();  // every thread has read part before out (may alias x) changes
    float* orow = out + t * H;
    for (int c = threadIdx.x * 4; c < H; c += 1024) {
        float4 v = *reinterpret_cast<const float4*>(xr + c);
        v.x *= inv; v.y *= inv; v.z *= inv; v.w *= inv;
        *reinterpret_cast<float4*>(orow + c) = v;
    }
}

// Byte copy between page-locked host memory (through its device mapping) and
// device memory, by SM loads and stores: for the few kilobytes of a decode
// step this avoids the copy engine's start-up and hand-off latency.  16-byte
// words when both pointers and the size allow, else 4-byte words (the sizes
// here are multiples of 4).
__global__ void __launch_bounds__(256)
stage_copy_kernel(const void* __restrict__ src, void* __restrict__ dst, int64_t bytes) {
    // the router (a programmatic dependent) may be scheduled now; it waits for
    // this grid before reading the staged tokens
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
    const int64_t stride = (int64_t)gridDim.x * blockDim.x;
    const int64_t i0 = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
    if (((reinterpret_cast<uintptr_t>(src) | reinterpret_cast<uintptr_t>(dst) | (uintptr_t)bytes) & 15) == 0) {
        const uint4* s = static_cast<const uint4*>(src);
        uint4* d = static_cast<uint4*>(dst);
        for (int64_t i = i0; i < bytes / 16; i += stride) d[i] = s[i];
    } else {
        const uint32_t* s = static_cast<const uint32_t*>(src);
        uint32_t* d = static_cast<uint32_t*>(dst);
        for (int64_t i = i0; i < bytes / 4; i += stride) d[i] = s[i];
    }
}

}  // namespace coli
