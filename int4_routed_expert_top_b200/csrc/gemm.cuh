// gemm.cuh - tcgen05 grouped-GEMM expert path for large batches.
#pragma once

#include "common.cuh"
#include "coli_moe.h"

namespace coli {

struct GemmCtx {
    const uint8_t* experts;
    int64_t blob_bytes;
    BlobLayout L;
    int H, I, group, E, n_shared, T, k;
    const int32_t* n_units;
    const int32_t* unit_expert;
    const int32_t* unit_begin;
    const int32_t* unit_end;
    const int32_t* pair_tok;
    const void* x;
    int x_bf16;
    float* o;           // [P, H]
};

inline bool gemm_path_preferred(const coli_moe_desc&, int) { return false; }

template <typename Mark>
inline int launch_gemm(const GemmCtx&, cudaStream_t, Mark&&) { return COLI_E_UNSUPPORTED; }

}  // namespace coli
