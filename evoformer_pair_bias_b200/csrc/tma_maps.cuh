// tma_maps.cuh -- host-side construction of TMA tensor maps (cuTensorMapEncodeTiled).
//
// The driver entry point is fetched once through cudaGetDriverEntryPoint, so
// the library needs no link-time dependency on libcuda.
#pragma once

#include <cuda.h>
#include <cudaTypedefs.h>
#include <cuda_runtime.h>

#include <algorithm>
#include <cstdint>
#include <mutex>

#include "evo_attn.h"

namespace evo {
namespace tma {

inline PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
    static std::once_flag once;
    static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
    std::call_once(once, [] {
        void* p = nullptr;
        cudaDriverEntryPointQueryResult q = cudaDriverEntryPointSymbolNotFound;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
    });
    return fn;
}

// Rank-r tiled map.  dims[0] is the contiguous dimension; strides_b[i-1] is
// the byte stride of dims[i].  A size-1 dimension is never stepped along, so
// it gets a stride that is always legal.
inline bool encode(CUtensorMap* m, CUtensorMapDataType dt, uint32_t elem_bytes, const void* ptr, int rank,
                   const uint64_t* dims, const uint64_t* strides_b, const uint32_t* box, CUtensorMapSwizzle sw) {
    auto fn = encode_fn();
    if (!fn) return false;
    cuuint64_t d[5];
    cuuint64_t s[4];
    cuuint32_t bx[5], es[5];
    uint64_t span = dims[0] * elem_bytes;
    for (int i = 0; i < rank; ++i) {
        d[i] = dims[i];
        bx[i] = box[i];
        es[i] = 1;
    }
    for (int i = 1; i < rank; ++i) span = std::max<uint64_t>(span, strides_b[i - 1] * dims[i]);
    for (int i = 1; i < rank; ++i) {
        uint64_t st = strides_b[i - 1];
        if (dims[i] == 1) st = (span + 15) / 16 * 16;
        if (st % 16 != 0 || st >= (1ull << 40)) return false;
        s[i - 1] = st;
    }
    CUresult r = fn(m, dt, (cuuint32_t)rank, const_cast<void*>(ptr), d, s, bx, es, CU_TENSOR_MAP_INTERLEAVE_NONE,
                    sw, CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS;
}

// bf16 per-row tensor, logical [B,S,N,H,C] with element strides st; box (C, rows, 1, 1, 1).
inline bool rows_bf16(CUtensorMap* m, const void* ptr, const evo_shape_t& sh, const evo_strides_t& st,
                      uint32_t rows, CUtensorMapSwizzle sw) {
    const uint64_t dims[5] = {(uint64_t)sh.C, (uint64_t)sh.N, (uint64_t)sh.H, (uint64_t)sh.S, (uint64_t)sh.B};
    const uint64_t str[4] = {(uint64_t)st.n * 2, (uint64_t)st.h * 2, (uint64_t)st.s * 2, (uint64_t)st.b * 2};
    const uint32_t box[5] = {(uint32_t)sh.C, rows, 1, 1, 1};
    return encode(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, ptr, 5, dims, str, box, sw);
}

// bf16 square [B,H,N,N] matrix (pair_bias, or its transpose) viewed as
// (col, row, h, b); box (64 cols, rows, 1, 1) with 128B swizzle.
inline bool square_bf16(CUtensorMap* m, const void* ptr, const evo_shape_t& sh, uint32_t rows) {
    const uint64_t N = (uint64_t)sh.N, H = (uint64_t)sh.H;
    const uint64_t dims[4] = {N, N, H, (uint64_t)sh.B};
    const uint64_t str[3] = {N * 2, N * N * 2, H * N * N * 2};
    const uint32_t box[4] = {64, rows, 1, 1};
    return encode(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, ptr, 4, dims, str, box, CU_TENSOR_MAP_SWIZZLE_128B);
}

// bf16 mask_bias [B,S,1,1,N] viewed as (j, s, b); box (keys, 1, 1).
inline bool mask_bf16(CUtensorMap* m, const void* ptr, const evo_shape_t& sh, uint32_t keys = 128) {
    const uint64_t N = (uint64_t)sh.N, S = (uint64_t)sh.S;
    const uint64_t dims[3] = {N, S, (uint64_t)sh.B};
    const uint64_t str[2] = {N * 2, S * N * 2};
    const uint32_t box[3] = {keys, 1, 1};
    return encode(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, ptr, 3, dims, str, box, CU_TENSOR_MAP_SWIZZLE_NONE);
}

// fp32 per-row scalar [B,S,H,n_row] viewed as (i, h, s, b); box (128, 1, 1, 1).
inline bool rowscalar_f32(CUtensorMap* m, const void* ptr, const evo_shape_t& sh, int64_t n_row) {
    const uint64_t N = (uint64_t)n_row, H = (uint64_t)sh.H, S = (uint64_t)sh.S;
    const uint64_t dims[4] = {N, H, S, (uint64_t)sh.B};
    const uint64_t str[3] = {N * 4, H * N * 4, S * H * N * 4};
    const uint32_t box[4] = {128, 1, 1, 1};
    return encode(m, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 4, ptr, 4, dims, str, box, CU_TENSOR_MAP_SWIZZLE_NONE);
}

// bf16 rank-term rows [B,S,H,2,n_row] (a high and a low row per (b,s,h))
// viewed as (i, row, h, s, b); box (64 queries, 2 rows, 1, 1, 1) with 128B
// swizzle, so each box lands as rows 0..1 of one 128B-swizzled operand atom.
inline bool rowterm_bf16(CUtensorMap* m, const void* ptr, const evo_shape_t& sh, int64_t n_row) {
    const uint64_t N = (uint64_t)n_row, H = (uint64_t)sh.H, S = (uint64_t)sh.S;
    const uint64_t dims[5] = {N, 2, H, S, (uint64_t)sh.B};
    const uint64_t str[4] = {N * 2, 2 * N * 2, H * 2 * N * 2, S * H * 2 * N * 2};
    const uint32_t box[5] = {64, 2, 1, 1, 1};
    return encode(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, ptr, 5, dims, str, box, CU_TENSOR_MAP_SWIZZLE_128B);
}

// bf16 row-major matrix [rows, cols] with row pitch ld (elements), viewed as
// (col, row); box (64 cols, box_rows) with 128B swizzle.
inline bool matrix_bf16(CUtensorMap* m, const void* ptr, int64_t rows, int64_t cols, int64_t ld, uint32_t box_rows) {
    const uint64_t dims[2] = {(uint64_t)cols, (uint64_t)rows};
    const uint64_t str[1] = {(uint64_t)ld * 2};
    const uint32_t box[2] = {64, box_rows};
    return encode(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, ptr, 2, dims, str, box, CU_TENSOR_MAP_SWIZZLE_128B);
}

// A stack of `batch` contiguous rows x cols bf16 matrices [batch][rows][cols],
// boxes of box0 (<= 64, one 128-byte swizzle span) x box1 rows of one matrix.
inline bool batch_bf16(CUtensorMap* m, const void* ptr, int64_t cols, int64_t rows, int64_t batch, uint32_t box0,
                       uint32_t box1) {
    const uint64_t dims[3] = {(uint64_t)cols, (uint64_t)rows, (uint64_t)batch};
    const uint64_t str[2] = {(uint64_t)cols * 2, (uint64_t)rows * cols * 2};
    const uint32_t box[3] = {box0, box1, 1};
    return encode(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, ptr, 3, dims, str, box, CU_TENSOR_MAP_SWIZZLE_128B);
}

}  // namespace tma
}  // namespace evo
