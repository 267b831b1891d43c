// Host-side TMA descriptors (cuTensorMapEncodeTiled through the runtime's driver
// entry point) for the bf16 operands of the tensor-core kernels.  Every box is 64
// elements (one 128-byte row) wide on K and stored with the 128-byte swizzle that
// the shared-memory matrix descriptors of sm100.cuh expect.
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>

namespace moe {
namespace tmap {

constexpr int kBoxK = 64;

typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                  const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                  const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                  CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

inline EncodeTiledFn encode_fn() {
    static EncodeTiledFn fn = nullptr;
    if (!fn) {
        void* p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) ==
                cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<EncodeTiledFn>(p);
    }
    return fn;
}

// bf16 matrix [rows, K] row-major; boxes of 64 (K) x box_rows.
inline bool matrix(CUtensorMap* m, const void* ptr, long long rows, int K, int box_rows) {
    EncodeTiledFn enc = encode_fn();
    if (!enc || rows <= 0) return false;
    cuuint64_t dims[2] = {static_cast<cuuint64_t>(K), static_cast<cuuint64_t>(rows)};
    cuuint64_t strides[1] = {static_cast<cuuint64_t>(K) * 2};
    cuuint32_t box[2] = {static_cast<cuuint32_t>(kBoxK), static_cast<cuuint32_t>(box_rows)};
    cuuint32_t estr[2] = {1, 1};
    return enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(ptr), dims, strides, box,
               estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
               CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// The weights of E experts, n = 2 n_pairs rows of K each per expert, as the 4-D tensor
// (k, s, i, e): element (k, s, i, e) is column k of the expert's row s_stride s +
// i_stride i.  A box of 64 (k) x 2 (s) x box_pairs (i) x 1 (e) lands in shared memory as
// 2 box_pairs rows of 128 bytes in the order of the row index 2i + s, whatever the
// layout in memory; coordinates (k0, 0, j0 / 2, e) for rows j0 .. of expert e.  Pairs
// i >= n_pairs read as zeros.
//   plain [E, n, K] (fc2; fc1 interleaved: row 2i = gate_i, 2i+1 = up_i):
//       s_stride 1, i_stride 2
//   fc1 chunked [E, 2I, K] (row i = gate_i, I+i = up_i): s_stride I, i_stride 1
//   int8 weights (u8 = true): one byte per element, 64-byte rows stored with the 64-byte
//       swizzle (logical 16-byte chunk c of row r at chunk c ^ ((r >> 1) & 3)), so that
//       the converting warps read one row per lane without bank conflicts
inline bool row_pairs(CUtensorMap* m, const void* w, int E, int n_pairs, int K, int box_pairs,
                      long long s_stride, long long i_stride, bool u8 = false) {
    EncodeTiledFn enc = encode_fn();
    if (!enc || E <= 0 || n_pairs <= 0) return false;
    const cuuint64_t row = static_cast<cuuint64_t>(K) * (u8 ? 1 : 2);
    cuuint64_t dims[4] = {static_cast<cuuint64_t>(K), 2, static_cast<cuuint64_t>(n_pairs),
                          static_cast<cuuint64_t>(E)};
    cuuint64_t strides[3] = {row * static_cast<cuuint64_t>(s_stride),
                             row * static_cast<cuuint64_t>(i_stride),
                             row * 2 * static_cast<cuuint64_t>(n_pairs)};
    cuuint32_t box[4] = {static_cast<cuuint32_t>(kBoxK), 2, static_cast<cuuint32_t>(box_pairs), 1};
    cuuint32_t estr[4] = {1, 1, 1, 1};
    return enc(m, u8 ? CU_TENSOR_MAP_DATA_TYPE_UINT8 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4,
               const_cast<void*>(w), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
               u8 ? CU_TENSOR_MAP_SWIZZLE_64B : CU_TENSOR_MAP_SWIZZLE_128B,
               CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// fc1 [E, 2I, H] of either layout, read in interleaved row order (gate_i, up_i pairs).
inline bool fc1_pairs(CUtensorMap* m, const void* fc1, int E, int I, int H, int box_pairs,
                      bool chunked, bool u8 = false) {
    return chunked ? row_pairs(m, fc1, E, I, H, box_pairs, I, 1, u8)
                   : row_pairs(m, fc1, E, I, H, box_pairs, 1, 2, u8);
}

// A plain [E, n, K] weight tensor (n even) in the same 4-D form, so that one load
// instruction serves both GEMMs of a kernel.
inline bool plain_pairs(CUtensorMap* m, const void* w, int E, int n, int K, int box_pairs,
                        bool u8 = false) {
    return n % 2 == 0 && row_pairs(m, w, E, n / 2, K, box_pairs, 1, 2, u8);
}

// bf16 weights in "fragment order" for an accumulator that the epilogue reads in 16x256b
// fragments (a thread holds lanes j, j + 8, j + 16, j + 24 of a 32-lane quadrant): a box
// of 128 weight rows from row r0 (a multiple of 32) of an expert lands in shared memory
// so that box row 32 Q + 8 q + j (Q, q = 0..3, j = 0..7) holds weight row
// r0 + 32 Q + 4 j + q, i.e. such a thread holds four consecutive weight rows.
//   plain [E, n, K] (fc2; fc1 interleaved, n = 2I): the 5-D tensor (k, j, q, Q, e) with
//       row strides (4, 1, 32, n); coordinates (k0, 0, 0, r0 / 32, e).  Rows past n of
//       the last expert read as zeros.
inline bool quad_rows(CUtensorMap* m, const void* w, int E, int n, int K) {
    EncodeTiledFn enc = encode_fn();
    if (!enc || E <= 0 || n <= 0 || n % 32 != 0) return false;
    const cuuint64_t row = static_cast<cuuint64_t>(K) * 2;
    cuuint64_t dims[5] = {static_cast<cuuint64_t>(K), 8, 4, static_cast<cuuint64_t>(n / 32),
                          static_cast<cuuint64_t>(E)};
    cuuint64_t strides[4] = {row * 4, row, row * 32, row * static_cast<cuuint64_t>(n)};
    cuuint32_t box[5] = {static_cast<cuuint32_t>(kBoxK), 8, 4, 4, 1};
    cuuint32_t estr[5] = {1, 1, 1, 1, 1};
    return enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 5, const_cast<void*>(w), dims, strides, box,
               estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
               CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

//   fc1 chunked [E, 2I, K] (row i = gate_i, I + i = up_i) in the same order over its
//       interleaved rows 2i + s: with q = 2 qq + s, interleaved row 32 Q + 4 j + 2 qq + s
//       of expert e is chunked row 2I e + s I + 16 Q + 2 j + qq.  The expert folds into
//       the last coordinate, X = e I / 8 + Q (16 X = 2I e + 16 Q): the 5-D tensor
//       (k, j, s, qq, X) with row strides (2, I, 1, 16); coordinates
//       (k0, 0, 0, 0, e I / 8 + r0 / 32).  X < (2E - 1) I / 16 keeps every element of
//       the tensor inside the weights; boxes past an expert's rows read another
//       expert's (or zeros past the last), whose outputs the kernel drops.
inline bool fc1_quad_rows_chunked(CUtensorMap* m, const void* fc1, int E, int I, int K) {
    EncodeTiledFn enc = encode_fn();
    if (!enc || E <= 0 || I <= 0 || I % 16 != 0) return false;
    const cuuint64_t row = static_cast<cuuint64_t>(K) * 2;
    cuuint64_t dims[5] = {static_cast<cuuint64_t>(K), 8, 2, 2,
                          static_cast<cuuint64_t>(2 * E - 1) * static_cast<cuuint64_t>(I / 16)};
    cuuint64_t strides[4] = {row * 2, row * static_cast<cuuint64_t>(I), row, row * 16};
    cuuint32_t box[5] = {static_cast<cuuint32_t>(kBoxK), 8, 2, 2, 4};
    cuuint32_t estr[5] = {1, 1, 1, 1, 1};
    return enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 5, const_cast<void*>(fc1), dims, strides, box,
               estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
               CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

}  // namespace tmap
}  // namespace moe
