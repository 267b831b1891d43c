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

// fc1 [E, 2I, H] as the 4-D tensor (h, s, i, e) with element (h, s, i, e) = gate_i
// (s = 0) or up_i (s = 1) of expert e at column h, whichever the layout stores it:
//   interleaved: row 2i + s (s stride one row, i stride two rows);
//   chunked:     row s I + i (s stride I rows, i stride one row).
// A box of 64 (h) x 2 (s) x box_pairs (i) x 1 (e) lands in shared memory as
// 2 box_pairs rows of 128 bytes in interleaved order (row 2i + s), whatever the
// layout in memory; coordinates (k0, 0, i0, e).  Pairs i >= I read as zeros.
inline bool fc1_pairs(CUtensorMap* m, const void* fc1, int E, int I, int H, int box_pairs,
                      bool chunked) {
    EncodeTiledFn enc = encode_fn();
    if (!enc || E <= 0 || I <= 0) return false;
    const cuuint64_t row = static_cast<cuuint64_t>(H) * 2;
    cuuint64_t dims[4] = {static_cast<cuuint64_t>(H), 2, static_cast<cuuint64_t>(I),
                          static_cast<cuuint64_t>(E)};
    cuuint64_t strides[3] = {chunked ? row * static_cast<cuuint64_t>(I) : row,
                             chunked ? row : 2 * row, 2 * row * static_cast<cuuint64_t>(I)};
    cuuint32_t box[4] = {static_cast<cuuint32_t>(kBoxK), 2, static_cast<cuuint32_t>(box_pairs), 1};
    cuuint32_t estr[4] = {1, 1, 1, 1};
    return enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, const_cast<void*>(fc1), dims, strides, box,
               estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
               CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

}  // namespace tmap
}  // namespace moe
