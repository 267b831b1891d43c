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

// The parameters of one tiled view, apart from its base address: rank, extents
// (innermost first), byte strides of dimensions 1 .. rank-1, box extents, element type
// and swizzle.  The *_view functions below only compute them (no driver call), so the
// host can check a view's footprint without a GPU; encode() turns one into a map.
struct View {
    int rank = 0;
    cuuint64_t dims[5] = {0, 0, 0, 0, 0};
    cuuint64_t strides[4] = {0, 0, 0, 0};
    cuuint32_t box[5] = {0, 0, 0, 0, 0};
    int elem_bytes = 2;
    bool u8 = false;                // uint8 with the 64-byte swizzle, else bf16 with the 128-byte one
};

inline bool encode(CUtensorMap* m, const View& v, const void* ptr) {
    EncodeTiledFn enc = encode_fn();
    if (!enc || v.rank <= 0) return false;
    cuuint32_t estr[5] = {1, 1, 1, 1, 1};
    return enc(m, v.u8 ? CU_TENSOR_MAP_DATA_TYPE_UINT8 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16,
               static_cast<cuuint32_t>(v.rank), const_cast<void*>(ptr), v.dims, v.strides, v.box,
               estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
               v.u8 ? CU_TENSOR_MAP_SWIZZLE_64B : CU_TENSOR_MAP_SWIZZLE_128B,
               CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// bf16 matrix [rows, K] row-major; boxes of 64 (K) x box_rows.
inline bool matrix_view(View* v, long long rows, int K, int box_rows) {
    if (rows <= 0 || K <= 0) return false;
    *v = View{};
    v->rank = 2;
    v->dims[0] = static_cast<cuuint64_t>(K);
    v->dims[1] = static_cast<cuuint64_t>(rows);
    v->strides[0] = static_cast<cuuint64_t>(K) * 2;
    v->box[0] = static_cast<cuuint32_t>(kBoxK);
    v->box[1] = static_cast<cuuint32_t>(box_rows);
    return true;
}

inline bool matrix(CUtensorMap* m, const void* ptr, long long rows, int K, int box_rows) {
    View v;
    return matrix_view(&v, rows, K, box_rows) && encode(m, v, ptr);
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
inline bool row_pairs_view(View* v, int E, int n_pairs, int K, int box_pairs, long long s_stride,
                           long long i_stride, bool u8 = false) {
    if (E <= 0 || n_pairs <= 0 || K <= 0) return false;
    const cuuint64_t row = static_cast<cuuint64_t>(K) * (u8 ? 1 : 2);
    *v = View{};
    v->rank = 4;
    v->u8 = u8;
    v->elem_bytes = u8 ? 1 : 2;
    v->dims[0] = static_cast<cuuint64_t>(K);
    v->dims[1] = 2;
    v->dims[2] = static_cast<cuuint64_t>(n_pairs);
    v->dims[3] = static_cast<cuuint64_t>(E);
    v->strides[0] = row * static_cast<cuuint64_t>(s_stride);
    v->strides[1] = row * static_cast<cuuint64_t>(i_stride);
    v->strides[2] = row * 2 * static_cast<cuuint64_t>(n_pairs);
    v->box[0] = static_cast<cuuint32_t>(kBoxK);
    v->box[1] = 2;
    v->box[2] = static_cast<cuuint32_t>(box_pairs);
    v->box[3] = 1;
    return true;
}

// fc1 [E, 2I, H] of either layout, read in interleaved row order (gate_i, up_i pairs).
inline bool fc1_pairs_view(View* v, int E, int I, int H, int box_pairs, bool chunked,
                           bool u8 = false) {
    return chunked ? row_pairs_view(v, E, I, H, box_pairs, I, 1, u8)
                   : row_pairs_view(v, E, I, H, box_pairs, 1, 2, u8);
}

inline bool fc1_pairs(CUtensorMap* m, const void* fc1, int E, int I, int H, int box_pairs,
                      bool chunked, bool u8 = false) {
    View v;
    return fc1_pairs_view(&v, E, I, H, box_pairs, chunked, u8) && encode(m, v, fc1);
}

// A plain [E, n, K] weight tensor (n even) in the same 4-D form, so that one load
// instruction serves both GEMMs of a kernel.
inline bool plain_pairs_view(View* v, int E, int n, int K, int box_pairs, bool u8 = false) {
    return n % 2 == 0 && row_pairs_view(v, E, n / 2, K, box_pairs, 1, 2, u8);
}

inline bool plain_pairs(CUtensorMap* m, const void* w, int E, int n, int K, int box_pairs,
                        bool u8 = false) {
    View v;
    return plain_pairs_view(&v, E, n, K, box_pairs, u8) && encode(m, v, w);
}

// bf16 weights in "fragment order" for an accumulator that the epilogue reads in 16x256b
// fragments (a thread holds lanes j, j + 8, j + 16, j + 24 of a 32-lane quadrant): a box
// of 128 weight rows from row r0 (a multiple of 32) of an expert lands in shared memory
// so that box row 32 Q + 8 q + j (Q, q = 0..3, j = 0..7) holds weight row
// r0 + 32 Q + 4 j + q, i.e. such a thread holds four consecutive weight rows.
//   plain [E, n, K] (fc2; fc1 interleaved, n = 2I): the 5-D tensor (k, j, q, Q, e) with
//       row strides (4, 1, 32, n); coordinates (k0, 0, 0, r0 / 32, e).  Rows past n of
//       the last expert read as zeros.
inline bool quad_rows_view(View* v, int E, int n, int K) {
    if (E <= 0 || n <= 0 || n % 32 != 0 || K <= 0) return false;
    const cuuint64_t row = static_cast<cuuint64_t>(K) * 2;
    *v = View{};
    v->rank = 5;
    v->dims[0] = static_cast<cuuint64_t>(K);
    v->dims[1] = 8;
    v->dims[2] = 4;
    v->dims[3] = static_cast<cuuint64_t>(n / 32);
    v->dims[4] = static_cast<cuuint64_t>(E);
    v->strides[0] = row * 4;
    v->strides[1] = row;
    v->strides[2] = row * 32;
    v->strides[3] = row * static_cast<cuuint64_t>(n);
    v->box[0] = static_cast<cuuint32_t>(kBoxK);
    v->box[1] = 8;
    v->box[2] = 4;
    v->box[3] = 4;
    v->box[4] = 1;
    return true;
}

inline bool quad_rows(CUtensorMap* m, const void* w, int E, int n, int K) {
    View v;
    return quad_rows_view(&v, E, n, K) && encode(m, v, w);
}

//   fc1 chunked [E, 2I, K] (row i = gate_i, I + i = up_i) in the same order over its
//       interleaved rows 2i + s: with q = 2 qq + s, interleaved row 32 Q + 4 j + 2 qq + s
//       of expert e is chunked row 2I e + s I + 16 Q + 2 j + qq.  The expert folds into
//       the last coordinate, X = e I / 8 + Q (16 X = 2I e + 16 Q): the 5-D tensor
//       (k, j, s, qq, X) with row strides (2, I, 1, 16); coordinates
//       (k0, 0, 0, 0, e I / 8 + r0 / 32).  X < (2E - 1) I / 16 keeps every element of
//       the tensor inside the weights; boxes past an expert's rows read another
//       expert's (or zeros past the last), whose outputs the kernel drops.
inline bool fc1_quad_rows_chunked_view(View* v, int E, int I, int K) {
    if (E <= 0 || I <= 0 || I % 16 != 0 || K <= 0) return false;
    const cuuint64_t row = static_cast<cuuint64_t>(K) * 2;
    *v = View{};
    v->rank = 5;
    v->dims[0] = static_cast<cuuint64_t>(K);
    v->dims[1] = 8;
    v->dims[2] = 2;
    v->dims[3] = 2;
    v->dims[4] = static_cast<cuuint64_t>(2 * E - 1) * static_cast<cuuint64_t>(I / 16);
    v->strides[0] = row * 2;
    v->strides[1] = row * static_cast<cuuint64_t>(I);
    v->strides[2] = row;
    v->strides[3] = row * 16;
    v->box[0] = static_cast<cuuint32_t>(kBoxK);
    v->box[1] = 8;
    v->box[2] = 2;
    v->box[3] = 2;
    v->box[4] = 4;
    return true;
}

inline bool fc1_quad_rows_chunked(CUtensorMap* m, const void* fc1, int E, int I, int K) {
    View v;
    return fc1_quad_rows_chunked_view(&v, E, I, K) && encode(m, v, fc1);
}

}  // namespace tmap
}  // namespace moe
