// Host side of TMA: encode tensor maps through the driver entry point that the
// CUDA runtime hands out, so the library needs no link against libcuda.
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>

#include <cstdint>

namespace sa {

using EncodeTiledFn = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                   const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                   CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

inline EncodeTiledFn encode_tiled_fn()
{
    static EncodeTiledFn fn = nullptr;
    if (!fn) {
        void* p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<EncodeTiledFn>(p);
    }
    return fn;
}

// Map over a contiguous bf16 tensor viewed as [outer][rows][cols] (cols
// innermost), loaded in boxes of 64 columns x box_rows rows x 1 with the
// 128-byte swizzle.  Reads past `rows` or `cols` return zeros.  Returns false
// when the driver rejects the map (alignment, strides, sizes).
inline bool make_map_bf16_3d(CUtensorMap* map, const void* base, uint64_t cols, uint64_t rows, uint64_t outer,
                             uint32_t box_rows)
{
    EncodeTiledFn enc = encode_tiled_fn();
    if (!enc) return false;
    cuuint64_t dims[3] = {cols, rows, outer};
    cuuint64_t strides[2] = {cols * 2, rows * cols * 2};
    cuuint32_t box[3] = {64, box_rows, 1};
    cuuint32_t estr[3] = {1, 1, 1};
    CUresult r = enc(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(base), dims, strides, box, estr,
                     CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                     CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS;
}

// Map over a contiguous bf16 tensor [outer][rows][cols] viewed in the
// residue-grouped order of its rows, P = (t mod s) * n + t / s with n = rows / s
// (token t = j s + g for P = g n + j): dimensions (cols, s, n, outer), that is
// (feature, g, j, plane) with strides of one row (g) and s rows (j), so that
// grouped rows P0 .. P0 + box_rows - 1 of one group are the box at (c0, P0 / n,
// P0 mod n, plane).  Needs rows % s == 0 and n a multiple of box_rows (a box
// never spans two groups).
inline bool make_map_bf16_grouped(CUtensorMap* map, const void* base, uint64_t cols, uint64_t rows, uint64_t outer,
                                  uint64_t s, uint32_t box_rows)
{
    EncodeTiledFn enc = encode_tiled_fn();
    if (!enc || s == 0 || rows % s != 0) return false;
    const uint64_t n = rows / s;
    if (n % box_rows != 0) return false;
    cuuint64_t dims[4] = {cols, s, n, outer};
    cuuint64_t strides[3] = {cols * 2, s * cols * 2, rows * cols * 2};
    cuuint32_t box[4] = {64, 1, box_rows, 1};
    cuuint32_t estr[4] = {1, 1, 1, 1};
    CUresult r = enc(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, const_cast<void*>(base), dims, strides, box, estr,
                     CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                     CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS;
}

}  // namespace sa
