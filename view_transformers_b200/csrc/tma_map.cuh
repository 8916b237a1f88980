// Host-side construction of the 2D TMA tensor maps of the tensor-core kernels: row-major
// matrices of 2-byte elements read in boxes 64 elements (128 bytes, one swizzle atom) wide,
// with the 128-byte swizzle that their MMA shared-memory descriptors expect.
#pragma once

#include <cuda.h>
#include <cudaTypedefs.h>
#include <cuda_runtime.h>

#include <cstdint>
#include <mutex>

namespace bsa {

// cuTensorMapEncodeTiled from the driver, looked up once per process (nullptr if the driver
// does not provide it).
inline PFN_cuTensorMapEncodeTiled_v12000 tensor_map_encoder() {
    static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
    static std::once_flag once;
    std::call_once(once, [] {
        void* p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
    });
    return fn;
}

// Map over a row-major [rows, cols] matrix of bf16 (or fp16) elements with a row pitch of
// cols * 2 bytes; a box is 64 columns x box_rows rows. Rows past the end read zeros. False
// when the driver rejects the map (alignment, sizes) or rows == 0.
inline bool make_tile_map(CUtensorMap* tm, const void* base, uint64_t rows, uint64_t cols, uint32_t box_rows,
                          bool fp16) {
    auto enc = tensor_map_encoder();
    if (enc == nullptr || rows == 0) return false;
    cuuint64_t dims[2] = {cols, rows};
    cuuint64_t strides[1] = {cols * 2};
    cuuint32_t box[2] = {64, box_rows};
    cuuint32_t estr[2] = {1, 1};
    return enc(tm, fp16 ? CU_TENSOR_MAP_DATA_TYPE_FLOAT16 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2,
               const_cast<void*>(base), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
               CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
               CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

}  // namespace bsa
