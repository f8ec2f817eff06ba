// Tensor-memory-accelerator (TMA) helpers shared by the kernels of libkda. Internal.
// Tensor maps are encoded on the host through the driver's cuTensorMapEncodeTiled, reached
// with cudaGetDriverEntryPoint (no link-time dependency on libcuda). No multicast anywhere.
#pragma once

#include <cuda.h>

#include "common.cuh"
#include "umma.cuh"

namespace kda {

typedef CUresult (*EncodeTiledFn)(CUtensorMap *, CUtensorMapDataType, cuuint32_t, void *, const cuuint64_t *,
                                  const cuuint64_t *, const cuuint32_t *, const cuuint32_t *, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

inline EncodeTiledFn encode_fn() {
    static EncodeTiledFn fn = nullptr;
    if (!fn) {
        void *p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) != cudaSuccess ||
            q != cudaDriverEntryPointSuccess)
            return nullptr;
        fn = reinterpret_cast<EncodeTiledFn>(p);
    }
    return fn;
}

// 3-D map over B streams of token rows (FP32 or BF16 elements of `esize` bytes): dims (cols,
// T, B), row stride `cols` elements, stream stride T_pad rows; box (box_cols, box_rows, 1),
// dense in shared memory. Rows t >= T of a stream lie outside the map and arrive as zeros
// (the pad guard of the chunked path).
inline int make_rows_map(CUtensorMap *tm, const void *base, CUtensorMapDataType dtype, int esize, int cols, int T,
                         int T_pad, int B, int box_cols, int box_rows) {
    EncodeTiledFn fn = encode_fn();
    if (!fn) return KDA_ERR_CUDA;
    const cuuint64_t dims[3] = {static_cast<cuuint64_t>(cols), static_cast<cuuint64_t>(T), static_cast<cuuint64_t>(B)};
    const cuuint64_t strides[2] = {static_cast<cuuint64_t>(cols) * esize,
                                   static_cast<cuuint64_t>(T_pad) * static_cast<cuuint64_t>(cols) * esize};
    const cuuint32_t box[3] = {static_cast<cuuint32_t>(box_cols), static_cast<cuuint32_t>(box_rows), 1};
    const cuuint32_t estr[3] = {1, 1, 1};
    const CUresult r = fn(tm, dtype, 3, const_cast<void *>(base), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                          CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                          CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS ? KDA_OK : KDA_ERR_INVALID_ARG;
}

// One thread: 3-D tiled TMA load of the box at (x, y, z) into shared memory, completing on
// `bar` (whose expected bytes the caller announced). x * 4 bytes must be a multiple of 16.
__device__ __forceinline__ void tma_load_3d(void *smem_dst, const CUtensorMap *tm, int x, int y, int z,
                                            uint64_t *bar) {
    asm volatile(
        "cp.async.bulk.tensor.3d.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1, {%2, %3, %4}], [%5];" ::
            "r"(umma::smem_u32(smem_dst)),
        "l"(reinterpret_cast<uint64_t>(tm)), "r"(x), "r"(y), "r"(z), "r"(umma::smem_u32(bar))
        : "memory");
}

__device__ __forceinline__ void mbar_expect_tx(uint64_t *bar, uint32_t bytes) {
    asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(umma::smem_u32(bar)), "r"(bytes)
                 : "memory");
}

}  // namespace kda
