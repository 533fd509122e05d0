// Host side of the TMA (tensor memory accelerator) tile loads: tensor maps over
// the [rows, H, d] bf16 input tensors, encoded with the driver's
// cuTensorMapEncodeTiled (looked up once through the runtime, so the library
// does not link libcuda directly).  The device side is sm100::tma_load_3d.
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include <mutex>

namespace kda {

using EncodeTiledFn = CUresult (*)(CUtensorMap *, CUtensorMapDataType, cuuint32_t, void *,
                                   const cuuint64_t *, const cuuint64_t *, const cuuint32_t *,
                                   const cuuint32_t *, CUtensorMapInterleave, CUtensorMapSwizzle,
                                   CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

inline EncodeTiledFn encode_tiled_fn() {
    static EncodeTiledFn fn = nullptr;
    static std::once_flag once;
    std::call_once(once, [] {
        void *p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) ==
                cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<EncodeTiledFn>(p);
    });
    return fn;
}

// A tensor map over a row-major bf16 tensor [rows, H, d] whose tiles are
// `box_rows` consecutive rows (tokens) of `box_cols` consecutive channels of one
// head: coordinates (channel, head, row).  The box lands in shared memory as
// box_rows lines of box_cols * 2 bytes with the given swizzle (the line length
// must equal the swizzle span: 128 B for SWIZZLE_128B, 64 B for SWIZZLE_64B).
// Rows past `rows` read as zero.  Returns false when the driver rejects the map
// (a base address that is not 16-byte aligned, for instance).
inline bool make_rows_heads_tmap(CUtensorMap *map, const void *base, int64_t rows, int H, int d,
                                 int box_cols, int box_rows, CUtensorMapSwizzle swizzle) {
    EncodeTiledFn fn = encode_tiled_fn();
    if (!fn || !base || rows <= 0) return false;
    if ((reinterpret_cast<uintptr_t>(base) & 15u) != 0) return false;
    const cuuint64_t dims[3] = {(cuuint64_t)d, (cuuint64_t)H, (cuuint64_t)rows};
    const cuuint64_t strides[2] = {(cuuint64_t)d * 2, (cuuint64_t)H * d * 2};   // bytes, dims 1..2
    const cuuint32_t box[3] = {(cuuint32_t)box_cols, 1u, (cuuint32_t)box_rows};
    const cuuint32_t estride[3] = {1u, 1u, 1u};
    return fn(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void *>(base), dims, strides, box,
              estride, CU_TENSOR_MAP_INTERLEAVE_NONE, swizzle, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
              CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

}  // namespace kda
