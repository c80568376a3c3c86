// tmap.cuh — TMA tensor maps: the driver's encoder (fetched at run time, so
// the library links against the runtime only) and the tiled-load instructions.
#pragma once

#include <cuda.h>   // CUtensorMap types
#include <cuda_runtime.h>

#include <cstdint>

#include "sync.cuh"

namespace moe {

typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                  const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

// cuTensorMapEncodeTiled, or nullptr if the driver does not provide it.
inline EncodeTiledFn encode_tiled() {
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

// A tensor of 8-byte words [slots][rows][row_bytes / 8] (row_bytes and
// slot_stride multiples of 16), loaded in boxes of box_bytes x box_rows with
// no swizzle: smem rows of box_bytes.  A box wider than the row reads zeros
// past the row's end, so box_bytes > row_bytes stages padded rows.
inline bool padded_rows_map(CUtensorMap* m, const void* base, uint64_t row_bytes, uint64_t rows, uint64_t slots,
                            uint64_t slot_stride, uint32_t box_bytes, uint32_t box_rows) {
    EncodeTiledFn fn = encode_tiled();
    if (!fn || row_bytes % 16 || slot_stride % 16 || box_bytes % 16 || box_bytes / 8 > 256 || box_rows > 256)
        return false;
    const cuuint64_t dims[3] = {row_bytes / 8, rows, slots};
    const cuuint64_t strides[2] = {row_bytes, slot_stride};
    const cuuint32_t box[3] = {box_bytes / 8, box_rows, 1};
    const cuuint32_t es[3] = {1, 1, 1};
    return fn(m, CU_TENSOR_MAP_DATA_TYPE_UINT64, 3, const_cast<void*>(base), dims, strides, box, es,
              CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
              CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// Tiled 3-D box load into shared memory (dst 128-byte aligned), completing
// the box's bytes on bar.
MOE_DEVINL void tma_box_3d(void* dst, const CUtensorMap* map, int x, int y, int z, uint64_t* bar) {
    asm volatile(
        "cp.async.bulk.tensor.3d.shared::cluster.global.tile.mbarrier::complete_tx::bytes [%0], [%1, {%2, %3, %4}], "
        "[%5];" ::"r"(smem_u32(dst)),
        "l"(map), "r"(x), "r"(y), "r"(z), "r"(smem_u32(bar))
        : "memory");
}

}  // namespace moe
