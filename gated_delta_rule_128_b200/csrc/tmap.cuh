// Host side: TMA tensor maps for the operator's [B, T, H, D] tensors, encoded
// through the driver entry point (no link against libcuda).
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>

#include <mutex>

namespace gdn2 {

typedef CUresult (*EncodeTiledFn)(CUtensorMap *, CUtensorMapDataType, cuuint32_t, void *,
                                  const cuuint64_t *, const cuuint64_t *, const cuuint32_t *,
                                  const cuuint32_t *, CUtensorMapInterleave, CUtensorMapSwizzle,
                                  CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

inline EncodeTiledFn encode_fn() {
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

// Map of a contiguous [B, T, H, D] tensor whose box is `rows` consecutive
// tokens x `cols` channels (starting at a channel multiple of cols) of one
// (b, h).  Coordinates (innermost first): {channel, h, t, b}.  Rows past T
// read as zero and are not written by stores.  With swizzle128 the box's
// rows (cols x element size = 128 bytes) land in shared memory with their
// 16-byte chunks XOR-ed by (row % 8), the layout of tc.cuh's sw128 tiles.
// Returns false if the driver refuses the map.
inline bool make_btHd_map(CUtensorMap *map, const void *base, bool bf16, int B, int T, int H,
                          int D, int rows, int cols, bool swizzle128 = false) {
    EncodeTiledFn fn = encode_fn();
    if (!fn) return false;
    const cuuint64_t es = bf16 ? 2 : 4;
    cuuint64_t dims[4] = {(cuuint64_t)D, (cuuint64_t)H, (cuuint64_t)T, (cuuint64_t)B};
    cuuint64_t strides[3] = {D * es, (cuuint64_t)H * D * es, (cuuint64_t)T * H * D * es};
    cuuint32_t box[4] = {(cuuint32_t)cols, 1, (cuuint32_t)rows, 1};
    cuuint32_t estr[4] = {1, 1, 1, 1};
    CUresult r = fn(map, bf16 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16 : CU_TENSOR_MAP_DATA_TYPE_FLOAT32,
                    4, const_cast<void *>(base), dims, strides, box, estr,
                    CU_TENSOR_MAP_INTERLEAVE_NONE,
                    swizzle128 ? CU_TENSOR_MAP_SWIZZLE_128B : CU_TENSOR_MAP_SWIZZLE_NONE,
                    CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS;
}

// Map of a contiguous [B, T, H, D] tensor (D = 128 channels) whose one box is
// a whole raw tile: `rows` consecutive tokens x all D channels of one (b, h),
// in the shared-memory layout of `make_btHd_map` boxes of 128-byte channel
// groups (32 float32 or 64 bf16) placed one after another (tc_common.cuh
// raw16 / raw32).  The group is a dimension of its own, outside the tokens:
// dims (innermost first) {group channel, h, t, group, b}, coordinates
// {0, h, t, 0, b}, so one copy replaces one per group.  Rows past T read as
// zero and are not written by stores.  Returns false if the driver refuses
// the map.
inline bool make_wide_map(CUtensorMap *map, const void *base, bool bf16, int B, int T, int H, int D,
                          int rows) {
    EncodeTiledFn fn = encode_fn();
    if (!fn) return false;
    const cuuint64_t es = bf16 ? 2 : 4, gc = 128 / es, ng = D / gc;
    if (ng * gc != (cuuint64_t)D) return false;
    cuuint64_t dims[5] = {gc, (cuuint64_t)H, (cuuint64_t)T, ng, (cuuint64_t)B};
    cuuint64_t strides[4] = {D * es, (cuuint64_t)H * D * es, 128, (cuuint64_t)T * H * D * es};
    cuuint32_t box[5] = {(cuuint32_t)gc, 1, (cuuint32_t)rows, (cuuint32_t)ng, 1};
    cuuint32_t estr[5] = {1, 1, 1, 1, 1};
    CUresult r = fn(map, bf16 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16 : CU_TENSOR_MAP_DATA_TYPE_FLOAT32,
                    5, const_cast<void *>(base), dims, strides, box, estr,
                    CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                    CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS;
}

}  // namespace gdn2
