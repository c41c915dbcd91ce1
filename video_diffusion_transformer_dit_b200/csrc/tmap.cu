// TMA tensor-map construction (host).  The driver entry point is fetched
// through the runtime so the library needs no link against libcuda.
#include <cudaTypedefs.h>

#include <mutex>

#include "kernels.h"

namespace wan {

static PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
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

// 2-D bf16 tensor [outer][inner] with row stride ld_elems, box box_outer x
// box_inner (box_inner * 2 bytes must be 128 for the 128-byte swizzle),
// out-of-range elements read as zero.
bool make_tmap_2d(CUtensorMap* m, const void* ptr, uint64_t inner, uint64_t outer, uint64_t ld_elems,
                  uint32_t box_inner, uint32_t box_outer) {
    auto fn = encode_fn();
    if (!fn) return false;
    cuuint64_t dims[2] = {inner, outer};
    cuuint64_t strides[1] = {ld_elems * 2};
    cuuint32_t box[2] = {box_inner, box_outer};
    cuuint32_t estr[2] = {1, 1};
    CUresult r = fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(ptr), dims, strides, box, estr,
                    CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                    CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS;
}

// 3-D bf16 tensor [d2][d1][inner] (strides ld1, ld2 in elements), box
// 1 x box1 x box_inner; rows past d1 inside a batch read as zero.
bool make_tmap_3d(CUtensorMap* m, const void* ptr, uint64_t inner, uint64_t d1, uint64_t d2, uint64_t ld1_elems,
                  uint64_t ld2_elems, uint32_t box_inner, uint32_t box1) {
    auto fn = encode_fn();
    if (!fn) return false;
    cuuint64_t dims[3] = {inner, d1, d2};
    cuuint64_t strides[2] = {ld1_elems * 2, ld2_elems * 2};
    cuuint32_t box[3] = {box_inner, box1, 1};
    cuuint32_t estr[3] = {1, 1, 1};
    CUresult r = fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(ptr), dims, strides, box, estr,
                    CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                    CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS;
}

// 5-D bf16 tensor [d4][d3][d2][d1][inner] (channels-last video: inner = channels,
// d1 = width, d2 = height, d3 = frames, d4 = batch), strides in elements, box
// 1 x 1 x box2 x box1 x box_inner; coordinates outside the tensor (negative
// included) read as zero.
bool make_tmap_5d(CUtensorMap* m, const void* ptr, const uint64_t (&dims)[5], const uint64_t (&strides_elems)[4],
                  uint32_t box_inner, uint32_t box1, uint32_t box2) {
    auto fn = encode_fn();
    if (!fn) return false;
    cuuint64_t d[5], st[4];
    for (int i = 0; i < 5; ++i) d[i] = dims[i];
    for (int i = 0; i < 4; ++i) st[i] = strides_elems[i] * 2;
    cuuint32_t box[5] = {box_inner, box1, box2, 1, 1};
    cuuint32_t estr[5] = {1, 1, 1, 1, 1};
    CUresult r = fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 5, const_cast<void*>(ptr), d, st, box, estr,
                    CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                    CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS;
}

}  // namespace wan
