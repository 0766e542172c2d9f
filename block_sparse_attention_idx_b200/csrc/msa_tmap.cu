// Tensor maps (TMA descriptors) for bf16 tensors, encoded through the driver entry point that the
// runtime exposes, so the library does not link libcuda directly.
#include <cudaTypedefs.h>

#include "msa_internal.h"

namespace msa {

static PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
    static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
    if (!fn) {
        void* p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
    }
    return fn;
}

static CUtensorMapSwizzle swizzle_of(int bytes) {
    switch (bytes) {
        case 128: return CU_TENSOR_MAP_SWIZZLE_128B;
        case 64: return CU_TENSOR_MAP_SWIZZLE_64B;
        case 32: return CU_TENSOR_MAP_SWIZZLE_32B;
        default: return CU_TENSOR_MAP_SWIZZLE_NONE;
    }
}

static bool encode(CUtensorMap* m, const void* base, int rank, const uint64_t* dims, const uint64_t* strides,
                   const uint32_t* box, int swizzle_bytes,
                   CUtensorMapDataType dtype = CU_TENSOR_MAP_DATA_TYPE_BFLOAT16) {
    auto fn = encode_fn();
    if (!fn) return false;
    cuuint32_t estr[5] = {1, 1, 1, 1, 1};
    CUresult r = fn(m, dtype, rank, const_cast<void*>(base),
                    reinterpret_cast<const cuuint64_t*>(dims), reinterpret_cast<const cuuint64_t*>(strides),
                    reinterpret_cast<const cuuint32_t*>(box), estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                    swizzle_of(swizzle_bytes), CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS;
}

bool make_tmap_2d(CUtensorMap* m, const void* base, uint64_t d0, uint64_t d1, uint64_t stride1, uint32_t box0,
                  uint32_t box1, int swizzle_bytes) {
    const uint64_t dims[2] = {d0, d1};
    const uint64_t strides[1] = {stride1};
    const uint32_t box[2] = {box0, box1};
    return encode(m, base, 2, dims, strides, box, swizzle_bytes);
}

bool make_tmap_3d(CUtensorMap* m, const void* base, uint64_t d0, uint64_t d1, uint64_t d2, uint64_t stride1,
                  uint64_t stride2, uint32_t box0, uint32_t box1, uint32_t box2, int swizzle_bytes) {
    const uint64_t dims[3] = {d0, d1, d2};
    const uint64_t strides[2] = {stride1, stride2};
    const uint32_t box[3] = {box0, box1, box2};
    return encode(m, base, 3, dims, strides, box, swizzle_bytes);
}

bool make_tmap_4d(CUtensorMap* m, const void* base, const uint64_t dims[4], const uint64_t strides[3],
                  const uint32_t box[4], int swizzle_bytes) {
    return encode(m, base, 4, dims, strides, box, swizzle_bytes);
}

bool make_tmap_3d_u8(CUtensorMap* m, const void* base, uint64_t d0, uint64_t d1, uint64_t d2, uint64_t stride1,
                     uint64_t stride2, uint32_t box0, uint32_t box1, int swizzle_bytes) {
    const uint64_t dims[3] = {d0, d1, d2};
    const uint64_t strides[2] = {stride1, stride2};
    const uint32_t box[3] = {box0, box1, 1};
    return encode(m, base, 3, dims, strides, box, swizzle_bytes, CU_TENSOR_MAP_DATA_TYPE_UINT8);
}

bool make_tmap_qrows(CUtensorMap* m, const void* q, int B, int N, int H_q, int d, int G) {
    // dims: column within a 64-column half, head within a group of 8, column half, group of 8 heads,
    // query (batch-major); one box = the G heads x d columns of one query in 8-row x 64-column atoms
    const uint64_t dims[5] = {64, 8, (uint64_t)d / 64, (uint64_t)H_q / 8, (uint64_t)B * N};
    const uint64_t strides[4] = {(uint64_t)d * 2, 128, (uint64_t)8 * d * 2, (uint64_t)H_q * d * 2};
    const uint32_t box[5] = {64, 8, (uint32_t)d / 64, (uint32_t)G / 8, 1};
    return encode(m, q, 5, dims, strides, box, 128);
}

}  // namespace msa
