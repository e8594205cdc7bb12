// Host helpers: TMA tensor-map encoding (driver entry point fetched at run time so the
// library loads on machines without a driver) and device queries.
#include <cstdint>
#include <cstring>
#include <cuda.h>
#include <cuda_runtime.h>
#include <cudaTypedefs.h>

#include "nf_internal.h"

namespace nf {

namespace {
PFN_cuTensorMapEncodeTiled_v12000 lookup_encode_fn() {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
        return reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
    return nullptr;
}

// Looked up once; a function-local static is initialised exactly once even when several host
// threads make their first call at the same time.
PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
    static const PFN_cuTensorMapEncodeTiled_v12000 fn = lookup_encode_fn();
    return fn;
}
}  // namespace

bool make_tmap_bf16_2d(CUtensorMap* map, const void* base, uint64_t rows, uint64_t cols, uint32_t box_rows) {
    std::memset(map, 0, sizeof(*map));
    auto fn = encode_fn();
    if (fn == nullptr || base == nullptr || rows == 0 || cols == 0) return false;
    if ((reinterpret_cast<uintptr_t>(base) & 15u) != 0 || (cols * 2) % 16 != 0) return false;
    cuuint64_t dims[2] = {cols, rows};
    cuuint64_t strides[1] = {cols * 2};
    cuuint32_t box[2] = {64, box_rows};
    cuuint32_t estr[2] = {1, 1};
    CUresult r = fn(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides, box, estr,
                    CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                    CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS;
}

bool make_tmap_bf16_3d_heads(CUtensorMap* map, const void* base, uint64_t tokens, uint64_t heads, uint64_t head_dim,
                             uint32_t box_tokens) {
    std::memset(map, 0, sizeof(*map));
    auto fn = encode_fn();
    if (fn == nullptr || base == nullptr || tokens == 0 || heads == 0 || head_dim == 0) return false;
    if ((reinterpret_cast<uintptr_t>(base) & 15u) != 0 || (head_dim * 2) % 16 != 0) return false;
    cuuint64_t dims[3] = {head_dim, heads, tokens};
    cuuint64_t strides[2] = {head_dim * 2, heads * head_dim * 2};
    cuuint32_t box[3] = {64, 1, box_tokens};
    cuuint32_t estr[3] = {1, 1, 1};
    CUresult r = fn(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(base), dims, strides, box, estr,
                    CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                    CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS;
}

int device_sm_count() {
    int dev = 0, sms = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return 0;
    if (cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) return 0;
    return sms;
}

}  // namespace nf
