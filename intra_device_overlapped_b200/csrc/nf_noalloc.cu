// Decode attention that allocates nothing (entry point nf_decode_attention_noalloc).
//
// For callers that cannot allocate device memory at the point of the call (code running
// between the capture calls of a CUDA graph, an allocator-free runtime, a process that has
// handed all device memory to its own pool): they cannot create an nf_model, whose
// workspace comes from cudaMalloc. This entry point runs the tensor-core decode attention of
// the serving iteration from plain device pointers. Its only scratch -- the per-request
// prefix of page counts that deals the requests to the persistent CTAs -- lives in the
// file-scope array below, so the call makes no cudaMalloc, cudaFree or allocating library
// call. Requests are not split along their keys here (split partials would need scratch
// proportional to the batch), so each request is one work item.
//
// Every call on a device shares that one array: two calls that overlap on the GPU (on
// different streams, or from different host threads) race on it and may produce wrong
// output. Serialise them.
#include <new>
#include <cmath>
#include <cstdint>
#include <cstring>
#include <mutex>

#include <cuda.h>
#include <cuda_runtime.h>

#include "nanoflow.h"
#include "nf_attention.h"
#include "nf_internal.h"

namespace {

// Scratch layout: item_off, NF_NOALLOC_MAX_REQUESTS + 1 ints, written in full by the schedule
// kernel before the attention kernel reads them; then the work-item claim counter, zeroed before each
// launch.
constexpr size_t kScratchBytes = 4 * (size_t)(NF_NOALLOC_MAX_REQUESTS + 64);
static_assert(kScratchBytes % 256 == 0, "scratch size");

__device__ __align__(256) unsigned char g_noalloc_scratch[kScratchBytes];

constexpr int kMaxDevices = 64;
std::mutex g_setup_mu;
void* g_scratch_ptr[kMaxDevices] = {};

// Device address of the scratch array on the current device, looked up once per device (and kept
// for the life of the process: after cudaDeviceReset the cached address is stale).
nf_status scratch_for_current_device(unsigned char** out) {
    int dev = -1;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return NF_ERR_CUDA;
    std::lock_guard<std::mutex> lock(g_setup_mu);
    if (g_scratch_ptr[dev] == nullptr) {
        void* p = nullptr;
        const cudaError_t e = cudaGetSymbolAddress(&p, g_noalloc_scratch);
        if (e != cudaSuccess || p == nullptr) return NF_ERR_CUDA;
        g_scratch_ptr[dev] = p;
    }
    *out = static_cast<unsigned char*>(g_scratch_ptr[dev]);
    return NF_OK;
}

}  // namespace

extern "C" nf_status nf_decode_attention_noalloc(const void* q, void* out, const void* kv_pool, int32_t num_pages,
                                                 const int32_t* ctx_len, const int32_t* page_indptr,
                                                 const int32_t* page_indices, int32_t num_requests,
                                                 int32_t n_q_heads, int32_t n_kv_heads, int32_t head_dim,
                                                 int32_t sm_count, int32_t* status_device, void* stream) try {
    if (!q || !out || !kv_pool || !ctx_len || !page_indptr || !page_indices || !status_device)
        return NF_ERR_INVALID_ARGUMENT;
    if (num_pages <= 0 || num_requests < 0 || sm_count < 0) return NF_ERR_INVALID_ARGUMENT;
    if (num_requests > NF_NOALLOC_MAX_REQUESTS) return NF_ERR_INVALID_ARGUMENT;  // scratch holds at most this many
    if (!nf::decode_tc_supported(n_q_heads, n_kv_heads, head_dim)) return NF_ERR_UNSUPPORTED;
    if (num_requests == 0) return NF_OK;

    unsigned char* scratch = nullptr;
    nf_status st = scratch_for_current_device(&scratch);
    if (st != NF_OK) return st;
    int* status = status_device;
    int* item_off = reinterpret_cast<int*>(scratch);
    int* claim = item_off + NF_NOALLOC_MAX_REQUESTS + 1;

    int dev = 0, sms = 0;
    if (cudaGetDevice(&dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || sms <= 0)
        return NF_ERR_CUDA;
    const int grid = sm_count > 0 ? (sm_count < sms ? sm_count : sms) : sms;

    CUtensorMap tmq;
    if (!nf::make_tmap_bf16_2d(&tmq, q, (uint64_t)num_requests * n_q_heads, (uint64_t)head_dim,
                               (uint32_t)n_q_heads))
        return NF_ERR_INVALID_ARGUMENT;

    cudaStream_t s = static_cast<cudaStream_t>(stream);
    if (nf::launch_decode_tc_schedule(ctx_len, num_requests, nf::kDecodeNoSplit, item_off, nullptr, status, s) !=
        cudaSuccess)
        return NF_ERR_CUDA;
    if (cudaMemsetAsync(claim, 0, sizeof(int), s) != cudaSuccess) return NF_ERR_CUDA;

    nf::DecodeArgs a;
    std::memset(&a, 0, sizeof(a));
    a.q = static_cast<const uint16_t*>(q);
    a.out = static_cast<uint16_t*>(out);
    a.ctx_len = ctx_len;
    a.page_indptr = page_indptr;
    a.page_indices = page_indices;
    a.item_off = item_off;
    a.kv_pool = static_cast<const uint16_t*>(kv_pool);
    a.req_begin = 0;
    a.req_end = num_requests;
    a.nq = n_q_heads;
    a.nkv = n_kv_heads;
    a.G = n_q_heads / n_kv_heads;
    a.num_pages = num_pages;
    a.split_pages = nf::kDecodeNoSplit;
    a.scale_log2 = (float)(1.4426950408889634 / std::sqrt((double)head_dim));
    a.status = status;
    a.claim_ctr = claim;
    if (nf::launch_decode_attention_tc(tmq, a, grid, s) != cudaSuccess) return NF_ERR_CUDA;
    return NF_OK;
} catch (const std::bad_alloc&) {
    return NF_ERR_OUT_OF_MEMORY;
} catch (...) {
    return NF_ERR_INVALID_ARGUMENT;
}
