// Causal attention of the prefill chunk on the 5th-generation tensor cores (head dim 128).
//
// The prefill chunk is the compute-bound part of attention in a NanoFlow iteration; it runs
// beside the GEMMs (README "Introduction"). Work unit = 128 consecutive query positions of one
// query head. For each key tile of 128 keys (8 pages of the chunk) one thread issues
//   S[128 q x 128 k]  = Q K^T        (A = Q, B = K, both K-major)
//   O[128 q x 128 d] += P V          (A = P from shared memory, B = V read MN-major)
// with fp32 accumulators in TMEM. Each softmax thread owns one query row (one TMEM lane), so
// the running maximum, the row sum and the lazy rescale of its O row (only when the maximum
// grows by more than 2^8) need no communication between threads.
//
// K and V of a key tile are gathered from the paged pool: in the page layout each (K|V, half of
// d, KV head) block of a page is 16 rows of 128 bytes already in the 128-byte-swizzled order, so
// eight 2 KB bulk copies per half build a [128 keys x 64 d] operand tile directly. Keys past the
// chunk (in the last page, or pages the chunk does not have) get zero V rows; their scores are
// masked by causality.
#include <cstdint>
#include <cuda.h>
#include <cuda_runtime.h>

#include "nf_attention.h"
#include "nf_prefill_body.cuh"
#include "nf_internal.h"
#include "nf_ptx.cuh"

namespace nf {
namespace {

using namespace prefill_impl;

__global__ void __launch_bounds__(THREADS, 1)
    prefill_attention_tc_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ PrefillArgs a) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    __shared__ uint32_t tmem_slot;
    const int warp = threadIdx.x >> 5;
    uint64_t t_start = 0;
    if (threadIdx.x == 0) t_start = globaltimer_ns();
    if (warp == 1) {
        tmem_alloc(&tmem_slot, TMEM_COLS);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = tmem_slot;
    prefill_body(&tmQ, a, smem, tmem, (int)blockIdx.x, (int)gridDim.x);
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem, TMEM_COLS);
    }
    if (threadIdx.x == 0 && a.trace != nullptr) {
        const int i = atomicAdd(a.trace_ctr, 1);
        if (i < a.trace_cap) {
            a.trace[i].kernel = NF_KERNEL_PREFILL_ATTN;
            a.trace[i].smid = (int32_t)smid();
            a.trace[i].t_start = t_start;
            a.trace[i].t_end = globaltimer_ns();
        }
    }
}

}  // namespace

bool prefill_tc_supported(int head_dim) { return head_dim == 128; }

cudaError_t launch_prefill_attention_tc(const CUtensorMap& tmQ, const PrefillArgs& a, int grid, cudaStream_t stream) {
    if (grid <= 0 || a.prefill_len <= 0) return cudaSuccess;
    static bool cfg = false;
    if (!cfg) {
        cudaError_t e = cudaFuncSetAttribute(prefill_attention_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                             (int)SMEM);
        if (e != cudaSuccess) return e;
        cfg = true;
    }
    const int units = ((a.prefill_len + ROWS - 1) / ROWS) * a.nq;
    if (grid > units) grid = units;
    prefill_attention_tc_kernel<<<grid, THREADS, SMEM, stream>>>(tmQ, a);
    return cudaGetLastError();
}

}  // namespace nf
