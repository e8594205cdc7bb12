// Paged GQA decode attention on the 5th-generation tensor cores (8 KV heads of dim 128).
//
// Decode attention is the memory-bound operation NanoFlow overlaps with the GEMMs of
// another nano-batch (README "Introduction"; arXiv abstract). For the overlap to pay, the
// attention kernel must pull HBM bandwidth from a minority of the SMs. On B200 an SM completes
// bulk copies at a nearly fixed number per second whatever their size (measured on 16 SMs with a
// ring of copies in flight: 23 GB/s per SM with 8 KB copies, 91 GB/s with 32 KB, 175 GB/s with
// 64 KB). The paged KV cache is therefore laid out so that one page of one layer -- K and V of all
// KV heads, 64 KB -- is a single contiguous block whose bytes are already the shared-memory image
// the tensor cores read:
//   [K|V][64-column half of d][KV head][16 tokens][8 chunks of 16 B, chunk c of row r at c ^ (r & 7)]
// and one bulk copy moves a page into a stage of the page ring.
//
// Split along KV. A request of n pages is cut into ceil(n / chunk_pages) chunks (chunk_pages = 64,
// so contexts above 1024 keys are split) whose page counts
// differ by at most one (chunk c = pages [c n / nch, (c + 1) n / nch)); the cut depends only on the
// request's context length, never on the grid. A work item is one chunk with all heads. Items are dealt to the persistent CTAs in
// contiguous ranges of equal page counts, so a CTA's share differs from the mean by less than
// one chunk. A request of one chunk writes its output directly; the chunks of a longer request
// each write their unnormalised partial (O, running maximum m, sum l per query head) and
// decode_merge_kernel combines them in chunk order. Every rescale factor 2^(m_c - M) is an exact
// power of two (the running maxima are integers), so the result is the same for every grid.
//
// Per page (16 keys x 8 KV heads = 128 rows) one thread issues
//   S^T[128 rows x nq] = K_page Q^T       (A = K, K-major; B = the request's nq query rows)
//   O^T[128 d x nq]   += V_page^T P^T     (A = V read MN-major; B = P, K-major)
// with fp32 accumulators in TMEM. A row (KV head h, key k) of S^T only pairs with the G query
// heads of head h, so P is block diagonal: each softmax thread owns one row, writes its G
// probabilities and leaves the other entries at the zero they were set to once. Per query
// head the running maximum moves only when a score exceeds it by more than 2^8 (O^T is then
// rescaled in TMEM).
#include <cstdint>
#include <cuda.h>
#include <cuda_runtime.h>

#include "nf_attention.h"
#include "nf_decode_body.cuh"
#include "nf_internal.h"
#include "nf_ptx.cuh"

namespace nf {
namespace {

using namespace decode_impl;

template <int NQ>
__global__ void __launch_bounds__(THREADS, 1)
    decode_attention_tc_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ DecodeArgs a) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    __shared__ uint32_t tmem_slot;
    const int warp = threadIdx.x >> 5;
    uint64_t t_start = 0;
    if (threadIdx.x == 0) t_start = globaltimer_ns();
    if (warp == 1) {
        tmem_alloc(&tmem_slot, TcCfg<NQ>::TMEM_COLS);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = tmem_slot;
    decode_body<NQ>(&tmQ, a, smem, tmem, (int)blockIdx.x, (int)gridDim.x);
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem, TcCfg<NQ>::TMEM_COLS);
    }
    if (threadIdx.x == 0 && a.trace != nullptr) {
        const int i = atomicAdd(a.trace_ctr, 1);
        if (i < a.trace_cap) {
            a.trace[i].kernel = NF_KERNEL_DECODE_ATTN;
            a.trace[i].smid = (int32_t)smid();
            a.trace[i].t_start = t_start;
            a.trace[i].t_end = globaltimer_ns();
        }
    }
}

// Warp w of CTA b merges units (request, group of MERGE_HEADS query heads) 8 b + w, 8 (b + grid) + w, ...
constexpr int MERGE_THREADS = 256;

template <int NQ>
__global__ void __launch_bounds__(MERGE_THREADS) decode_merge_kernel(const __grid_constant__ DecodeArgs a) {
    constexpr int NG = NQ / MERGE_HEADS;
    const int units = (a.req_end - a.req_begin) * NG;
    const int wpc = MERGE_THREADS / 32;
    for (int u = blockIdx.x * wpc + (threadIdx.x >> 5); u < units; u += gridDim.x * wpc)
        merge_heads_warp<NQ>(a, a.req_begin + u / NG, (u % NG) * MERGE_HEADS, threadIdx.x & 31);
}

template <int NQ>
cudaError_t launch_nq(const CUtensorMap& tmQ, const DecodeArgs& a, int grid, cudaStream_t stream) {
    static bool cfg = false;
    if (!cfg) {
        cudaError_t e = cudaFuncSetAttribute(decode_attention_tc_kernel<NQ>,
                                             cudaFuncAttributeMaxDynamicSharedMemorySize, (int)TcCfg<NQ>::SMEM);
        if (e != cudaSuccess) return e;
        cfg = true;
    }
    decode_attention_tc_kernel<NQ><<<grid, THREADS, TcCfg<NQ>::SMEM, stream>>>(tmQ, a);
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess || a.split_pages >= kDecodeNoSplit || !a.any_split) return e;
    const int units = (a.req_end - a.req_begin) * (NQ / MERGE_HEADS);
    const int blocks = (units + MERGE_THREADS / 32 - 1) / (MERGE_THREADS / 32);
    decode_merge_kernel<NQ><<<blocks < 2048 ? blocks : 2048, MERGE_THREADS, 0, stream>>>(a);
    return cudaGetLastError();
}

// Page prefix (item_off) and chunk prefix (chunk_off, optional) of requests [0, R): request r has
// ceil((ctx + 1) / 16) pages in ceil(pages / split_pages) chunks. A negative context length is
// recorded as NF_ERR_DEVICE_BOUNDS and read as 0.
__global__ void decode_tc_schedule_kernel(const int* ctx_len, int R, int split_pages, int* item_off, int* chunk_off,
                                          int* status) {
    __shared__ long long carry[2];
    __shared__ int warp_sums[2][32];
    if (threadIdx.x < 2) carry[threadIdx.x] = 0;
    __syncthreads();
    const int lane = threadIdx.x & 31, w = threadIdx.x >> 5, nw = blockDim.x >> 5;
    for (int base = 0; base < R; base += blockDim.x) {
        const int r = base + threadIdx.x;
        int v[2] = {0, 0};
        if (r < R) {
            int c = ctx_len[r];
            if (c < 0) { set_status(status, NF_ERR_DEVICE_BOUNDS); c = 0; }
            v[0] = (c + 1 + 15) >> 4;
            v[1] = ceil_div(v[0], split_pages);
        }
        int incl[2];
#pragma unroll
        for (int k = 0; k < 2; ++k) {
            int x = v[k];
#pragma unroll
            for (int o = 1; o < 32; o <<= 1) {
                const int y = __shfl_up_sync(0xffffffffu, x, o);
                if (lane >= o) x += y;
            }
            if (lane == 31) warp_sums[k][w] = x;
            incl[k] = x;
        }
        __syncthreads();
        if (w == 0) {
#pragma unroll
            for (int k = 0; k < 2; ++k) {
                int s = lane < nw ? warp_sums[k][lane] : 0;
#pragma unroll
                for (int o = 1; o < 32; o <<= 1) {
                    const int y = __shfl_up_sync(0xffffffffu, s, o);
                    if (lane >= o) s += y;
                }
                if (lane < nw) warp_sums[k][lane] = s;
            }
        }
        __syncthreads();
#pragma unroll
        for (int k = 0; k < 2; ++k) incl[k] += (w > 0 ? warp_sums[k][w - 1] : 0);
        if (r < R) {
            item_off[r] = (int)(carry[0] + incl[0] - v[0]);
            if (chunk_off) chunk_off[r] = (int)(carry[1] + incl[1] - v[1]);
        }
        __syncthreads();
        if (threadIdx.x == blockDim.x - 1) { carry[0] += incl[0]; carry[1] += incl[1]; }
        __syncthreads();
    }
    if (threadIdx.x == 0) {
        item_off[R] = (int)carry[0];
        if (chunk_off) chunk_off[R] = (int)carry[1];
    }
}

}  // namespace

bool decode_tc_supported(int nq, int nkv, int head_dim) {
    return head_dim == 128 && nkv == 8 && (nq == 32 || nq == 64);
}

cudaError_t launch_decode_tc_schedule(const int* ctx_len, int R, int split_pages, int* item_off, int* chunk_off,
                                      int* status, cudaStream_t stream) {
    if (R <= 0) return cudaSuccess;
    decode_tc_schedule_kernel<<<1, 1024, 0, stream>>>(ctx_len, R, split_pages, item_off, chunk_off, status);
    return cudaGetLastError();
}

cudaError_t launch_decode_attention_tc(const CUtensorMap& tmQ, const DecodeArgs& a, int grid, cudaStream_t stream) {
    if (grid <= 0 || a.req_end <= a.req_begin) return cudaSuccess;
    if (a.nq == 32) return launch_nq<32>(tmQ, a, grid, stream);
    if (a.nq == 64) return launch_nq<64>(tmQ, a, grid, stream);
    return cudaErrorInvalidValue;
}

}  // namespace nf
