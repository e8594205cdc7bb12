// Mixture-of-experts pieces of a Mixtral-style layer (arXiv abstract: Mixtral 8x7B is
// one of the evaluated models): router logits + top-k + softmax over the selected
// logits, a stable counting sort of the (token, k) assignments by expert, the row
// gather that feeds the grouped expert GEMMs, and the weighted combine + residual.
#include <cstdint>
#include <cuda_runtime.h>

#include "nf_misc.h"
#include "nf_ptx.cuh"

namespace nf {
namespace {

constexpr int kMaxExperts = 16;
constexpr int kSortThreads = 1024;

__device__ __forceinline__ float warp_sum(float x) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) x += __shfl_xor_sync(0xffffffffu, x, o);
    return x;
}

// One warp per token: z[e] = rs * <h, Wr'[e]> + b[e] in fp32 from the fp32 residual,
// top-k by value (ties: lower expert index), weights = softmax over the k selected logits.
__global__ void moe_route_kernel(const MoeArgs a) {
    const int lane = threadIdx.x & 31;
    const int warps = (gridDim.x * blockDim.x) >> 5;
    for (int r = (blockIdx.x * blockDim.x + threadIdx.x) >> 5; r < a.rows; r += warps) {
        const int t = a.tok0 + r;
        const float* h = a.resid + (size_t)t * a.H;
        float acc[kMaxExperts];
#pragma unroll
        for (int e = 0; e < kMaxExperts; ++e) acc[e] = 0.f;
        for (int k = lane; k < a.H; k += 32) {
            const float x = h[k];
#pragma unroll
            for (int e = 0; e < kMaxExperts; ++e)
                if (e < a.E) acc[e] += x * a.router[(size_t)e * a.H + k];
        }
        float ss = 0.f;
        for (int j = lane; j < a.n_part; j += 32) ss += a.partials[(size_t)t * a.n_part + j];
        ss = warp_sum(ss);
        const float rs = rsqrtf(ss * a.inv_dim + a.eps);
        float z[kMaxExperts];
#pragma unroll
        for (int e = 0; e < kMaxExperts; ++e) z[e] = warp_sum(acc[e]) * rs + (e < a.E ? a.router_bias[e] : 0.f);
        if (lane == 0) {
            bool taken[kMaxExperts];
#pragma unroll
            for (int e = 0; e < kMaxExperts; ++e) taken[e] = false;
            float sel[kMaxExperts];
            int idx[kMaxExperts];
            for (int k = 0; k < a.K; ++k) {
                int best = -1;
                for (int e = 0; e < a.E; ++e)
                    if (!taken[e] && (best < 0 || z[e] > z[best])) best = e;
                taken[best] = true;
                idx[k] = best;
                sel[k] = z[best];
            }
            float den = 0.f;
            for (int k = 0; k < a.K; ++k) den += __expf(sel[k] - sel[0]);
            for (int k = 0; k < a.K; ++k) {
                const float w = __expf(sel[k] - sel[0]) / den;
                a.topk_idx[(size_t)r * a.K + k] = idx[k];
                a.topk_w[(size_t)r * a.K + k] = w;
                if (a.dbg_idx) a.dbg_idx[(size_t)r * a.K + k] = idx[k];
                if (a.dbg_w) a.dbg_w[(size_t)r * a.K + k] = w;
            }
            if (a.dbg_logits)
                for (int e = 0; e < a.E; ++e) a.dbg_logits[(size_t)r * a.E + e] = z[e];
        }
    }
}

// Stable counting sort of assignments a = r*K + k by expert (single CTA).
// counts[e] = first sorted slot of expert e, counts[E] = total; perm[slot] = a; inv[a] = slot.
__global__ void __launch_bounds__(kSortThreads) moe_sort_kernel(const MoeArgs a) {
    extern __shared__ int sh[];  // [kSortThreads][E] per-thread counts, then [E+1] offsets
    const int E = a.E;
    const int n = a.rows * a.K;
    const int tid = threadIdx.x;
    const int per = (n + kSortThreads - 1) / kSortThreads;
    const int c0 = min(n, tid * per), c1 = min(n, c0 + per);
    int* cnt = sh + tid * E;
    for (int e = 0; e < E; ++e) cnt[e] = 0;
    for (int i = c0; i < c1; ++i) cnt[a.topk_idx[i]]++;
    __syncthreads();
    int* off = sh + kSortThreads * E;
    if (tid < E) {  // exclusive prefix of expert `tid` over threads, in thread order
        int run = 0;
        for (int t = 0; t < kSortThreads; ++t) {
            const int c = sh[t * E + tid];
            sh[t * E + tid] = run;
            run += c;
        }
        off[tid] = run;  // total of expert tid (turned into offsets below)
    }
    __syncthreads();
    if (tid == 0) {
        int run = 0;
        for (int e = 0; e < E; ++e) {
            const int c = off[e];
            off[e] = run;
            a.counts[e] = run;
            run += c;
        }
        off[E] = run;
        a.counts[E] = run;
    }
    __syncthreads();
    for (int i = c0; i < c1; ++i) {
        const int e = a.topk_idx[i];
        const int slot = off[e] + cnt[e]++;
        a.perm[slot] = i;
        a.inv[i] = slot;
    }
}

__global__ void moe_gather_kernel(const MoeArgs a) {
    const int per_row = a.H / 8;
    const int n = a.rows * a.K;
    for (int i = blockIdx.x * blockDim.x + threadIdx.x; i < n * per_row; i += gridDim.x * blockDim.x) {
        const int slot = i / per_row, c = i - slot * per_row;
        const int t = a.tok0 + a.perm[slot] / a.K;
        reinterpret_cast<uint4*>(a.a_sorted + (size_t)slot * a.H)[c] =
            reinterpret_cast<const uint4*>(a.xb + (size_t)t * a.H)[c];
        if (c < a.n_part) a.part_sorted[(size_t)slot * a.n_part + c] = a.partials[(size_t)t * a.n_part + c];
    }
}

// x' = h + sum_k w_k y[slot(t, k)] (k ascending), with bf16 copy and per-segment sums of squares.
__global__ void moe_combine_kernel(const MoeArgs a) {
    const int lane = threadIdx.x & 31;
    const int nseg = a.H / 256;
    const int warps = (gridDim.x * blockDim.x) >> 5;
    for (int w = (blockIdx.x * blockDim.x + threadIdx.x) >> 5; w < a.rows * nseg; w += warps) {
        const int r = w / nseg, seg = w - r * nseg;
        const int t = a.tok0 + r;
        const int c = seg * 256 + lane * 8;
        float v[8];
        const float4* h4 = reinterpret_cast<const float4*>(a.resid + (size_t)t * a.H + c);
        const float4 h0 = h4[0], h1 = h4[1];
        v[0] = h0.x; v[1] = h0.y; v[2] = h0.z; v[3] = h0.w; v[4] = h1.x; v[5] = h1.y; v[6] = h1.z; v[7] = h1.w;
        for (int k = 0; k < a.K; ++k) {
            const float wk = a.topk_w[(size_t)r * a.K + k];
            const int slot = a.inv[r * a.K + k];
            const float4* y4 = reinterpret_cast<const float4*>(a.y_sorted + (size_t)slot * a.H + c);
            const float4 y0 = y4[0], y1 = y4[1];
            v[0] += wk * y0.x; v[1] += wk * y0.y; v[2] += wk * y0.z; v[3] += wk * y0.w;
            v[4] += wk * y1.x; v[5] += wk * y1.y; v[6] += wk * y1.z; v[7] += wk * y1.w;
        }
        float ss = 0.f;
#pragma unroll
        for (int i = 0; i < 8; ++i) ss += v[i] * v[i];
        float4* o4 = reinterpret_cast<float4*>(a.resid_out + (size_t)t * a.H + c);
        o4[0] = make_float4(v[0], v[1], v[2], v[3]);
        o4[1] = make_float4(v[4], v[5], v[6], v[7]);
        if (a.out_f32) {
            float4* f4 = reinterpret_cast<float4*>(a.out_f32 + (size_t)t * a.H + c);
            f4[0] = make_float4(v[0], v[1], v[2], v[3]);
            f4[1] = make_float4(v[4], v[5], v[6], v[7]);
        }
        uint4 b;
        b.x = pack_bf16x2(v[0], v[1]); b.y = pack_bf16x2(v[2], v[3]);
        b.z = pack_bf16x2(v[4], v[5]); b.w = pack_bf16x2(v[6], v[7]);
        *reinterpret_cast<uint4*>(a.xb_out + (size_t)t * a.H + c) = b;
        ss = warp_sum(ss);
        if (lane == 0) a.partials_out[(size_t)t * nseg + seg] = ss;
    }
}

int blocks_for(size_t work, int per_block, int max_blocks) {
    size_t g = (work + per_block - 1) / per_block;
    if (g < 1) g = 1;
    if (g > (size_t)max_blocks) g = max_blocks;
    return (int)g;
}

}  // namespace

cudaError_t launch_moe_route(const MoeArgs& a, int max_blocks, cudaStream_t s) {
    if (a.rows <= 0) return cudaSuccess;
    if (a.E > kMaxExperts || a.K > a.E || a.K < 1) return cudaErrorInvalidValue;
    moe_route_kernel<<<blocks_for((size_t)a.rows, 8, max_blocks), 256, 0, s>>>(a);
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return e;
    const int smem = (kSortThreads * a.E + a.E + 1) * (int)sizeof(int);
    static bool cfg = false;
    if (!cfg) {
        e = cudaFuncSetAttribute(moe_sort_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 (kSortThreads * kMaxExperts + kMaxExperts + 1) * (int)sizeof(int));
        if (e != cudaSuccess) return e;
        cfg = true;
    }
    moe_sort_kernel<<<1, kSortThreads, smem, s>>>(a);
    return cudaGetLastError();
}

cudaError_t launch_moe_gather(const MoeArgs& a, int max_blocks, cudaStream_t s) {
    if (a.rows <= 0) return cudaSuccess;
    moe_gather_kernel<<<blocks_for((size_t)a.rows * a.K * (a.H / 8), 256, max_blocks), 256, 0, s>>>(a);
    return cudaGetLastError();
}

cudaError_t launch_moe_combine(const MoeArgs& a, int max_blocks, cudaStream_t s) {
    if (a.rows <= 0) return cudaSuccess;
    moe_combine_kernel<<<blocks_for((size_t)a.rows * (a.H / 256), 8, max_blocks), 256, 0, s>>>(a);
    return cudaGetLastError();
}

}  // namespace nf
