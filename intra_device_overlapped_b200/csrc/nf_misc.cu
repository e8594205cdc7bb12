// Small kernels around the GEMMs and attention: residual-stream set-up (input hidden
// or token embedding), LM-head row gather, argmax reduction, weight repacking, and a
// bounded device wait used to test the timeout path.
#include <cstdint>
#include <cuda_runtime.h>

#include "nf_misc.h"
#include "nf_ptx.cuh"

namespace nf {
namespace {

__device__ __forceinline__ float warp_sum(float x) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) x += __shfl_xor_sync(0xffffffffu, x, o);
    return x;
}

// One warp per (row, 256-column segment): fp32 residual, bf16 copy and the segment's sum of squares.
__device__ __forceinline__ void residual_segment(const uint16_t* src, int row_out, int seg, int H, float* resid,
                                                 uint16_t* xb, float* partials, int lane) {
    const int c = seg * 256 + lane * 8;
    const uint4 w = *reinterpret_cast<const uint4*>(src + c);
    const uint32_t ws[4] = {w.x, w.y, w.z, w.w};
    float v[8];
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        v[2 * i] = __uint_as_float(ws[i] << 16);
        v[2 * i + 1] = __uint_as_float(ws[i] & 0xFFFF0000u);
    }
    float ss = 0.f;
#pragma unroll
    for (int i = 0; i < 8; ++i) ss += v[i] * v[i];
    float4* r4 = reinterpret_cast<float4*>(resid + (size_t)row_out * H + c);
    r4[0] = make_float4(v[0], v[1], v[2], v[3]);
    r4[1] = make_float4(v[4], v[5], v[6], v[7]);
    *reinterpret_cast<uint4*>(xb + (size_t)row_out * H + c) = w;
    ss = warp_sum(ss);
    if (lane == 0) partials[(size_t)row_out * (H / 256) + seg] = ss;
}

__global__ void prep_hidden_kernel(const uint16_t* __restrict__ in, int T, int H, float* resid, uint16_t* xb,
                                   float* partials) {
    const int lane = threadIdx.x & 31;
    const int nseg = H / 256;
    const int warps = (gridDim.x * blockDim.x) >> 5;
    for (int w = (blockIdx.x * blockDim.x + threadIdx.x) >> 5; w < T * nseg; w += warps) {
        const int row = w / nseg, seg = w - row * nseg;
        residual_segment(in + (size_t)row * H, row, seg, H, resid, xb, partials, lane);
    }
}

__global__ void embed_kernel(const int* __restrict__ tokens, const uint16_t* __restrict__ table, int T, int H,
                             int V, float* resid, uint16_t* xb, float* partials, int* status) {
    const int lane = threadIdx.x & 31;
    const int nseg = H / 256;
    const int warps = (gridDim.x * blockDim.x) >> 5;
    for (int w = (blockIdx.x * blockDim.x + threadIdx.x) >> 5; w < T * nseg; w += warps) {
        const int row = w / nseg, seg = w - row * nseg;
        int tok = tokens[row];
        if (tok < 0 || tok >= V) {
            if (lane == 0) set_status(status, NF_ERR_DEVICE_BOUNDS);
            tok = 0;
        }
        residual_segment(table + (size_t)tok * H, row, seg, H, resid, xb, partials, lane);
    }
}

// Token feedback: out[t] = prev_token[src[t]] for src[t] >= 0 (the previous iteration's greedy
// token of that request), else token_ids[t] (a prompt token).
__global__ void gather_tokens_kernel(const int* __restrict__ token_ids, const int* __restrict__ src,
                                     const int* __restrict__ prev_token, int prev_rows, int T, int* out,
                                     int* status) {
    for (int t = blockIdx.x * blockDim.x + threadIdx.x; t < T; t += gridDim.x * blockDim.x) {
        const int s = src[t];
        int tok;
        if (s < 0) {
            tok = token_ids[t];
        } else if (s < prev_rows) {
            tok = prev_token[s];
        } else {
            set_status(status, NF_ERR_DEVICE_BOUNDS);
            tok = 0;
        }
        out[t] = tok;
    }
}

// LM-head input rows: every decode row, then (if present) the chunk's last row.
__global__ void lm_gather_kernel(const uint16_t* __restrict__ xb, const float* __restrict__ partials, int R,
                                 int T, int rows, int H, uint16_t* out, float* out_partials) {
    const int nseg = H / 256;
    const int per_row = H / 8;  // uint4 per row
    for (int i = blockIdx.x * blockDim.x + threadIdx.x; i < rows * per_row; i += gridDim.x * blockDim.x) {
        const int r = i / per_row, c = i - r * per_row;
        const int src = r < R ? r : T - 1;
        reinterpret_cast<uint4*>(out + (size_t)r * H)[c] = reinterpret_cast<const uint4*>(xb + (size_t)src * H)[c];
        if (c < nseg) out_partials[(size_t)r * nseg + c] = partials[(size_t)src * nseg + c];
    }
}

// next[r] = argmax over the row's per-tile maxima; strict '>' in tile order keeps the lowest index.
__global__ void argmax_reduce_kernel(const float* __restrict__ tile_max, const int* __restrict__ tile_arg,
                                     int rows, int ntiles, int* next) {
    const int lane = threadIdx.x & 31;
    const int warps = (gridDim.x * blockDim.x) >> 5;
    for (int r = (blockIdx.x * blockDim.x + threadIdx.x) >> 5; r < rows; r += warps) {
        float best = -INFINITY;
        int arg = 0x7fffffff;
        for (int t = lane; t < ntiles; t += 32) {
            const float v = tile_max[(size_t)r * ntiles + t];
            const int a = tile_arg[(size_t)r * ntiles + t];
            if (v > best || (v == best && a < arg)) { best = v; arg = a; }
        }
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) {
            const float ov = __shfl_xor_sync(0xffffffffu, best, o);
            const int oa = __shfl_xor_sync(0xffffffffu, arg, o);
            if (ov > best || (ov == best && oa < arg)) { best = ov; arg = oa; }
        }
        if (lane == 0) next[r] = arg;
    }
}

// dst row of source row r: (r / blk) * dst_blk_stride + dst_blk_off + r % blk; optional column scale.
__global__ void pack_rows_kernel(const uint16_t* __restrict__ src, uint16_t* __restrict__ dst, int rows, int cols,
                                 const uint16_t* __restrict__ gamma, int blk, int dst_blk_stride, int dst_blk_off) {
    const size_t n = (size_t)rows * cols;
    for (size_t i = (size_t)blockIdx.x * blockDim.x + threadIdx.x; i < n; i += (size_t)gridDim.x * blockDim.x) {
        const int r = (int)(i / cols), c = (int)(i - (size_t)r * cols);
        const int dr = (r / blk) * dst_blk_stride + dst_blk_off + r % blk;
        uint16_t v = src[i];
        if (gamma != nullptr) v = f2bf(bf2f(v) * bf2f(gamma[c]));
        dst[(size_t)dr * cols + c] = v;
    }
}

// fp32 copy of a bf16 matrix with an optional column scale (exact: bf16 x bf16 fits fp32).
__global__ void widen_scaled_kernel(const uint16_t* __restrict__ src, float* __restrict__ dst, int rows, int cols,
                                    const uint16_t* __restrict__ gamma) {
    const size_t n = (size_t)rows * cols;
    for (size_t i = (size_t)blockIdx.x * blockDim.x + threadIdx.x; i < n; i += (size_t)gridDim.x * blockDim.x) {
        const int c = (int)(i % cols);
        float v = bf2f(src[i]);
        if (gamma != nullptr) v *= bf2f(gamma[c]);
        dst[i] = v;
    }
}

// Page i of the list lands at dst + i * page_bytes; 16-byte loads that stream through L2 (the pages
// are read once), one CTA per page at a time.
__global__ void gather_pages_kernel(const uint4* __restrict__ pool, const int* __restrict__ ids, int n,
                                    size_t page_vec, uint4* __restrict__ dst) {
    for (int i = blockIdx.x; i < n; i += gridDim.x) {
        const uint4* src = pool + (size_t)ids[i] * page_vec;
        uint4* out = dst + (size_t)i * page_vec;
        for (size_t v = threadIdx.x; v < page_vec; v += blockDim.x) out[v] = __ldcs(src + v);
    }
}

__global__ void wait_flag_kernel(volatile int* flag, uint64_t limit_ns, int* status) {
    const uint64_t t0 = globaltimer_ns();
    while (*flag == 0) {
        if (globaltimer_ns() - t0 > limit_ns) {
            set_status(status, NF_ERR_DEVICE_TIMEOUT);
            return;
        }
        __nanosleep(1000);
    }
}

int grid_for(size_t work, int per_block, int max_blocks) {
    size_t g = (work + per_block - 1) / per_block;
    if (g < 1) g = 1;
    if (g > (size_t)max_blocks) g = max_blocks;
    return (int)g;
}

}  // namespace

cudaError_t launch_prep_hidden(const uint16_t* in, int T, int H, float* resid, uint16_t* xb, float* partials,
                               int max_blocks, cudaStream_t s) {
    if (T <= 0) return cudaSuccess;
    prep_hidden_kernel<<<grid_for((size_t)T * (H / 256), 8, max_blocks), 256, 0, s>>>(in, T, H, resid, xb, partials);
    return cudaGetLastError();
}

cudaError_t launch_embed(const int* tokens, const uint16_t* table, int T, int H, int V, float* resid, uint16_t* xb,
                         float* partials, int* status, int max_blocks, cudaStream_t s) {
    if (T <= 0) return cudaSuccess;
    embed_kernel<<<grid_for((size_t)T * (H / 256), 8, max_blocks), 256, 0, s>>>(tokens, table, T, H, V, resid, xb,
                                                                                  partials, status);
    return cudaGetLastError();
}

cudaError_t launch_gather_tokens(const int* token_ids, const int* src, const int* prev_token, int prev_rows, int T,
                                 int* out, int* status, cudaStream_t s) {
    if (T <= 0) return cudaSuccess;
    gather_tokens_kernel<<<(T + 255) / 256, 256, 0, s>>>(token_ids, src, prev_token, prev_rows, T, out, status);
    return cudaGetLastError();
}

cudaError_t launch_lm_gather(const uint16_t* xb, const float* partials, int R, int T, int rows, int H, uint16_t* out,
                             float* out_partials, int max_blocks, cudaStream_t s) {
    if (rows <= 0) return cudaSuccess;
    lm_gather_kernel<<<grid_for((size_t)rows * (H / 8), 256, max_blocks), 256, 0, s>>>(xb, partials, R, T, rows, H,
                                                                                        out, out_partials);
    return cudaGetLastError();
}

cudaError_t launch_argmax_reduce(const float* tile_max, const int* tile_arg, int rows, int ntiles, int* next,
                                 int max_blocks, cudaStream_t s) {
    if (rows <= 0) return cudaSuccess;
    argmax_reduce_kernel<<<grid_for((size_t)rows, 8, max_blocks), 256, 0, s>>>(tile_max, tile_arg, rows, ntiles,
                                                                                 next);
    return cudaGetLastError();
}

cudaError_t launch_pack_rows(const uint16_t* src, uint16_t* dst, int rows, int cols, const uint16_t* gamma, int blk,
                             int dst_blk_stride, int dst_blk_off, cudaStream_t s) {
    pack_rows_kernel<<<grid_for((size_t)rows * cols, 256, 4096), 256, 0, s>>>(src, dst, rows, cols, gamma, blk,
                                                                              dst_blk_stride, dst_blk_off);
    return cudaGetLastError();
}

cudaError_t launch_widen_scaled(const uint16_t* src, float* dst, int rows, int cols, const uint16_t* gamma,
                                cudaStream_t s) {
    widen_scaled_kernel<<<grid_for((size_t)rows * cols, 256, 4096), 256, 0, s>>>(src, dst, rows, cols, gamma);
    return cudaGetLastError();
}

cudaError_t launch_wait_flag(int* flag, uint64_t limit_ns, int* status, cudaStream_t s) {
    wait_flag_kernel<<<1, 1, 0, s>>>(flag, limit_ns, status);
    return cudaGetLastError();
}

}  // namespace nf

namespace nf {
cudaError_t launch_gather_pages(const void* pool, const int* ids, int n, size_t page_bytes, void* dst, int max_blocks,
                                cudaStream_t s) {
    if (n <= 0) return cudaSuccess;
    const int grid = n < max_blocks ? n : max_blocks;
    gather_pages_kernel<<<grid, 256, 0, s>>>(static_cast<const uint4*>(pool), ids, n, page_bytes / 16,
                                             static_cast<uint4*>(dst));
    return cudaGetLastError();
}
}  // namespace nf
