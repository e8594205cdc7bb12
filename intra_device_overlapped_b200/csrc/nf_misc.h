// Launchers of the small kernels (nf_misc.cu, nf_moe.cu).
#pragma once
#include <cstdint>
#include <cuda_runtime.h>

namespace nf {

cudaError_t launch_prep_hidden(const uint16_t* in, int T, int H, float* resid, uint16_t* xb, float* partials,
                               int max_blocks, cudaStream_t s);
cudaError_t launch_embed(const int* tokens, const uint16_t* table, int T, int H, int V, float* resid, uint16_t* xb,
                         float* partials, int* status, int max_blocks, cudaStream_t s);
cudaError_t launch_gather_tokens(const int* token_ids, const int* src, const int* prev_token, int prev_rows, int T,
                                 int* out, int* status, cudaStream_t s);
cudaError_t launch_lm_gather(const uint16_t* xb, const float* partials, int R, int T, int rows, int H, uint16_t* out,
                             float* out_partials, int max_blocks, cudaStream_t s);
cudaError_t launch_argmax_reduce(const float* tile_max, const int* tile_arg, int rows, int ntiles, int* next,
                                 int max_blocks, cudaStream_t s);
cudaError_t launch_pack_rows(const uint16_t* src, uint16_t* dst, int rows, int cols, const uint16_t* gamma, int blk,
                             int dst_blk_stride, int dst_blk_off, cudaStream_t s);
cudaError_t launch_widen_scaled(const uint16_t* src, float* dst, int rows, int cols, const uint16_t* gamma,
                                cudaStream_t s);
cudaError_t launch_wait_flag(int* flag, uint64_t limit_ns, int* status, cudaStream_t s);
// Pack pages ids[0..n) of a pool (page_bytes each, a multiple of 16) contiguously into dst.
cudaError_t launch_gather_pages(const void* pool, const int* ids, int n, size_t page_bytes, void* dst, int max_blocks,
                                cudaStream_t s);

// --- mixture of experts (nf_moe.cu) ---
struct MoeArgs {
    const float* resid;      // [T x H] fp32 residual h (rows of the launch start at tok0)
    const float* partials;   // [T x H/256]
    const float* router;     // [E x H] fp32, ffn-norm gamma folded
    const float* router_bias;  // [E]
    int tok0, rows, H, E, K, n_part;
    float inv_dim, eps;
    float* logits;           // [rows x E] (workspace)
    int* topk_idx;           // [rows x K]
    float* topk_w;           // [rows x K]
    int* counts;             // [E + 1] group offsets (output of the sort)
    int* perm;               // [rows*K] sorted slot -> assignment (token * K + k), local to the launch
    int* inv;                // [rows*K] assignment -> sorted slot
    const uint16_t* xb;      // [T x H] bf16 residual copy
    uint16_t* a_sorted;      // [rows*K x H] gathered rows
    float* part_sorted;      // [rows*K x H/256]
    const float* y_sorted;   // [rows*K x H] expert outputs
    float* resid_out;        // [T x H] updated residual (may alias resid)
    uint16_t* xb_out;        // [T x H]
    float* partials_out;     // [T x H/256]
    float* out_f32;          // nullable final fp32 copy
    int* dbg_idx;            // nullable [rows x K] copy of the routing for the caller
    float* dbg_w;
    float* dbg_logits;
};

cudaError_t launch_moe_route(const MoeArgs& a, int max_blocks, cudaStream_t s);
cudaError_t launch_moe_gather(const MoeArgs& a, int max_blocks, cudaStream_t s);
cudaError_t launch_moe_combine(const MoeArgs& a, int max_blocks, cudaStream_t s);

}  // namespace nf
