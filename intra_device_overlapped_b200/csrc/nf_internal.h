// Internal interfaces between the C ABI layer and the kernels.
#pragma once
#include <cstdint>
#include <cuda.h>
#include <cuda_runtime.h>

#include "nanoflow.h"

namespace nf {

constexpr int kGemmBM = 128;
constexpr int kGemmBN = 256;
constexpr int kGemmBK = 64;
constexpr int kGemmStages = 4;
constexpr int kGemmThreads = 192;
constexpr int kGemmBarrierBytes = 256;
constexpr int kGemmStagingBytes = 4 * 32 * 32 * 4;  // residual epilogue: 32 x 32 fp32 per epilogue warp
constexpr int kGemmSmemBytes =
    kGemmStages * (kGemmBM + kGemmBN) * kGemmBK * 2 + 1024 + kGemmBarrierBytes + kGemmStagingBytes;
// CTA-pair kernel: per CTA a stage holds 128 A rows and 128 B rows (its half of the 256-wide tile)
constexpr int kGemm2Stages = 6;
constexpr int kGemm2SmemBytes = kGemm2Stages * 256 * kGemmBK * 2 + 1024 + kGemmBarrierBytes + kGemmStagingBytes;
// rows of the boxes of every B (weight) tensor map: both kernels load B in 128-row boxes
constexpr int kGemmBBoxRows = 128;

enum EpiKind : int {
    EPI_F32 = 0,     // out_f32 = acc (* rs if partials)
    EPI_QKV = 1,     // rs, RoPE on q/k heads, q -> q_out, k/v -> paged cache slots
    EPI_RESID = 2,   // resid += acc; bf16 copy; per-(row, N-tile) sum of squares
    EPI_SWIGLU = 3,  // rs; silu(gate) * up over interleaved 128-col halves -> bf16
    EPI_LMHEAD = 4,  // rs; bf16 logits (optional); per-(row, N-tile) max and first argmax
};

struct GemmArgs {
    int M;         // rows of the launch (grouped: rows of all groups)
    int a_row0;    // TMA row coordinate of launch row 0 in A
    int tok0;      // per-row parameter index of launch row 0
    int N;         // output columns (grouped: per group)
    int K;
    int m_tiles, n_tiles, k_blocks;
    int grouped;   // 1: rows split by group_offsets, B rows of group g start at g * N
    const int* group_offsets;  // [num_groups + 1], launch-row offsets (device)
    int num_groups;
    // RMSNorm row scale: rs = rsqrt(sum(partials[row][0..n_part)) * inv_dim + eps)
    const float* partials;
    int n_part;
    float inv_dim;
    float eps;
    // outputs
    float* out_f32;
    int ld_f32;
    uint16_t* out_bf16;
    int ld_bf16;
    float* resid;         // EPI_RESID: [rows x N] fp32 residual, updated in place
    float* out_partials;  // EPI_RESID: [rows x n_tiles]
    // EPI_QKV
    const int* positions;
    const float* rope_cos;  // [max_position x d/2]
    const float* rope_sin;
    int max_position;
    uint16_t* q_out;        // [rows x nq x d]
    int nq, nkv, head_dim;
    uint16_t* kv_pool;      // [num_pages][2][nkv][16][d]
    int num_pages;
    const int* page_indptr;
    const int* page_indices;
    int num_decode;
    // split-K (EPI_RESID only): with k_split = 2 work unit u < tiles is the first half of the k
    // blocks of tile u and writes its fp32 partial to splitk_ws, publishing splitk_flags[u] =
    // splitk_epoch; unit tiles + u is the second half and adds that partial (in this fixed order)
    // before the residual epilogue. Units of first halves come first in every CTA's order.
    int k_split;
    float* splitk_ws;     // [tiles x BM x BN] fp32
    int* splitk_flags;    // [tiles]
    int splitk_epoch;
    // EPI_LMHEAD
    float* tile_max;  // [rows x n_tiles]
    int* tile_arg;
    // Work order: nullptr = static (CTA b takes units b, b + grid, ...); else a zeroed counter from
    // which CTAs claim units in increasing order, so that a launch whose CTAs start at different
    // times (SMs freed by a kernel on another stream) still shares the units evenly.
    int* tile_ctr;
    // diagnostics
    int* status;
    int* trace_ctr;
    nf_trace_entry* trace;
    int trace_cap;
};

// Encode a 2-D bf16 tensor map over a row-major [rows x cols] matrix with a box of
// box_rows x 64 columns and 128-byte swizzle. Returns false on failure.
bool make_tmap_bf16_2d(CUtensorMap* map, const void* base, uint64_t rows, uint64_t cols, uint32_t box_rows);
// [tokens][heads][head_dim] bf16 viewed as a 3-D map with boxes of 64 elements x 1 head x
// box_tokens tokens (128-byte swizzle): one head's rows of consecutive tokens.
bool make_tmap_bf16_3d_heads(CUtensorMap* map, const void* base, uint64_t tokens, uint64_t heads, uint64_t head_dim,
                             uint32_t box_tokens);

// Dense launches (not grouped) with a grid of at least 2 run on CTA pairs with 256 x 256 tiles; grouped
// launches and single-CTA grids on single CTAs with 128 x 256 tiles.
cudaError_t launch_gemm(int epi, const CUtensorMap& tmA, const CUtensorMap& tmB, const GemmArgs& args, int grid,
                        cudaStream_t stream);
bool gemm_uses_pairs(const GemmArgs& a);
// work units (output tiles, times 2 with split K) of a launch on the kernel launch_gemm picks for grids >= 2
int gemm_units(const GemmArgs& a);

int device_sm_count();

}  // namespace nf
