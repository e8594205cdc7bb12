// Argument blocks and launchers of the attention kernels.
#pragma once
#include <cstdint>
#include <cuda.h>
#include <cuda_runtime.h>

#include "nanoflow.h"

namespace nf {

// Decode keys are split into chunks of at most this many pages; the split of a request depends only
// on its ctx_len. The warp-level kernel splits every request longer than 512 keys; the tensor-core
// kernel, whose chunks cost a hand-off and a merge, splits contexts longer than 1024 keys.
constexpr int kDecodeSplitPages = 32;
constexpr int kDecodeSplitPagesTc = 64;
// split_pages value that keeps every request in one chunk (no partials, no merge pass)
constexpr int kDecodeNoSplit = 1 << 30;

struct DecodeArgs {
    const uint16_t* q;   // [rows x nq x d] bf16; decode request r is row r
    uint16_t* out;       // [rows x nq x d] bf16
    float* part_o;       // [items x G x d] split partials (normalised)
    float* part_lse;     // [items x G] log2-sum-exp of each split
    const int* ctx_len;  // [R]
    const int* page_indptr;
    const int* page_indices;
    const int* item_off;  // [R + 1] first work item of each request
    const void* item_tab; // [items] int4 work-item table (decode_items_kernel)
    const uint16_t* kv_pool;  // the layer's pool, physical page layout (see store_kv_row32 / nanoflow.h)
    int req_begin, req_end;
    int nq, nkv, G;
    int num_pages;
    int split_pages;
    float scale_log2;     // log2(e) / sqrt(d)
    int* merge_cnt;       // [R x nkv] split arrival counters (zeroed by decode_items_kernel)
    const int* chunk_off; // tensor-core kernel: [R + 1] first partial slot of each request
    float* part_ml;       // tensor-core kernel: [chunks x nq x 2] running maximum and row sum per query head
    int any_split;        // tensor-core kernel: 0 when no request of the launch has more than one chunk
    int* claim_ctr;       // tensor-core kernel: zeroed counter from which the CTAs claim work items in
                          // order (nullptr: each CTA takes an equal share of the page prefix)
    int* status;
    int* trace_ctr;
    nf_trace_entry* trace;
    int trace_cap;
};

struct PrefillArgs {
    const uint16_t* q;   // [rows x nq x d]; chunk row i is row num_decode + i
    uint16_t* out;
    const uint16_t* kv_pool;
    const int* page_indptr;
    const int* page_indices;
    int num_decode;      // index of the prefill request in the page table
    int prefill_len;
    int nq, nkv, G;
    int num_pages;
    float scale_log2;
    int* status;
    int* trace_ctr;
    nf_trace_entry* trace;
    int trace_cap;
};

int decode_smem_bytes(int head_dim);
int prefill_smem_bytes(int head_dim);

cudaError_t launch_decode_schedule(const int* ctx_len, int R, int nkv, int split_pages, int* item_off,
                                   cudaStream_t stream);
cudaError_t launch_decode_items(const int* ctx_len, const int* page_indptr, int R, int nkv, int split_pages,
                                const int* item_off, void* item_tab, int* merge_cnt, cudaStream_t stream);
cudaError_t launch_decode_attention(const DecodeArgs& a, int head_dim, int grid, cudaStream_t stream);
cudaError_t launch_prefill_attention(const PrefillArgs& a, int head_dim, int grid, cudaStream_t stream);

// Tensor-core (tcgen05) decode attention for 8 KV heads of dim 128 and 32 or 64 query heads:
// one request (all heads) per work item, one 64 KB page per pipeline stage. a.item_off holds
// the per-request prefix of page counts (decode_schedule with nkv = 1, split_pages = 1); tmQ
// maps q as [rows * nq x d] with boxes of nq rows.
bool decode_tc_supported(int nq, int nkv, int head_dim);
// item_off[r] = pages of requests [0, r), chunk_off[r] = chunks of requests [0, r) (nullable), for
// requests [0, R] (one CTA; a negative ctx_len is recorded in *status and read as 0).
cudaError_t launch_decode_tc_schedule(const int* ctx_len, int R, int split_pages, int* item_off, int* chunk_off,
                                      int* status, cudaStream_t stream);
cudaError_t launch_decode_attention_tc(const CUtensorMap& tmQ, const DecodeArgs& a, int grid, cudaStream_t stream);

// Tensor-core (tcgen05) causal attention of the prefill chunk for head dim 128 (any G):
// 128 query positions of one head per unit; tmQ maps q as [tokens][nq][128] (3-D, boxes of
// 64 x 1 x 128).
bool prefill_tc_supported(int head_dim);
cudaError_t launch_prefill_attention_tc(const CUtensorMap& tmQ, const PrefillArgs& a, int grid, cudaStream_t stream);

}  // namespace nf
