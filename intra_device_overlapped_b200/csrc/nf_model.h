// Internal model state behind the opaque nf_model handle.
#pragma once
#include <cstdint>
#include <vector>
#include <cuda.h>
#include <cuda_runtime.h>

#include "nanoflow.h"
#include "nf_schedule.h"

namespace nf {

constexpr int kDecodeSplitPagesHost = 32;     // must equal kDecodeSplitPages (nf_attention.h)
constexpr int kDecodeSplitPagesTcHost = 64;  // must equal kDecodeSplitPagesTc (nf_attention.h)

// Decode attention work items of a batch (sizes the split-KV partials): chunks of at most
// kDecodeSplitPagesHost pages, one per request chunk for the tensor-core kernel, one per KV head
// and chunk for the warp-level kernel.
int64_t decode_work_items(const ModelDims& d, const int32_t* ctx_len, int R);

// ops of one forward that can have a work counter (later elastic ops run on the GEMM share statically)
constexpr int kMaxCountedOps = 4096;

struct LayerWeights {
    uint16_t* wqkv = nullptr;  // [(nq + 2 nkv) d x H], attn-norm gamma folded
    uint16_t* wo = nullptr;    // [H x nq d]
    uint16_t* wgu = nullptr;   // dense: [2F x H]; MoE: [E x 2F x H]; gate/up interleaved per 128 rows, gamma folded
    uint16_t* wd = nullptr;    // dense: [H x F]; MoE: [E x H x F]
    float* router = nullptr;   // MoE: [E x H] fp32, gamma folded
    float* router_bias = nullptr;  // MoE: [E]
    CUtensorMap tm_qkv, tm_o, tm_gu, tm_d;
    bool loaded = false;
};

}  // namespace nf

struct nf_model {
    nf_model_config cfg;
    nf::ModelDims dims;
    int sm_count = 0;
    int n_part = 0;  // H / 256 partial sums of squares per row
    std::vector<nf::LayerWeights> layers;
    bool globals_loaded = false;
    uint16_t* embed = nullptr;    // [V x H]
    uint16_t* lm_head = nullptr;  // [V x H], final-norm gamma folded
    CUtensorMap tm_lm;

    // workspace (rows sized by max_tokens; MoE rows by max_tokens * top_k)
    float* resid = nullptr;       // [T x H] fp32 residual stream
    uint16_t* xb = nullptr;       // [T x H] bf16 copy: A operand of QKV / gate-up
    float* partials = nullptr;    // [T x H/256] sums of squares for the next RMSNorm
    uint16_t* q = nullptr;        // [T x nq d]
    uint16_t* attn_o = nullptr;   // [T x nq d]
    uint16_t* act = nullptr;      // [T(*K) x F] SwiGLU output
    float* rope_cos = nullptr;    // [max_position x d/2]
    float* rope_sin = nullptr;
    int* item_off = nullptr;      // [max_requests + 1] page prefix (tensor-core decode) or item prefix
    int* chunk_off = nullptr;     // [max_requests + 1] split-KV chunk prefix (tensor-core decode)
    int* tile_ctr = nullptr;      // [kMaxCountedOps] work counters of elastic GEMM and decode ops, zeroed per forward
    int* op_claim = nullptr;      // work counter of the single-op decode attention entry point
    int* mega_ctr = nullptr;      // [n_layers x kMegaCountersPerLayer] completion and work counters of the
                                  // persistent layer kernel, zeroed per forward
    bool decode_any_split = true; // some request of the current batch spans several decode chunks
    // KV offload: two staging buffers of offload_cap pages and the device copy of the page list
    uint8_t* offload_stage = nullptr;
    int* offload_ids = nullptr;
    int64_t offload_cap = 0;
    int* tok_feedback = nullptr;  // [T] token ids gathered from the previous iteration's next_token
    float* splitk_ws = nullptr;   // split-K partials of the residual GEMMs: [tiles x 128 x 256] fp32
    int* splitk_flags = nullptr;  // [tiles]: epoch of the last published first half
    int splitk_epoch = 0;         // incremented per split-K launch
    int* merge_cnt = nullptr;     // [max_requests x nkv] split-KV arrival counters
    float* part_o = nullptr;      // split-KV partials
    float* part_lse = nullptr;
    void* item_tab = nullptr;     // [part_capacity] int4 decode work items
    int64_t part_capacity = 0;    // items
    // LM head
    uint16_t* lm_in = nullptr;    // [max_requests + 1 x H]
    float* lm_partials = nullptr;
    float* tile_max = nullptr;    // [rows x V/256]
    int* tile_arg = nullptr;
    // MoE
    float* moe_logits = nullptr;  // [T x E]
    int* moe_idx = nullptr;       // [T x K]
    float* moe_w = nullptr;
    int* moe_counts = nullptr;    // [E + 1]
    int* moe_perm = nullptr;      // [T K]
    int* moe_inv = nullptr;
    uint16_t* moe_a = nullptr;    // [T K x H]
    float* moe_part = nullptr;    // [T K x H/256]
    float* moe_y = nullptr;       // [T K x H]
    CUtensorMap tm_xb, tm_attn_o, tm_act, tm_lm_in, tm_moe_a;
    CUtensorMap tm_q;             // q as [T * nq rows x d], nq-row boxes (tensor-core decode attention Q loads)
    bool decode_tc = false;       // the tensor-core decode kernel handles this model's head shape
    CUtensorMap tm_q3;            // q as [T][nq][d], 128-token boxes of one head (tensor-core prefill Q loads)
    bool prefill_tc = false;      // the tensor-core prefill kernel handles this model's head dim

    int* status = nullptr;        // device status word
    int* trace_ctr = nullptr;
    nf_trace_entry* trace = nullptr;
    int trace_cap = 0;
    bool trace_on = false;

    cudaStream_t s_attn = nullptr;
    cudaEvent_t ev_fork = nullptr, ev_join = nullptr;
    std::vector<cudaEvent_t> events;


    // per-op event timing
    bool timing_on = false;
    std::vector<cudaEvent_t> t_ev;
    std::vector<nf_op_time> t_ops;

    nf::CostModel cost;
    std::vector<void*> allocations;
};
