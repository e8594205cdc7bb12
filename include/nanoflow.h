/*
 * nanoflow.h — C ABI of a B200 (sm_100a) implementation of one NanoFlow-style
 * serving iteration with intra-device overlap.
 *
 * What the library computes. One batched serving iteration of a Llama-style
 * transformer (NanoFlow README "Feasibility": Llama2-70B, Llama3-8B, Mixtral 8x7B)
 * over a mixed batch: R decode requests (one new token each, attending to their
 * paged KV cache) followed by one prefill chunk of C tokens. Per layer:
 * RMSNorm -> QKV projection -> RoPE -> K/V written into the paged cache ->
 * paged GQA decode attention and causal prefill attention -> output projection
 * + residual -> RMSNorm -> SwiGLU FFN (or top-k mixture of SwiGLU experts) +
 * residual; full models add the token embedding, the final norm, the LM head
 * and greedy argmax.
 *
 * How it is scheduled. "Nano-batching" splits the batch into smaller
 * nano-batches and duplicates each operation per nano-batch so that operations
 * of different nano-batches no longer depend on one another (arXiv abstract of
 * "NanoFlow: Towards Optimal Large Language Model Serving Throughput"; README
 * "Abstract"). A pipeline inside the device then assigns execution units so that
 * the compute-bound GEMMs of one nano-batch run on one part of the GPU while
 * the memory-bound attention of another runs on the rest (README
 * "Introduction" and "Abstract"). The number, size, order and GPU resource
 * split of the nano-batches are chosen automatically, taking interference into
 * account (arXiv abstract). Here the split is a set of SMs: GEMM kernels and
 * attention kernels are persistent and launched with grids that claim disjoint
 * SM sets on two CUDA streams; nf_plan_iteration picks the plan by exhaustive
 * search over per-kernel costs.
 *
 * Conventions.
 *  - Every call returns an nf_status; nothing aborts or prints. No C++ exception leaves the
 *    library: a failed host allocation returns NF_ERR_OUT_OF_MEMORY.
 *  - bf16 tensors are passed as raw 16-bit patterns (void*), row-major.
 *  - Device pointers are owned by the caller unless stated otherwise; the model
 *    owns its packed weights and workspace (freed by nf_destroy_model).
 *  - `stream` arguments are cudaStream_t values passed as void* (NULL = legacy
 *    default stream). Work is asynchronous on that stream.
 *  - A model is not thread-safe: one forward at a time per model.
 *  - Errors detected on the device (page index out of range, token id out of
 *    range, a wait that timed out) are latched in a device status word and
 *    returned by nf_sync_status().
 *  - Token order within an iteration: decode rows first (request order), then
 *    the prefill chunk. Decode request r has ctx_len[r] cached tokens; its new
 *    token sits at position ctx_len[r] and its K/V go to that slot. The chunk is
 *    a fresh prompt at positions 0..C-1.
 */
#ifndef NANOFLOW_H
#define NANOFLOW_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
    NF_OK = 0,
    NF_ERR_INVALID_ARGUMENT = 1, /* a null pointer, a size out of range, an inconsistent descriptor */
    NF_ERR_UNSUPPORTED = 2,      /* a shape the kernels do not handle (see nf_init_model) */
    NF_ERR_OUT_OF_MEMORY = 3,    /* device allocation failed */
    NF_ERR_CUDA = 4,             /* a CUDA runtime call failed (no device, launch failure, ...) */
    NF_ERR_DEVICE_TIMEOUT = 5,   /* a device-side wait exceeded its time limit and gave up */
    NF_ERR_DEVICE_BOUNDS = 6     /* a device-side index check failed; the access was skipped */
} nf_status;

/* Static description of the string of a status code (never NULL). */
const char* nf_status_string(int status);

/* ------------------------------------------------------------------ model */

typedef struct nf_model nf_model; /* opaque */

typedef struct {
    int32_t n_layers;
    int32_t hidden;       /* H, multiple of 256 */
    int32_t n_q_heads;    /* nq */
    int32_t n_kv_heads;   /* nkv; nq % nkv == 0 and nq / nkv <= 8 */
    int32_t head_dim;     /* d: 64 or 128 */
    int32_t ffn;          /* F (per expert for MoE), multiple of 128 */
    int32_t vocab;        /* 0: layer slice (hidden in/out); >0: embedding + final norm + LM head, multiple of 256 */
    int32_t n_experts;    /* 0: dense SwiGLU FFN; 1..16: mixture of experts */
    int32_t top_k;        /* experts per token (MoE), 1..n_experts */
    float rms_eps;        /* RMSNorm epsilon */
    float rope_theta;     /* RoPE base */
    int32_t page_size;    /* tokens per KV page; must be 16 */
    int32_t max_tokens;   /* upper bound on T = R + C per iteration (workspace sizing) */
    int32_t max_requests; /* upper bound on R */
    int32_t max_position; /* positions must be < max_position (RoPE table length) */
} nf_model_config;

/* A Llama-style model of the families the NanoFlow README benchmarks ("Feasibility": LLaMA-2-70B,
 * LLaMA-3-8B, Mixtral 8x7B; dense SwiGLU or top-k mixture of experts, grouped-query attention).
 * Validate `cfg`, allocate the model's packed-weight buffers and workspace and
 * build the RoPE table (angles pos * theta^(-2i/d) in double, stored as fp32). The weights
 * are handed over afterwards, layer by layer, with nf_set_layer_weights / nf_set_global_weights
 * (a model of 34 GB of weights need not exist twice on the device at any moment).
 * On success *out owns device memory until nf_destroy_model. Requirements:
 * (nq + 2 nkv) d, nq d, H and 2F divisible by 256; H divisible by 64. */
nf_status nf_init_model(const nf_model_config* cfg, nf_model** out);

/* Weights of one layer, canonical Hugging Face layout: device pointers to bf16,
 * linear weights [out_features x in_features] row-major. The library copies and
 * repacks them (QKV concatenated, gate/up interleaved per 128-row tile, RMSNorm
 * gamma folded into the columns of the following projection); the caller may
 * free its buffers once the stream has passed the copy. */
typedef struct {
    const void* attn_norm; /* [H] */
    const void* wq;        /* [nq*d x H] */
    const void* wk;        /* [nkv*d x H] */
    const void* wv;        /* [nkv*d x H] */
    const void* wo;        /* [H x nq*d] */
    const void* ffn_norm;  /* [H] */
    const void* w_gate;    /* [F x H] (dense) */
    const void* w_up;      /* [F x H] (dense) */
    const void* w_down;    /* [H x F] (dense) */
    const void* router;      /* [E x H] (MoE) */
    const void* router_bias; /* [E] (MoE) */
    const void* const* expert_gate; /* host array of E device pointers, each [F x H] (MoE) */
    const void* const* expert_up;   /* host array of E device pointers, each [F x H] (MoE) */
    const void* const* expert_down; /* host array of E device pointers, each [H x F] (MoE) */
} nf_layer_weights;

nf_status nf_set_layer_weights(nf_model* m, int32_t layer, const nf_layer_weights* w, void* stream);

/* Embedding, final norm and LM head (models with vocab > 0): device bf16 pointers. */
typedef struct {
    const void* embed;      /* [V x H] */
    const void* final_norm; /* [H] */
    const void* lm_head;    /* [V x H] */
} nf_global_weights;

nf_status nf_set_global_weights(nf_model* m, const nf_global_weights* w, void* stream);

void nf_destroy_model(nf_model* m);

/* ------------------------------------------------------------------ plan */

/* Host-side description of the iteration's batch (host copies of the page table that the
 * device copies in nf_iter_io hold). nf_plan_iteration, nf_tune_plan and nf_calibrate validate
 * it before anything is launched: every request holds at least ceil(keys / 16) pages
 * (keys = ctx_len[r] + 1 for a decode request, C for the chunk), the offsets start at 0 and
 * grow, and every page id of every request lies in [0, num_pages); else
 * NF_ERR_INVALID_ARGUMENT. */
typedef struct {
    int32_t num_decode;        /* R >= 0 */
    int32_t prefill_len;       /* C >= 0 */
    int32_t prefix_len;        /* must be 0 (fresh prompt) */
    const int32_t* ctx_len;    /* host [R]: cached tokens per decode request (>= 0) */
    const int32_t* page_indptr; /* host [R + 2]: CSR offsets of each request's pages (prefill last) */
    int32_t num_pages;         /* pages in each layer's pool */
    const int32_t* page_indices; /* host [page_indptr[R + 1]]: the page ids (required) */
} nf_batch_desc;

#define NF_MAX_NANO 4

typedef struct {
    int32_t force_nano;     /* 0: search; 1..4: this many nano-batches */
    int32_t force_sm_attn;  /* 0: search; >0: SMs given to attention kernels (overlapped plans) */
    int32_t force_template; /* -1: search; else an NF_TEMPLATE_* value */
    int32_t sm_total;       /* 0: every SM of the device */
} nf_plan_opts;

enum {
    NF_TEMPLATE_SEQUENTIAL = 0,       /* one nano-batch after another, each op on all SMs (no overlap) */
    NF_TEMPLATE_PIPELINED = 1,        /* attention of nano-batch j co-runs with the GEMMs of the others */
    NF_TEMPLATE_PREFILL_ON_GEMM = 2,  /* as PIPELINED, but the compute-bound prefill attention runs on the
                                         GEMM stream and SMs; only decode attention co-runs */
};

typedef struct {
    int32_t n_nano;
    int32_t tok_begin[NF_MAX_NANO]; /* nano-batch j = tokens [tok_begin[j], tok_end[j]) */
    int32_t tok_end[NF_MAX_NANO];
    int32_t nano_order[NF_MAX_NANO]; /* pipeline order of the nano-batches (O / FFN phase) */
    int32_t order_template;       /* NF_TEMPLATE_* */
    int32_t sm_attn;              /* SMs claimed by attention kernels while overlapped */
    int32_t sm_gemm;              /* SMs claimed by GEMM kernels while overlapped */
    int32_t sm_total;
    float predicted_us;           /* simulated iteration time of this plan */
    float predicted_serial_us;    /* simulated time of the same work without overlap */
    int32_t num_decode, prefill_len, num_tokens; /* copied from the batch */
    int64_t kv_pages_read;        /* decode + prefill KV pages (all KV heads) read per layer */
    int64_t decode_items;         /* decode attention work items (sizes the split-KV workspace) */
} nf_plan;

/* Choose nano-batch count, sizes (token ranges cut at request boundaries, the
 * prefill chunk whole), op order and SM split minimising the simulated two-stream
 * makespan over the model's per-kernel cost tables (arXiv abstract: the search
 * covers the count, size and order of nano-batches and their share of the GPU).
 * Host only. */
nf_status nf_plan_iteration(const nf_model* m, const nf_batch_desc* b, const nf_plan_opts* opts, nf_plan* out);

/* The same search for a model configuration without a device or a model handle:
 * uses the built-in default cost tables and `sm_count` SMs (> 0). Host only. */
nf_status nf_plan_for_config(const nf_model_config* cfg, int32_t sm_count, const nf_batch_desc* b,
                             const nf_plan_opts* opts, nf_plan* out);

/* ------------------------------------------------------------------ forward */

/* Per-iteration inputs and outputs, all device pointers owned by the caller. */
typedef struct {
    const int32_t* token_ids;    /* [T] (vocab > 0) */
    const void* hidden_in;       /* [T x H] bf16 (vocab == 0) */
    const int32_t* positions;    /* [T] */
    const int32_t* ctx_len;      /* [R] */
    const int32_t* page_indptr;  /* [R + 2] */
    const int32_t* page_indices; /* [page_indptr[R+1]] page ids < num_pages */
    void* const* kv_pools;       /* host array [n_layers]: device pool of num_pages pages, updated in place.
                                  * Page layout (bf16): [K|V][half of d (64 columns)][KV head][16 slots]
                                  * [8 chunks of 8 columns], logical chunk c of slot r stored at c ^ (r % 8);
                                  * one page holds 2 * nkv * 16 * d elements. */
    int32_t num_pages;
    void* hidden_out;            /* [T x H] bf16, nullable */
    float* hidden_out_f32;       /* [T x H] fp32 residual stream after the last layer, nullable */
    void* logits;                /* [rows x V] bf16, nullable; rows = R + (C > 0) */
    int32_t* next_token;         /* [rows], nullable */
    int32_t* topk_idx;           /* MoE: [n_layers x T x top_k] expert ids, nullable */
    float* topk_w;               /* MoE: [n_layers x T x top_k] routing weights, nullable */
    float* router_logits;        /* MoE: [n_layers x T x E] fp32, nullable */
    float* layer_hidden_out;     /* [n_layers x T x H] fp32 residual stream after each layer, nullable
                                  * (verification: copied row range by row range as each nano-batch
                                  * finishes a layer) */
    /* Token feedback on the device (vocab > 0), for a CPU that forms iteration i+1 before it has
     * read iteration i's tokens. token_src NULL: every token comes from token_ids. Otherwise
     * row t's token is prev_token[token_src[t]] when token_src[t] >= 0 (prev_token: the previous
     * iteration's next_token, prev_rows entries), else token_ids[t]. A token_src entry >=
     * prev_rows latches NF_ERR_DEVICE_BOUNDS and reads token 0. */
    const int32_t* token_src;    /* [T] device, nullable */
    const int32_t* prev_token;   /* [prev_rows] device */
    int32_t prev_rows;
} nf_iter_io;

/* Run the iteration described by `plan` (made by nf_plan_iteration for the same
 * batch): NanoFlow's nano-batched serving iteration (arXiv abstract of "NanoFlow: Towards Optimal
 * Large Language Model Serving Throughput": the batch is split into nano-batches and each
 * operation is duplicated per nano-batch so that operations bound by different resources overlap
 * inside the device; README "Introduction": compute-bound GEMMs beside memory-bound attention).
 * GEMMs run on `stream`, attention on a model-owned second stream (the higher-priority one) that
 * forks from and joins back into `stream`; the result does not depend on the plan (bit for bit).
 * Page ids of the device page table are checked on the device (an id outside the pool is recorded
 * as NF_ERR_DEVICE_BOUNDS and the access skipped); nf_plan_iteration checks the host copy before
 * anything runs. Asynchronous. */
nf_status nf_forward_iteration(nf_model* m, const nf_plan* plan, const nf_iter_io* io, void* stream);

/* The same iteration with each layer run as ONE persistent kernel on `stream` instead of one launch
 * per operation on two streams (NanoFlow's device-level pipeline, arXiv abstract: operations of
 * different nano-batches run in parallel inside the device, here scheduled by the device itself).
 * One CTA per SM (plan->sm_total of them) walks the layer's operations in the plan's issue order:
 * attention-stream operations on the plan's sm_attn CTAs, GEMM-stream operations inside an attention
 * window on the others, all other operations on every CTA. Before an operation a CTA waits until every
 * CTA has finished each operation it depends on (completion counters in device memory, acquire/release,
 * every wait bounded: NF_ERR_DEVICE_TIMEOUT on expiry); GEMM tiles and decode items are claimed from
 * work counters, so a CTA that runs out of work in one operation moves on to the next at once. The
 * GEMMs run on one-CTA 128 x 256 tiles (the stream executor pairs CTAs), so results equal those of
 * nf_forward_iteration up to the rounding of the fp32 accumulation order in the tensor cores (in
 * practice bit for bit). Same inputs, outputs and checks as nf_forward_iteration; NF_ERR_UNSUPPORTED
 * for models whose attention does not run on the tensor-core kernels (head dim 128, 8 KV heads, 32 or
 * 64 query heads) and for MoE models. Per-op timing (nf_set_timing) records nothing for the layers.
 * Asynchronous. */
nf_status nf_forward_iteration_persistent(nf_model* m, const nf_plan* plan, const nf_iter_io* io, void* stream);

/* The iteration of one plan as a CUDA graph: every launch, copy and cross-stream dependency of
 * nf_forward_iteration(m, plan, io) recorded once and replayed with one launch. nf_graph_create runs
 * the iteration once normally on `stream` (so that workspaces are sized before the capture), then
 * captures it on `stream` (a stream other than the legacy default stream; the model's attention
 * stream joins the capture) and instantiates the graph. The graph holds the plan and the pointers of
 * `io` (and their device contents are read at replay), so a caller reuses the same buffers from
 * iteration to iteration; a new plan needs a new graph. nf_graph_launch replays it on `stream`,
 * asynchronously, with the same results as nf_forward_iteration. NF_ERR_INVALID_ARGUMENT for null
 * pointers, the default stream, or per-op timing switched on; the errors of nf_forward_iteration;
 * NF_ERR_CUDA if the capture or instantiation fails. A graph must be destroyed before its model. */
typedef struct nf_graph nf_graph; /* opaque */
nf_status nf_graph_create(nf_model* m, const nf_plan* plan, const nf_iter_io* io, void* stream, nf_graph** out);
nf_status nf_graph_launch(nf_graph* g, void* stream);
void nf_graph_destroy(nf_graph* g);

/* Plan choice by measurement. After about 0.3 s of sequential iterations (the clock a power-capped
 * GPU holds under load is lower than its first burst), for each template and nano-batch count the
 * planner's best plan (the SM split chosen by the cost model) is run on this batch: one warm-up and
 * `reps` timed iterations (CUDA events on `stream`). The three fastest (the sequential plan always
 * among them) are then each run alone for about 0.8 s and timed over the next 0.2 s (a short run
 * inherits the clock its predecessors left under the power cap, and the GPU's power control settles
 * over a large fraction of a second); the fastest is written to `out` and its time, in
 * microseconds, to `best_us` (nullable). The sequential plan is kept unless another beats it by
 * more than 1%. Takes a few seconds. This is the search over
 * measured costs that the arXiv abstract describes, with the final choice between templates
 * and counts made on the device, where the interference of co-running kernels is real.
 * Runs nf_forward_iteration with `io` repeatedly: the new tokens' K/V slots are rewritten
 * with the same values and the outputs are overwritten. Synchronizes `stream`. */
nf_status nf_tune_plan(nf_model* m, const nf_batch_desc* b, const nf_iter_io* io, int32_t reps, void* stream,
                       nf_plan* out, float* best_us);

/* Wait for the model's streams and return (and clear) the latched device status. */
nf_status nf_sync_status(nf_model* m);

/* Time the model's own kernels at the sizes of `b` on several SM shares and GEMM + decode-attention
 * co-runs at three shares, then two whole plans in steady state (the sequential one for
 * iter_scale, one overlapped plan for power_floor), and store the fitted rates as the planner's
 * cost model (synchronous; about half a second, longer for deep models). Reads the KV pools of
 * `io`; the whole-plan timings run nf_forward_iteration with `io` (the new tokens' K/V slots are
 * rewritten with the same values, the outputs overwritten). */
nf_status nf_calibrate(nf_model* m, const nf_batch_desc* b, const nf_iter_io* io, void* stream);

/* The planner's per-kernel cost model (defaults until nf_calibrate has run). */
typedef struct {
    double gemm_flops_per_sm;  /* sustained tensor FLOP/s of one SM in the GEMM main loop */
    double gemm_tile_us;       /* fixed cost per 128 x 256 output tile */
    double gemm_launch_us;
    double hbm_bw;             /* bytes/s the decode attention reaches on every SM */
    double attn_bw_per_sm;     /* bytes/s one SM of decode attention pulls */
    double attn_launch_us;
    double attn_flops_per_sm;  /* prefill attention FLOP/s per SM */
    double interference;       /* fractional slow-down of a GEMM and an attention kernel co-running (mean of
                                * the tables below; used where a table entry is missing) */
    int32_t calibrated;
    /* Measured by nf_calibrate (zero = not measured): decode attention bytes/s on grids of 1/8, 1/4,
     * 1/2, 3/4 and all of the SMs, and the fractional slow-downs of decode attention and of a GEMM on
     * the remaining SMs when the two co-run with attention on 1/4, 1/2 and 3/4 of the SMs. The
     * planner interpolates them linearly in the attention share. */
    double attn_bw_at[5];
    double interf_attn[3];
    double interf_gemm[3];
    /* Measured over predicted time of the sequential one-nano-batch plan on the calibration batch
     * (1 = not measured). The kernel rates above are timed in bursts of a few launches; an iteration
     * that runs for tens of milliseconds settles at the lower clock of the power cap, and this factor
     * carries that into every prediction. */
    double iter_scale;
    /* Power floor (0 = none): a plan's predicted time is at least power_floor x its serial time (the
     * sum of its kernels' times on all SMs, scaled like every prediction). Under a power cap the GPU
     * trades the idle SM time that overlap removes for a lower clock, so an overlapped plan cannot
     * run much faster than its kernels' energy allows. nf_calibrate sets it from one overlapped plan
     * timed in steady state (its measured time over its serial time). */
    double power_floor;
} nf_cost_model;

nf_status nf_get_cost_model(const nf_model* m, nf_cost_model* out);
nf_status nf_set_cost_model(nf_model* m, const nf_cost_model* in);

/* Per-CTA placement trace of the last forward (enabled with nf_set_trace):
 * entries of {kernel id, sm id, start ns, end ns}. Returns the entry count
 * written (<= capacity), or a negative nf_status. */
typedef struct {
    int32_t kernel;   /* NF_KERNEL_* */
    int32_t smid;
    uint64_t t_start; /* %globaltimer ns */
    uint64_t t_end;
} nf_trace_entry;

enum { NF_KERNEL_GEMM = 1, NF_KERNEL_DECODE_ATTN = 2, NF_KERNEL_PREFILL_ATTN = 3 };

nf_status nf_set_trace(nf_model* m, int32_t enable);
int64_t nf_get_trace(nf_model* m, nf_trace_entry* out, int64_t capacity);

/* Per-operation CUDA-event timing (enabled with nf_set_timing, which also clears the
 * record): one entry per operation of every forward since, in issue order, with the duration
 * between events recorded around it on its own stream (a co-running op on the other
 * stream is included in the wall time it sees, not excluded). */
typedef struct {
    int32_t kind;   /* NF_OP_* */
    int32_t nano;   /* nano-batch index (-1 for the LM head) */
    int32_t layer;
    int32_t stream; /* 0: GEMM stream, 1: attention stream */
    int32_t grid;   /* CTAs launched (SMs claimed) */
    float us;
} nf_op_time;

enum { NF_OP_QKV = 0, NF_OP_DECODE_ATTN = 1, NF_OP_O = 2, NF_OP_GATE_UP = 3, NF_OP_DOWN = 4, NF_OP_MOE = 5,
       NF_OP_LM_HEAD = 6, NF_OP_PREFILL_ATTN = 7 };

nf_status nf_set_timing(nf_model* m, int32_t enable);
/* Waits for the model's streams; returns the number of entries written (<= capacity) or a negative nf_status. */
int64_t nf_get_op_times(nf_model* m, nf_op_time* out, int64_t capacity);

/* ------------------------------------------------------------------ single ops
 * The kernels of the hot path, callable one at a time (tests, calibration,
 * isolated timing). Same kernels as nf_forward_iteration uses.
 */

/* C[M x N] (fp32) = A[M x K] * B[N x K]^T with bf16 A, B (device, row-major) on the
 * tcgen05 tensor cores with TMEM accumulation. M >= 1, N % 256 == 0, K % 64 == 0,
 * A and B 16-byte aligned. `sm_count` = CTAs of the persistent grid (0 = all SMs). */
nf_status nf_op_gemm_bf16(const void* A, const void* B, float* C, int32_t M, int32_t N, int32_t K,
                          int32_t sm_count, void* stream);

/* Paged GQA decode attention of requests [req_begin, req_end) of layer `layer`'s
 * pool: out[r][h][:] = softmax(q[r][h] K_r^T / sqrt(d)) V_r over the ctx_len[r]+1
 * keys of request r, K/V of kv head h / (nq / nkv). q and out are [R x nq x d]
 * bf16 rows of the iteration (decode rows). Uses the model's workspace for the
 * split-KV partial results. */
nf_status nf_op_decode_attention(nf_model* m, const void* q, void* out, const nf_iter_io* io, int32_t layer,
                                 int32_t req_begin, int32_t req_end, int32_t sm_count, void* stream);

/* Causal attention of the prefill chunk (positions 0..C-1) reading its K/V from
 * the pages of request R (the prefill request) of layer `layer`. q and out are
 * [C x nq x d] bf16. */
nf_status nf_op_prefill_attention(nf_model* m, const void* q, void* out, const nf_iter_io* io, int32_t layer,
                                  int32_t num_decode, int32_t prefill_len, int32_t sm_count, void* stream);

/* Device-wait self test: one CTA waits on a flag in device memory that nothing sets,
 * with a time limit of `limit_ns`; returns NF_ERR_DEVICE_TIMEOUT (the expected
 * outcome) after the kernel has given up and exited, or NF_OK if the flag was set. */
nf_status nf_op_wait_flag_test(int32_t* flag_device, uint64_t limit_ns, void* stream);

/* Self test of the persistent layer kernel's dependency waits: the kernel is launched on a few CTAs
 * with an operation list whose first operation depends on its second (which every CTA reaches only
 * after the first), each wait limited to `limit_ns` (1 ns .. 10 s). Every CTA's wait must expire:
 * returns NF_ERR_DEVICE_TIMEOUT (the expected outcome) once the kernel has exited, NF_OK if a wait
 * did not expire, NF_ERR_CUDA on a launch or copy error. Blocks the host until done. */
nf_status nf_op_persistent_wait_test(uint64_t limit_ns, void* stream);

/* ------------------------------------------------------------------ KV offload
 *
 * Offload of a finished request's KV cache to host memory (hysenlabs review, "KV-cache offload to
 * SSD": NanoFlow moves the KV cache of finished requests off the GPU so that a later turn of the
 * same conversation can resume from it; only the device-to-host half is built here, the storage
 * tiers are not). For every layer l in [layer_begin, layer_end), the n_pages pages listed in
 * pages_host (host int32, each in [0, num_pool_pages)) of kv_pools[l] are copied, in list order,
 * to host_dst + ((l - layer_begin) * n_pages + i) * page_bytes, page_bytes = 2 * nkv * 16 * d * 2
 * (the physical page image described for nf_iter_io.kv_pools). Layer by layer, a gather kernel
 * packs the pages into a model-owned staging buffer and one cudaMemcpyAsync moves them to the host,
 * all on `stream`: issued on a stream of its own, the offload runs on the copy engine beside the
 * next iterations. host_dst must be pinned (page-locked) host memory for the copies to overlap.
 * The caller must not let an iteration rewrite the pages before the offload has completed (e.g.
 * keep them out of the free pool until an event recorded on `stream` has passed). Asynchronous;
 * NF_ERR_INVALID_ARGUMENT for a page id outside the pool, an empty or out-of-range layer range or
 * a null pointer; NF_ERR_OUT_OF_MEMORY if the staging buffer cannot grow. Not thread-safe per model. */
nf_status nf_offload_kv(nf_model* m, void* const* kv_pools, int32_t num_pool_pages, const int32_t* pages_host,
                        int32_t n_pages, int32_t layer_begin, int32_t layer_end, void* host_dst, void* stream);

/* Largest num_requests nf_decode_attention_noalloc accepts (size of its static scratch). */
#define NF_NOALLOC_MAX_REQUESTS 16384

/* Decode attention that allocates nothing. The paper has no counterpart: this entry point
 * exists for callers that cannot allocate device memory where they call it (code between
 * the capture calls of a CUDA graph, allocator-free runtimes, processes whose device memory
 * all belongs to their own pool), and therefore cannot create an nf_model.
 *
 * Computes, for each decode request r < num_requests and query head h, the softmax
 * attention of q[r][h] over the ctx_len[r] + 1 cached keys of KV head h / (nq / nkv),
 * gathered through the page table (the operation nf_forward_iteration runs as its decode
 * attention step), with the same tensor-core kernel as nf_op_decode_attention. Each request is
 * one work item here (no split along the keys, whose partials would need scratch that grows
 * with the batch), so the result equals nf_op_decode_attention's bit for bit for requests of at
 * most 1024 keys (which that entry point does not split either) and within rounding otherwise.
 *   q, out        device bf16 [num_requests x n_q_heads x head_dim], row r = request r.
 *   kv_pool       device bf16 pool of one layer, num_pages pages in the physical page layout
 *                 described for nf_iter_io.kv_pools.
 *   ctx_len       device int32 [num_requests]; page_indptr device int32 [num_requests + 1];
 *   page_indices  device int32 (CSR page table; request r owns page_indices[page_indptr[r] ..],
 *                 at least ceil((ctx_len[r] + 1) / 16) entries).
 *   sm_count      persistent grid (0 = every SM).
 *   status_device device int32 the caller zeroes (required; NULL gives NF_ERR_INVALID_ARGUMENT);
 *                 receives the first device-detected error: NF_ERR_DEVICE_BOUNDS for a page id
 *                 outside the pool, a request row shorter than its keys need (page 0 is read in
 *                 its place) or a negative ctx_len (read as 0); NF_ERR_DEVICE_TIMEOUT for a
 *                 pipeline wait that passed its limit.
 * Supported shapes: head_dim 128, n_kv_heads 8, n_q_heads 32 or 64 (else NF_ERR_UNSUPPORTED).
 * num_requests > NF_NOALLOC_MAX_REQUESTS returns NF_ERR_INVALID_ARGUMENT.
 * Scratch: a static device array of 64 KB per device (the per-request page prefix and the work
 * counter from which the CTAs claim requests), shared by
 * every call: calls that overlap on the GPU race on it and must be serialised. The first call
 * on each device looks up the array's address (cudaGetSymbolAddress) and keeps it for the life
 * of the process; make that first call before any stream capture, and do not call the entry
 * point again on a device after cudaDeviceReset (the kept address would be stale). Asynchronous
 * on `stream`; no call allocates device or pinned memory. */
nf_status nf_decode_attention_noalloc(const void* q, void* out, const void* kv_pool, int32_t num_pages,
                                      const int32_t* ctx_len, const int32_t* page_indptr,
                                      const int32_t* page_indices, int32_t num_requests, int32_t n_q_heads,
                                      int32_t n_kv_heads, int32_t head_dim, int32_t sm_count,
                                      int32_t* status_device, void* stream);

/* ------------------------------------------------------------------ serving scheduler (host)
 *
 * The CPU control flow around nf_forward_iteration for a stream of requests (prompt, then greedy
 * decoding). The CPU forms iteration i+1 while the GPU runs iteration i (README "Abstract",
 * arXiv abstract: NanoFlow's asynchronous CPU scheduling), so a request whose last token comes out
 * of iteration i is decoded once more in iteration i+1; that token is dropped and the request
 * leaves the batch from iteration i+2 on. Decode rows take their input token from the previous
 * iteration's next_token on the device (nf_iter_io.token_src), so forming a batch never waits for
 * the GPU. Host only: no call touches a device.
 *
 * Policy: first come first served; one prompt per iteration, whole, as the prefill chunk; a
 * request is admitted when a running slot and ceil((prompt_len + max_new_tokens) / 16) free pages
 * exist, and keeps those pages until the host learns that it finished. Admitted requests decode
 * in every iteration (rows in admission order), so none waits for a page or is preempted. */
typedef struct nf_sched nf_sched; /* opaque */

typedef struct {
    int32_t num_pages;    /* pages in each layer's KV pool, numbered 0 .. num_pages - 1 */
    int32_t max_running;  /* decode rows per iteration at most (<= the model's max_requests) */
    int32_t chunk_len;    /* prefill tokens per iteration at most; a prompt must fit one chunk.
                           * The model's max_tokens must be >= max_running + chunk_len. */
    int32_t max_position; /* prompt_len + max_new_tokens must not exceed it (the model's RoPE table) */
    int32_t lag;          /* 1: iteration i+1 is formed before iteration i completes (asynchronous);
                           * 0: after (synchronous) */
} nf_sched_config;

/* One formed iteration. The arrays belong to the scheduler and stay valid until the next
 * nf_sched_next call; they map one to one onto nf_batch_desc and nf_iter_io. */
typedef struct {
    int64_t iteration;           /* sequence number (0, 1, ...), -1 when num_tokens == 0 */
    int32_t num_decode;          /* R */
    int32_t prefill_len;         /* C (0: no prompt this iteration) */
    int32_t num_tokens;          /* T = R + C; 0: nothing to run now */
    int32_t rows;                /* next_token rows: R + (C > 0) */
    int32_t num_page_entries;    /* page_indptr[R + 1] */
    const int32_t* ctx_len;      /* [R] cached tokens per decode row */
    const int32_t* positions;    /* [T] */
    const int32_t* token_ids;    /* [T] prompt tokens on the chunk rows, -1 on decode rows */
    const int32_t* token_src;    /* [T] decode rows: their row in the previous iteration's next_token;
                                  * chunk rows: -1 */
    const int32_t* page_indptr;  /* [R + 2], prefill request last */
    const int32_t* page_indices; /* [num_page_entries] */
    const int64_t* row_request;  /* [rows] request id of each next_token row */
} nf_sched_iter;

typedef struct {
    int32_t waiting, running, finished, free_pages, inflight;
    int64_t iterations;       /* iterations formed */
    int64_t discarded_tokens; /* tokens decoded after a request's last one (one per request at lag 1) */
} nf_sched_stats;

/* NF_ERR_INVALID_ARGUMENT for a bad configuration. After NF_ERR_OUT_OF_MEMORY from any
 * nf_sched_* call the scheduler's state is unspecified: destroy it. */
nf_status nf_sched_create(const nf_sched_config* cfg, nf_sched** out);
void nf_sched_destroy(nf_sched* s);

/* Queue a request; the prompt is copied. eos_token < 0: none. NF_ERR_INVALID_ARGUMENT when
 * the request could never run (prompt longer than a chunk, prompt_len + max_new_tokens above
 * max_position, more pages than the pool). */
nf_status nf_sched_add_request(nf_sched* s, const int32_t* prompt, int32_t prompt_len, int32_t max_new_tokens,
                               int32_t eos_token, int64_t* id_out);

/* Form the next iteration. Iteration k may be formed only after iteration k - 1 - lag was
 * completed (else NF_ERR_INVALID_ARGUMENT). num_tokens == 0: nothing can run before another
 * completion (or every request has finished). */
nf_status nf_sched_next(nf_sched* s, nf_sched_iter* out);

/* Hand over the host copy of an iteration's next_token ([rows]); iterations complete in the
 * order they were formed. Finished requests release their pages. */
nf_status nf_sched_complete(nf_sched* s, int64_t iteration, const int32_t* next_token, int32_t rows);

/* Tokens generated so far for request `id` (the first min(cap, *len) are copied to out), and
 * whether it has finished (nullable). */
nf_status nf_sched_request_tokens(const nf_sched* s, int64_t id, int32_t* out, int32_t cap, int32_t* len,
                                  int32_t* finished);

nf_status nf_sched_get_stats(const nf_sched* s, nf_sched_stats* out);

/* Library version string. */
const char* nf_version(void);

#ifdef __cplusplus
}
#endif

#endif /* NANOFLOW_H */
