// The persistent device-scheduled layer kernel: one launch runs every operation of one layer of a
// plan, in the plan's issue order, on every SM, with completion counters in device memory in place of
// streams and events.
//
// NanoFlow's device-level pipeline (arXiv abstract; README "Introduction") runs the operations of
// different nano-batches in parallel inside one GPU. The stream executor (nf_forward_iteration) does
// that with one kernel launch per operation on two streams ordered by events, and with grids that
// claim disjoint SM sets. Here the same operations become the work of one persistent kernel: CTA b
// walks the layer's operation list, skips those of the other lane (attention CTAs: b < n_attn; GEMM
// CTAs: the rest; operations of LANE_ALL are run by every CTA), waits (bounded) until every CTA of
// the lane of each operation it depends on has finished that operation, runs its share (GEMM tiles
// and decode items are claimed from counters, so a CTA that finishes early takes more), and then
// counts itself finished. A CTA therefore moves on to the next operation as soon as it runs out of
// work in the current one, without waiting for a kernel boundary.
#pragma once
#include <cstdint>
#include <cuda.h>
#include <cuda_runtime.h>

#include "nf_attention.h"
#include "nf_internal.h"

namespace nf {

enum MegaKind : int {
    MEGA_QKV = 0,      // GEMM, EPI_QKV
    MEGA_RESID = 1,    // GEMM, EPI_RESID (O and down projections)
    MEGA_SWIGLU = 2,   // GEMM, EPI_SWIGLU (gate/up)
    MEGA_DECODE = 3,   // tensor-core decode attention
    MEGA_MERGE = 4,    // split-KV merge of the decode chunks
    MEGA_PREFILL = 5,  // tensor-core causal attention of the prefill chunk
    MEGA_NOP = 6,      // no work (self tests of the scheduling)
};

enum MegaLane : int { LANE_ALL = 0, LANE_GEMM = 1, LANE_ATTN = 2 };

constexpr int kMegaMaxOps = 28;      // 7 operations per nano-batch, NF_MAX_NANO nano-batches
constexpr int kMegaMaxDeps = 3;
constexpr int kMegaThreads = 256;
constexpr uint32_t kMegaTmemCols = 512;
constexpr int kMegaCountersPerLayer = 64;  // done[kMegaMaxOps] then claim[kMegaMaxOps], padded

struct alignas(64) MegaOp {
    CUtensorMap tmA;  // GEMM: A operand; attention: q
    CUtensorMap tmB;  // GEMM: B operand (weights); unused otherwise
    int kind;         // MegaKind
    int lane;         // MegaLane
    int dep[kMegaMaxDeps];  // earlier operations of the launch that must be finished, -1 = none
    union {
        GemmArgs g;
        DecodeArgs d;
        PrefillArgs p;
    };
};

struct MegaParams {
    MegaOp ops[kMegaMaxOps];
    int n_ops;
    int n_attn;     // CTAs [0, n_attn) form the attention lane (0: every operation is LANE_ALL)
    int* done;      // [n_ops], zeroed: CTAs of the operation's lane that have finished it
    int* status;
    unsigned long long wait_limit_ns;  // limit of each dependency wait (0: NF_WAIT_LIMIT_NS)
    int* trace_ctr;  // per-CTA, per-operation trace (nullable)
    nf_trace_entry* trace;
    int trace_cap;
};
static_assert(sizeof(MegaParams) <= 32000, "kernel parameters");

// Dynamic shared memory of the kernel (the largest of its bodies).
int mega_smem_bytes(int nq);
// Launches the layer kernel on `grid` CTAs (at most one per SM, all resident at once). nq: 32 or 64.
cudaError_t launch_mega(const MegaParams& p, int nq, int grid, cudaStream_t stream);

}  // namespace nf
