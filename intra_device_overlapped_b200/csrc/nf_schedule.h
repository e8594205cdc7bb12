// The iteration as a list of operations on two streams, shared by the planner's
// simulator and the executor so that what is simulated is exactly what runs.
#pragma once
#include <cstdint>
#include <vector>

#include "nanoflow.h"

namespace nf {

enum OpKind : int { OP_QKV = 0, OP_DATT = 1, OP_O = 2, OP_GU = 3, OP_D = 4, OP_MOE = 5, OP_PATT = 6 };
enum StreamId : int { STREAM_GEMM = 0, STREAM_ATTN = 1 };

struct Op {
    int kind;
    int stream;
    int nano;
    int layer;
    int full_sm;  // 1: no attention can co-run, the op may use every SM
    int elastic;  // 1: a GEMM launched on every SM with work claimed from a counter: it runs on the SMs
                  // the one attention kernel open beside it leaves free and grows onto the rest when
                  // that kernel ends (never set where another attention kernel could start meanwhile)
    int wait;     // index (in issue order) of an op on the other stream to wait for, -1 = none
    int signal;   // 1: some later op waits for this one
};

// Issue order of every operation of the iteration (excluding the prologue and the LM head).
// `order` lists the nano-batches in pipeline order; has_dec[j] / has_pre[j] say whether
// nano-batch j holds decode rows / the prefill chunk.
std::vector<Op> build_ops(int tmpl, int n_nano, const int* order, int n_layers, bool moe, const bool* has_dec,
                          const bool* has_pre);

// has_dec / has_pre of every nano-batch of a plan
void nano_content(const nf_plan& p, bool* has_dec, bool* has_pre);

// Per-kernel cost model used by the planner (microseconds, bytes, FLOPs).
struct CostModel {
    double gemm_flops_per_sm;   // sustained tensor FLOP/s of one SM in the GEMM main loop
    double gemm_tile_us;        // fixed per-tile cost (epilogue tail, pipeline fill)
    double gemm_launch_us;
    double hbm_bw;              // bytes/s, whole device
    double attn_bw_per_sm;      // bytes/s one attention SM can pull
    double attn_launch_us;
    double attn_flops_per_sm;   // prefill attention tensor FLOP/s per SM
    double interference;        // fractional slow-down of two co-running kernels (fallback)
    int calibrated;
    double attn_bw_at[5];       // decode bytes/s on 1/8, 1/4, 1/2, 3/4, 1 of the SMs (0 = not measured)
    double interf_attn[3];      // decode slow-down beside GEMMs, attention on 1/4, 1/2, 3/4 of the SMs
    double interf_gemm[3];      // GEMM slow-down beside decode attention, same shares
    double iter_scale;          // measured / predicted sequential iteration (sustained clock), 1 = none
    double power_floor;         // predicted time >= power_floor x serial time (0 = none)
};

// Decode attention bytes/s on `grid` of `sms` SMs (measured table, else the per-SM / HBM model) and
// the co-run slow-downs at attention share `sm_attn` / `sms`.
double attn_bw(const CostModel& c, int grid, int sms);
double interf_attn(const CostModel& c, int sm_attn, int sms);
double interf_gemm(const CostModel& c, int sm_attn, int sms);

CostModel default_cost_model(int sm_count);

struct ModelDims {
    int L, H, nq, nkv, d, F, E, K, qkv;
};

struct BatchInfo {
    int R, C, T;
    std::vector<int64_t> req_kv_bytes;  // decode KV bytes read per request per layer
    std::vector<int64_t> req_kv_prefix; // prefix sums of req_kv_bytes
};

// Simulated makespan (us) of a plan; also returns the no-overlap time.
double simulate_plan(const nf_plan& p, const ModelDims& m, const BatchInfo& b, const CostModel& c,
                     double* serial_us);

int op_grid(const nf_plan& p, const Op& o);

double op_time_us(int kind, int nano, const nf_plan& p, const ModelDims& m, const BatchInfo& b, const CostModel& c,
                  int grid);

}  // namespace nf
