// Planner: nano-batch count, sizes, pipeline order and SM split by exhaustive search
// over a per-kernel cost model, replacing the external MILP solver of the reference
// design. NanoFlow picks how many nano-batches to use, how large each is, the order
// of their operations and how the GPU is divided between them so that the iteration
// is shortest, taking into account how concurrent operations slow one another
// (arXiv abstract; README "Abstract": an offline parameter search configures the
// pipeline).
//
// Candidates: n in 1..4 nano-batches; decode rows cut at request boundaries into
// groups of equal KV bytes; the prefill chunk either its own nano-batch or joined to
// the last decode group; pipeline order natural or prefill first; SM split for
// attention in steps of 4; template sequential or pipelined. With one nano-batch the
// prefill-on-GEMM template still overlaps something: the decode attention (HBM-bound) on
// sm_attn SMs beside the prefill attention (tensor-bound) on the others. Each candidate's
// op list (build_ops) is simulated on two streams; the minimum makespan wins.
#include <new>
#include <algorithm>
#include <cmath>
#include <cstring>
#include <vector>

#include "nf_attention.h"
#include "nf_model.h"
#include "nf_schedule.h"

namespace nf {

int64_t decode_work_items(const ModelDims& d, const int32_t* ctx_len, int R) {
    const bool tc = decode_tc_supported(d.nq, d.nkv, d.d);
    const int per = tc ? 1 : d.nkv;
    const int split = tc ? kDecodeSplitPagesTcHost : kDecodeSplitPagesHost;
    int64_t items = 0;
    for (int r = 0; r < R; ++r) {
        const int np = (std::max(ctx_len[r], 0) + 1 + 15) / 16;
        items += (int64_t)per * ((np + split - 1) / split);
    }
    return items;
}

void nano_content(const nf_plan& p, bool* has_dec, bool* has_pre) {
    for (int j = 0; j < p.n_nano; ++j) {
        has_dec[j] = p.tok_begin[j] < p.num_decode;
        has_pre[j] = p.tok_end[j] > p.num_decode && p.prefill_len > 0;
    }
}

void mark_elastic(std::vector<Op>& ops);

std::vector<Op> build_ops(int tmpl, int n, const int* order, int L, bool moe, const bool* has_dec,
                          const bool* has_pre) {
    std::vector<Op> ops;
    auto push = [&](int kind, int stream, int j, int l) {
        Op o{kind, stream, j, l, 0, 0, -1, 0};
        ops.push_back(o);
        return (int)ops.size() - 1;
    };
    auto push_ffn = [&](int j, int l) {
        if (moe) {
            push(OP_MOE, STREAM_GEMM, j, l);
        } else {
            push(OP_GU, STREAM_GEMM, j, l);
            push(OP_D, STREAM_GEMM, j, l);
        }
    };
    if (tmpl == NF_TEMPLATE_SEQUENTIAL) {
        for (int l = 0; l < L; ++l)
            for (int i = 0; i < n; ++i) {
                const int j = order[i];
                push(OP_QKV, STREAM_GEMM, j, l);
                if (has_dec[j]) push(OP_DATT, STREAM_GEMM, j, l);
                if (has_pre[j]) push(OP_PATT, STREAM_GEMM, j, l);
                push(OP_O, STREAM_GEMM, j, l);
                push_ffn(j, l);
            }
        for (auto& o : ops) o.full_sm = 1;
        return ops;
    }
    // Pipelined: decode attention of (j, l) on the attention stream right after QKV(j, l);
    // prefill attention on the attention stream too, or (NF_TEMPLATE_PREFILL_ON_GEMM) on the
    // GEMM stream right before O(j, l). O(j, l) waits for the attention-stream ops of (j, l);
    // QKV(j, l+1) follows the FFN of (j, l) on the GEMM stream.
    const bool pre_on_gemm = tmpl == NF_TEMPLATE_PREFILL_ON_GEMM;
    std::vector<int> last_a((size_t)n * L, -1);
    auto issue_qkv = [&](int j, int l) {
        const int q = push(OP_QKV, STREAM_GEMM, j, l);
        int prev = q;
        if (has_dec[j]) {
            const int a = push(OP_DATT, STREAM_ATTN, j, l);
            ops[a].wait = q;
            ops[q].signal = 1;
            prev = a;
            last_a[(size_t)l * n + j] = a;
        }
        if (has_pre[j] && !pre_on_gemm) {
            const int a = push(OP_PATT, STREAM_ATTN, j, l);
            if (prev == q) { ops[a].wait = q; ops[q].signal = 1; }
            last_a[(size_t)l * n + j] = a;
        }
    };
    // first layer: nano-batches with attention-stream work get their QKV first
    for (int pass = 0; pass < 2; ++pass)
        for (int i = 0; i < n; ++i) {
            const int j = order[i];
            const bool a_work = has_dec[j] || (has_pre[j] && !pre_on_gemm);
            if ((pass == 0) == a_work) issue_qkv(j, 0);
        }
    for (int l = 0; l < L; ++l) {
        for (int i = 0; i < n; ++i) {
            const int j = order[i];
            if (has_pre[j] && pre_on_gemm) push(OP_PATT, STREAM_GEMM, j, l);
            const int o = push(OP_O, STREAM_GEMM, j, l);
            const int a = last_a[(size_t)l * n + j];
            if (a >= 0) { ops[o].wait = a; ops[a].signal = 1; }
            push_ffn(j, l);
            if (l + 1 < L) issue_qkv(j, l + 1);
        }
    }
    // A GEMM-stream op may take every SM iff it lies in no attention window: an
    // attention-stream op can only run between the end of its QKV and the start of its O.
    std::vector<int> gpos(ops.size(), -1);
    int g = 0;
    for (size_t i = 0; i < ops.size(); ++i)
        if (ops[i].stream == STREAM_GEMM) gpos[i] = g++;
    std::vector<int> covered(g + 1, 0);
    for (size_t i = 0; i < ops.size(); ++i) {
        if (ops[i].stream != STREAM_ATTN) continue;
        int q = -1;  // QKV of the same (j, l)
        for (int k = (int)i - 1; k >= 0; --k)
            if (ops[k].kind == OP_QKV && ops[k].nano == ops[i].nano && ops[k].layer == ops[i].layer) { q = k; break; }
        int o = -1;
        for (size_t k = i + 1; k < ops.size(); ++k)
            if (ops[k].kind == OP_O && ops[k].nano == ops[i].nano && ops[k].layer == ops[i].layer) { o = (int)k; break; }
        const int lo = gpos[q] + 1, hi = (o >= 0 ? gpos[o] : g);  // G ops in [lo, hi) may overlap
        for (int x = lo; x < hi; ++x) covered[x] = 1;
    }
    for (size_t i = 0; i < ops.size(); ++i)
        if (ops[i].stream == STREAM_GEMM) ops[i].full_sm = covered[gpos[i]] ? 0 : 1;
    mark_elastic(ops);
    return ops;
}

// A dense GEMM op inside an attention window may run elastically when that window holds exactly one
// attention op A that is already resident when the GEMM starts: A's QKV is not the GEMM's immediate
// predecessor on the GEMM stream (A is launched the moment that QKV completes), and the attention op
// queued before A on its stream was consumed by a GEMM-stream op that completes before the GEMM's
// predecessor does (so A started earlier). A GEMM holding every free SM then cannot delay any
// attention kernel's start, since none starts while it runs.
void mark_elastic(std::vector<Op>& ops) {
    const int n = (int)ops.size();
    std::vector<int> consumer(n, n), prev_attn(n, -1), prev_gemm(n, -1);
    int last_a = -1, last_g = -1;
    for (int i = 0; i < n; ++i) {
        if (ops[i].wait >= 0) consumer[ops[i].wait] = std::min(consumer[ops[i].wait], i);
        if (ops[i].stream == STREAM_ATTN) { prev_attn[i] = last_a; last_a = i; }
        else { prev_gemm[i] = last_g; last_g = i; }
    }
    // consumer of an attention op: the first GEMM-stream op that waits for it
    for (int g = 0; g < n; ++g) {
        Op& o = ops[g];
        if (o.stream != STREAM_GEMM || o.full_sm) continue;
        if (!(o.kind == OP_QKV || o.kind == OP_O || o.kind == OP_GU || o.kind == OP_D)) continue;
        int open = 0, a = -1;
        for (int i = 0; i < g; ++i)
            if (ops[i].stream == STREAM_ATTN && consumer[i] > g) { ++open; a = i; }
        if (open != 1) continue;
        const int trigger = ops[a].wait;  // the QKV that A waits for
        if (prev_gemm[g] < 0 || prev_gemm[g] == trigger) continue;
        const int pa = prev_attn[a];
        if (pa >= 0 && !(consumer[pa] < prev_gemm[g])) continue;
        o.elastic = 1;
    }
}

namespace {
// piecewise-linear interpolation of y at x over increasing knots xs (clamped at the ends)
double interp(const double* xs, const double* ys, int n, double x) {
    if (x <= xs[0]) return ys[0];
    for (int i = 1; i < n; ++i)
        if (x <= xs[i]) return ys[i - 1] + (ys[i] - ys[i - 1]) * (x - xs[i - 1]) / (xs[i] - xs[i - 1]);
    return ys[n - 1];
}
constexpr double kBwShares[5] = {0.125, 0.25, 0.5, 0.75, 1.0};
constexpr double kCoShares[3] = {0.25, 0.5, 0.75};
}  // namespace

double attn_bw(const CostModel& c, int grid, int sms) {
    const double model = std::min(c.hbm_bw, grid * c.attn_bw_per_sm);
    for (int i = 0; i < 5; ++i)
        if (c.attn_bw_at[i] <= 0) return model;
    const double x = (double)grid / std::max(1, sms);
    if (x < kBwShares[0]) return c.attn_bw_at[0] * x / kBwShares[0];  // per-SM-bound below the table
    return interp(kBwShares, c.attn_bw_at, 5, x);
}

double interf_attn(const CostModel& c, int sm_attn, int sms) {
    if (c.interf_attn[0] <= 0 && c.interf_attn[1] <= 0 && c.interf_attn[2] <= 0) return c.interference;
    return interp(kCoShares, c.interf_attn, 3, (double)sm_attn / std::max(1, sms));
}

double interf_gemm(const CostModel& c, int sm_attn, int sms) {
    if (c.interf_gemm[0] <= 0 && c.interf_gemm[1] <= 0 && c.interf_gemm[2] <= 0) return c.interference;
    return interp(kCoShares, c.interf_gemm, 3, (double)sm_attn / std::max(1, sms));
}

CostModel default_cost_model(int sms) {
    CostModel c;
    for (int i = 0; i < 5; ++i) c.attn_bw_at[i] = 0;
    for (int i = 0; i < 3; ++i) c.interf_attn[i] = c.interf_gemm[i] = 0;
    if (sms <= 0) sms = 148;
    c.gemm_flops_per_sm = 1.30e15 / 148.0;  // ~78% of the measured cuBLAS bf16 peak
    c.gemm_tile_us = 0.8;
    c.gemm_launch_us = 3.0;
    c.hbm_bw = 6.0e12;
    c.attn_bw_per_sm = 110e9;
    c.attn_launch_us = 4.0;
    c.attn_flops_per_sm = 2.0e12;
    c.interference = 0.08;
    c.calibrated = 0;
    c.iter_scale = 1.0;
    c.power_floor = 0.0;
    return c;
}

namespace {

double gemm_us(const CostModel& c, int M, int N, int K, int grid, int64_t weight_bytes) {
    if (M <= 0) return 0.0;
    // dense GEMMs run on CTA pairs with 256 x 256 tiles: two 128-row halves per pair tile
    const int64_t tiles = (int64_t)2 * ((M + 255) / 256) * (N / 256);
    const int g = std::max(1, std::min<int>(grid, (int)tiles));
    const int64_t waves = (tiles + g - 1) / g;
    const double t_tile = 2.0 * 128 * 256 * (double)K / c.gemm_flops_per_sm * 1e6 + c.gemm_tile_us;
    const double t_compute = waves * t_tile;
    const double bw = std::min(c.hbm_bw, g * c.attn_bw_per_sm * 1.2);
    const double t_mem = (double)weight_bytes / bw * 1e6;
    return c.gemm_launch_us + std::max(t_compute, t_mem);
}

}  // namespace

int op_grid(const nf_plan& p, const Op& o) {
    if (p.order_template == NF_TEMPLATE_SEQUENTIAL) return p.sm_total;
    if (o.stream == STREAM_ATTN) return p.sm_attn;
    return (o.full_sm || o.elastic) ? p.sm_total : p.sm_gemm;
}

double op_time_us(int kind, int j, const nf_plan& p, const ModelDims& m, const BatchInfo& b, const CostModel& c,
                  int grid) {
    const int t0 = p.tok_begin[j], t1 = p.tok_end[j];
    const int M = t1 - t0;
    if (M <= 0) return 0.0;
    switch (kind) {
        case OP_QKV: return gemm_us(c, M, m.qkv, m.H, grid, (int64_t)m.qkv * m.H * 2);
        case OP_O: return gemm_us(c, M, m.H, m.nq * m.d, grid, (int64_t)m.H * m.nq * m.d * 2);
        case OP_GU: return gemm_us(c, M, 2 * m.F, m.H, grid, (int64_t)2 * m.F * m.H * 2);
        case OP_D: return gemm_us(c, M, m.H, m.F, grid, (int64_t)m.H * m.F * 2);
        case OP_MOE: {
            const int rows = M * m.K;
            const int per = std::max(1, rows / std::max(1, m.E));
            double t = 0;
            // E groups of ~rows/E rows; weights of every expert are read once
            t += gemm_us(c, per, 2 * m.F, m.H, std::max(1, grid / std::max(1, m.E)), (int64_t)2 * m.F * m.H * 2);
            t += gemm_us(c, per, m.H, m.F, std::max(1, grid / std::max(1, m.E)), (int64_t)m.H * m.F * 2);
            return t + 20.0;
        }
        case OP_DATT: {
            const int r0 = std::min(t0, b.R), r1 = std::min(t1, b.R);
            const int64_t bytes = b.req_kv_prefix[r1] - b.req_kv_prefix[r0];
            if (bytes <= 0) return 0.0;
            return c.attn_launch_us + (double)bytes / attn_bw(c, grid, p.sm_total) * 1e6;
        }
        case OP_PATT: {
            if (!(t1 > b.R && b.C > 0)) return 0.0;
            const double flops = 4.0 * m.nq * m.d * (double)b.C * (b.C + 1) / 2.0;
            return c.attn_launch_us + flops / (grid * c.attn_flops_per_sm) * 1e6;
        }
    }
    return 0.0;
}

double simulate_plan(const nf_plan& p, const ModelDims& m, const BatchInfo& b, const CostModel& c,
                     double* serial_us) {
    int order[NF_MAX_NANO];
    for (int i = 0; i < p.n_nano; ++i) order[i] = p.nano_order[i];
    bool has_dec[NF_MAX_NANO], has_pre[NF_MAX_NANO];
    nano_content(p, has_dec, has_pre);
    const std::vector<Op> ops = build_ops(p.order_template, p.n_nano, order, m.L, m.E > 0, has_dec, has_pre);
    const int S = p.sm_total;
    const bool pipelined = p.order_template != NF_TEMPLATE_SEQUENTIAL;
    std::vector<double> dur(ops.size()), beg(ops.size()), end(ops.size());
    double serial = 0.0;
    std::vector<double> dur_gemm_share(ops.size(), 0.0);  // elastic ops: time on the GEMM share alone
    for (size_t i = 0; i < ops.size(); ++i) {
        const Op& o = ops[i];
        const int grid = op_grid(p, o);
        dur[i] = op_time_us(o.kind, o.nano, p, m, b, c, grid);
        if (o.elastic) dur_gemm_share[i] = op_time_us(o.kind, o.nano, p, m, b, c, p.sm_gemm);
        serial += op_time_us(o.kind, o.nano, p, m, b, c, S);
    }
    const double scale = c.iter_scale > 0 ? c.iter_scale : 1.0;
    if (serial_us) *serial_us = serial * scale;
    double makespan = 0.0;
    for (int pass = 0; pass < 2; ++pass) {
        double free_t[2] = {0.0, 0.0};
        double attn_end = 0.0;  // end of the latest attention op scheduled so far
        for (size_t i = 0; i < ops.size(); ++i) {
            const Op& o = ops[i];
            double st = free_t[o.stream];
            if (o.wait >= 0) st = std::max(st, end[o.wait]);
            beg[i] = st;
            double d = dur[i];
            if (o.elastic && st < attn_end && dur_gemm_share[i] > 0) {
                // on the GEMM share until the open attention op ends, then on every SM
                const double full = dur[i], part = dur_gemm_share[i];
                const double span = attn_end - st;
                d = span >= part ? part : span + (1.0 - span / part) * full;
            }
            end[i] = st + d;
            free_t[o.stream] = end[i];
            if (o.stream == STREAM_ATTN) attn_end = std::max(attn_end, end[i]);
        }
        makespan = std::max(free_t[0], free_t[1]);
        if (pass == 0 && pipelined) {
            // inflate each op by the interference factor times the fraction of it that overlaps the other stream
            std::vector<std::pair<double, double>> other[2];
            for (size_t i = 0; i < ops.size(); ++i) other[ops[i].stream].push_back({beg[i], end[i]});
            for (size_t i = 0; i < ops.size(); ++i) {
                if (dur[i] <= 0) continue;
                double ov = 0;
                for (auto& iv : other[1 - ops[i].stream])
                    ov += std::max(0.0, std::min(end[i], iv.second) - std::max(beg[i], iv.first));
                const double k = ops[i].stream == STREAM_ATTN ? interf_attn(c, p.sm_attn, p.sm_total)
                                                              : interf_gemm(c, p.sm_attn, p.sm_total);
                const double f = 1.0 + k * std::min(1.0, ov / dur[i]);
                dur[i] *= f;
                dur_gemm_share[i] *= f;
            }
        } else {
            break;
        }
    }
    // energy bound: under a power cap the plan runs no faster than its kernels' energy allows
    if (c.power_floor > 0) makespan = std::max(makespan, c.power_floor * serial);
    return makespan * scale;
}

}  // namespace nf

// ------------------------------------------------------------------ C ABI entry point

namespace {

nf::BatchInfo batch_info(const nf_model* m, const nf_batch_desc* b) {
    nf::BatchInfo bi;
    bi.R = b->num_decode;
    bi.C = b->prefill_len;
    bi.T = bi.R + bi.C;
    bi.req_kv_bytes.resize(bi.R);
    bi.req_kv_prefix.assign(bi.R + 1, 0);
    const int64_t page_bytes = 2LL * 16 * m->dims.d * 2 * m->dims.nkv;  // K and V of all KV heads
    for (int r = 0; r < bi.R; ++r) {
        const int64_t pages = (b->ctx_len[r] + 1 + 15) / 16;
        bi.req_kv_bytes[r] = pages * page_bytes;
        bi.req_kv_prefix[r + 1] = bi.req_kv_prefix[r] + bi.req_kv_bytes[r];
    }
    return bi;
}

// Cut decode requests [0, R) into `groups` contiguous ranges of near-equal KV bytes.
std::vector<int> split_requests(const nf::BatchInfo& bi, int groups) {
    std::vector<int> cut(groups + 1, 0);
    cut[groups] = bi.R;
    const int64_t total = bi.req_kv_prefix[bi.R];
    for (int g = 1; g < groups; ++g) {
        const int64_t target = total * g / groups;
        int r = (int)(std::lower_bound(bi.req_kv_prefix.begin(), bi.req_kv_prefix.end(), target) -
                      bi.req_kv_prefix.begin());
        r = std::max(cut[g - 1], std::min(r, bi.R));
        cut[g] = r;
    }
    return cut;
}

}  // namespace

namespace {
nf_status plan_impl(const nf_model* m, const nf_batch_desc* b, const nf_plan_opts* opts, nf_plan* out);
}

extern "C" nf_status nf_plan_iteration(const nf_model* m, const nf_batch_desc* b, const nf_plan_opts* opts,
                                       nf_plan* out) try {
    return plan_impl(m, b, opts, out);
} catch (const std::bad_alloc&) {
    return NF_ERR_OUT_OF_MEMORY;
} catch (...) {
    return NF_ERR_INVALID_ARGUMENT;
}

extern "C" nf_status nf_plan_for_config(const nf_model_config* cfg, int32_t sm_count, const nf_batch_desc* b,
                                        const nf_plan_opts* opts, nf_plan* out) try {
    if (cfg == nullptr || sm_count <= 0) return NF_ERR_INVALID_ARGUMENT;
    nf_model m;
    m.cfg = *cfg;
    m.dims.L = cfg->n_layers;
    m.dims.H = cfg->hidden;
    m.dims.nq = cfg->n_q_heads;
    m.dims.nkv = cfg->n_kv_heads;
    m.dims.d = cfg->head_dim;
    m.dims.F = cfg->ffn;
    m.dims.E = cfg->n_experts;
    m.dims.K = cfg->n_experts > 0 ? cfg->top_k : 1;
    m.dims.qkv = (cfg->n_q_heads + 2 * cfg->n_kv_heads) * cfg->head_dim;
    m.sm_count = sm_count;
    m.cost = nf::default_cost_model(sm_count);
    if (m.dims.nkv <= 0 || m.dims.L <= 0) return NF_ERR_INVALID_ARGUMENT;
    return plan_impl(&m, b, opts, out);
} catch (const std::bad_alloc&) {
    return NF_ERR_OUT_OF_MEMORY;
} catch (...) {
    return NF_ERR_INVALID_ARGUMENT;
}

namespace {
nf_status plan_impl(const nf_model* m, const nf_batch_desc* b, const nf_plan_opts* opts, nf_plan* out) {
    if (m == nullptr || b == nullptr || out == nullptr) return NF_ERR_INVALID_ARGUMENT;
    const int R = b->num_decode, C = b->prefill_len;
    if (R < 0 || C < 0 || R + C <= 0 || b->prefix_len != 0) return NF_ERR_INVALID_ARGUMENT;
    if (R + C > m->cfg.max_tokens || R > m->cfg.max_requests) return NF_ERR_INVALID_ARGUMENT;
    if (R > 0 && (b->ctx_len == nullptr)) return NF_ERR_INVALID_ARGUMENT;
    if (b->page_indptr == nullptr) return NF_ERR_INVALID_ARGUMENT;
    // Page-table validation: every request holds enough pages, offsets are monotone.
    for (int r = 0; r <= R; ++r) {
        const int keys = r < R ? b->ctx_len[r] + 1 : C;
        if (r < R && (b->ctx_len[r] < 0 || b->ctx_len[r] + 1 > m->cfg.max_position)) return NF_ERR_INVALID_ARGUMENT;
        const int have = b->page_indptr[r + 1] - b->page_indptr[r];
        if (have < 0 || have < (keys + 15) / 16) return NF_ERR_INVALID_ARGUMENT;
    }
    if (b->page_indptr[0] != 0 || b->num_pages <= 0) return NF_ERR_INVALID_ARGUMENT;
    // every page id a request owns must address the pool (checked here, before any launch)
    if (b->page_indices == nullptr && b->page_indptr[R + 1] > 0) return NF_ERR_INVALID_ARGUMENT;
    for (int i = 0; i < b->page_indptr[R + 1]; ++i)
        if (b->page_indices[i] < 0 || b->page_indices[i] >= b->num_pages) return NF_ERR_INVALID_ARGUMENT;

    nf_plan_opts o;
    if (opts) o = *opts; else { std::memset(&o, 0, sizeof(o)); o.force_template = -1; }
    const int S = o.sm_total > 0 ? std::min(o.sm_total, m->sm_count) : m->sm_count;
    const nf::BatchInfo bi = batch_info(m, b);
    const nf::CostModel& cm = m->cost;

    nf_plan best;
    std::memset(&best, 0, sizeof(best));
    double best_t = 1e30;
    int n_lo = 1, n_hi = NF_MAX_NANO;
    if (o.force_nano > 0) n_lo = n_hi = std::min(o.force_nano, NF_MAX_NANO);

    for (int n = n_lo; n <= n_hi; ++n) {
        for (int prefill_alone = 0; prefill_alone <= 1; ++prefill_alone) {
            if (prefill_alone && (C == 0 || R == 0 || n < 2)) continue;
            const int dgroups = prefill_alone ? n - 1 : n;
            if (dgroups > std::max(R, 1)) continue;
            if (R == 0 && n > 1) continue;
            nf_plan p;
            std::memset(&p, 0, sizeof(p));
            p.n_nano = n;
            p.num_decode = R;
            p.prefill_len = C;
            p.num_tokens = R + C;
            p.sm_total = S;
            const std::vector<int> cut = split_requests(bi, std::max(dgroups, 1));
            for (int g = 0; g < dgroups; ++g) {
                p.tok_begin[g] = cut[g];
                p.tok_end[g] = cut[g + 1];
            }
            if (prefill_alone) {
                p.tok_begin[n - 1] = R;
                p.tok_end[n - 1] = R + C;
            } else {
                p.tok_end[dgroups - 1] = R + C;
            }
            bool degenerate = false;
            for (int j = 0; j < n; ++j)
                if (p.tok_end[j] <= p.tok_begin[j]) degenerate = true;
            if (degenerate) continue;
            int perm[NF_MAX_NANO];
            for (int i = 0; i < n; ++i) perm[i] = i;
            do {
                for (int i = 0; i < n; ++i) p.nano_order[i] = perm[i];
                for (int tmpl = 0; tmpl <= 2; ++tmpl) {
                    if (o.force_template >= 0 && tmpl != o.force_template) continue;
                    // one nano-batch overlaps only with the prefill attention on the GEMM stream beside
                    // the decode attention (two attention kernels bound by different units)
                    if (tmpl != NF_TEMPLATE_SEQUENTIAL && n < 2 && !(tmpl == NF_TEMPLATE_PREFILL_ON_GEMM && R > 0))
                        continue;
                    if (tmpl == NF_TEMPLATE_PREFILL_ON_GEMM && C == 0) continue;
                    if (tmpl == NF_TEMPLATE_SEQUENTIAL && perm[0] != 0) continue;  // order is irrelevant
                    p.order_template = tmpl;
                    int a_lo = 8, a_hi = S - 8, a_step = 4;
                    if (tmpl == NF_TEMPLATE_SEQUENTIAL) { a_lo = a_hi = 0; }
                    if (o.force_sm_attn > 0 && tmpl != NF_TEMPLATE_SEQUENTIAL)
                        a_lo = a_hi = std::min(o.force_sm_attn, S - 4);
                    for (int sa = a_lo; sa <= a_hi; sa += a_step) {
                        p.sm_attn = tmpl == NF_TEMPLATE_SEQUENTIAL ? S : sa;
                        p.sm_gemm = tmpl == NF_TEMPLATE_SEQUENTIAL ? S : S - sa;
                        double serial = 0;
                        const double t = nf::simulate_plan(p, m->dims, bi, cm, &serial);
                        if (t < best_t) {
                            best_t = t;
                            best = p;
                            best.predicted_us = (float)t;
                            best.predicted_serial_us = (float)serial;
                        }
                    }
                }
            } while (std::next_permutation(perm, perm + n));
        }
    }
    if (best.n_nano == 0) return NF_ERR_INVALID_ARGUMENT;
    int64_t pages = 0;
    for (int r = 0; r < R; ++r) pages += (b->ctx_len[r] + 1 + 15) / 16;
    pages += (C + 15) / 16;
    best.kv_pages_read = pages;
    best.decode_items = nf::decode_work_items(m->dims, b->ctx_len, R);
    *out = best;
    return NF_OK;
}
}  // namespace
