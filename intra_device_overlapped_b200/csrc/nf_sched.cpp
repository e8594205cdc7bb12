// Host-side serving scheduler: the CPU control flow around nf_forward_iteration.
//
// NanoFlow keeps the GPU busy by scheduling iteration i+1 on the CPU while the GPU still runs
// iteration i. The CPU therefore forms a batch before it knows which requests the previous
// iteration finished. A request that produced its end-of-sequence token (or its last allowed
// token) in iteration i is still decoded once more in iteration i+1, and that extra token is
// dropped; it leaves the batch from iteration i+2 on (README "Abstract" and arXiv abstract:
// asynchronous CPU scheduling hides the CPU's share of an iteration). `lag` = 1 gives that
// order, `lag` = 0 the synchronous one (iteration i completes before i+1 is formed).
//
// Policy (the pages fix none of it): requests are admitted first come first served, one
// prompt per iteration as the prefill chunk, when a running slot and the pages for the
// request's whole life (prompt + max_new_tokens slots, the extra token included) are free.
// Admitted requests decode every iteration until they finish; their pages return to the pool
// when the host learns that they finished. Reserving at admission means no request ever
// waits for a page or is preempted once it runs.
#include <algorithm>
#include <cstring>
#include <deque>
#include <new>
#include <unordered_map>
#include <vector>

#include "nanoflow.h"

struct nf_sched {
    struct Request {
        int64_t id;
        std::vector<int32_t> prompt;
        int32_t max_new;
        int32_t eos;
        std::vector<int32_t> pages;   // reserved at admission, page j holds slots 16 j .. 16 j + 15
        std::vector<int32_t> out;     // generated tokens known on the host
        int32_t n_cached = 0;         // slots whose K/V the scheduled iterations write
        int32_t last_row = -1;        // row of this request in the last scheduled iteration's next_token
        bool admitted = false;
        bool finished = false;        // known on the host (EOS or max_new reached)
    };
    struct Inflight {
        int64_t iteration;
        std::vector<int64_t> row_request;
    };

    nf_sched_config cfg;
    std::unordered_map<int64_t, Request> reqs;
    std::deque<int64_t> waiting;      // FIFO of requests not yet admitted
    std::vector<int64_t> running;     // admitted and not known finished, in admission order
    std::vector<int32_t> free_pages;  // stack of free page ids
    std::deque<Inflight> inflight;    // scheduled, not yet completed (in iteration order)
    int64_t next_id = 0;
    int64_t next_iter = 0;            // sequence number of the next iteration to form
    int64_t next_complete = 0;        // the next iteration nf_sched_complete must receive
    int64_t discarded = 0;
    int64_t finished_count = 0;

    // arrays of the last formed iteration
    std::vector<int32_t> ctx_len, positions, token_ids, token_src, page_indptr, page_indices;
    std::vector<int64_t> row_request;

    int32_t pages_for(const Request& r) const {
        return (int32_t)((r.prompt.size() + (size_t)r.max_new + 15) / 16);
    }
};

namespace {

bool valid_config(const nf_sched_config& c) {
    return c.num_pages > 0 && c.max_running > 0 && c.chunk_len > 0 && c.max_position > 1 &&
           (c.lag == 0 || c.lag == 1);
}

}  // namespace

extern "C" nf_status nf_sched_create(const nf_sched_config* cfg, nf_sched** out) try {
    if (!cfg || !out || !valid_config(*cfg)) return NF_ERR_INVALID_ARGUMENT;
    nf_sched* s = new (std::nothrow) nf_sched();
    if (!s) return NF_ERR_OUT_OF_MEMORY;
    s->cfg = *cfg;
    s->free_pages.reserve((size_t)cfg->num_pages);
    for (int32_t p = cfg->num_pages - 1; p >= 0; --p) s->free_pages.push_back(p);  // page 0 handed out first
    *out = s;
    return NF_OK;
} catch (const std::bad_alloc&) {
    return NF_ERR_OUT_OF_MEMORY;
} catch (...) {
    return NF_ERR_INVALID_ARGUMENT;
}

extern "C" void nf_sched_destroy(nf_sched* s) { delete s; }

extern "C" nf_status nf_sched_add_request(nf_sched* s, const int32_t* prompt, int32_t prompt_len,
                                          int32_t max_new_tokens, int32_t eos_token, int64_t* id_out) try {
    if (!s || !prompt || !id_out || prompt_len < 1 || max_new_tokens < 1) return NF_ERR_INVALID_ARGUMENT;
    if (prompt_len > s->cfg.chunk_len) return NF_ERR_INVALID_ARGUMENT;          // one prompt = one chunk
    if ((int64_t)prompt_len + max_new_tokens > s->cfg.max_position) return NF_ERR_INVALID_ARGUMENT;
    nf_sched::Request r;
    r.id = s->next_id++;
    r.prompt.assign(prompt, prompt + prompt_len);
    r.max_new = max_new_tokens;
    r.eos = eos_token;
    if (s->pages_for(r) > s->cfg.num_pages) return NF_ERR_INVALID_ARGUMENT;     // could never be admitted
    const int64_t id = r.id;
    s->reqs.emplace(id, std::move(r));
    s->waiting.push_back(id);
    *id_out = id;
    return NF_OK;
} catch (const std::bad_alloc&) {
    return NF_ERR_OUT_OF_MEMORY;
} catch (...) {
    return NF_ERR_INVALID_ARGUMENT;
}

extern "C" nf_status nf_sched_next(nf_sched* s, nf_sched_iter* out) try {
    if (!s || !out) return NF_ERR_INVALID_ARGUMENT;
    // the batch of iteration k may only be formed once iteration k - 1 - lag has completed
    if (s->next_complete < s->next_iter - s->cfg.lag) return NF_ERR_INVALID_ARGUMENT;
    const int64_t k = s->next_iter;
    s->ctx_len.clear();
    s->positions.clear();
    s->token_ids.clear();
    s->token_src.clear();
    s->page_indptr.assign(1, 0);
    s->page_indices.clear();
    s->row_request.clear();

    // decode rows: every admitted request not known to have finished, in admission order
    for (int64_t id : s->running) {
        nf_sched::Request& r = s->reqs.at(id);
        const int32_t ctx = r.n_cached;
        const int32_t need = ctx / 16 + 1;  // pages holding slots 0 .. ctx
        if (need > (int32_t)r.pages.size()) return NF_ERR_INVALID_ARGUMENT;  // cannot happen: see the reservation
        s->ctx_len.push_back(ctx);
        s->positions.push_back(ctx);
        s->token_ids.push_back(-1);
        s->token_src.push_back(r.last_row);
        s->page_indices.insert(s->page_indices.end(), r.pages.begin(), r.pages.begin() + need);
        s->page_indptr.push_back((int32_t)s->page_indices.size());
        s->row_request.push_back(id);
    }
    const int32_t R = (int32_t)s->ctx_len.size();
    for (int32_t row = 0; row < R; ++row) {
        nf_sched::Request& r = s->reqs.at(s->row_request[row]);
        r.n_cached += 1;
        r.last_row = row;
    }

    // at most one prompt as the prefill chunk: the head of the queue, if it fits
    int32_t C = 0;
    if (!s->waiting.empty() && R < s->cfg.max_running) {
        nf_sched::Request& r = s->reqs.at(s->waiting.front());
        const int32_t np = s->pages_for(r);
        if (np <= (int32_t)s->free_pages.size()) {
            s->waiting.pop_front();
            for (int32_t j = 0; j < np; ++j) {
                r.pages.push_back(s->free_pages.back());
                s->free_pages.pop_back();
            }
            r.admitted = true;
            C = (int32_t)r.prompt.size();
            for (int32_t t = 0; t < C; ++t) {
                s->positions.push_back(t);
                s->token_ids.push_back(r.prompt[t]);
                s->token_src.push_back(-1);
            }
            const int32_t need = (C + 15) / 16;
            s->page_indices.insert(s->page_indices.end(), r.pages.begin(), r.pages.begin() + need);
            r.n_cached = C;
            r.last_row = R;  // the chunk's last row is next_token row R
            s->row_request.push_back(r.id);
            s->running.push_back(r.id);
        }
    }
    s->page_indptr.push_back((int32_t)s->page_indices.size());

    out->iteration = k;
    out->num_decode = R;
    out->prefill_len = C;
    out->num_tokens = R + C;
    out->rows = R + (C > 0 ? 1 : 0);
    out->num_page_entries = (int32_t)s->page_indices.size();
    out->ctx_len = s->ctx_len.data();
    out->positions = s->positions.data();
    out->token_ids = s->token_ids.data();
    out->token_src = s->token_src.data();
    out->page_indptr = s->page_indptr.data();
    out->page_indices = s->page_indices.data();
    out->row_request = s->row_request.data();
    if (out->num_tokens > 0) {
        s->inflight.push_back(nf_sched::Inflight{k, s->row_request});
        s->next_iter = k + 1;
    } else {
        out->iteration = -1;  // nothing to run: no sequence number is used
    }
    return NF_OK;
} catch (const std::bad_alloc&) {
    return NF_ERR_OUT_OF_MEMORY;
} catch (...) {
    return NF_ERR_INVALID_ARGUMENT;
}

extern "C" nf_status nf_sched_complete(nf_sched* s, int64_t iteration, const int32_t* next_token, int32_t rows) try {
    if (!s || !next_token || s->inflight.empty()) return NF_ERR_INVALID_ARGUMENT;
    const nf_sched::Inflight& it = s->inflight.front();
    if (iteration != it.iteration || rows != (int32_t)it.row_request.size()) return NF_ERR_INVALID_ARGUMENT;
    for (int32_t row = 0; row < rows; ++row) {
        nf_sched::Request& r = s->reqs.at(it.row_request[row]);
        if (r.finished) {  // decoded once more after its last token: dropped
            s->discarded += 1;
            continue;
        }
        const int32_t tok = next_token[row];
        r.out.push_back(tok);
        if (tok == r.eos || (int32_t)r.out.size() >= r.max_new) {
            r.finished = true;
            s->finished_count += 1;
            s->running.erase(std::find(s->running.begin(), s->running.end(), r.id));
            // iterations already formed that still use these pages run before any later one
            // that may receive them (one stream), so they can be handed out again now
            for (int32_t p : r.pages) s->free_pages.push_back(p);
            r.pages.clear();
        }
    }
    s->inflight.pop_front();
    s->next_complete = iteration + 1;
    return NF_OK;
} catch (const std::bad_alloc&) {
    return NF_ERR_OUT_OF_MEMORY;
} catch (...) {
    return NF_ERR_INVALID_ARGUMENT;
}

extern "C" nf_status nf_sched_request_tokens(const nf_sched* s, int64_t id, int32_t* out, int32_t cap, int32_t* len,
                                             int32_t* finished) try {
    if (!s || !len || cap < 0 || (cap > 0 && !out)) return NF_ERR_INVALID_ARGUMENT;
    auto f = s->reqs.find(id);
    if (f == s->reqs.end()) return NF_ERR_INVALID_ARGUMENT;
    const std::vector<int32_t>& o = f->second.out;
    const int32_t n = std::min<int32_t>(cap, (int32_t)o.size());
    if (n > 0) std::memcpy(out, o.data(), (size_t)n * sizeof(int32_t));
    *len = (int32_t)o.size();
    if (finished) *finished = f->second.finished ? 1 : 0;
    return NF_OK;
} catch (const std::bad_alloc&) {
    return NF_ERR_OUT_OF_MEMORY;
} catch (...) {
    return NF_ERR_INVALID_ARGUMENT;
}

extern "C" nf_status nf_sched_get_stats(const nf_sched* s, nf_sched_stats* out) try {
    if (!s || !out) return NF_ERR_INVALID_ARGUMENT;
    out->waiting = (int32_t)s->waiting.size();
    out->running = (int32_t)s->running.size();
    out->finished = (int32_t)s->finished_count;
    out->free_pages = (int32_t)s->free_pages.size();
    out->inflight = (int32_t)s->inflight.size();
    out->iterations = s->next_iter;
    out->discarded_tokens = s->discarded;
    return NF_OK;
} catch (const std::bad_alloc&) {
    return NF_ERR_OUT_OF_MEMORY;
} catch (...) {
    return NF_ERR_INVALID_ARGUMENT;
}
