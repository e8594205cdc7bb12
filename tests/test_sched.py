"""Serving scheduler (nf_sched_*): batch formation, page reservation, delayed retirement.

A fake device stands in for the GPU and keeps its stream semantics: iterations run in launch
order, decode rows read their input token from the previous iteration's next_token through
token_src (as the gather kernel does), and every K/V slot an iteration writes is recorded in a
page pool. Each decode row checks that all the slots it attends to still hold its own request's
entries, so a page handed to another request while still in use fails the test. The generated
tokens are a fixed function of the prompt and the position, so each request's expected stream is
known without any batching.
"""
import numpy as np
import pytest

import intra_device_overlapped_b200 as nf

V = 1000


def first_token(prompt):
    h = 17
    for t in prompt:
        h = (h * 131 + int(t) + 7) % V
    return h


def next_tok(tok, pos):
    return (tok * 37 + pos * 11 + 5) % V


def expected(prompt, max_new, eos):
    out = [first_token(prompt)]
    while out[-1] != eos and len(out) < max_new:
        out.append(next_tok(out[-1], len(prompt) + len(out) - 1))
    return out


class FakeDevice:
    def __init__(self, num_pages):
        self.pool = np.full((num_pages, 16, 2), -1, dtype=np.int64)  # (request id, position) per slot
        self.prev = None

    def run(self, it):
        R, C, T, rows = it.num_decode, it.prefill_len, it.num_tokens, it.rows
        arr = lambda p, n: np.ctypeslib.as_array(p, shape=(n,)).copy() if n else np.zeros(0, np.int64)
        tok, src, pos = arr(it.token_ids, T), arr(it.token_src, T), arr(it.positions, T)
        ctx, indptr = arr(it.ctx_len, R), arr(it.page_indptr, R + 2)
        pages, req = arr(it.page_indices, it.num_page_entries), arr(it.row_request, rows)
        inp = np.where(src >= 0, 0, tok)
        for t in range(T):
            if src[t] >= 0:
                assert self.prev is not None and src[t] < len(self.prev)
                inp[t] = self.prev[src[t]]
        out = np.zeros(rows, dtype=np.int64)
        for r in range(R):
            pl = pages[indptr[r]:indptr[r + 1]]
            assert len(pl) == ctx[r] // 16 + 1 and pos[r] == ctx[r]
            self.pool[pl[ctx[r] // 16], ctx[r] % 16] = (req[r], ctx[r])
            keys = np.arange(ctx[r] + 1)  # the keys this row attends to are its own
            held = self.pool[pl[keys // 16], keys % 16]
            assert (held[:, 0] == req[r]).all() and (held[:, 1] == keys).all()
            out[r] = next_tok(inp[r], pos[r])
        if C:
            pl = pages[indptr[R]:indptr[R + 1]]
            assert len(pl) == (C + 15) // 16 and list(pos[R:]) == list(range(C)) and (src[R:] == -1).all()
            for p in range(C):
                self.pool[pl[p // 16], p % 16] = (req[R], p)
            out[R] = first_token(tok[R:])
        self.prev = out
        return out


def serve(requests, lag, num_pages=64, max_running=4, chunk_len=32, max_position=512):
    st, s = nf.nf_sched_create(nf.nf_sched_config(num_pages, max_running, chunk_len, max_position, lag))
    assert st == 0
    try:
        ids = []
        for prompt, max_new, eos in requests:
            st, rid = nf.nf_sched_add_request(s, prompt, max_new, eos)
            assert st == 0
            ids.append(rid)
        dev, inflight, iters = FakeDevice(num_pages), [], 0
        while True:
            _, stats = nf.nf_sched_get_stats(s)
            if stats.finished == len(ids) and not inflight:
                break
            st, it = nf.nf_sched_next(s)
            assert st == 0
            if it.num_tokens == 0:
                assert inflight
                k, out = inflight.pop(0)
                assert nf.nf_sched_complete(s, k, out.tolist()) == 0
                continue
            assert it.num_decode <= max_running and it.prefill_len <= chunk_len
            inflight.append((it.iteration, dev.run(it)))
            iters += 1
            while len(inflight) > lag:
                k, out = inflight.pop(0)
                assert nf.nf_sched_complete(s, k, out.tolist()) == 0
            assert iters < 10000
        toks = [nf.nf_sched_request_tokens(s, r)[1] for r in ids]
        _, stats = nf.nf_sched_get_stats(s)
        assert stats.free_pages == num_pages and stats.running == 0 and stats.waiting == 0
        return toks, stats.as_dict()
    finally:
        nf.nf_sched_destroy(s)


def random_requests(seed, n, vocab=V):
    rng = np.random.default_rng(seed)
    reqs = []
    for _ in range(n):
        L = int(rng.integers(1, 33))
        prompt = rng.integers(0, vocab, L).tolist()
        max_new = int(rng.integers(1, 40))
        full = expected(prompt, 10 ** 6, -1)[:max_new]
        # half of the requests stop at an end token that their stream actually produces
        eos = int(full[int(rng.integers(0, len(full)))]) if rng.random() < 0.5 else -1
        reqs.append((prompt, max_new, eos))
    return reqs


@pytest.mark.parametrize("lag", [0, 1])
@pytest.mark.parametrize("seed,num_pages,max_running", [(0, 64, 4), (1, 12, 3), (2, 200, 8), (3, 6, 2)])
def test_streams_match_per_request_reference(lag, seed, num_pages, max_running):
    reqs = random_requests(seed, 25)
    toks, stats = serve(reqs, lag, num_pages=num_pages, max_running=max_running)
    for (prompt, max_new, eos), got in zip(reqs, toks):
        assert got == expected(prompt, max_new, eos)
    # at lag 1 every request is decoded exactly once after its last token, and that token is dropped
    assert stats["discarded_tokens"] == (len(reqs) if lag == 1 else 0)


def test_async_and_sync_agree_and_async_runs_one_extra_row_per_request():
    reqs = random_requests(7, 40)
    a, sa = serve(reqs, 1, num_pages=40, max_running=6)
    b, sb = serve(reqs, 0, num_pages=40, max_running=6)
    assert a == b
    assert sa["discarded_tokens"] == len(reqs) and sb["discarded_tokens"] == 0


def test_fifo_admission_waits_for_pages():
    # each request needs ceil((16 + 16) / 16) = 2 pages; a 4-page pool holds two at a time
    reqs = [([i + 1] * 16, 16, -1) for i in range(5)]
    toks, stats = serve(reqs, 1, num_pages=4, max_running=8)
    assert [t for t in toks] == [expected(p, m, e) for p, m, e in reqs]


def test_rejects_requests_that_could_never_run():
    st, s = nf.nf_sched_create(nf.nf_sched_config(3, 2, 8, 64, 1))
    assert st == 0
    try:
        assert nf.nf_sched_add_request(s, [1] * 9, 4)[0] == nf.NF_ERR_INVALID_ARGUMENT   # longer than a chunk
        assert nf.nf_sched_add_request(s, [1] * 8, 57)[0] == nf.NF_ERR_INVALID_ARGUMENT  # past max_position
        assert nf.nf_sched_add_request(s, [1] * 8, 41)[0] == nf.NF_ERR_INVALID_ARGUMENT  # 49 slots: 4 pages > 3
        assert nf.nf_sched_add_request(s, [1] * 8, 40)[0] == 0                            # 48 slots: 3 pages
        assert nf.nf_sched_add_request(s, [], 4)[0] == nf.NF_ERR_INVALID_ARGUMENT
        assert nf.nf_sched_add_request(s, [1], 0)[0] == nf.NF_ERR_INVALID_ARGUMENT
    finally:
        nf.nf_sched_destroy(s)
    for bad in (nf.nf_sched_config(0, 2, 8, 64, 1), nf.nf_sched_config(4, 0, 8, 64, 1),
                nf.nf_sched_config(4, 2, 0, 64, 1), nf.nf_sched_config(4, 2, 8, 64, 2)):
        assert nf.nf_sched_create(bad)[0] == nf.NF_ERR_INVALID_ARGUMENT


@pytest.mark.parametrize("lag", [0, 1])
def test_next_refuses_to_run_ahead_of_completions(lag):
    st, s = nf.nf_sched_create(nf.nf_sched_config(16, 4, 8, 64, lag))
    try:
        for i in range(3):
            assert nf.nf_sched_add_request(s, [i + 1, 2, 3], 5)[0] == 0
        dev = FakeDevice(16)
        outs = []
        for k in range(lag + 1):  # lag + 1 iterations may be formed before the first completion
            st, it = nf.nf_sched_next(s)
            assert st == 0 and it.iteration == k
            outs.append(dev.run(it))
        assert nf.nf_sched_next(s)[0] == nf.NF_ERR_INVALID_ARGUMENT
        assert nf.nf_sched_complete(s, 1, outs[0].tolist()) == nf.NF_ERR_INVALID_ARGUMENT  # out of order
        assert nf.nf_sched_complete(s, 0, outs[0].tolist()[:-1] + [0, 0]) == nf.NF_ERR_INVALID_ARGUMENT  # rows
        assert nf.nf_sched_complete(s, 0, outs[0].tolist()) == 0
        assert nf.nf_sched_next(s)[0] == 0
    finally:
        nf.nf_sched_destroy(s)


def test_batch_layout_matches_the_forward_contract():
    st, s = nf.nf_sched_create(nf.nf_sched_config(32, 4, 20, 128, 1))
    try:
        p0, p1 = list(range(1, 18)), [5, 6, 7]
        assert nf.nf_sched_add_request(s, p0, 8)[0] == 0
        assert nf.nf_sched_add_request(s, p1, 8)[0] == 0
        st, it = nf.nf_sched_next(s)           # iteration 0: prompt 0 alone
        a = lambda p, n: np.ctypeslib.as_array(p, shape=(n,)).tolist()
        assert (it.num_decode, it.prefill_len, it.rows) == (0, 17, 1)
        assert a(it.token_ids, 17) == p0 and a(it.positions, 17) == list(range(17))
        assert a(it.page_indptr, 2) == [0, 2] and a(it.page_indices, 2) == [0, 1]
        st, it = nf.nf_sched_next(s)           # iteration 1: request 0 decodes, prompt 1 prefills
        assert (it.num_decode, it.prefill_len, it.rows, it.num_tokens) == (1, 3, 2, 4)
        assert a(it.ctx_len, 1) == [17] and a(it.positions, 4) == [17, 0, 1, 2]
        assert a(it.token_src, 4) == [0, -1, -1, -1] and a(it.token_ids, 4)[1:] == p1
        # request 0 reserved ceil((17 + 8) / 16) = 2 pages, request 1 ceil(11 / 16) = 1
        assert a(it.page_indptr, 3) == [0, 2, 3] and a(it.page_indices, 3) == [0, 1, 2]
        assert np.ctypeslib.as_array(it.row_request, shape=(2,)).tolist() == [0, 1]
    finally:
        nf.nf_sched_destroy(s)


def test_serving_plan_shape_policy():
    """Decode attention beside prefill attention only when both are present; one nano-batch."""
    from intra_device_overlapped_b200.serving import default_plan_opts
    pick = default_plan_opts(148, prefill_sms=8)
    both, dec, pre = pick(7, 20), pick(8, 0), pick(0, 32)
    assert (both.force_nano, both.force_template, both.force_sm_attn) == (1, nf.NF_TEMPLATE_PREFILL_ON_GEMM, 140)
    for o in (dec, pre):
        assert (o.force_nano, o.force_template) == (1, nf.NF_TEMPLATE_SEQUENTIAL)
    assert default_plan_opts(12)(4, 4).force_template == nf.NF_TEMPLATE_SEQUENTIAL  # too few SMs to split
