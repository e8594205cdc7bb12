"""The decode attention entry point that allocates nothing (nf_decode_attention_noalloc).

Some callers cannot allocate device memory at the point where they run attention (code between
the capture calls of a CUDA graph, runtimes without an allocator, processes whose device memory all
belongs to their own pool), so they cannot create a model. This entry point runs the same
tensor-core decode attention from plain device pointers, with its scratch in a static device array.

Checked here: two calls in a row (the scratch is reused, not cleared, between them) each give the
bits of the model-based entry point nf_op_decode_attention (every request here has at most 1024 keys,
which neither entry point splits) and match the oracle within the parity bar; a request whose page
row is too short, or whose context length is negative, is reported through the status word with a
finite output; the size limit, a missing status word and unsupported shapes are rejected. This file
is collected last so that it also runs after every other GPU test in the same process.
"""
import numpy as np
import pytest
import torch

import synth
from synth import weights as SW
from synth.workloads import ModelShape, Workload

pytestmark = pytest.mark.gpu

DEV = "cuda:0"
ATT_ABS = 2e-2  # max-abs, as the attention parity tests


@pytest.fixture(scope="module")
def case():
    import intra_device_overlapped_b200 as nf
    from intra_device_overlapped_b200.harness import DeviceWorkload
    # 8 KV heads x 128, 32 query heads: ragged contexts up to 511 keys, many requests per CTA
    w = Workload(ModelShape("noalloc_tc32", 1, 1024, 32, 8, 128, 512), 37, 0, 510, prefill_len=16)
    dw = DeviceWorkload(w, DEV)
    rng = np.random.default_rng(3)
    q = torch.from_numpy(rng.standard_normal((dw.T, 32, 128)).astype(np.float32)).to(DEV).to(torch.bfloat16)
    yield nf, dw, q
    dw.close()


def _noalloc(nf, dw, q, out, R, sm, status, ctx_ptr=None, indptr_ptr=None):
    io = dw.io
    return nf.nf_decode_attention_noalloc(q.data_ptr(), out.data_ptr(), dw.kv[0].data_ptr(),
                                          dw.batch.num_pages, ctx_ptr or io.ctx_len, indptr_ptr or io.page_indptr,
                                          io.page_indices, R, 32, 8, 128, sm, status.data_ptr(), 0)


def test_noalloc_equals_model_entry_point_and_oracle_twice(case):
    from oracle import forward as F
    nf, dw, q = case
    b = dw.batch
    R = b.num_decode
    ref = torch.zeros_like(q)
    nf.check(nf.nf_op_decode_attention(dw.model, q.data_ptr(), ref.data_ptr(), dw.io, 0, 0, R, 0), "model entry")
    nf.check(dw.sync(), "status")
    status = torch.zeros(1, dtype=torch.int32, device=DEV)
    qd = q.double().cpu().numpy()
    for call, sm in enumerate((0, 11)):
        out = torch.full_like(q, float("nan"))
        nf.check(_noalloc(nf, dw, q, out, R, sm, status), f"noalloc call {call}")
        torch.cuda.synchronize()
        assert int(status.item()) == 0
        assert torch.equal(out[:R].view(torch.int16), ref[:R].view(torch.int16)), f"call {call}"
        got = out[:R].float().cpu().numpy()
        worst = 0.0
        for r in range(R):
            pages = b.page_indices[b.page_indptr[r]:b.page_indptr[r + 1]]
            kv = F.PagedKV(lambda layer, pg: synth.bf16_to_f64(SW.host_kv_pages(dw.shape, layer, pg)), 16)
            K, V = kv.read(0, pages, int(b.ctx_lens[r]) + 1)
            for bf in (True, False):
                worst = max(worst, float(np.abs(got[r] - F.decode_attention(qd[r], K, V, bf16_p=bf)).max()))
        print(f"no-alloc call {call} (grid {sm or 'all'}): max-abs {worst:.4g} against the oracle")
        assert worst <= ATT_ABS, (call, worst)


@pytest.mark.parametrize("fault", ["short_row", "negative_ctx"])
def test_noalloc_reports_bad_page_rows_and_contexts(case, fault):
    """A request whose row of the page table holds fewer pages than its keys need reads page 0 in
    place of the missing ones; a negative context length is read as 0. Both are reported as
    NF_ERR_DEVICE_BOUNDS, and the output stays finite."""
    nf, dw, q = case
    b = dw.batch
    R = b.num_decode
    ctx = torch.from_numpy(np.ascontiguousarray(b.ctx_lens, dtype=np.int32)).to(DEV)
    r = int(np.argmax(b.ctx_lens))
    if fault == "short_row":
        ctx[r] += 16 * 3                       # three pages more than the request's row holds
    else:
        ctx[r] = -5
    status = torch.zeros(1, dtype=torch.int32, device=DEV)
    out = torch.full_like(q, float("nan"))
    nf.check(_noalloc(nf, dw, q, out, R, 0, status, ctx_ptr=ctx.data_ptr()), "noalloc")
    torch.cuda.synchronize()
    assert int(status.item()) == nf.NF_ERR_DEVICE_BOUNDS
    assert torch.isfinite(out[:R].float()).all()


def test_noalloc_rejects_oversize_missing_status_and_unsupported(case):
    nf, dw, q = case
    out = torch.zeros_like(q)
    status = torch.zeros(1, dtype=torch.int32, device=DEV)
    R = nf.NF_NOALLOC_MAX_REQUESTS + 1
    assert _noalloc(nf, dw, q, out, R, 0, status) == nf.NF_ERR_INVALID_ARGUMENT
    io = dw.io
    st = nf.nf_decode_attention_noalloc(q.data_ptr(), out.data_ptr(), dw.kv[0].data_ptr(), dw.batch.num_pages,
                                        io.ctx_len, io.page_indptr, io.page_indices, 4, 32, 8, 128, 0, 0, 0)
    assert st == nf.NF_ERR_INVALID_ARGUMENT           # no status word
    st = nf.nf_decode_attention_noalloc(q.data_ptr(), out.data_ptr(), dw.kv[0].data_ptr(), dw.batch.num_pages,
                                        io.ctx_len, io.page_indptr, io.page_indices, 4, 32, 8, 64, 0,
                                        status.data_ptr(), 0)
    assert st == nf.NF_ERR_UNSUPPORTED
