"""The decode attention entry point that allocates nothing (nf_decode_attention_noalloc).

It runs the same tensor-core decode attention as nf_op_decode_attention, with its scratch in
a static device array instead of model-owned buffers. Two calls in a row must each match the
model-based entry point within the tests' tolerance (the scratch is reused, not re-zeroed,
between calls), and the size limit and unsupported shapes must be rejected. This file is
collected last so that it also runs after every other GPU test in the same process.
"""
import numpy as np
import pytest
import torch

from synth.workloads import ModelShape, Workload

pytestmark = pytest.mark.gpu

DEV = "cuda:0"
TOL = 1.5e-2  # max-abs, as the decode attention parity tests


@pytest.fixture(scope="module")
def case():
    import intra_device_overlapped_b200 as nf
    from intra_device_overlapped_b200.harness import DeviceWorkload
    # 8 KV heads x 128, 32 query heads: ragged contexts, many requests per CTA
    w = Workload(ModelShape("noalloc_tc32", 1, 1024, 32, 8, 128, 512), 37, 0, 700, prefill_len=16)
    dw = DeviceWorkload(w, DEV)
    rng = np.random.default_rng(3)
    q = torch.from_numpy(rng.standard_normal((dw.T, 32, 128)).astype(np.float32)).to(DEV).to(torch.bfloat16)
    yield nf, dw, q
    dw.close()


def _noalloc(nf, dw, q, out, R, sm, status):
    io = dw.io
    return nf.nf_decode_attention_noalloc(q.data_ptr(), out.data_ptr(), dw.kv[0].data_ptr(),
                                          dw.batch.num_pages, io.ctx_len, io.page_indptr, io.page_indices, R,
                                          32, 8, 128, sm, status.data_ptr(), 0)


def test_noalloc_matches_model_entry_point_twice(case):
    nf, dw, q = case
    R = dw.batch.num_decode
    ref = torch.zeros_like(q)
    nf.check(nf.nf_op_decode_attention(dw.model, q.data_ptr(), ref.data_ptr(), dw.io, 0, 0, R, 0), "model entry")
    nf.check(dw.sync(), "status")
    status = torch.zeros(1, dtype=torch.int32, device=DEV)
    for call, sm in enumerate((0, 11)):
        out = torch.full_like(q, float("nan"))
        nf.check(_noalloc(nf, dw, q, out, R, sm, status), f"noalloc call {call}")
        torch.cuda.synchronize()
        assert int(status.item()) == 0
        got, want = out[:R].float(), ref[:R].float()
        assert torch.isfinite(got).all()
        assert float((got - want).abs().max()) <= TOL, f"call {call}"


def test_noalloc_rejects_oversize_and_unsupported(case):
    nf, dw, q = case
    out = torch.zeros_like(q)
    status = torch.zeros(1, dtype=torch.int32, device=DEV)
    R = nf.NF_NOALLOC_MAX_REQUESTS + 1
    assert _noalloc(nf, dw, q, out, R, 0, status) == nf.NF_ERR_INVALID_ARGUMENT
    io = dw.io
    st = nf.nf_decode_attention_noalloc(q.data_ptr(), out.data_ptr(), dw.kv[0].data_ptr(), dw.batch.num_pages,
                                        io.ctx_len, io.page_indptr, io.page_indices, 4, 32, 8, 64, 0, 0, 0)
    assert st == nf.NF_ERR_UNSUPPORTED
