"""KV offload of a finished request to host memory (nf_offload_kv), on the GPU.

The pages a request owns are copied, layer by layer, to pinned host memory on a stream of their own;
the host copy must equal the pool's pages bit for bit, in the listed order, for every layer. The
offload runs beside an iteration without changing the iteration's result. Page ids outside the
pool are rejected on the host.
"""
import numpy as np
import pytest
import torch

pytestmark = pytest.mark.gpu
DEV = "cuda:0"


def test_offloaded_pages_equal_the_pool_and_leave_the_iteration_unchanged():
    import intra_device_overlapped_b200 as nf
    from intra_device_overlapped_b200.harness import DeviceWorkload
    from synth.workloads import TEST_WORKLOADS
    dw = DeviceWorkload(TEST_WORKLOADS["small_gqa8"], DEV)
    try:
        b, s = dw.batch, dw.shape
        plan = dw.plan(nano=2, template=1, sm_attn=20)
        dw.forward(plan)
        assert dw.sync() == 0
        ref = dw.hidden_out_f32.clone()
        r = int(np.argmax(b.ctx_lens))
        pages = [int(p) for p in b.page_indices[b.page_indptr[r]:b.page_indptr[r + 1]]][::-1]  # any order
        page_elems = dw.kv[0].shape[1]
        host = torch.empty((s.n_layers, len(pages), page_elems), dtype=torch.bfloat16).pin_memory()
        side = torch.cuda.Stream(DEV, priority=0)
        # the offload on its own stream beside an iteration on the default stream
        st = nf.nf_offload_kv(dw.model, dw._kv_ptrs, b.num_pages, pages, 0, s.n_layers, host.data_ptr(),
                              side.cuda_stream)
        assert st == nf.NF_OK
        dw.forward(plan)
        side.synchronize()
        assert dw.sync() == 0
        assert torch.equal(dw.hidden_out_f32.view(torch.int32), ref.view(torch.int32))
        for layer in range(s.n_layers):
            want = dw.kv[layer][pages].cpu()
            assert torch.equal(host[layer].view(torch.int16), want.view(torch.int16)), layer
        # one layer only, into a fresh buffer
        host1 = torch.zeros((1, 3, page_elems), dtype=torch.bfloat16).pin_memory()
        assert nf.nf_offload_kv(dw.model, dw._kv_ptrs, b.num_pages, pages[:3], 1, 2, host1.data_ptr(), 0) == nf.NF_OK
        torch.cuda.synchronize()
        assert torch.equal(host1[0].view(torch.int16), dw.kv[1][pages[:3]].cpu().view(torch.int16))
        # rejected on the host
        bad = [pages[0], b.num_pages]
        assert nf.nf_offload_kv(dw.model, dw._kv_ptrs, b.num_pages, bad, 0, 1, host.data_ptr(), 0) == \
            nf.NF_ERR_INVALID_ARGUMENT
        assert nf.nf_offload_kv(dw.model, dw._kv_ptrs, b.num_pages, pages, 1, 1, host.data_ptr(), 0) == \
            nf.NF_ERR_INVALID_ARGUMENT
    finally:
        dw.close()
