"""The iteration replayed as a CUDA graph (nf_graph_create / nf_graph_launch).

A graph of one plan, captured on a side stream with the model's attention stream joining it, gives
the bits of nf_forward_iteration for that plan, on every replay, for the sequential plan and for an
overlapped two-nano-batch plan whose decode attention runs on the attention stream. The default
stream is rejected.
"""
import pytest
import torch

pytestmark = pytest.mark.gpu
DEV = "cuda:0"


@pytest.mark.parametrize("opts", [dict(nano=1, template=0), dict(nano=2, template=2, sm_attn=36)])
def test_graph_replay_equals_stream_forward(opts):
    import intra_device_overlapped_b200 as nf
    from intra_device_overlapped_b200.harness import DeviceWorkload
    from synth.workloads import TEST_WORKLOADS
    dw = DeviceWorkload(TEST_WORKLOADS["small_gqa8"], DEV)
    try:
        plan = dw.plan(**opts)
        side = torch.cuda.Stream(DEV)
        dw.forward(plan, side)
        side.synchronize()
        assert dw.sync() == 0
        ref = dw.hidden_out_f32.clone()
        g = dw.graph(plan, side)
        for _ in range(3):
            dw.hidden_out_f32.zero_()
            nf.check(nf.nf_graph_launch(g, side.cuda_stream), "nf_graph_launch")
            side.synchronize()
            assert dw.sync() == 0
            assert torch.equal(dw.hidden_out_f32.view(torch.int32), ref.view(torch.int32)), plan.describe()
        st, _ = nf.nf_graph_create(dw.model, plan, dw.io, 0)
        assert st == nf.NF_ERR_INVALID_ARGUMENT
    finally:
        dw.close()
