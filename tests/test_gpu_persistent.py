"""The iteration with each layer as one persistent kernel (nf_forward_iteration_persistent).

The persistent kernel runs the same operations as the stream executor, scheduled on the device: CTAs
wait on completion counters instead of kernel boundaries and events, and its GEMMs use one-CTA tiles
instead of CTA pairs. Checked here, on the tensor-core attention shapes (8 KV heads of 128, 32 and 64
query heads):
- the result equals the stream executor's bit for bit (fp32 residual stream after every layer, and
  the KV slots written), for the sequential plan and for plans of two to four nano-batches in both
  overlapped templates, including batches whose long requests are split along KV (merge operation);
- against the oracle, within the parity bars (so the bitwise equality above is not two equal
  mistakes);
- the per-CTA trace of an overlapped plan shows GEMM and decode attention work running at the same
  time on different SMs inside the one launch;
- the full-size Llama-3-8B-shaped layer (512 decode requests, contexts U[1024, 1536], 1024-token
  chunk) matches the stream executor bit for bit;
- models the kernel does not cover (head dim 64) are refused with NF_ERR_UNSUPPORTED;
- a dependency wait that cannot be satisfied (an operation list whose first operation waits on its
  second) expires with NF_ERR_DEVICE_TIMEOUT on every CTA, the kernel exits, and the context stays
  usable.
"""
import numpy as np
import pytest
import torch

from synth import weights as SW
from synth.workloads import WORKLOADS, TEST_WORKLOADS, ModelShape, Workload

from parity import check_readings

pytestmark = pytest.mark.gpu
DEV = "cuda:0"

# 2 layers, 40 decode requests with contexts up to 2100 keys (the longer ones are split in chunks
# of 1024 keys and merged), a 200-token chunk
LONG = Workload(ModelShape("gqa8_long", 2, 1024, 32, 8, 128, 1024, rope_theta=500000.0, norm_sigma=0.1),
                40, 900, 2100, prefill_len=200)
# 64 query heads (the Llama-2-70B head shape), some requests split
Q64 = Workload(ModelShape("gqa8_q64", 1, 2048, 64, 8, 128, 1024, rope_theta=10000.0, norm_sigma=0.1),
               16, 1, 1300, prefill_len=40)

# up to four nano-batches: 7 operations each fill the layer kernel's list of 28
PLANS = [dict(nano=1, template=0), dict(nano=2, template=1, sm_attn=36), dict(nano=2, template=2, sm_attn=40),
         dict(nano=3, template=1, sm_attn=48), dict(nano=4, template=2, sm_attn=64)]


def _reset_kv(dw):
    for layer, pool in enumerate(dw.kv):
        SW.gpu_fill_kv_pool(dw.shape, layer, pool)
    torch.cuda.synchronize()


def _run(dw, plan, persistent):
    _reset_kv(dw)
    dw.layer_hidden.zero_()
    dw.forward(plan, persistent=persistent)
    st = dw.sync()
    assert st == 0, f"device status {st}"
    return (dw.layer_hidden.clone(), [p.clone() for p in dw.kv])


def _assert_same(a, b, what):
    ha, kva = a
    hb, kvb = b
    assert torch.equal(ha.view(torch.int32), hb.view(torch.int32)), f"{what}: residual stream differs"
    for layer, (x, y) in enumerate(zip(kva, kvb)):
        assert torch.equal(x.view(torch.int16), y.view(torch.int16)), f"{what}: KV pool of layer {layer} differs"


@pytest.mark.parametrize("wname", ["small_gqa8", "long", "q64"])
def test_persistent_equals_stream_executor(wname):
    from intra_device_overlapped_b200.harness import DeviceWorkload
    w = {"small_gqa8": TEST_WORKLOADS["small_gqa8"], "long": LONG, "q64": Q64}[wname]
    dw = DeviceWorkload(w, DEV, layer_outputs=True)
    try:
        if wname == "long":
            assert int(dw.batch.ctx_lens.max()) + 1 > 1024  # some requests are split along KV
        for opts in PLANS:
            plan = dw.plan(**opts)
            ref = _run(dw, plan, False)
            for rep in range(2):
                _assert_same(_run(dw, plan, True), ref, f"{wname} {plan.describe()} run {rep}")
    finally:
        dw.close()


def test_persistent_matches_oracle():
    from intra_device_overlapped_b200.harness import DeviceWorkload
    from oracle.run import run_oracle
    w = TEST_WORKLOADS["small_gqa8"]
    dw = DeviceWorkload(w, DEV)
    try:
        _, res, _ = run_oracle(w, batch=dw.batch)
        f64 = run_oracle(w, batch=dw.batch, bf16_act=False)[1]["hidden"]
        plan = dw.plan(nano=2, template=1, sm_attn=36)
        _reset_kv(dw)
        dw.forward(plan, persistent=True)
        assert dw.sync() == 0
        hid = dw.hidden_out_f32.cpu().numpy().astype(np.float64)
        check_readings(hid, {"bf16 model": res["hidden"], "float64 activations": f64},
                       f"small_gqa8 persistent, plan {plan.describe()}")
    finally:
        dw.close()


def test_persistent_trace_shows_gemm_beside_decode():
    import intra_device_overlapped_b200 as nf
    from intra_device_overlapped_b200.harness import DeviceWorkload
    dw = DeviceWorkload(LONG, DEV)
    try:
        plan = dw.plan(nano=2, template=1, sm_attn=36)
        dw.trace(True)
        dw.forward(plan, persistent=True)
        assert dw.sync() == 0
        tr = list(dw.get_trace())  # (kernel, smid, t_start, t_end) per CTA and operation
        dw.trace(False)
        gemm = [e for e in tr if e[0] == nf.NF_KERNEL_GEMM]
        dec = [e for e in tr if e[0] == nf.NF_KERNEL_DECODE_ATTN]
        assert gemm and dec
        # some GEMM interval overlaps some decode interval, on different SMs
        both = [(g, a) for g in gemm for a in dec if g[2] < a[3] and a[2] < g[3] and g[1] != a[1]]
        assert both, "no GEMM work ran beside decode attention"
        # decode attention ran only on the attention lane's SMs, which also ran GEMM work after it
        dec_sms = {e[1] for e in dec}
        assert len(dec_sms) <= plan.sm_attn
    finally:
        dw.close()


def test_full_size_layer_persistent_equals_stream_executor():
    from intra_device_overlapped_b200.harness import DeviceWorkload
    dw = DeviceWorkload(WORKLOADS["llama3_8b_layer"], DEV, keep_logits=False, layer_outputs=True)
    try:
        for opts in (dict(nano=1, template=0), dict(nano=2, template=2, sm_attn=100)):
            plan = dw.plan(**opts)
            _assert_same(_run(dw, plan, True), _run(dw, plan, False), f"llama3_8b_layer {plan.describe()}")
    finally:
        dw.close()


def test_persistent_refuses_uncovered_models():
    import intra_device_overlapped_b200 as nf
    from intra_device_overlapped_b200.harness import DeviceWorkload
    dw = DeviceWorkload(TEST_WORKLOADS["tiny_gamma"], DEV)  # head dim 64
    try:
        plan = dw.plan(nano=1, template=0)
        st = nf.nf_forward_iteration_persistent(dw.model, plan, dw.io, torch.cuda.current_stream().cuda_stream)
        assert st == nf.NF_ERR_UNSUPPORTED
    finally:
        dw.close()


def test_persistent_dependency_wait_times_out_cleanly():
    import intra_device_overlapped_b200 as nf
    from intra_device_overlapped_b200.harness import DeviceWorkload
    torch.cuda.set_device(DEV)
    assert nf.nf_op_persistent_wait_test(10_000_000) == nf.NF_ERR_DEVICE_TIMEOUT
    assert nf.nf_op_persistent_wait_test(0) == nf.NF_ERR_INVALID_ARGUMENT
    # the context is usable afterwards: a persistent forward still equals the stream executor
    dw = DeviceWorkload(TEST_WORKLOADS["small_gqa8"], DEV, layer_outputs=True)
    try:
        plan = dw.plan(nano=1, template=0)
        _assert_same(_run(dw, plan, True), _run(dw, plan, False), "after the timeout test")
    finally:
        dw.close()
