"""The device-level pipeline on the GPU: co-running kernels split the SMs and overlap in time.

NanoFlow runs the compute-bound GEMMs of one nano-batch beside the memory-bound decode attention
of another by giving each its own part of the GPU (README "Introduction"; arXiv abstract). Here
the parts are SMs: every kernel is persistent with one CTA per SM, decode attention takes sm_attn
SMs, and the GEMMs beside it take the others (growing onto the attention SMs once the attention
kernel has finished, for elastic GEMM launches). The library's per-CTA trace (kernel, %smid, start
and end in %globaltimer ns) shows both properties on the Llama-3-8B-shaped layer:

* no SM ever holds a decode-attention CTA and a GEMM CTA at the same time;
* decode-attention CTAs and GEMM CTAs do run at the same time, on different SMs;

and the overlapped plan gives the sequential plan's bits.
"""
import numpy as np
import pytest
import torch

pytestmark = pytest.mark.gpu
DEV = "cuda:0"


def _intervals(entries, kind):
    return [(e[1], e[2], e[3]) for e in entries if e[0] == kind]   # (smid, start, end)


def test_decode_and_gemm_ctas_split_the_sms_and_overlap():
    import intra_device_overlapped_b200 as nf
    from intra_device_overlapped_b200.harness import DeviceWorkload
    from synth.workloads import WORKLOADS
    from synth import weights as SW
    dw = DeviceWorkload(WORKLOADS["llama3_8b_layer"], DEV, keep_logits=False)
    try:
        seq = dw.plan(nano=1, template=0)
        dw.forward(seq)
        assert dw.sync() == 0
        ref = dw.hidden_out_f32.clone()
        for layer, pool in enumerate(dw.kv):
            SW.gpu_fill_kv_pool(dw.shape, layer, pool)
        plan = dw.plan(nano=2, template=nf.NF_TEMPLATE_PREFILL_ON_GEMM, sm_attn=80)
        dw.trace(True)
        dw.forward(plan)
        assert dw.sync() == 0
        entries = list(dw.get_trace())   # (kernel, smid, t_start, t_end)
        dw.trace(False)
        assert torch.equal(dw.hidden_out_f32.view(torch.int32), ref.view(torch.int32)), plan.describe()

        dec = _intervals(entries, nf.NF_KERNEL_DECODE_ATTN)
        gem = _intervals(entries, nf.NF_KERNEL_GEMM)
        assert len(dec) == plan.sm_attn and gem
        # exclusive occupancy of every SM
        by_sm = {}
        for sm, a, b in dec:
            by_sm.setdefault(sm, []).append((a, b))
        clashes = [(sm, a, b) for sm, a, b in gem for (c, d) in by_sm.get(sm, []) if a < d and c < b]
        assert not clashes, clashes[:4]
        # decode CTAs co-run with GEMM CTAs on other SMs
        d0, d1 = min(a for _, a, _ in dec), max(b for _, _, b in dec)
        corun = [(sm, a, b) for sm, a, b in gem if a < d1 and d0 < b]
        corun_sms = {sm for sm, _, _ in corun}
        overlap_ns = sum(min(b, d1) - max(a, d0) for _, a, b in corun)
        print(f"{plan.describe()}: decode window {(d1 - d0) / 1e3:.1f} us on {len(dec)} SMs; "
              f"{len(corun)} GEMM CTAs on {len(corun_sms)} other SMs overlap it "
              f"({overlap_ns / 1e3 / max(len(corun_sms), 1):.1f} us per SM on average)")
        assert corun, "no GEMM CTA ran beside the decode attention"
        assert len(corun_sms) >= plan.sm_gemm // 2, (len(corun_sms), plan.sm_gemm)
    finally:
        dw.close()
