"""Parity at the workloads' full sizes, in the bench's launch configuration, on sampled rows.

Each test builds the whole workload on the GPU (every layer's weights and paged KV pool, every
request), runs one serving iteration through nf_plan_iteration + nf_forward_iteration, and checks
sampled decode rows (and, for the single layer, the whole prefill chunk) against the float64
oracle computed for those rows only. Decode rows are independent of one another (their attention
reads only their own pages), so the oracle's sub-batch reproduces them exactly.

Reference: the oracle's bf16 model (every tensor handed from one operation to the next is bf16,
everything else float64). Bars: max-abs <= 2e-2 and relative L1 <= 5e-3, with hidden states
divided row by row by the oracle row's RMS before the max-abs (the residual stream's scale is
several units, where one bf16 ulp of an intermediate already moves outputs by about 2e-2).
Deep stacks are checked layer by layer with teacher forcing: the oracle layer runs on the GPU's
own input to that layer (the GPU exports its residual after every layer), so errors are measured
per layer instead of compounding over 20-32 layers. Greedy tokens and MoE routing are compared
exactly wherever the oracle's decision margin exceeds twice the observed error of its inputs.
"""
import gc

import numpy as np
import pytest
import torch

from synth.workloads import WORKLOADS
from parity import MAX_ABS, MEAN_REL, errors, row_scaled_max_abs

pytestmark = pytest.mark.gpu
DEV = "cuda:0"


def _dw(name, **kw):
    from intra_device_overlapped_b200.harness import DeviceWorkload
    return DeviceWorkload(WORKLOADS[name], DEV, **kw)


def _release(dw):
    # the workloads hold up to ~100 GB: return it before the next test builds its own
    dw.close()
    dw.__dict__.clear()
    gc.collect()
    torch.cuda.empty_cache()


def _forward(dw, plan):
    dw.forward(plan)
    st = dw.sync()
    assert st == 0, f"device status {st}"


def _check_rows(got, ref, what):
    mx = row_scaled_max_abs(got, ref)
    raw, rel = errors(got, ref)
    print(f"{what}: row-scaled max-abs {mx:.4g}, raw max-abs {raw:.4g}, relative L1 {rel:.4g}")
    assert mx <= MAX_ABS and rel <= MEAN_REL, (what, mx, rel)


def _layer_input_rows(name, dw, reqs):
    """Input of layer 0 for the sampled decode rows: the hidden input, or the token embeddings."""
    from synth import bf16_to_f64
    from synth import weights as SW
    s = WORKLOADS[name].shape
    if s.vocab > 0:
        toks = np.asarray(dw.batch.tokens)[reqs]
        return bf16_to_f64(SW.host_rows(SW.global_specs(s)["embed"], toks))
    return bf16_to_f64(SW.host_input_rows(s, np.asarray(reqs)))


def _teacher_forced_layers(name, dw, reqs, layers):
    """Each sampled layer: the oracle layer on the GPU's input rows against the GPU's output rows."""
    from oracle.forward import layer_forward, sub_batch
    from oracle.run import layer_weights_f64, make_kv
    s = WORKLOADS[name].shape
    sb = sub_batch(dw.batch, reqs, keep_prefill=False)
    lh = dw.layer_hidden
    extras = {}
    for layer in layers:
        x_in = _layer_input_rows(name, dw, reqs) if layer == 0 else \
            lh[layer - 1].cpu().numpy().astype(np.float64)[reqs]
        out, ex = layer_forward(s, layer_weights_f64(s, layer), x_in, sb, make_kv(s), layer)
        got = lh[layer].cpu().numpy().astype(np.float64)[reqs]
        _check_rows(got, out, f"layer {layer}")
        extras[layer] = ex
    return extras


def test_llama3_8b_layer_full_size_planner_plan():
    """512 decode requests (context U[1024,1536]) + a 1024-token chunk, the planner's plan."""
    from oracle.run import run_oracle
    dw = _dw("llama3_8b_layer", keep_logits=False)
    try:
        dw.calibrate()
        plan = dw.plan()
        _forward(dw, plan)
        got = dw.hidden_out_f32.cpu().numpy().astype(np.float64)
        reqs = [0, 1, 255, 511]
        R = dw.batch.num_decode
        rows = reqs + list(range(R, dw.T))
        w = WORKLOADS["llama3_8b_layer"]
        ref = run_oracle(w, batch=dw.batch, requests=reqs, keep_prefill=True)[1]["hidden"]
        _check_rows(got[rows], ref, plan.describe())
        # against the model with float64 activations the relative error stays within the bar too
        ref64 = run_oracle(w, batch=dw.batch, requests=reqs, keep_prefill=True, bf16_act=False)[1]["hidden"]
        assert errors(got[rows], ref64)[1] <= MEAN_REL
    finally:
        _release(dw)


def test_llama2_70b_slice_full_size_nano_2_and_4():
    """20 layers of the 70B shape at nano-batch counts 2 and 4: bitwise the same, layers match the oracle."""
    from synth import weights as SW
    dw = _dw("llama2_70b_slice", keep_logits=False, layer_outputs=True)
    try:
        outs = []
        for n in (2, 2, 4):
            for layer, pool in enumerate(dw.kv):   # fresh cache: the iteration writes its new K/V
                SW.gpu_fill_kv_pool(dw.shape, layer, pool)
            plan = dw.plan(nano=n)
            _forward(dw, plan)
            outs.append((plan.describe(), dw.hidden_out_f32.cpu().numpy()))
        for desc, o in outs[1:]:
            if not np.array_equal(o, outs[0][1]):
                bad = np.nonzero(np.any(o != outs[0][1], axis=1))[0]
                pytest.fail(f"plans {outs[0][0]} / {desc}: {bad.size} rows differ (first {bad[:8].tolist()}), "
                            f"max diff {np.abs(o - outs[0][1]).max():.3e}")
        _teacher_forced_layers("llama2_70b_slice", dw, [0, 511], [0, 10, 19])
    finally:
        _release(dw)


def test_mixtral_slice_full_size_routing_and_layers():
    """8 MoE layers, 1024 decode requests with lognormal contexts: routing and layer outputs."""
    dw = _dw("mixtral_8x7b_slice", keep_logits=False, moe_debug=True, layer_outputs=True)
    try:
        _forward(dw, dw.plan())
        reqs = [0, 1023]
        s = dw.shape
        layers = [0, 4, 7]
        extras = _teacher_forced_layers("mixtral_8x7b_slice", dw, reqs, layers)
        for layer in layers:
            z_gpu = dw.router_logits[layer].cpu().numpy().astype(np.float64)[reqs]
            z_ref = extras[layer]["router_logits"]
            zerr = np.abs(z_gpu - z_ref).max()
            idx = dw.topk_idx[layer].cpu().numpy()[reqs]
            srt = np.sort(z_ref, axis=1)[:, ::-1]
            for t in range(len(reqs)):
                own = sorted(range(s.n_experts), key=lambda e: (-z_gpu[t, e], e))[:s.top_k]
                assert idx[t].tolist() == own
                if srt[t, 1] - srt[t, 2] > 2 * zerr and srt[t, 0] - srt[t, 1] > 2 * zerr:
                    assert idx[t].tolist() == extras[layer]["topk_idx"][t].tolist(), (layer, t)
    finally:
        _release(dw)


def test_llama3_8b_full_model_layers_logits_and_greedy_tokens():
    """32 layers + LM head (vocabulary 128256), 512 decode requests + a 512-token chunk."""
    from oracle.forward import lm_head_argmax
    from synth import bf16_to_f64
    from synth import weights as SW
    dw = _dw("llama3_8b_full", keep_logits=True, layer_outputs=True)
    try:
        _forward(dw, dw.plan())
        reqs = [0, 511]
        _teacher_forced_layers("llama3_8b_full", dw, reqs, [0, 16, 31])
        s = dw.shape
        g = SW.global_specs(s)
        x_last = dw.layer_hidden[s.n_layers - 1].cpu().numpy().astype(np.float64)[reqs]
        ref, ref_tok = lm_head_argmax(x_last, bf16_to_f64(SW.host_tensor(g["final_norm"])),
                                      bf16_to_f64(SW.host_tensor(g["lm_head"])), s.rms_eps, bf16_act=True)
        logits = dw.logits.float().cpu().numpy()[reqs]
        mx, rel = errors(logits, ref)
        print(f"logits given the GPU's final hidden state: max-abs {mx:.4g}, relative L1 {rel:.4g}")
        assert mx <= MAX_ABS and rel <= MEAN_REL, (mx, rel)
        nxt = dw.next_token.cpu().numpy()[reqs]
        for i, tok in enumerate(nxt):
            top = np.sort(ref[i])[::-1]
            if top[0] - top[1] > 2 * mx:
                assert tok == ref_tok[i]
            else:
                assert ref[i, tok] >= top[0] - 2 * mx
    finally:
        _release(dw)
