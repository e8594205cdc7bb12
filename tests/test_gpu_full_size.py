"""Parity at the workloads' full sizes, in the bench's launch configuration, on sampled rows.

Each test builds the whole workload on the GPU (every layer's weights and paged KV pool, every
request), runs one serving iteration through nf_plan_iteration + nf_forward_iteration, and checks
sampled rows against the float64 oracle computed for those rows only:

* decode rows: the first and last request, the longest and shortest contexts, and the requests on
  both sides of several boundaries of the decode attention's work partition (the page-prefix
  fractions k / grid that the persistent kernel deals out). Decode rows are independent of one
  another (their attention reads only their own pages), so the oracle's sub-batch reproduces them.
* prefill-chunk rows: the first, a middle, the last and the rows on both sides of a 128-row tile
  boundary. The oracle projects K/V for every chunk row (causal attention reads them) and runs
  attention, the output projection and the FFN only for the sampled rows.

Two precision readings of the oracle are checked, each against the bars max-abs <= 2e-2 and
relative L1 <= 5e-3: the bf16 model (every tensor handed from one operation to the next is bf16)
and float64 activations. Hidden states are divided row by row by the oracle row's RMS before the
max-abs (residual values reach about 11 in these random-weight stacks, where one bf16 ulp of an
intermediate already moves outputs by about 2e-2); raw max-abs is printed beside it. Deep stacks are
checked layer by layer with teacher forcing (the oracle layer runs on the GPU's own input to that
layer), on every fourth layer and the last. Greedy tokens and MoE routing are compared exactly
wherever the oracle's decision margin exceeds twice the observed error of its inputs.
"""
import gc

import numpy as np
import pytest
import torch

from synth.workloads import WORKLOADS
from parity import MAX_ABS, MEAN_REL, errors, check_readings

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


def _forward(dw, plan, persistent=False):
    dw.forward(plan, persistent=persistent)
    st = dw.sync()
    assert st == 0, f"device status {st}"


def _decode_samples(batch, grid):
    """Decode requests to check: ends, extreme contexts, both sides of partition boundaries."""
    R = batch.num_decode
    ctx = np.asarray(batch.ctx_lens)
    pages = (ctx + 1 + 15) // 16
    prefix = np.concatenate([[0], np.cumsum(pages)])
    W = int(prefix[-1])
    picks = {0, R - 1, int(np.argmax(ctx)), int(np.argmin(ctx))}
    g = max(int(grid), 1)
    for b in sorted({1, g // 3, g // 2, (2 * g) // 3, g - 1}):
        if 0 < b < g:
            r = int(np.searchsorted(prefix, W * b // g, side="right")) - 1   # request holding that page
            picks.update({max(r - 1, 0), r, min(r + 1, R - 1)})
    return sorted(picks)


def _chunk_samples(batch):
    R, C = batch.num_decode, batch.prefill_len
    rows = {0, C // 2, C - 1, min(127, C - 1), min(128, C - 1)}
    return [R + r for r in sorted(rows)]


def _oracle_layer(name, dw, lw, layer, x_rows, reqs, chunk_rows, bf16_act):
    """Oracle layer on a sub-batch (sampled decode requests + the whole chunk); returns the rows
    of the sampled requests followed by the sampled chunk rows."""
    from oracle.forward import layer_forward, sub_batch
    from oracle.run import make_kv
    s = WORKLOADS[name].shape
    sb = sub_batch(dw.batch, reqs, keep_prefill=True)
    R = dw.batch.num_decode
    rows = list(range(len(reqs))) + [len(reqs) + (t - R) for t in chunk_rows]
    return layer_forward(s, lw, x_rows, sb, make_kv(s), layer, bf16_act, rows=rows)


def _input_rows(name, dw, reqs, layer):
    """GPU input of `layer` for the sampled requests and every chunk row (teacher forcing)."""
    from synth import bf16_to_f64
    from synth import weights as SW
    s = WORKLOADS[name].shape
    R, T = dw.batch.num_decode, dw.T
    rows = list(reqs) + list(range(R, T))
    if layer > 0:
        return dw.layer_hidden[layer - 1].cpu().numpy().astype(np.float64)[rows]
    if s.vocab > 0:
        return bf16_to_f64(SW.host_rows(SW.global_specs(s)["embed"], np.asarray(dw.batch.tokens)[rows]))
    return bf16_to_f64(SW.host_input_rows(s, np.asarray(rows)))


def _teacher_forced(name, dw, reqs, chunk_rows, layers):
    """Each listed layer: both oracle readings on the GPU's input rows against the GPU's output rows."""
    from oracle.run import layer_weights_f64
    extras = {}
    for layer in layers:
        x_rows = _input_rows(name, dw, reqs, layer)
        got = dw.layer_hidden[layer].cpu().numpy().astype(np.float64)[list(reqs) + list(chunk_rows)]
        lw = layer_weights_f64(WORKLOADS[name].shape, layer)
        refs = {}
        for label, bf in (("bf16 model", True), ("float64 activations", False)):
            out, ex = _oracle_layer(name, dw, lw, layer, x_rows, reqs, chunk_rows, bf)
            refs[label] = out
            if bf:
                extras[layer] = ex
        check_readings(got, refs, f"{name} layer {layer} ({len(reqs)} decode + {len(chunk_rows)} chunk rows)")
    return extras


def _every_fourth(n_layers):
    return sorted(set(range(0, n_layers, 4)) | {n_layers - 1})


def test_llama3_8b_layer_full_size_planner_plan():
    """512 decode requests (context U[1024,1536]) + a 1024-token chunk, the planner's plan: sampled
    decode rows and the whole chunk against both oracle readings."""
    from oracle.run import run_oracle
    name = "llama3_8b_layer"
    dw = _dw(name, keep_logits=False)
    try:
        dw.calibrate()
        plan = dw.plan()
        _forward(dw, plan)
        got = dw.hidden_out_f32.cpu().numpy().astype(np.float64)
        reqs = _decode_samples(dw.batch, plan.sm_attn)
        R = dw.batch.num_decode
        rows = reqs + list(range(R, dw.T))
        w = WORKLOADS[name]
        refs = {label: run_oracle(w, batch=dw.batch, requests=reqs, keep_prefill=True, bf16_act=bf)[1]["hidden"]
                for label, bf in (("bf16 model", True), ("float64 activations", False))}
        check_readings(got[rows], refs, f"{name}, {len(reqs)} decode rows + whole chunk, {plan.describe()}")
    finally:
        _release(dw)


def test_llama2_70b_slice_full_size_nano_2_and_4():
    """20 layers of the 70B shape (64 query heads) at nano-batch counts 2 and 4, and the 2-nano-batch
    plan again with each layer as one persistent kernel: bitwise the same; every fourth layer
    matches the oracle on sampled decode and chunk rows."""
    from synth import weights as SW
    name = "llama2_70b_slice"
    dw = _dw(name, keep_logits=False, layer_outputs=True)
    try:
        outs = []
        for n, persistent in ((2, False), (2, False), (4, False), (2, True)):
            for layer, pool in enumerate(dw.kv):   # fresh cache: the iteration writes its new K/V
                SW.gpu_fill_kv_pool(dw.shape, layer, pool)
            plan = dw.plan(nano=n)
            _forward(dw, plan, persistent)
            outs.append((str(plan.describe()) + (" persistent" if persistent else ""), dw.hidden_out_f32.cpu().numpy()))
        for desc, o in outs[1:]:
            if not np.array_equal(o, outs[0][1]):
                bad = np.nonzero(np.any(o != outs[0][1], axis=1))[0]
                pytest.fail(f"plans {outs[0][0]} / {desc}: {bad.size} rows differ (first {bad[:8].tolist()}), "
                            f"max diff {np.abs(o - outs[0][1]).max():.3e}")
        reqs = _decode_samples(dw.batch, plan.sm_attn)
        _teacher_forced(name, dw, reqs, _chunk_samples(dw.batch), _every_fourth(dw.shape.n_layers))
    finally:
        _release(dw)


def test_mixtral_slice_full_size_routing_and_layers():
    """8 MoE layers, 1024 decode requests with lognormal contexts (up to 4097 keys): routing and
    layer outputs on sampled decode rows (the longest context among them) and chunk rows."""
    name = "mixtral_8x7b_slice"
    dw = _dw(name, keep_logits=False, moe_debug=True, layer_outputs=True)
    try:
        plan = dw.plan()
        _forward(dw, plan)
        reqs = _decode_samples(dw.batch, plan.sm_attn)
        chunk = _chunk_samples(dw.batch)
        s = dw.shape
        layers = [0, 2, 4, 6, 7]
        extras = _teacher_forced(name, dw, reqs, chunk, layers)
        rows = list(reqs) + list(chunk)
        for layer in layers:
            z_gpu = dw.router_logits[layer].cpu().numpy().astype(np.float64)[rows]
            z_ref = extras[layer]["router_logits"]
            zerr = np.abs(z_gpu - z_ref).max()
            idx = dw.topk_idx[layer].cpu().numpy()[rows]
            srt = np.sort(z_ref, axis=1)[:, ::-1]
            for t in range(len(rows)):
                own = sorted(range(s.n_experts), key=lambda e: (-z_gpu[t, e], e))[:s.top_k]
                assert idx[t].tolist() == own
                if srt[t, 1] - srt[t, 2] > 2 * zerr and srt[t, 0] - srt[t, 1] > 2 * zerr:
                    assert idx[t].tolist() == extras[layer]["topk_idx"][t].tolist(), (layer, t)
    finally:
        _release(dw)


def test_llama3_8b_full_model_layers_logits_and_greedy_tokens():
    """32 layers + LM head (vocabulary 128256), 512 decode requests + a 512-token chunk: every fourth
    layer teacher-forced on sampled decode and chunk rows, then the logits and greedy tokens of the
    sampled LM-head rows from the GPU's final hidden state."""
    from oracle.forward import lm_head_argmax
    from synth import bf16_to_f64
    from synth import weights as SW
    name = "llama3_8b_full"
    dw = _dw(name, keep_logits=True, layer_outputs=True)
    try:
        plan = dw.plan()
        _forward(dw, plan)
        reqs = _decode_samples(dw.batch, plan.sm_attn)
        _teacher_forced(name, dw, reqs, _chunk_samples(dw.batch), _every_fourth(dw.shape.n_layers))
        s = dw.shape
        g = SW.global_specs(s)
        R, T = dw.batch.num_decode, dw.T
        lm_rows = list(reqs) + [T - 1]                      # the chunk's last row produces a token too
        out_rows = list(reqs) + [R]                         # its logits row is row R
        x_last = dw.layer_hidden[s.n_layers - 1].cpu().numpy().astype(np.float64)[lm_rows]
        fn, head = bf16_to_f64(SW.host_tensor(g["final_norm"])), bf16_to_f64(SW.host_tensor(g["lm_head"]))
        refs = {}
        for label, bf in (("bf16 model", True), ("float64 activations", False)):
            refs[label], tok = lm_head_argmax(x_last, fn, head, s.rms_eps, bf16_act=bf)
            if bf:
                ref, ref_tok = refs[label], tok
        logits = dw.logits.float().cpu().numpy()[out_rows]
        check_readings(logits, refs, "logits given the GPU's final hidden state", row_scaled=False)
        mx = errors(logits, ref)[0]
        nxt = dw.next_token.cpu().numpy()[out_rows]
        for i, tok in enumerate(nxt):
            top = np.sort(ref[i])[::-1]
            if top[0] - top[1] > 2 * mx:
                assert tok == ref_tok[i]
            else:
                assert ref[i, tok] >= top[0] - 2 * mx
    finally:
        _release(dw)
