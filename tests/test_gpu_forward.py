"""Whole-iteration parity on the GPU: nf_plan_iteration + nf_forward_iteration against the
float64 oracle, plus the nano-batching invariant (every plan gives bitwise the same result).
"""
import numpy as np
import pytest
import torch

from synth.workloads import WORKLOADS, TEST_WORKLOADS
from synth import weights as SW
import synth

from parity import MAX_ABS, MEAN_REL, errors, check_readings

pytestmark = pytest.mark.gpu
DEV = "cuda:0"


def _bits(t):
    return t.detach().contiguous().view(torch.int16).cpu().numpy()


def _run(dw, plan):
    dw.forward(plan)
    st = dw.sync()
    assert st == 0, f"device status {st}"
    return dw.hidden_out_f32.cpu().numpy().astype(np.float64)


def _reset_kv(dw):
    for layer, pool in enumerate(dw.kv):
        SW.gpu_fill_kv_pool(dw.shape, layer, pool)
    torch.cuda.synchronize()


@pytest.fixture(scope="module")
def tiny():
    from intra_device_overlapped_b200.harness import DeviceWorkload
    from oracle.run import run_oracle
    w = TEST_WORKLOADS["tiny_gamma"]
    dw = DeviceWorkload(w, DEV)
    b, res, kv = run_oracle(w, batch=dw.batch)
    res["hidden_f64"] = run_oracle(w, batch=dw.batch, bf16_act=False)[1]["hidden"]
    yield dw, res, kv
    dw.close()


PLANS = [dict(nano=1, template=0), dict(nano=2, template=1, sm_attn=16), dict(nano=3, template=1, sm_attn=40),
         dict(nano=4, template=1, sm_attn=64), dict(nano=2, template=0), dict(nano=2, template=2, sm_attn=24),
         dict(nano=3, template=2, sm_attn=52), dict(nano=1, template=2, sm_attn=120)]


@pytest.mark.parametrize("opts", PLANS)
def test_tiny_iteration_matches_oracle(tiny, opts):
    dw, res, _ = tiny
    _reset_kv(dw)
    plan = dw.plan(**opts)
    hid = _run(dw, plan)
    check_readings(hid, {"bf16 model": res["hidden"], "float64 activations": res["hidden_f64"]},
                   f"tiny layer, plan {plan.describe()}")
    # bf16 output copy is the rounded fp32 residual
    hb = dw.hidden_out.float().cpu().numpy()
    assert np.abs(hb - hid).max() <= np.abs(hid).max() * 2 ** -8


def test_tiny_nano_batching_is_bitwise_invariant(tiny):
    dw, _, _ = tiny
    outs, kvs = [], []
    for opts in PLANS + [dict()]:
        _reset_kv(dw)
        plan = dw.plan(**opts)
        _run(dw, plan)
        outs.append(_bits(dw.hidden_out_f32))
        kvs.append(_bits(dw.kv[0]))
    for o, k in zip(outs[1:], kvs[1:]):
        assert np.array_equal(o, outs[0])
        assert np.array_equal(k, kvs[0])


def test_tiny_kv_slots_written_and_others_untouched(tiny):
    dw, res, kv_oracle = tiny
    _reset_kv(dw)
    _run(dw, dw.plan(nano=2, template=1, sm_attn=20))
    from intra_device_overlapped_b200.harness import kv_logical
    s, b = dw.shape, dw.batch
    got = synth.bf16_to_f64(kv_logical(dw, 0))
    init = synth.bf16_to_f64(SW.host_kv_pool(s, 0, b.num_pages))
    written = res["layers"][0]["written"]
    mask = np.zeros(got.shape, dtype=bool)
    worst = 0.0
    for t, (page, slot) in written.items():
        mask[page, :, :, slot, :] = True
        ref = kv_oracle.pages[(0, page)][:, :, slot, :]
        worst = max(worst, float(np.abs(got[page, :, :, slot, :] - ref).max()))
    assert worst <= MAX_ABS, worst
    assert np.array_equal(got[~mask], init[~mask])          # every other slot bit-identical


def test_tiny_iteration_is_idempotent(tiny):
    dw, _, _ = tiny
    _reset_kv(dw)
    plan = dw.plan(nano=2, template=1, sm_attn=24)
    a = _run(dw, plan).copy()
    b = _run(dw, plan)          # same K/V rewritten into the same slots
    assert np.array_equal(a, b)


@pytest.mark.parametrize("name", ["tiny_decode_only", "tiny_prefill_only"])
def test_degenerate_batches(name):
    from intra_device_overlapped_b200.harness import DeviceWorkload
    from oracle.run import run_oracle
    w = TEST_WORKLOADS[name]
    dw = DeviceWorkload(w, DEV)
    try:
        _, res, _ = run_oracle(w, batch=dw.batch)
        ref64 = run_oracle(w, batch=dw.batch, bf16_act=False)[1]["hidden"]
        for opts in (dict(nano=1, template=0), dict()):
            _reset_kv(dw)
            hid = _run(dw, dw.plan(**opts))
            check_readings(hid, {"bf16 model": res["hidden"], "float64 activations": ref64}, f"{name} {opts}")
    finally:
        dw.close()


def test_tiny_lm_head_and_argmax():
    from intra_device_overlapped_b200.harness import DeviceWorkload
    from oracle.run import run_oracle
    w = TEST_WORKLOADS["tiny_lm"]
    dw = DeviceWorkload(w, DEV)
    try:
        _, res, _ = run_oracle(w, batch=dw.batch)
        res64 = run_oracle(w, batch=dw.batch, bf16_act=False)[1]
        _run(dw, dw.plan(nano=2, template=1, sm_attn=32))
        logits = dw.logits.float().cpu().numpy()
        check_readings(logits, {"bf16 model": res["logits"], "float64 activations": res64["logits"]},
                       "tiny LM logits", row_scaled=False)
        mx, rel = errors(logits, res["logits"])
        nxt = dw.next_token.cpu().numpy()
        ref = res["logits"]
        for r, tok in enumerate(nxt):
            top = np.sort(ref[r])[::-1]
            if top[0] - top[1] > 2 * mx:
                assert tok == res["next_token"][r]
            else:  # inside the error margin: the GPU's choice must be a near-maximum
                assert ref[r, tok] >= top[0] - 2 * mx
    finally:
        dw.close()


def test_tiny_moe_routing_and_output():
    from intra_device_overlapped_b200.harness import DeviceWorkload
    from oracle.run import run_oracle
    w = TEST_WORKLOADS["tiny_moe"]
    dw = DeviceWorkload(w, DEV, moe_debug=True)
    try:
        _, res, _ = run_oracle(w, batch=dw.batch)
        res64 = run_oracle(w, batch=dw.batch, bf16_act=False)[1]
        hid = _run(dw, dw.plan(nano=2, template=1, sm_attn=24))
        check_readings(hid, {"bf16 model": res["hidden"], "float64 activations": res64["hidden"]}, "tiny MoE")
        for layer in range(w.shape.n_layers):
            z_gpu = dw.router_logits[layer].cpu().numpy().astype(np.float64)
            z_ref = res["layers"][layer]["router_logits"]
            zerr = np.abs(z_gpu - z_ref).max()
            idx = dw.topk_idx[layer].cpu().numpy()
            srt = np.sort(z_ref, axis=1)[:, ::-1]
            for t in range(dw.T):
                # routing function on the GPU's own logits is exact (top-2, ties to the lower index)
                own = sorted(range(w.shape.n_experts), key=lambda e: (-z_gpu[t, e], e))[:2]
                assert idx[t].tolist() == own
                if srt[t, 1] - srt[t, 2] > 2 * zerr and srt[t, 0] - srt[t, 1] > 2 * zerr:
                    assert idx[t].tolist() == res["layers"][layer]["topk_idx"][t].tolist()
    finally:
        dw.close()


def test_gqa8_iteration_matches_oracle_and_is_invariant():
    """Head shape of the Llama-3-8B layer (32 query / 8 KV heads of 128): tensor-core decode path."""
    from intra_device_overlapped_b200.harness import DeviceWorkload
    from oracle.run import run_oracle
    w = TEST_WORKLOADS["small_gqa8"]
    dw = DeviceWorkload(w, DEV)
    try:
        _, res, _ = run_oracle(w, batch=dw.batch)
        ref64 = run_oracle(w, batch=dw.batch, bf16_act=False)[1]["hidden"]
        outs = []
        for opts in (dict(nano=1, template=0), dict(nano=2, template=1, sm_attn=20),
                     dict(nano=3, template=2, sm_attn=36), dict()):
            _reset_kv(dw)
            hid = _run(dw, dw.plan(**opts))
            check_readings(hid, {"bf16 model": res["hidden"], "float64 activations": ref64}, f"small_gqa8 {opts}")
            outs.append(_bits(dw.hidden_out_f32))
        for o in outs[1:]:
            assert np.array_equal(o, outs[0])
    finally:
        dw.close()


def test_tuned_plan_is_bitwise_equal_to_sequential():
    """nf_tune_plan returns one of the planner's plans, timed on the device; any plan gives the same bits."""
    from intra_device_overlapped_b200.harness import DeviceWorkload
    w = TEST_WORKLOADS["small_gqa8"]
    dw = DeviceWorkload(w, DEV)
    try:
        _reset_kv(dw)
        _run(dw, dw.plan(nano=1, template=0))
        ref = _bits(dw.hidden_out_f32)
        plan, us = dw.tune(reps=2)
        assert us > 0 and 1 <= plan.n_nano <= 4
        _reset_kv(dw)
        _run(dw, plan)
        assert np.array_equal(_bits(dw.hidden_out_f32), ref)
    finally:
        dw.close()


# --- bit-exact decisions: planted exact ties and the embedding gather -------------------------------

def test_lm_head_exact_ties_pick_the_lower_index():
    """LM head with every row zero except rows 5 and 900, which are equal: the fp32 logits of those two
    columns are identical and every other logit is exactly 0. The greedy token must be 5 where that
    shared logit is positive and 0 (the first of the zero logits) where it is negative: ties go to
    the lower index, bit-exactly, across the tile-wise maximum and its reduction."""
    from intra_device_overlapped_b200.harness import DeviceWorkload
    w = TEST_WORKLOADS["tiny_lm"]
    dw = DeviceWorkload(w, DEV)
    try:
        def edit(t):
            head = t["lm_head"]
            row = head[5].clone()
            head.zero_()
            head[5] = row
            head[900] = row
        dw.load_globals(edit)
        _run(dw, dw.plan(nano=2, template=1, sm_attn=32))
        logits = dw.logits.float().cpu().numpy()
        nxt = dw.next_token.cpu().numpy()
        assert np.array_equal(logits[:, 5], logits[:, 900])
        others = np.delete(logits, [5, 900], axis=1)
        assert np.all(others == 0.0)
        expect = np.where(logits[:, 5] > 0, 5, 0)
        assert np.any(expect == 5) and np.any(expect == 0)   # both tie kinds occur
        assert np.array_equal(nxt, expect), (nxt, expect)
    finally:
        dw.close()


@pytest.mark.parametrize("tie", ["all_equal", "pair"])
def test_router_exact_ties_pick_the_lower_experts(tie):
    """Router rows made equal: 'all_equal' gives every expert the same logit (top-2 must be experts
    0 and 1 with weights 1/2 each); 'pair' gives experts 1 and 3 the same row and a bias above the
    others (top-2 must be [1, 3]). Routing is compared bit-exactly on every token and layer."""
    from intra_device_overlapped_b200.harness import DeviceWorkload
    w = TEST_WORKLOADS["tiny_moe"]
    dw = DeviceWorkload(w, DEV, moe_debug=True)
    try:
        def edit(t):
            r, b = t["router"], t["router_bias"]
            if tie == "all_equal":
                r[:] = r[0].clone()
                b[:] = b[0].clone()
            else:
                r[3] = r[1].clone()
                b[:] = -8.0
                b[1] = 8.0
                b[3] = 8.0
        for layer in range(w.shape.n_layers):
            dw.load_layer(layer, edit)
        _run(dw, dw.plan(nano=2, template=1, sm_attn=24))
        want = [0, 1] if tie == "all_equal" else [1, 3]
        for layer in range(w.shape.n_layers):
            idx = dw.topk_idx[layer].cpu().numpy()
            assert np.all(idx == np.array(want)[None, :]), (layer, idx[:4])
            if tie == "all_equal":
                assert np.all(dw.topk_w[layer].cpu().numpy() == 0.5)
    finally:
        dw.close()


def test_embedding_gather_is_bit_exact():
    """With the output and down projections zeroed, every layer adds exact zeros to the residual
    stream, so the fp32 hidden state leaving the model is the gathered embedding row of each token:
    compared bit for bit with the bf16 table widened to fp32."""
    from intra_device_overlapped_b200.harness import DeviceWorkload
    w = TEST_WORKLOADS["tiny_lm"]
    dw = DeviceWorkload(w, DEV)
    try:
        def zero_out(t):
            t["wo"].zero_()
            t["w_down"].zero_()
        for layer in range(w.shape.n_layers):
            dw.load_layer(layer, zero_out)
        _run(dw, dw.plan(nano=2, template=1, sm_attn=32))
        got = dw.hidden_out_f32.cpu().numpy()
        emb = synth.bf16_to_f64(SW.host_rows(SW.global_specs(w.shape)["embed"], np.asarray(dw.batch.tokens)))
        assert np.array_equal(got.astype(np.float64), emb)
    finally:
        dw.close()
