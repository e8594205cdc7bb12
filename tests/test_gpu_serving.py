"""Greedy serving through the scheduler and nf_forward_iteration on the GPU.

The same requests are served with the CPU one iteration ahead of the GPU (lag 1: tokens fed back on
the device, one dropped token per request) and in lock step (lag 0); the streams must be identical.
End tokens taken from those streams must cut them at their first occurrence. Every generated token
is checked against the float64 oracle run as plain greedy decoding: the whole sequence so far
(prompt + the GPU's own earlier tokens) as one fresh prompt, no KV cache, next token = argmax of the
last row's logits. A token passes if its oracle logit is within twice the logit tolerance of the
maximum (the decision is exact wherever the oracle's margin is wider than that).
"""
import gc

import numpy as np
import pytest
import torch

from parity import MAX_ABS
from synth.workloads import TEST_WORKLOADS, Batch

pytestmark = pytest.mark.gpu
DEV = "cuda:0"


def oracle_next_logits(shape, tokens):
    from oracle.forward import iteration_forward
    from oracle.run import layer_weights_f64, make_kv
    from synth import bf16_to_f64
    from synth import weights as SW
    L = len(tokens)
    n_pages = (L + shape.page_size - 1) // shape.page_size
    b = Batch(num_decode=0, prefill_len=L, ctx_lens=np.zeros(0, np.int32), page_size=shape.page_size,
              num_pages=n_pages, page_indptr=np.array([0, n_pages], np.int32),
              page_indices=np.arange(n_pages, dtype=np.int32), positions=np.arange(L, dtype=np.int32),
              tokens=np.asarray(tokens, np.int32))
    g = SW.global_specs(shape)
    res = iteration_forward(shape, b, lambda l: layer_weights_f64(shape, l), make_kv(shape),
                            embed_rows=lambda t: bf16_to_f64(SW.host_rows(g["embed"], t)),
                            final_norm=bf16_to_f64(SW.host_tensor(g["final_norm"])),
                            lm_head=bf16_to_f64(SW.host_tensor(g["lm_head"])), bf16_act=True)
    return res["logits"][0]


def _serve(dw, reqs, lag, num_pages=24):
    from intra_device_overlapped_b200.serving import ServingSession
    sess = ServingSession(dw.model, dw.shape, DEV, num_pages=num_pages, max_running=dw.R, chunk_len=dw.C,
                          max_position=4096, lag=lag)
    try:
        ids = [sess.add(p, m, e) for p, m, e in reqs]
        stats = sess.run()
        assert dw.sync() == 0
        return [sess.tokens(i) for i in ids], stats
    finally:
        sess.close()


def test_async_serving_matches_lockstep_and_greedy_oracle():
    from intra_device_overlapped_b200.harness import DeviceWorkload
    w = TEST_WORKLOADS["tiny_lm"]
    dw = DeviceWorkload(w, DEV, keep_logits=False)
    try:
        s = w.shape
        rng = np.random.default_rng(5)
        reqs = [(rng.integers(0, s.vocab, int(rng.integers(1, 33))).tolist(), int(rng.integers(1, 25)), -1)
                for _ in range(12)]
        a, sa = _serve(dw, reqs, 1)
        b, sb = _serve(dw, reqs, 0)
        assert a == b
        assert [len(t) for t in a] == [m for _, m, _ in reqs]
        assert sa["discarded_tokens"] == len(reqs) and sb["discarded_tokens"] == 0
        assert sa["free_pages"] == 24 and sb["free_pages"] == 24

        # end tokens: request i stops at the first occurrence of its stream's token at index j_i
        eos_reqs, want = [], []
        for (p, m, _), full in zip(reqs, a):
            e = full[int(rng.integers(0, len(full)))]
            eos_reqs.append((p, m, e))
            want.append(full[:full.index(e) + 1])
        c, _ = _serve(dw, eos_reqs, 1)
        assert c == want

        worst = 0.0
        exact = total = 0
        for (p, _, _), got in list(zip(reqs, a))[:5]:
            for j, tok in enumerate(got):
                z = oracle_next_logits(s, list(p) + got[:j])
                gap = float(z.max() - z[tok])
                worst = max(worst, gap)
                exact += int(gap == 0.0)
                total += 1
                assert gap <= 2 * MAX_ABS, (j, tok, int(np.argmax(z)), gap)
        print(f"greedy tokens equal to the oracle's argmax: {exact}/{total}; worst logit gap {worst:.3g}")
    finally:
        dw.close()
        dw.__dict__.clear()
        gc.collect()
        torch.cuda.empty_cache()
