"""Assemble the oracle's inputs from the seeded generator and run one iteration.

Test infrastructure only. Weights and cached K/V are regenerated on the host
from the same element-indexed streams the device fills, so sampled rows of even
the largest workloads can be recomputed without holding the whole model.
"""
from __future__ import annotations

import numpy as np

from synth import bf16_to_f64
from synth.workloads import Workload, make_batch
from synth import weights as W

from .forward import PagedKV, iteration_forward, sub_batch


def layer_weights_f64(shape, layer: int) -> dict:
    return {k: bf16_to_f64(v) for k, v in W.host_layer(shape, layer).items()}


def make_kv(shape) -> PagedKV:
    return PagedKV(lambda layer, pages: bf16_to_f64(W.host_kv_pages(shape, layer, pages)), shape.page_size)


def run_oracle(work: Workload, batch=None, requests=None, keep_prefill: bool = True,
               keep_layer_inputs: bool = False, weights_cache: dict | None = None, bf16_act: bool = True):
    """Oracle outputs for ``work``; with ``requests`` only those decode rows (and the chunk if kept).

    Returns (sub-batch actually computed, result dict, kv cache object).
    """
    s = work.shape
    full = batch if batch is not None else make_batch(work)
    b = full if requests is None else sub_batch(full, requests, keep_prefill)
    kv = make_kv(s)

    def lw(layer):
        if weights_cache is not None:
            if layer not in weights_cache:
                weights_cache[layer] = layer_weights_f64(s, layer)
            return weights_cache[layer]
        return layer_weights_f64(s, layer)

    kwargs = {}
    if s.vocab > 0:
        g = W.global_specs(s)
        kwargs["embed_rows"] = lambda toks: bf16_to_f64(W.host_rows(g["embed"], toks))
        kwargs["final_norm"] = bf16_to_f64(W.host_tensor(g["final_norm"]))
        kwargs["lm_head"] = bf16_to_f64(W.host_tensor(g["lm_head"]))
        x_in = None
    else:
        if requests is None:
            x_in = bf16_to_f64(W.host_input_hidden(s, full.num_tokens))
        else:
            rows = list(requests)
            if keep_prefill:
                rows += list(range(full.num_decode, full.num_tokens))
            x_in = bf16_to_f64(W.host_input_rows(s, np.array(rows, dtype=np.int64)))
    res = iteration_forward(s, b, lw, kv, x_in=x_in, keep_layer_inputs=keep_layer_inputs, bf16_act=bf16_act,
                            **kwargs)
    return b, res, kv
