"""CPU oracle of one batched serving iteration (test infrastructure only).

This package is the slow, plain reference that the CUDA path is checked
against. Only the test suite, the smoke check of ``__graft_entry__`` and the
CPU-baseline leg of ``bench.py`` may import it; the library itself never does.
It shares no code with the CUDA path: its only dependency besides numpy is the
``synth`` input generator, which holds none of the iteration's arithmetic.

Everything is computed in float64 (numpy; dense contractions go through numpy's
matmul as a library primitive) from bf16 inputs widened exactly. The paged KV
cache's element type is bf16: newly written K and V are rounded when stored and
attention reads them back from the cache. Two precision readings of the
activations are offered (``bf16_act``): the bf16 model, in which every tensor one
operation hands to the next is rounded to bf16 (the default), and float64
activations throughout (``bf16_act=False``), the stricter reference the parity
bars are also checked against.
"""
from .forward import (bf16_round, rmsnorm, rope_cos_sin, apply_rope, attention, decode_attention,
                      prefill_attention, silu, swiglu_ffn, moe_route, moe_ffn, lm_head_argmax,
                      PagedKV, layer_forward, iteration_forward, sub_batch)

__all__ = ["bf16_round", "rmsnorm", "rope_cos_sin", "apply_rope", "attention", "decode_attention",
           "prefill_attention", "silu", "swiglu_ffn", "moe_route", "moe_ffn", "lm_head_argmax",
           "PagedKV", "layer_forward", "iteration_forward", "sub_batch"]
