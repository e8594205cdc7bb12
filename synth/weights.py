"""Seeded random-init weights, cached K/V pages and input activations.

Every tensor is an element-indexed stream of the generator in ``synth_cpu.c``
(host) / ``synth_gpu.cu`` (device): element i of tensor (seed, tid) is the same
bf16 value on both, so the oracle can regenerate any slice of an input that the
device filled in HBM.

Layouts are the ones the library's C ABI accepts: linear weights are
[out_features x in_features] row-major, norms are [hidden]. The paged KV pool of one
layer holds, per page, the physical image described by ``kv_phys_to_logical``; the
generator fills the physical pool element by element, and the host helpers below hand
the oracle the logical view [pages, 2 (K, V), n_kv_heads, page_size, head_dim].
"""
from __future__ import annotations

import math

import numpy as np

from . import (SEED_WEIGHTS, SEED_KV, SEED_INPUTS, IN_HIDDEN, W_Q, W_K, W_V, W_O, W_GATE, W_UP,
               W_DOWN, W_ATTN_NORM, W_FFN_NORM, W_ROUTER, W_ROUTER_BIAS, GLOBAL_LAYER, G_EMBED,
               G_LM_HEAD, G_FINAL_NORM, weight_tid, expert_kind, normal_bf16, ranges_normal_bf16,
               gpu_fill_normal_bf16)
from .workloads import ModelShape


def layer_specs(s: ModelShape, layer: int):
    """name -> (tensor id, shape, sigma, mean) of one transformer layer."""
    H, d, F = s.hidden, s.head_dim, s.ffn
    specs = {
        "wq": (weight_tid(layer, W_Q), (s.n_q_heads * d, H), s.w_sigma, 0.0),
        "wk": (weight_tid(layer, W_K), (s.n_kv_heads * d, H), s.w_sigma, 0.0),
        "wv": (weight_tid(layer, W_V), (s.n_kv_heads * d, H), s.w_sigma, 0.0),
        "wo": (weight_tid(layer, W_O), (H, s.n_q_heads * d), s.w_sigma, 0.0),
        "attn_norm": (weight_tid(layer, W_ATTN_NORM), (H,), s.norm_sigma, 1.0),
        "ffn_norm": (weight_tid(layer, W_FFN_NORM), (H,), s.norm_sigma, 1.0),
    }
    if s.n_experts == 0:
        specs["w_gate"] = (weight_tid(layer, W_GATE), (F, H), s.w_sigma, 0.0)
        specs["w_up"] = (weight_tid(layer, W_UP), (F, H), s.w_sigma, 0.0)
        specs["w_down"] = (weight_tid(layer, W_DOWN), (H, F), s.w_sigma, 0.0)
    else:
        rs = s.router_sigma if s.router_sigma > 0 else 1.0 / math.sqrt(H)
        specs["router"] = (weight_tid(layer, W_ROUTER), (s.n_experts, H), rs, 0.0)
        specs["router_bias"] = (weight_tid(layer, W_ROUTER_BIAS), (s.n_experts,), s.router_bias_sigma, 0.0)
        for e in range(s.n_experts):
            specs[f"e{e}_gate"] = (weight_tid(layer, expert_kind(e, 0)), (F, H), s.w_sigma, 0.0)
            specs[f"e{e}_up"] = (weight_tid(layer, expert_kind(e, 1)), (F, H), s.w_sigma, 0.0)
            specs[f"e{e}_down"] = (weight_tid(layer, expert_kind(e, 2)), (H, F), s.w_sigma, 0.0)
    return specs


def global_specs(s: ModelShape):
    if s.vocab <= 0:
        return {}
    g = lambda k: weight_tid(GLOBAL_LAYER, k)
    return {
        "embed": (g(G_EMBED), (s.vocab, s.hidden), s.w_sigma, 0.0),
        "lm_head": (g(G_LM_HEAD), (s.vocab, s.hidden), s.w_sigma, 0.0),
        "final_norm": (g(G_FINAL_NORM), (s.hidden,), s.norm_sigma, 1.0),
    }


def host_tensor(spec) -> np.ndarray:
    tid, shape, sigma, mean = spec
    n = int(np.prod(shape))
    return normal_bf16(SEED_WEIGHTS, tid, n, sigma, mean).reshape(shape)


def host_rows(spec, rows: np.ndarray) -> np.ndarray:
    """Selected rows of a 2-D weight (e.g. embedding rows of given token ids)."""
    tid, shape, sigma, mean = spec
    rows = np.asarray(rows, dtype=np.uint64)
    return ranges_normal_bf16(SEED_WEIGHTS, tid, rows * np.uint64(shape[1]), shape[1], sigma, mean)


def host_layer(s: ModelShape, layer: int) -> dict:
    return {k: host_tensor(v) for k, v in layer_specs(s, layer).items()}


def host_globals(s: ModelShape) -> dict:
    return {k: host_tensor(v) for k, v in global_specs(s).items()}


def kv_page_elems(s: ModelShape) -> int:
    return 2 * s.n_kv_heads * s.page_size * s.head_dim


def kv_phys_to_logical(phys: np.ndarray, s: ModelShape) -> np.ndarray:
    """Logical view [n, 2, nkv, 16, d] of physical page images [n, page elements].

    Physical order within a page: K|V, then 64-column half of the head dimension, then KV
    head, then the 16 rows (tokens), then eight 16-byte chunks of 8 elements, where logical
    chunk c of row r is stored at chunk position c XOR (r mod 8). Each (K|V, half, head)
    block is thus the 2 KB image of a 16 x 64 tile in 128-byte-swizzled form, and all heads
    of a half are one contiguous region.
    """
    n = phys.shape[0]
    nkv, d, P = s.n_kv_heads, s.head_dim, s.page_size
    h2 = d // 64
    a = np.asarray(phys).reshape(n, 2, h2, nkv, P, 8, 8)
    rows = np.arange(P)[:, None]
    src = np.arange(8)[None, :] ^ (rows & 7)
    a = a[:, :, :, :, rows, src, :]                       # [n, 2, h2, nkv, P, 8, 8], logical chunks
    return a.transpose(0, 1, 3, 4, 2, 5, 6).reshape(n, 2, nkv, P, d)


def host_kv_pool(s: ModelShape, layer: int, num_pages: int) -> np.ndarray:
    """Initial contents of a whole pool, logical view [num_pages, 2, nkv, P, d]."""
    n = num_pages * kv_page_elems(s)
    return kv_phys_to_logical(normal_bf16(SEED_KV, layer, n).reshape(num_pages, -1), s)


def host_kv_pages(s: ModelShape, layer: int, pages: np.ndarray) -> np.ndarray:
    """Initial contents of the listed pages of one layer's pool, logical view [len(pages), 2, nkv, P, d]."""
    pe = kv_page_elems(s)
    starts = np.asarray(pages, dtype=np.uint64) * np.uint64(pe)
    out = ranges_normal_bf16(SEED_KV, layer, starts, pe)
    return kv_phys_to_logical(out, s)


def host_input_hidden(s: ModelShape, num_tokens: int) -> np.ndarray:
    return normal_bf16(SEED_INPUTS, IN_HIDDEN, num_tokens * s.hidden).reshape(num_tokens, s.hidden)


def host_input_rows(s: ModelShape, rows: np.ndarray) -> np.ndarray:
    rows = np.asarray(rows, dtype=np.uint64)
    return ranges_normal_bf16(SEED_INPUTS, IN_HIDDEN, rows * np.uint64(s.hidden), s.hidden)


# --- device fills (torch tensors as plain device memory) ----------------------------------------

def gpu_fill(spec, tensor) -> None:
    tid, shape, sigma, mean = spec
    n = int(np.prod(shape))
    assert tensor.numel() == n and tensor.element_size() == 2 and tensor.is_contiguous()
    gpu_fill_normal_bf16(tensor.data_ptr(), n, SEED_WEIGHTS, tid, sigma, mean)


def gpu_fill_kv_pool(s: ModelShape, layer: int, tensor) -> None:
    assert tensor.element_size() == 2 and tensor.is_contiguous()
    gpu_fill_normal_bf16(tensor.data_ptr(), tensor.numel(), SEED_KV, layer)


def gpu_fill_input_hidden(tensor) -> None:
    gpu_fill_normal_bf16(tensor.data_ptr(), tensor.numel(), SEED_INPUTS, IN_HIDDEN)
