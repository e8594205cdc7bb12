"""Float64 CPU forward of one mixed prefill + decode serving iteration.

Test infrastructure only (see the package docstring). The iteration is the one
the NanoFlow pages schedule: a batch of decode requests plus a prefill chunk
through a Llama-style transformer (arXiv abstract and README "Feasibility":
LLaMA-2-70B, LLaMA-3-8B, Mixtral 8x7B). The pages give no equations; the layer
is the standard Llama / Mixtral layer, written out here step by step:

    n  = RMSNorm(x) * gamma_attn
    q, k, v = n Wq^T, n Wk^T, n Wv^T             rotate-half RoPE on q and k
    K/V of the new tokens -> paged cache (bf16)
    o  = softmax(q K^T / sqrt(d)) V               per request, GQA head map h -> h // G
    h  = x + o Wo^T
    n2 = RMSNorm(h) * gamma_ffn
    x' = h + (silu(n2 Wg^T) * (n2 Wu^T)) Wd^T     dense SwiGLU, or
    x' = h + sum_k w_k E_{i_k}(n2)                top-k mixture of SwiGLU experts

NanoFlow's nano-batching cuts the batch into smaller pieces and runs a copy of
each operation on every piece on its own (arXiv abstract of the NanoFlow paper):
a schedule, not an approximation. The oracle therefore computes the
unsplit batch; every nano-batch plan must reproduce it.

Precision. The model runs in bf16 with fp32 accumulation, so every tensor one
operation hands to the next is a bf16 tensor. With ``bf16_act`` (the default) the
oracle rounds exactly those tensors to bf16 and computes everything else in
float64: the operand of each projection is the bf16 copy of the residual stream x
(RMSNorm's 1/rms and gamma scale the product, so n = bf16(x) / rms(x) * gamma with
rms taken over the unrounded x); q after RoPE; K and V in the cache; the attention
output; the SwiGLU activation; and the attention weights that multiply V (see
``attention``). The residual stream itself, the router logits, the softmax sums and
all accumulations stay unrounded. With ``bf16_act=False`` nothing but the inputs,
weights and cache is bf16.
"""
from __future__ import annotations

import math
from typing import Callable, Dict, Optional, Sequence

import numpy as np


# --- elementwise definitions ----------------------------------------------------------------------

def bf16_round(x) -> np.ndarray:
    """Round float64 values to the nearest bf16 value (8 significant bits, ties to even).

    Applied where the data format is bf16: the paged KV cache, and (bf16 model) the tensors one
    operation hands to the next.
    """
    x = np.asarray(x, dtype=np.float64)
    m, e = np.frexp(x)                      # x = m * 2**e with 0.5 <= |m| < 1
    return np.ldexp(np.round(np.ldexp(m, 8)), e - 8)


def rmsnorm(x: np.ndarray, gamma: np.ndarray, eps: float) -> np.ndarray:
    """RMSNorm (Zhang & Sennrich, 2019) over the last axis: x / sqrt(mean(x^2) + eps) * gamma."""
    ms = np.mean(x * x, axis=-1, keepdims=True)
    return x / np.sqrt(ms + eps) * gamma


def rope_cos_sin(positions: np.ndarray, head_dim: int, theta: float):
    """cos/sin of the rotary angles pos * theta^(-2i/d), i in [0, d/2) (RoFormer, Su et al. 2021)."""
    i = np.arange(head_dim // 2, dtype=np.float64)
    inv_freq = theta ** (-2.0 * i / head_dim)
    ang = np.asarray(positions, dtype=np.float64)[:, None] * inv_freq[None, :]
    return np.cos(ang), np.sin(ang)


def apply_rope(x: np.ndarray, cos: np.ndarray, sin: np.ndarray) -> np.ndarray:
    """Rotate-half RoPE: dimension i pairs with i + d/2. x is [T, heads, d]; cos/sin are [T, d/2]."""
    half = x.shape[-1] // 2
    x1, x2 = x[..., :half], x[..., half:]
    c, s = cos[:, None, :], sin[:, None, :]
    return np.concatenate([x1 * c - x2 * s, x2 * c + x1 * s], axis=-1)


def silu(z: np.ndarray) -> np.ndarray:
    """SiLU / swish: z * sigmoid(z) = z / (1 + exp(-z))."""
    return z / (1.0 + np.exp(-z))


# --- attention ------------------------------------------------------------------------------------

def attention(q: np.ndarray, k: np.ndarray, v: np.ndarray, q_pos: np.ndarray, k_pos: np.ndarray,
              bf16_p: bool = False) -> np.ndarray:
    """Scaled dot-product attention with a position mask (key j visible to query i iff k_pos[j] <= q_pos[i]).

    q is [Tq, nq, d]; k, v are [Tk, nkv, d]; query head h reads KV head h // (nq // nkv) (GQA).
    Softmax with max subtraction, all in float64. Returns [Tq, nq, d].

    With bf16_p, the weights that multiply V form a bf16 matrix, as in a bf16 model: in the log2
    domain x = s * log2(e), P = bf16(2^(x - M)) with M the integer ceiling of the row maximum, and
    the output is (P V) / sum 2^(x - M) (the sum unrounded). For any integer M the bf16 rounding of
    2^(x - M) differs only by the exact power of two 2^(M' - M), so this P is defined independently
    of how an implementation blocks the keys, as long as its running maximum stays integral.
    """
    Tq, nq, d = q.shape
    nkv = k.shape[1]
    G = nq // nkv
    visible = np.asarray(k_pos)[None, :] <= np.asarray(q_pos)[:, None]
    out = np.zeros((Tq, nq, v.shape[2]), dtype=np.float64)
    for h in range(nq):
        g = h // G
        s = (q[:, h, :] @ k[:, g, :].T) / math.sqrt(d)
        s = np.where(visible, s, -np.inf)
        if bf16_p:
            x = s * math.log2(math.e)
            p = np.exp2(x - np.ceil(x.max(axis=1, keepdims=True)))
            out[:, h, :] = (bf16_round(p) @ v[:, g, :]) / p.sum(axis=1, keepdims=True)
            continue
        s = s - s.max(axis=1, keepdims=True)
        p = np.exp(s)
        p = p / p.sum(axis=1, keepdims=True)
        out[:, h, :] = p @ v[:, g, :]
    return out


def decode_attention(q: np.ndarray, k: np.ndarray, v: np.ndarray, bf16_p: bool = False) -> np.ndarray:
    """One decode query [nq, d] over all of its request's keys [n, nkv, d] (its own new key included)."""
    n = k.shape[0]
    return attention(q[None], k, v, np.array([n - 1]), np.arange(n), bf16_p)[0]


def prefill_attention(q: np.ndarray, k: np.ndarray, v: np.ndarray, prefix_len: int = 0,
                      bf16_p: bool = False) -> np.ndarray:
    """Causal attention of a prefill chunk: query at position prefix+i sees keys 0..prefix+i."""
    C = q.shape[0]
    return attention(q, k, v, prefix_len + np.arange(C), np.arange(k.shape[0]), bf16_p)


# --- feed-forward ---------------------------------------------------------------------------------

def swiglu_ffn(n: np.ndarray, w_gate: np.ndarray, w_up: np.ndarray, w_down: np.ndarray,
               bf16_act: bool = False) -> np.ndarray:
    """SwiGLU FFN (Shazeer 2020): (silu(n Wg^T) * (n Wu^T)) Wd^T; with bf16_act the activation
    silu(n Wg^T) * (n Wu^T), the tensor handed to the down projection, is a bf16 tensor."""
    act = silu(n @ w_gate.T) * (n @ w_up.T)
    if bf16_act:
        act = bf16_round(act)
    return act @ w_down.T


def moe_route(z: np.ndarray, top_k: int):
    """Top-k experts per row of router logits z [T, E] (ties: lower expert index first),
    with weights softmax over the selected logits (Mixtral routing)."""
    order = np.argsort(-z, axis=1, kind="stable")
    idx = order[:, :top_k]
    zs = np.take_along_axis(z, idx, axis=1)
    zs = zs - zs.max(axis=1, keepdims=True)
    w = np.exp(zs)
    w = w / w.sum(axis=1, keepdims=True)
    return idx, w


def moe_ffn(n: np.ndarray, experts: Sequence, idx: np.ndarray, w: np.ndarray, bf16_act: bool = False) -> np.ndarray:
    """sum_k w[t,k] * SwiGLU_{idx[t,k]}(n[t]) with k ascending; experts[e] = (w_gate, w_up, w_down)."""
    T, K = idx.shape
    y = np.zeros((T, experts[0][2].shape[0]), dtype=np.float64)
    for e, (wg, wu, wd) in enumerate(experts):
        for kk in range(K):
            rows = np.nonzero(idx[:, kk] == e)[0]
            if rows.size:
                y[rows] += w[rows, kk:kk + 1] * swiglu_ffn(n[rows], wg, wu, wd, bf16_act)
    return y


def norm_operand(x: np.ndarray, gamma: np.ndarray, eps: float, bf16_act: bool) -> np.ndarray:
    """RMSNorm(x) * gamma as a projection consumes it: with bf16_act the product's operand is the
    bf16 copy of x, scaled by 1/rms of the unrounded x and by gamma."""
    if not bf16_act:
        return rmsnorm(x, gamma, eps)
    x = np.asarray(x, dtype=np.float64)
    rs = 1.0 / np.sqrt(np.mean(x * x, axis=-1, keepdims=True) + eps)
    return bf16_round(x) * rs * gamma


def lm_head_argmax(x: np.ndarray, final_norm: np.ndarray, lm_head: np.ndarray, eps: float,
                   bf16_act: bool = False):
    """logits = RMSNorm(x) * gamma_final  E_out^T; greedy next token = first index of the maximum."""
    logits = norm_operand(x, final_norm, eps, bf16_act) @ lm_head.T
    return logits, np.argmax(logits, axis=1).astype(np.int64)


# --- paged KV cache -------------------------------------------------------------------------------

class PagedKV:
    """Paged KV cache of all layers: page p of a layer is [2 (K, V), nkv, page_size, d] bf16 values.

    Initial page contents come from ``initial(layer, pages) -> array [len, 2, nkv, P, d]`` (float64
    holding bf16 values); pages written during the iteration are kept here. Writes round to bf16,
    the cache's element type.
    """

    def __init__(self, initial: Callable[[int, np.ndarray], np.ndarray], page_size: int):
        self.initial = initial
        self.page_size = page_size
        self.pages: Dict[tuple, np.ndarray] = {}

    def _load(self, layer: int, pages: np.ndarray) -> None:
        missing = [int(p) for p in pages if (layer, int(p)) not in self.pages]
        if missing:
            uniq = np.array(sorted(set(missing)), dtype=np.int64)
            data = self.initial(layer, uniq)
            for i, p in enumerate(uniq):
                self.pages[(layer, int(p))] = np.array(data[i], dtype=np.float64)

    def write(self, layer: int, page: int, slot: int, k: np.ndarray, v: np.ndarray) -> None:
        self._load(layer, np.array([page]))
        buf = self.pages[(layer, int(page))]
        buf[0, :, slot, :] = bf16_round(k)
        buf[1, :, slot, :] = bf16_round(v)

    def read(self, layer: int, pages: np.ndarray, n_keys: int):
        """Keys/values of positions 0..n_keys-1 stored in the page list, as [n_keys, nkv, d]."""
        pages = np.asarray(pages)
        self._load(layer, pages)
        blk = np.stack([self.pages[(layer, int(p))] for p in pages])      # [np, 2, nkv, P, d]
        kv = blk.transpose(1, 0, 3, 2, 4).reshape(2, -1, blk.shape[2], blk.shape[4])
        return kv[0, :n_keys], kv[1, :n_keys]


# --- one layer, one iteration ---------------------------------------------------------------------

def _request_of_token(t: int, R: int) -> int:
    return t if t < R else R


def layer_forward(s, lw: dict, x: np.ndarray, batch, kv: PagedKV, layer: int, bf16_act: bool = True,
                  rows: Optional[Sequence[int]] = None):
    """One transformer layer over the whole batch (decode rows first, then the prefill chunk).

    With ``rows`` only those token rows of the output are computed (and returned, in that order):
    K/V of every token are still projected and written, since attention reads them, but attention,
    the output projection and the FFN run on the listed rows only. Rows are independent after
    attention, so these rows equal the same rows of the full computation.
    """
    T, R, C = batch.num_tokens, batch.num_decode, batch.prefill_len
    sel = np.arange(T) if rows is None else np.asarray(rows, dtype=np.int64)
    nq, nkv, d, P = s.n_q_heads, s.n_kv_heads, s.head_dim, s.page_size
    pos = np.asarray(batch.positions, dtype=np.int64)

    n = norm_operand(x, lw["attn_norm"], s.rms_eps, bf16_act)
    q = (n @ lw["wq"].T).reshape(T, nq, d)
    k = (n @ lw["wk"].T).reshape(T, nkv, d)
    v = (n @ lw["wv"].T).reshape(T, nkv, d)
    cos, sin = rope_cos_sin(pos, d, s.rope_theta)
    q = apply_rope(q, cos, sin)
    k = apply_rope(k, cos, sin)
    if bf16_act:
        q = bf16_round(q)

    # New K/V of every token go to slot pos % P of page page_table[req][pos // P].
    written = {}
    for t in range(T):
        r = _request_of_token(t, R)
        page = int(batch.page_indices[batch.page_indptr[r] + pos[t] // P])
        kv.write(layer, page, int(pos[t] % P), k[t], v[t])
        written[t] = (page, int(pos[t] % P))

    o = np.zeros((len(sel), nq, d), dtype=np.float64)
    for i, t in enumerate(sel):
        if t < R:
            pages = batch.page_indices[batch.page_indptr[t]:batch.page_indptr[t + 1]]
            K, V = kv.read(layer, pages, int(pos[t]) + 1)
            o[i] = decode_attention(q[t], K, V, bf16_act)
    pre = np.nonzero(sel >= R)[0]
    if C > 0 and pre.size:
        pages = batch.page_indices[batch.page_indptr[R]:batch.page_indptr[R + 1]]
        K, V = kv.read(layer, pages, C)
        if rows is None:
            o[pre] = prefill_attention(q[R:], K, V, bf16_p=bf16_act)
        else:  # chunk rows at positions sel - R, causal over the chunk's keys
            o[pre] = attention(q[sel[pre]], K, V, sel[pre] - R, np.arange(C), bf16_act)

    if bf16_act:
        o = bf16_round(o)
    x = x[sel]
    T = len(sel)
    h = x + o.reshape(T, nq * d) @ lw["wo"].T
    n2 = norm_operand(h, lw["ffn_norm"], s.rms_eps, bf16_act)
    extras = {"written": written}
    if s.n_experts == 0:
        y = swiglu_ffn(n2, lw["w_gate"], lw["w_up"], lw["w_down"], bf16_act)
    else:
        # router logits from the unrounded residual
        z = rmsnorm(h, lw["ffn_norm"], s.rms_eps) @ lw["router"].T + lw["router_bias"]
        idx, w = moe_route(z, s.top_k)
        experts = [(lw[f"e{e}_gate"], lw[f"e{e}_up"], lw[f"e{e}_down"]) for e in range(s.n_experts)]
        y = moe_ffn(n2, experts, idx, w, bf16_act)
        extras.update(router_logits=z, topk_idx=idx, topk_w=w)
    return h + y, extras


def iteration_forward(s, batch, layer_weights: Callable[[int], dict], kv: PagedKV,
                      x_in: Optional[np.ndarray] = None,
                      embed_rows: Optional[Callable[[np.ndarray], np.ndarray]] = None,
                      final_norm: Optional[np.ndarray] = None, lm_head: Optional[np.ndarray] = None,
                      keep_layer_inputs: bool = False, bf16_act: bool = True):
    """The whole iteration. Layer slices take ``x_in`` [T, H]; full models embed ``batch.tokens``
    and finish with the final norm, the LM head over the decode rows plus the chunk's last row,
    and greedy argmax."""
    if s.vocab > 0:
        x = embed_rows(np.asarray(batch.tokens))
    else:
        x = np.asarray(x_in, dtype=np.float64)
    out = {"layers": []}
    for layer in range(s.n_layers):
        if keep_layer_inputs:
            out.setdefault("layer_inputs", []).append(x.copy())
        x, extras = layer_forward(s, layer_weights(layer), x, batch, kv, layer, bf16_act)
        out["layers"].append(extras)
    out["hidden"] = x
    if s.vocab > 0:
        rows = lm_rows(batch)
        out["lm_rows"] = rows
        out["logits"], out["next_token"] = lm_head_argmax(x[rows], final_norm, lm_head, s.rms_eps, bf16_act)
    return out


def lm_rows(batch) -> np.ndarray:
    """Rows that produce a next token: every decode row, plus the prefill chunk's last row."""
    rows = list(range(batch.num_decode))
    if batch.prefill_len > 0:
        rows.append(batch.num_tokens - 1)
    return np.array(rows, dtype=np.int64)


def sub_batch(batch, requests: Sequence[int], keep_prefill: bool):
    """The batch restricted to the listed decode requests (and the prefill chunk if kept).

    Decode rows are independent of one another and of the chunk, so the oracle's rows of a
    sub-batch equal those of the full batch.
    """
    import dataclasses
    requests = list(requests)
    R = batch.num_decode
    counts, idx = [], []
    for r in requests + ([R] if keep_prefill else []):
        a, b = int(batch.page_indptr[r]), int(batch.page_indptr[r + 1])
        counts.append(b - a)
        idx.extend(batch.page_indices[a:b].tolist())
    if not keep_prefill:
        counts.append(0)
    indptr = np.zeros(len(requests) + 2, dtype=np.int32)
    indptr[1:] = np.cumsum(counts)
    C = batch.prefill_len if keep_prefill else 0
    pos = np.concatenate([batch.positions[requests], batch.positions[R:R + C]]).astype(np.int32)
    tokens = None
    if batch.tokens is not None:
        tokens = np.concatenate([batch.tokens[requests], batch.tokens[R:R + C]]).astype(np.int32)
    return dataclasses.replace(batch, num_decode=len(requests), prefill_len=C,
                               ctx_lens=batch.ctx_lens[requests], page_indptr=indptr,
                               page_indices=np.array(idx, dtype=np.int32), positions=pos, tokens=tokens)
