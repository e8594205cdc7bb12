"""Model shapes and seeded batch recipes of the five serving workloads.

Shapes follow the Llama / Mixtral definitions the pages name (NanoFlow README,
"Introduction" and "Feasibility" benchmark: Llama2-70B, Llama3-8B, Mixtral 8x7B
at input 1024 / output 512). The batch recipe is synthetic: decode requests with
drawn context lengths plus one prefill chunk, a paged KV cache with page size 16
and a seeded random page permutation.

Token order inside an iteration: decode rows first, in request order, then the
prefill chunk. The new decode token of request r sits at position ctx_len[r];
the prefill chunk is a fresh prompt at positions 0..C-1.
"""
from __future__ import annotations

from dataclasses import dataclass, field, replace
from typing import Optional

import numpy as np

from . import (SEED_BATCH, SEED_INPUTS, B_CTX_UNIFORM, B_CTX_LOGNORMAL, B_PAGE_PERM, IN_TOKENS,
               normal_f32, uniform_int)


@dataclass(frozen=True)
class ModelShape:
    name: str
    n_layers: int
    hidden: int
    n_q_heads: int
    n_kv_heads: int
    head_dim: int
    ffn: int
    vocab: int = 0              # 0: layer slice (hidden in, hidden out); >0: embed + final norm + LM head
    n_experts: int = 0          # 0: dense SwiGLU FFN
    top_k: int = 2
    rms_eps: float = 1e-5
    rope_theta: float = 10000.0
    page_size: int = 16
    w_sigma: float = 0.02       # linear / embedding weights
    norm_sigma: float = 0.0     # RMSNorm gamma = 1 + N(0, norm_sigma)
    router_sigma: float = -1.0  # <0: 1/sqrt(hidden)
    router_bias_sigma: float = 0.5

    @property
    def qkv_dim(self) -> int:
        return (self.n_q_heads + 2 * self.n_kv_heads) * self.head_dim

    @property
    def group(self) -> int:
        return self.n_q_heads // self.n_kv_heads


@dataclass(frozen=True)
class Workload:
    shape: ModelShape
    num_decode: int
    ctx_lo: int = 0
    ctx_hi: int = 0
    ctx_lognormal_median: float = 0.0   # >0: lognormal context lengths
    ctx_lognormal_sigma: float = 1.0
    prefill_len: int = 0
    nano: tuple = (2,)
    description: str = ""


@dataclass
class Batch:
    """Host-side batch descriptor with its paged-KV page table (CSR)."""
    num_decode: int
    prefill_len: int
    ctx_lens: np.ndarray          # int32 [R]: tokens already cached per decode request
    page_size: int
    num_pages: int
    page_indptr: np.ndarray       # int32 [R + 2]: decode requests, then the prefill request
    page_indices: np.ndarray      # int32 [num_pages]
    positions: np.ndarray         # int32 [T]
    tokens: Optional[np.ndarray] = None  # int32 [T] when the model has an embedding

    @property
    def num_tokens(self) -> int:
        return self.num_decode + self.prefill_len


def pages_needed(n_keys: int, page_size: int) -> int:
    return (int(n_keys) + page_size - 1) // page_size


def make_batch(w: Workload, seed: int = SEED_BATCH) -> Batch:
    s = w.shape
    R, C, P = w.num_decode, w.prefill_len, s.page_size
    if w.ctx_lognormal_median > 0:
        z = normal_f32(seed, B_CTX_LOGNORMAL, R).astype(np.float64)
        ctx = np.rint(w.ctx_lognormal_median * np.exp(w.ctx_lognormal_sigma * z))
        ctx = np.clip(ctx, w.ctx_lo, w.ctx_hi).astype(np.int64)
    else:
        ctx = uniform_int(seed, B_CTX_UNIFORM, R, w.ctx_lo, w.ctx_hi)
    return batch_for_contexts(s, ctx, C, seed)


def batch_for_contexts(s: ModelShape, ctx, C: int, seed: int = SEED_BATCH) -> Batch:
    """Batch of decode requests with the given context lengths plus a C-token prefill chunk, with the
    seeded page permutation of ``make_batch`` (edge cases: empty contexts, page and chunk boundaries)."""
    ctx = np.asarray(ctx, dtype=np.int64)
    R, P = len(ctx), s.page_size
    # Pages: decode request r holds ctx+1 keys (its new token included); the prefill request C keys.
    counts = [pages_needed(c + 1, P) for c in ctx] + [pages_needed(C, P)]
    num_pages = int(sum(counts))
    # Seeded Fisher-Yates: for i = P-1 .. 1 swap a[i] with a[j_i], j_i = (word_i * (i + 1)) >> 32,
    # word_i being the 32-bit uniform of counter i.
    perm = np.arange(num_pages, dtype=np.int64)
    words = uniform_int(seed, B_PAGE_PERM, num_pages, 0, 0xFFFFFFFF)
    for i in range(num_pages - 1, 0, -1):
        j = (int(words[i]) * (i + 1)) >> 32
        perm[i], perm[j] = perm[j], perm[i]
    indptr = np.zeros(R + 2, dtype=np.int64)
    indptr[1:] = np.cumsum(counts)
    positions = np.concatenate([ctx, np.arange(C, dtype=np.int64)]).astype(np.int32)
    tokens = None
    if s.vocab > 0:
        tokens = uniform_int(SEED_INPUTS, IN_TOKENS, R + C, 0, s.vocab - 1).astype(np.int32)
    return Batch(num_decode=R, prefill_len=C, ctx_lens=ctx.astype(np.int32), page_size=P,
                 num_pages=num_pages, page_indptr=indptr.astype(np.int32),
                 page_indices=perm.astype(np.int32), positions=positions, tokens=tokens)


# --- the five workloads -------------------------------------------------------------------------

TINY = ModelShape("tiny", 1, 256, 4, 2, 64, 512, rope_theta=10000.0)
LLAMA3_8B = ModelShape("llama3-8b", 32, 4096, 32, 8, 128, 14336, rope_theta=500000.0)
LLAMA2_70B = ModelShape("llama2-70b", 80, 8192, 64, 8, 128, 28672, rope_theta=10000.0)
MIXTRAL_8X7B = ModelShape("mixtral-8x7b", 32, 4096, 32, 8, 128, 14336, n_experts=8, top_k=2,
                          rope_theta=1000000.0)

WORKLOADS = {
    "tiny_layer": Workload(TINY, 8, 16, 64, prefill_len=32, nano=(2,),
                           description="tiny Llama-style layer, 8 decode + 32-token prefill chunk"),
    "llama3_8b_layer": Workload(replace(LLAMA3_8B, n_layers=1), 512, 1024, 1536, prefill_len=1024,
                                nano=(1, 2, 4),
                                description="Llama-3-8B-shaped layer, 512 decode (ctx U[1024,1536]) + 1024 prefill"),
    "llama3_8b_full": Workload(replace(LLAMA3_8B, vocab=128256), 512, 1024, 1536, prefill_len=512,
                               nano=(2,),
                               description="Llama-3-8B-shaped 32 layers + LM head, 512 decode + 512 prefill"),
    "llama2_70b_slice": Workload(replace(LLAMA2_70B, n_layers=20), 512, 1024, 1536, prefill_len=1024,
                                 nano=(2, 4),
                                 description="Llama-2-70B-shaped 20-layer slice, 512 decode + 1024 prefill"),
    "mixtral_8x7b_slice": Workload(replace(MIXTRAL_8X7B, n_layers=8), 1024, 64, 4096, ctx_lognormal_median=768.0,
                                   prefill_len=1024, nano=(2,),
                                   description="Mixtral-8x7B-shaped 8-layer MoE slice, 1024 decode "
                                               "(ctx lognormal median 768 in [64,4096]) + 1024 prefill"),
}

# Small variants used by parity tests (same structure, sizes the oracle finishes in seconds).
TEST_WORKLOADS = {
    "tiny_gamma": Workload(replace(TINY, norm_sigma=0.1), 8, 16, 64, prefill_len=32),
    "tiny_lm": Workload(replace(TINY, n_layers=2, vocab=1024, norm_sigma=0.1), 8, 16, 64, prefill_len=32),
    "tiny_moe": Workload(replace(TINY, n_layers=2, n_experts=4, top_k=2, norm_sigma=0.1), 8, 16, 64,
                         prefill_len=32),
    "tiny_decode_only": Workload(TINY, 6, 1, 40, prefill_len=0),
    # 8 KV heads of dim 128 with 32 query heads: the head shape of the Llama-3-8B / Mixtral layers
    "small_gqa8": Workload(ModelShape("small_gqa8", 2, 1024, 32, 8, 128, 1024, rope_theta=500000.0,
                                      norm_sigma=0.1), 24, 1, 300, prefill_len=70),
    "tiny_prefill_only": Workload(TINY, 0, prefill_len=45),
}
