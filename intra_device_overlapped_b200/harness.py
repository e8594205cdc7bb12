"""Device set-up of a serving workload for the C ABI: seeded weights and KV cache in HBM,
the batch descriptor and the per-iteration I/O block.

PyTorch is used only to own device memory and streams; weights, cached K/V and inputs
are written by the seeded device generator (``synth``), then handed to the library
through ``nf_set_layer_weights`` / ``nf_set_global_weights`` and ``nf_iter_io``.
"""
from __future__ import annotations

import ctypes
from typing import Optional

import numpy as np
import torch

import synth
from synth import weights as SW
from synth.workloads import Workload, make_batch

from . import (NF_OK, check, nf_calibrate, nf_get_cost_model, nf_batch_desc, nf_destroy_model, nf_forward_iteration, nf_global_weights,
               nf_init_model, nf_iter_io, nf_layer_weights, nf_model_config, nf_plan_iteration, nf_plan_opts,
               nf_tune_plan, nf_graph_create, nf_graph_destroy, nf_forward_iteration_persistent,
               nf_set_global_weights, nf_set_layer_weights, nf_sync_status, nf_set_trace, nf_get_trace)

_vp = ctypes.c_void_p


def _dev_i32(a: np.ndarray, device) -> torch.Tensor:
    return torch.from_numpy(np.ascontiguousarray(a, dtype=np.int32)).to(device)


def _empty_bf16(shape, device) -> torch.Tensor:
    return torch.empty(tuple(shape), dtype=torch.bfloat16, device=device)


def model_config(work: Workload, max_tokens: Optional[int] = None, max_position: int = 8192) -> nf_model_config:
    s = work.shape
    T = work.num_decode + work.prefill_len
    return nf_model_config(n_layers=s.n_layers, hidden=s.hidden, n_q_heads=s.n_q_heads, n_kv_heads=s.n_kv_heads,
                           head_dim=s.head_dim, ffn=s.ffn, vocab=s.vocab, n_experts=s.n_experts,
                           top_k=s.top_k if s.n_experts else 0, rms_eps=s.rms_eps, rope_theta=s.rope_theta,
                           page_size=s.page_size, max_tokens=max_tokens or max(T, 1),
                           max_requests=max(work.num_decode, 1), max_position=max_position)


class DeviceWorkload:
    """One workload resident on a GPU: model (packed weights), KV pools, inputs and outputs."""

    def __init__(self, work: Workload, device: str = "cuda:0", batch=None, keep_logits: bool = True,
                 moe_debug: bool = False, layer_outputs: bool = False):
        self.work = work
        self.shape = s = work.shape
        self.device = torch.device(device)
        self.batch = b = batch if batch is not None else make_batch(work)
        T, R, C = b.num_tokens, b.num_decode, b.prefill_len
        self.T, self.R, self.C = T, R, C
        max_pos = int(max(int(b.positions.max()) + 1 if T else 1, 16))
        cfg = model_config(work, max_tokens=T, max_position=max(max_pos, 4096 + 16))
        st, self.model = nf_init_model(cfg)
        check(st, "nf_init_model")
        self._load_weights()
        # paged KV pools, one per layer (physical page images, see synth.weights.kv_phys_to_logical)
        self.kv = [_empty_bf16((b.num_pages, SW.kv_page_elems(s)), self.device) for _ in range(s.n_layers)]
        for layer, pool in enumerate(self.kv):
            SW.gpu_fill_kv_pool(s, layer, pool)
        self._kv_ptrs = (_vp * s.n_layers)(*[p.data_ptr() for p in self.kv])
        # inputs
        self.positions = _dev_i32(b.positions, self.device)
        self.ctx_len = _dev_i32(b.ctx_lens if R else np.zeros(1), self.device)
        self.page_indptr = _dev_i32(b.page_indptr, self.device)
        self.page_indices = _dev_i32(b.page_indices, self.device)
        self.hidden_in = None
        self.tokens = None
        if s.vocab > 0:
            self.tokens = _dev_i32(b.tokens, self.device)
        else:
            self.hidden_in = _empty_bf16((T, s.hidden), self.device)
            synth.gpu_fill_normal_bf16(self.hidden_in.data_ptr(), T * s.hidden, synth.SEED_INPUTS, synth.IN_HIDDEN)
        # outputs
        self.hidden_out = _empty_bf16((T, s.hidden), self.device)
        self.hidden_out_f32 = torch.empty((T, s.hidden), dtype=torch.float32, device=self.device)
        self.rows = R + (1 if C > 0 else 0)
        self.logits = None
        self.next_token = None
        if s.vocab > 0:
            self.next_token = torch.empty((self.rows,), dtype=torch.int32, device=self.device)
            if keep_logits:
                self.logits = _empty_bf16((self.rows, s.vocab), self.device)
        self.topk_idx = self.topk_w = self.router_logits = None
        # fp32 residual after every layer (verification of deep stacks layer by layer)
        self.layer_hidden = (torch.empty((s.n_layers, T, s.hidden), dtype=torch.float32, device=self.device)
                             if layer_outputs else None)
        if s.n_experts > 0 and moe_debug:
            self.topk_idx = torch.empty((s.n_layers, T, s.top_k), dtype=torch.int32, device=self.device)
            self.topk_w = torch.empty((s.n_layers, T, s.top_k), dtype=torch.float32, device=self.device)
            self.router_logits = torch.empty((s.n_layers, T, s.n_experts), dtype=torch.float32, device=self.device)
        self.io = self.make_io()
        self._ctx_host = np.ascontiguousarray(b.ctx_lens, dtype=np.int32)
        self._indptr_host = np.ascontiguousarray(b.page_indptr, dtype=np.int32)
        self._pages_host = np.ascontiguousarray(b.page_indices, dtype=np.int32)
        self.desc = nf_batch_desc(num_decode=R, prefill_len=C, prefix_len=0,
                                  ctx_len=self._ctx_host.ctypes.data_as(ctypes.POINTER(ctypes.c_int32)),
                                  page_indptr=self._indptr_host.ctypes.data_as(ctypes.POINTER(ctypes.c_int32)),
                                  num_pages=b.num_pages,
                                  page_indices=self._pages_host.ctypes.data_as(ctypes.POINTER(ctypes.c_int32)))
        torch.cuda.synchronize(self.device)

    # -- set-up -----------------------------------------------------------------------------------
    def _load_weights(self):
        for layer in range(self.shape.n_layers):
            self.load_layer(layer)
        if self.shape.vocab > 0:
            self.load_globals()

    def _seeded(self, specs: dict, edit=None) -> dict:
        tens = {}
        for name, spec in specs.items():
            t = _empty_bf16(spec[1], self.device)
            SW.gpu_fill(spec, t)
            tens[name] = t
        if edit is not None:  # tests: change the seeded tensors in place before they are handed over
            edit(tens)
        return tens

    def load_layer(self, layer: int, edit=None) -> None:
        """Seeded weights of one layer through nf_set_layer_weights; `edit(tensors)` may change them first."""
        s = self.shape
        tens = self._seeded(SW.layer_specs(s, layer), edit)
        w = nf_layer_weights()
        for f in ("attn_norm", "wq", "wk", "wv", "wo", "ffn_norm"):
            setattr(w, f, tens[f].data_ptr())
        keep = []
        if s.n_experts == 0:
            w.w_gate, w.w_up, w.w_down = (tens["w_gate"].data_ptr(), tens["w_up"].data_ptr(),
                                          tens["w_down"].data_ptr())
        else:
            w.router, w.router_bias = tens["router"].data_ptr(), tens["router_bias"].data_ptr()
            E = s.n_experts
            g = (_vp * E)(*[tens[f"e{e}_gate"].data_ptr() for e in range(E)])
            u = (_vp * E)(*[tens[f"e{e}_up"].data_ptr() for e in range(E)])
            dn = (_vp * E)(*[tens[f"e{e}_down"].data_ptr() for e in range(E)])
            keep = [g, u, dn]
            w.expert_gate, w.expert_up, w.expert_down = g, u, dn
        check(nf_set_layer_weights(self.model, layer, w, 0), f"nf_set_layer_weights({layer})")
        torch.cuda.synchronize(self.device)
        del tens, keep

    def load_globals(self, edit=None) -> None:
        """Seeded embedding, final norm and LM head through nf_set_global_weights (see load_layer)."""
        tens = self._seeded(SW.global_specs(self.shape), edit)
        g = nf_global_weights(embed=tens["embed"].data_ptr(), final_norm=tens["final_norm"].data_ptr(),
                              lm_head=tens["lm_head"].data_ptr())
        check(nf_set_global_weights(self.model, g, 0), "nf_set_global_weights")
        torch.cuda.synchronize(self.device)
        del tens

    def make_io(self, hidden_in: Optional[torch.Tensor] = None, hidden_out: Optional[torch.Tensor] = None,
                next_token: Optional[torch.Tensor] = None) -> nf_iter_io:
        p = lambda t: t.data_ptr() if t is not None else None
        io = nf_iter_io()
        io.token_ids = p(self.tokens)
        io.hidden_in = p(hidden_in if hidden_in is not None else self.hidden_in)
        io.positions = p(self.positions)
        io.ctx_len = p(self.ctx_len)
        io.page_indptr = p(self.page_indptr)
        io.page_indices = p(self.page_indices)
        io.kv_pools = self._kv_ptrs
        io.num_pages = self.batch.num_pages
        io.hidden_out = p(hidden_out if hidden_out is not None else self.hidden_out)
        io.hidden_out_f32 = p(self.hidden_out_f32)
        io.logits = p(self.logits)
        io.next_token = p(next_token if next_token is not None else self.next_token)
        io.topk_idx = p(self.topk_idx)
        io.topk_w = p(self.topk_w)
        io.router_logits = p(self.router_logits)
        io.layer_hidden_out = p(self.layer_hidden)
        return io

    # -- running ----------------------------------------------------------------------------------
    def plan(self, nano: int = 0, sm_attn: int = 0, template: int = -1, sm_total: int = 0):
        opts = nf_plan_opts(force_nano=nano, force_sm_attn=sm_attn, force_template=template, sm_total=sm_total)
        st, plan = nf_plan_iteration(self.model, self.desc, opts)
        check(st, "nf_plan_iteration")
        return plan

    def tune(self, reps: int = 5, stream: Optional[torch.cuda.Stream] = None):
        """Fastest plan measured on this batch (nf_tune_plan) and its iteration time in us."""
        s = stream if stream is not None else torch.cuda.current_stream(self.device)
        st, plan, us = nf_tune_plan(self.model, self.desc, self.io, reps, s.cuda_stream)
        check(st, "nf_tune_plan")
        return plan, us

    def forward(self, plan, stream: Optional[torch.cuda.Stream] = None, io: Optional[nf_iter_io] = None,
                persistent: bool = False) -> None:
        """One iteration of `plan`: one launch per operation on two streams (nf_forward_iteration), or
        with persistent=True one persistent kernel per layer (nf_forward_iteration_persistent)."""
        s = stream.cuda_stream if stream is not None else torch.cuda.current_stream(self.device).cuda_stream
        fn = nf_forward_iteration_persistent if persistent else nf_forward_iteration
        check(fn(self.model, plan, io if io is not None else self.io, s), fn.__name__)

    def graph(self, plan, stream: torch.cuda.Stream) -> int:
        """The iteration of `plan` on this workload's buffers as a CUDA graph (nf_graph_create); the
        handle is destroyed with the workload."""
        st, g = nf_graph_create(self.model, plan, self.io, stream.cuda_stream)
        check(st, "nf_graph_create")
        self._graphs = getattr(self, "_graphs", []) + [g]
        return g

    def calibrate(self, stream: Optional[torch.cuda.Stream] = None) -> dict:
        """Time the model's kernels on this batch and install the fitted cost model for planning."""
        s = stream.cuda_stream if stream is not None else torch.cuda.current_stream(self.device).cuda_stream
        check(nf_calibrate(self.model, self.desc, self.io, s), "nf_calibrate")
        st, c = nf_get_cost_model(self.model)
        check(st, "nf_get_cost_model")
        return c.as_dict()

    def sync(self) -> int:
        return nf_sync_status(self.model)

    def trace(self, enable: bool = True):
        check(nf_set_trace(self.model, enable), "nf_set_trace")

    def get_trace(self):
        st, entries = nf_get_trace(self.model)
        check(st, "nf_get_trace")
        return entries

    def close(self):
        for g in getattr(self, "_graphs", []):
            nf_graph_destroy(g)
        self._graphs = []
        if getattr(self, "model", None):
            nf_destroy_model(self.model)
            self.model = None

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass


def kv_logical(dw: "DeviceWorkload", layer: int) -> np.ndarray:
    """Host copy of a layer's pool as bf16 bit patterns in the logical view [pages, 2, nkv, P, d]."""
    return SW.kv_phys_to_logical(bf16_bits(dw.kv[layer]), dw.shape)


def bf16_bits(t: torch.Tensor) -> np.ndarray:
    """uint16 bit patterns of a bf16 tensor (host copy)."""
    return t.detach().contiguous().view(torch.int16).cpu().numpy().view(np.uint16)
