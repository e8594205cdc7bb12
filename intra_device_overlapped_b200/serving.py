"""Greedy serving of a request stream: the CPU control flow around nf_forward_iteration.

The scheduler (``nf_sched_*``, C++ in the library) forms each iteration's batch: the decode rows of
every running request plus at most one new prompt as the prefill chunk, with the KV pages each
request reserved at admission. This module only marshals: it copies the scheduler's host arrays
into pinned buffers, issues the host-to-device copies, the plan and the forward on one stream, and
reads each iteration's greedy tokens back.

With ``lag=1`` the CPU forms and launches iteration i+1 before it has read iteration i's tokens,
so the host's work for i+1 (batch formation, planning, copies, launch) overlaps the GPU's work on
i; decode rows take their input token from iteration i's ``next_token`` on the device
(``nf_iter_io.token_src``). A request whose last token came out of iteration i is decoded once more
in i+1 and that token is dropped (NanoFlow's asynchronous scheduling; README "Abstract" and the
arXiv abstract). ``lag=0`` waits for each iteration before forming the next. Both give the same
tokens.
"""
from __future__ import annotations

import ctypes
import time
from collections import deque
from typing import Callable, Optional

import numpy as np
import torch

from . import (check, nf_batch_desc, nf_forward_iteration, nf_iter_io, nf_plan_iteration, nf_plan_opts,
               nf_sched_add_request, nf_sched_complete, nf_sched_config, nf_sched_create, nf_sched_destroy,
               nf_sched_get_stats, nf_sched_next, nf_sched_request_tokens, NF_TEMPLATE_PREFILL_ON_GEMM,
               NF_TEMPLATE_SEQUENTIAL)

_vp = ctypes.c_void_p


def default_plan_opts(sm_count: int, prefill_sms: int = 8) -> Callable[[int, int], nf_plan_opts]:
    """Plan shape per batch without the full search: one nano-batch; decode attention beside the
    prefill attention (prefill on `prefill_sms` SMs) when both are present, else every op on all SMs."""
    def opts(num_decode: int, prefill_len: int) -> nf_plan_opts:
        if num_decode > 0 and prefill_len > 0 and sm_count > prefill_sms + 8:
            return nf_plan_opts(force_nano=1, force_sm_attn=sm_count - prefill_sms,
                                force_template=NF_TEMPLATE_PREFILL_ON_GEMM)
        return nf_plan_opts(force_nano=1, force_template=NF_TEMPLATE_SEQUENTIAL)
    return opts


class ServingSession:
    """A model (with embedding and LM head), its own KV pools and a scheduler."""

    def __init__(self, model: int, shape, device: str, num_pages: int, max_running: int, chunk_len: int,
                 max_position: int, lag: int = 1, plan_opts: Optional[Callable[[int, int], nf_plan_opts]] = None):
        from synth import weights as SW
        if shape.vocab <= 0:
            raise ValueError("serving needs a model with an embedding and an LM head")
        self.model = model
        self.device = torch.device(device)
        self.lag = lag
        st, self.sched = nf_sched_create(nf_sched_config(num_pages=num_pages, max_running=max_running,
                                                         chunk_len=chunk_len, max_position=max_position, lag=lag))
        check(st, "nf_sched_create")
        sm = torch.cuda.get_device_properties(self.device).multi_processor_count
        self.plan_opts = plan_opts or default_plan_opts(sm)
        self.num_pages = num_pages
        self.kv = [torch.zeros((num_pages, SW.kv_page_elems(shape)), dtype=torch.bfloat16, device=self.device)
                   for _ in range(shape.n_layers)]
        self._kv_ptrs = (_vp * shape.n_layers)(*[p.data_ptr() for p in self.kv])
        T, R = max_running + chunk_len, max_running
        i32 = dict(dtype=torch.int32)
        # two buffer sets: iteration k uses set k % 2 (its copies must land before k + 2 reuses it)
        self._dev = [dict(tok=torch.empty(T, device=self.device, **i32), src=torch.empty(T, device=self.device, **i32),
                          pos=torch.empty(T, device=self.device, **i32), ctx=torch.empty(max(R, 1), device=self.device, **i32),
                          indptr=torch.empty(R + 2, device=self.device, **i32),
                          pages=torch.empty(num_pages, device=self.device, **i32),
                          next=torch.empty(R + 1, device=self.device, **i32)) for _ in range(2)]
        self._host = [{k: torch.empty(v.shape, pin_memory=True, **i32) for k, v in d.items()} for d in self._dev]
        self._events = [torch.cuda.Event(), torch.cuda.Event()]
        self._inflight: deque = deque()  # (iteration, rows, buffer set)
        self._prev_rows = 0
        self.requests: list[int] = []
        self.iterations = 0
        self.host_launch_s = 0.0

    def add(self, prompt, max_new_tokens: int, eos_token: int = -1) -> int:
        st, rid = nf_sched_add_request(self.sched, list(prompt), max_new_tokens, eos_token)
        check(st, "nf_sched_add_request")
        self.requests.append(rid)
        return rid

    def _launch(self, it, stream) -> None:
        t0 = time.perf_counter()
        b = it.iteration % 2
        h, d = self._host[b], self._dev[b]
        T, R, C, rows, P = it.num_tokens, it.num_decode, it.prefill_len, it.rows, it.num_page_entries
        arr = lambda p, n: np.ctypeslib.as_array(p, shape=(n,))
        h["tok"].numpy()[:T] = arr(it.token_ids, T)
        h["src"].numpy()[:T] = arr(it.token_src, T)
        h["pos"].numpy()[:T] = arr(it.positions, T)
        if R:
            h["ctx"].numpy()[:R] = arr(it.ctx_len, R)
        h["indptr"].numpy()[:R + 2] = arr(it.page_indptr, R + 2)
        h["pages"].numpy()[:P] = arr(it.page_indices, P)
        with torch.cuda.stream(stream):
            for key, n in (("tok", T), ("src", T), ("pos", T), ("ctx", R), ("indptr", R + 2), ("pages", P)):
                if n:
                    d[key][:n].copy_(h[key][:n], non_blocking=True)
        desc = nf_batch_desc(num_decode=R, prefill_len=C, prefix_len=0, ctx_len=it.ctx_len,
                             page_indptr=it.page_indptr, num_pages=self.num_pages,
                             page_indices=it.page_indices)
        st, plan = nf_plan_iteration(self.model, desc, self.plan_opts(R, C))
        check(st, "nf_plan_iteration")
        io = nf_iter_io()
        io.token_ids = d["tok"].data_ptr()
        io.positions = d["pos"].data_ptr()
        io.ctx_len = d["ctx"].data_ptr()
        io.page_indptr = d["indptr"].data_ptr()
        io.page_indices = d["pages"].data_ptr()
        io.kv_pools = self._kv_ptrs
        io.num_pages = self.num_pages
        io.next_token = d["next"].data_ptr()
        io.token_src = d["src"].data_ptr()
        io.prev_token = self._dev[1 - b]["next"].data_ptr()
        io.prev_rows = self._prev_rows
        check(nf_forward_iteration(self.model, plan, io, stream.cuda_stream), "nf_forward_iteration")
        with torch.cuda.stream(stream):
            h["next"][:rows].copy_(d["next"][:rows], non_blocking=True)
        self._events[b].record(stream)
        self._inflight.append((it.iteration, rows, b))
        self._prev_rows = rows
        self.iterations += 1
        self.host_launch_s += time.perf_counter() - t0

    def _complete_oldest(self) -> None:
        k, rows, b = self._inflight.popleft()
        self._events[b].synchronize()
        check(nf_sched_complete(self.sched, k, self._host[b]["next"].numpy()[:rows].tolist()), "nf_sched_complete")

    def run(self, stream: Optional[torch.cuda.Stream] = None) -> dict:
        """Serve every added request to completion; returns wall time and counters."""
        stream = stream or torch.cuda.current_stream(self.device)
        t0 = time.perf_counter()
        while True:
            st, stats = nf_sched_get_stats(self.sched)
            check(st, "nf_sched_get_stats")
            if stats.finished == len(self.requests) and not self._inflight:
                break
            st, it = nf_sched_next(self.sched)
            check(st, "nf_sched_next")
            if it.num_tokens == 0:
                if not self._inflight:
                    raise RuntimeError("scheduler has unfinished requests but nothing to run")
                self._complete_oldest()
                continue
            self._launch(it, stream)
            while len(self._inflight) > self.lag:
                self._complete_oldest()
        wall = time.perf_counter() - t0
        st, stats = nf_sched_get_stats(self.sched)
        out = stats.as_dict()
        out.update(wall_s=wall, launched=self.iterations, host_launch_s=self.host_launch_s,
                   generated=sum(len(self.tokens(r)) for r in self.requests))
        return out

    def tokens(self, rid: int) -> list:
        st, toks, _ = nf_sched_request_tokens(self.sched, rid)
        check(st, "nf_sched_request_tokens")
        return toks

    def close(self) -> None:
        if getattr(self, "sched", None):
            nf_sched_destroy(self.sched)
            self.sched = None

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass
