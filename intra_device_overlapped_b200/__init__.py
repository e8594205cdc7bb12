"""Python binding of the NanoFlow-style B200 serving-iteration library (``include/nanoflow.h``).

Argument marshalling only: every function here has the name of the C entry point it
calls through ctypes, takes plain integers (device pointers, e.g. ``tensor.data_ptr()``)
or the ctypes structures below, and returns the C status code. All computation runs
in the sm_100a kernels of ``libnanoflow.so``; there is no other implementation. If the
shared library is missing, importing the binding fails loudly.
"""
from __future__ import annotations

import ctypes
import os

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libnanoflow.so")

NF_OK = 0
NF_ERR_INVALID_ARGUMENT = 1
NF_ERR_UNSUPPORTED = 2
NF_ERR_OUT_OF_MEMORY = 3
NF_ERR_CUDA = 4
NF_ERR_DEVICE_TIMEOUT = 5
NF_ERR_DEVICE_BOUNDS = 6

NF_MAX_NANO = 4
NF_TEMPLATE_SEQUENTIAL = 0
NF_TEMPLATE_PIPELINED = 1
NF_TEMPLATE_PREFILL_ON_GEMM = 2
NF_KERNEL_GEMM, NF_KERNEL_DECODE_ATTN, NF_KERNEL_PREFILL_ATTN = 1, 2, 3

_i32, _i64, _u64, _f32, _vp = ctypes.c_int32, ctypes.c_int64, ctypes.c_uint64, ctypes.c_float, ctypes.c_void_p


class nf_model_config(ctypes.Structure):
    _fields_ = [("n_layers", _i32), ("hidden", _i32), ("n_q_heads", _i32), ("n_kv_heads", _i32),
                ("head_dim", _i32), ("ffn", _i32), ("vocab", _i32), ("n_experts", _i32), ("top_k", _i32),
                ("rms_eps", _f32), ("rope_theta", _f32), ("page_size", _i32), ("max_tokens", _i32),
                ("max_requests", _i32), ("max_position", _i32)]


class nf_layer_weights(ctypes.Structure):
    _fields_ = [("attn_norm", _vp), ("wq", _vp), ("wk", _vp), ("wv", _vp), ("wo", _vp), ("ffn_norm", _vp),
                ("w_gate", _vp), ("w_up", _vp), ("w_down", _vp), ("router", _vp), ("router_bias", _vp),
                ("expert_gate", ctypes.POINTER(_vp)), ("expert_up", ctypes.POINTER(_vp)),
                ("expert_down", ctypes.POINTER(_vp))]


class nf_global_weights(ctypes.Structure):
    _fields_ = [("embed", _vp), ("final_norm", _vp), ("lm_head", _vp)]


class nf_batch_desc(ctypes.Structure):
    _fields_ = [("num_decode", _i32), ("prefill_len", _i32), ("prefix_len", _i32),
                ("ctx_len", ctypes.POINTER(_i32)), ("page_indptr", ctypes.POINTER(_i32)), ("num_pages", _i32),
                ("page_indices", ctypes.POINTER(_i32))]


class nf_plan_opts(ctypes.Structure):
    _fields_ = [("force_nano", _i32), ("force_sm_attn", _i32), ("force_template", _i32), ("sm_total", _i32)]


class nf_plan(ctypes.Structure):
    _fields_ = [("n_nano", _i32), ("tok_begin", _i32 * NF_MAX_NANO), ("tok_end", _i32 * NF_MAX_NANO),
                ("nano_order", _i32 * NF_MAX_NANO), ("order_template", _i32), ("sm_attn", _i32),
                ("sm_gemm", _i32), ("sm_total", _i32), ("predicted_us", _f32), ("predicted_serial_us", _f32),
                ("num_decode", _i32), ("prefill_len", _i32), ("num_tokens", _i32), ("kv_pages_read", _i64),
                ("decode_items", _i64)]

    def describe(self) -> dict:
        n = self.n_nano
        return {"n_nano": n, "tokens": [(self.tok_begin[j], self.tok_end[j]) for j in range(n)],
                "order": [self.nano_order[i] for i in range(n)],
                "template": ["sequential", "pipelined", "prefill_on_gemm"][self.order_template],
                "sm_attn": self.sm_attn, "sm_gemm": self.sm_gemm, "sm_total": self.sm_total,
                "predicted_us": round(self.predicted_us, 1), "predicted_serial_us": round(self.predicted_serial_us, 1)}


class nf_iter_io(ctypes.Structure):
    _fields_ = [("token_ids", _vp), ("hidden_in", _vp), ("positions", _vp), ("ctx_len", _vp),
                ("page_indptr", _vp), ("page_indices", _vp), ("kv_pools", ctypes.POINTER(_vp)),
                ("num_pages", _i32), ("hidden_out", _vp), ("hidden_out_f32", _vp), ("logits", _vp),
                ("next_token", _vp), ("topk_idx", _vp), ("topk_w", _vp), ("router_logits", _vp),
                ("layer_hidden_out", _vp), ("token_src", _vp), ("prev_token", _vp), ("prev_rows", _i32)]


class nf_sched_config(ctypes.Structure):
    _fields_ = [("num_pages", _i32), ("max_running", _i32), ("chunk_len", _i32), ("max_position", _i32),
                ("lag", _i32)]


class nf_sched_iter(ctypes.Structure):
    _fields_ = [("iteration", _i64), ("num_decode", _i32), ("prefill_len", _i32), ("num_tokens", _i32),
                ("rows", _i32), ("num_page_entries", _i32), ("ctx_len", ctypes.POINTER(_i32)),
                ("positions", ctypes.POINTER(_i32)), ("token_ids", ctypes.POINTER(_i32)),
                ("token_src", ctypes.POINTER(_i32)), ("page_indptr", ctypes.POINTER(_i32)),
                ("page_indices", ctypes.POINTER(_i32)), ("row_request", ctypes.POINTER(_i64))]


class nf_sched_stats(ctypes.Structure):
    _fields_ = [("waiting", _i32), ("running", _i32), ("finished", _i32), ("free_pages", _i32), ("inflight", _i32),
                ("iterations", _i64), ("discarded_tokens", _i64)]

    def as_dict(self) -> dict:
        return {f: getattr(self, f) for f, _ in self._fields_}


class nf_op_time(ctypes.Structure):
    _fields_ = [("kind", _i32), ("nano", _i32), ("layer", _i32), ("stream", _i32), ("grid", _i32),
                ("us", _f32)]


NF_OP_NAMES = ("qkv", "decode_attention", "o_proj", "gate_up", "down", "moe", "lm_head", "prefill_attention")


class nf_cost_model(ctypes.Structure):
    _fields_ = [("gemm_flops_per_sm", ctypes.c_double), ("gemm_tile_us", ctypes.c_double),
                ("gemm_launch_us", ctypes.c_double), ("hbm_bw", ctypes.c_double),
                ("attn_bw_per_sm", ctypes.c_double), ("attn_launch_us", ctypes.c_double),
                ("attn_flops_per_sm", ctypes.c_double), ("interference", ctypes.c_double), ("calibrated", _i32),
                ("attn_bw_at", ctypes.c_double * 5), ("interf_attn", ctypes.c_double * 3),
                ("interf_gemm", ctypes.c_double * 3), ("iter_scale", ctypes.c_double),
                ("power_floor", ctypes.c_double)]

    def as_dict(self) -> dict:
        out = {}
        for f, _ in self._fields_:
            v = getattr(self, f)
            out[f] = list(v) if isinstance(v, ctypes.Array) else v
        return out


class nf_trace_entry(ctypes.Structure):
    _fields_ = [("kernel", _i32), ("smid", _i32), ("t_start", _u64), ("t_end", _u64)]


def _load():
    if not os.path.exists(LIB_PATH):
        raise RuntimeError(
            f"{LIB_PATH} is missing: the CUDA library has not been built "
            "(python -m intra_device_overlapped_b200.build, or __graft_entry__.build()).")
    lib = ctypes.CDLL(LIB_PATH)
    P = ctypes.POINTER
    sig = {
        "nf_status_string": ([ctypes.c_int], ctypes.c_char_p),
        "nf_version": ([], ctypes.c_char_p),
        "nf_init_model": ([P(nf_model_config), P(_vp)], ctypes.c_int),
        "nf_set_layer_weights": ([_vp, _i32, P(nf_layer_weights), _vp], ctypes.c_int),
        "nf_set_global_weights": ([_vp, P(nf_global_weights), _vp], ctypes.c_int),
        "nf_destroy_model": ([_vp], None),
        "nf_plan_iteration": ([_vp, P(nf_batch_desc), P(nf_plan_opts), P(nf_plan)], ctypes.c_int),
        "nf_plan_for_config": ([P(nf_model_config), _i32, P(nf_batch_desc), P(nf_plan_opts), P(nf_plan)],
                               ctypes.c_int),
        "nf_forward_iteration": ([_vp, P(nf_plan), P(nf_iter_io), _vp], ctypes.c_int),
        "nf_forward_iteration_persistent": ([_vp, P(nf_plan), P(nf_iter_io), _vp], ctypes.c_int),
        "nf_graph_create": ([_vp, P(nf_plan), P(nf_iter_io), _vp, P(_vp)], ctypes.c_int),
        "nf_graph_launch": ([_vp, _vp], ctypes.c_int),
        "nf_graph_destroy": ([_vp], None),
        "nf_tune_plan": ([_vp, P(nf_batch_desc), P(nf_iter_io), _i32, _vp, P(nf_plan), P(_f32)], ctypes.c_int),
        "nf_sync_status": ([_vp], ctypes.c_int),
        "nf_calibrate": ([_vp, P(nf_batch_desc), P(nf_iter_io), _vp], ctypes.c_int),
        "nf_get_cost_model": ([_vp, P(nf_cost_model)], ctypes.c_int),
        "nf_set_cost_model": ([_vp, P(nf_cost_model)], ctypes.c_int),
        "nf_set_trace": ([_vp, _i32], ctypes.c_int),
        "nf_set_timing": ([_vp, _i32], ctypes.c_int),
        "nf_get_op_times": ([_vp, P(nf_op_time), _i64], _i64),
        "nf_get_trace": ([_vp, P(nf_trace_entry), _i64], _i64),
        "nf_op_gemm_bf16": ([_vp, _vp, _vp, _i32, _i32, _i32, _i32, _vp], ctypes.c_int),
        "nf_op_decode_attention": ([_vp, _vp, _vp, P(nf_iter_io), _i32, _i32, _i32, _i32, _vp], ctypes.c_int),
        "nf_op_prefill_attention": ([_vp, _vp, _vp, P(nf_iter_io), _i32, _i32, _i32, _i32, _vp], ctypes.c_int),
        "nf_op_wait_flag_test": ([_vp, _u64, _vp], ctypes.c_int),
        "nf_op_persistent_wait_test": ([_u64, _vp], ctypes.c_int),
        "nf_decode_attention_noalloc": ([_vp, _vp, _vp, _i32, _vp, _vp, _vp, _i32, _i32, _i32, _i32, _i32, _vp, _vp],
                                        ctypes.c_int),
        "nf_offload_kv": ([_vp, P(_vp), _i32, P(_i32), _i32, _i32, _i32, _vp, _vp], ctypes.c_int),
        "nf_sched_create": ([P(nf_sched_config), P(_vp)], ctypes.c_int),
        "nf_sched_destroy": ([_vp], None),
        "nf_sched_add_request": ([_vp, P(_i32), _i32, _i32, _i32, P(_i64)], ctypes.c_int),
        "nf_sched_next": ([_vp, P(nf_sched_iter)], ctypes.c_int),
        "nf_sched_complete": ([_vp, _i64, P(_i32), _i32], ctypes.c_int),
        "nf_sched_request_tokens": ([_vp, _i64, P(_i32), _i32, P(_i32), P(_i32)], ctypes.c_int),
        "nf_sched_get_stats": ([_vp, P(nf_sched_stats)], ctypes.c_int),
    }
    for name, (args, res) in sig.items():
        f = getattr(lib, name)
        f.argtypes = args
        f.restype = res
    return lib


_lib = _load()
EXPORTED = ("nf_status_string", "nf_version", "nf_init_model", "nf_set_layer_weights", "nf_set_global_weights",
            "nf_destroy_model", "nf_plan_iteration", "nf_plan_for_config", "nf_forward_iteration", "nf_forward_iteration_persistent", "nf_tune_plan", "nf_sync_status", "nf_calibrate",
            "nf_graph_create", "nf_graph_launch", "nf_graph_destroy",
            "nf_get_cost_model", "nf_set_cost_model",
            "nf_set_trace", "nf_get_trace", "nf_set_timing", "nf_get_op_times", "nf_op_gemm_bf16", "nf_op_decode_attention",
            "nf_offload_kv",
            "nf_op_prefill_attention", "nf_op_wait_flag_test", "nf_op_persistent_wait_test", "nf_decode_attention_noalloc",
            "nf_sched_create", "nf_sched_destroy", "nf_sched_add_request", "nf_sched_next", "nf_sched_complete",
            "nf_sched_request_tokens", "nf_sched_get_stats")


NF_NOALLOC_MAX_REQUESTS = 16384


def nf_decode_attention_noalloc(q_ptr: int, out_ptr: int, kv_pool_ptr: int, num_pages: int, ctx_len_ptr: int,
                                page_indptr_ptr: int, page_indices_ptr: int, num_requests: int, n_q_heads: int,
                                n_kv_heads: int, head_dim: int, sm_count: int = 0, status_ptr: int = 0,
                                stream: int = 0) -> int:
    """Decode attention from plain device pointers; allocates nothing (static scratch, see nanoflow.h)."""
    return _lib.nf_decode_attention_noalloc(q_ptr, out_ptr, kv_pool_ptr, num_pages, ctx_len_ptr, page_indptr_ptr,
                                            page_indices_ptr, num_requests, n_q_heads, n_kv_heads, head_dim,
                                            sm_count, status_ptr or None, stream or None)


def nf_offload_kv(model: int, kv_pools, num_pool_pages: int, pages, layer_begin: int, layer_end: int,
                  host_dst_ptr: int, stream: int = 0) -> int:
    """KV pages of layers [layer_begin, layer_end) to pinned host memory (see nanoflow.h)."""
    ids = (_i32 * len(pages))(*[int(p) for p in pages])
    return _lib.nf_offload_kv(model, kv_pools, num_pool_pages, ids, len(pages), layer_begin, layer_end,
                              host_dst_ptr, stream)


class NanoflowError(RuntimeError):
    def __init__(self, status: int, what: str = ""):
        super().__init__(f"{what}: {nf_status_string(status)} ({status})")
        self.status = status


def check(status: int, what: str = "nanoflow call") -> None:
    if status != NF_OK:
        raise NanoflowError(status, what)


def nf_status_string(status: int) -> str:
    return _lib.nf_status_string(int(status)).decode()


def nf_version() -> str:
    return _lib.nf_version().decode()


def nf_init_model(cfg: nf_model_config):
    """Returns (status, model handle as int)."""
    h = _vp()
    st = _lib.nf_init_model(ctypes.byref(cfg), ctypes.byref(h))
    return st, h.value


def nf_set_layer_weights(model: int, layer: int, w: nf_layer_weights, stream: int = 0) -> int:
    return _lib.nf_set_layer_weights(model, layer, ctypes.byref(w), stream)


def nf_set_global_weights(model: int, w: nf_global_weights, stream: int = 0) -> int:
    return _lib.nf_set_global_weights(model, ctypes.byref(w), stream)


def nf_destroy_model(model: int) -> None:
    _lib.nf_destroy_model(model)


def nf_plan_iteration(model: int, batch: nf_batch_desc, opts: nf_plan_opts | None = None):
    """Returns (status, nf_plan)."""
    plan = nf_plan()
    st = _lib.nf_plan_iteration(model, ctypes.byref(batch), ctypes.byref(opts) if opts is not None else None,
                                ctypes.byref(plan))
    return st, plan


def nf_plan_for_config(cfg: nf_model_config, sm_count: int, batch: nf_batch_desc,
                       opts: nf_plan_opts | None = None):
    """Host-only planning for a configuration (default cost tables). Returns (status, nf_plan)."""
    plan = nf_plan()
    st = _lib.nf_plan_for_config(ctypes.byref(cfg), sm_count, ctypes.byref(batch),
                                 ctypes.byref(opts) if opts is not None else None, ctypes.byref(plan))
    return st, plan


def nf_forward_iteration(model: int, plan: nf_plan, io: nf_iter_io, stream: int = 0) -> int:
    return _lib.nf_forward_iteration(model, ctypes.byref(plan), ctypes.byref(io), stream)


def nf_forward_iteration_persistent(model: int, plan: nf_plan, io: nf_iter_io, stream: int = 0) -> int:
    return _lib.nf_forward_iteration_persistent(model, ctypes.byref(plan), ctypes.byref(io), stream)


def nf_graph_create(model: int, plan: nf_plan, io: nf_iter_io, stream: int):
    """Returns (status, graph handle as int)."""
    h = _vp()
    st = _lib.nf_graph_create(model, ctypes.byref(plan), ctypes.byref(io), stream, ctypes.byref(h))
    return st, h.value


def nf_graph_launch(graph: int, stream: int) -> int:
    return _lib.nf_graph_launch(graph, stream)


def nf_graph_destroy(graph: int) -> None:
    _lib.nf_graph_destroy(graph)


def nf_tune_plan(model: int, desc: nf_batch_desc, io: nf_iter_io, reps: int = 5, stream: int = 0):
    """(status, fastest measured plan, its mean iteration time in us)."""
    plan = nf_plan()
    us = ctypes.c_float(0.0)
    st = _lib.nf_tune_plan(model, ctypes.byref(desc), ctypes.byref(io), reps, stream, ctypes.byref(plan),
                           ctypes.byref(us))
    return st, plan, us.value


def nf_sync_status(model: int) -> int:
    return _lib.nf_sync_status(model)


def nf_calibrate(model: int, batch: nf_batch_desc, io: nf_iter_io, stream: int = 0) -> int:
    return _lib.nf_calibrate(model, ctypes.byref(batch), ctypes.byref(io), stream)


def nf_get_cost_model(model: int):
    c = nf_cost_model()
    st = _lib.nf_get_cost_model(model, ctypes.byref(c))
    return st, c


def nf_set_cost_model(model: int, c: nf_cost_model) -> int:
    return _lib.nf_set_cost_model(model, ctypes.byref(c))


def nf_set_trace(model: int, enable: bool) -> int:
    return _lib.nf_set_trace(model, 1 if enable else 0)


def nf_get_trace(model: int, capacity: int = 65536):
    buf = (nf_trace_entry * capacity)()
    n = _lib.nf_get_trace(model, buf, capacity)
    if n < 0:
        return int(-n), []
    return NF_OK, [(e.kernel, e.smid, e.t_start, e.t_end) for e in buf[:n]]


def nf_set_timing(model: int, enable: bool) -> int:
    return _lib.nf_set_timing(model, 1 if enable else 0)


def nf_get_op_times(model: int, capacity: int = 8192):
    """Returns (status, [(op name, nano, layer, stream, grid, us), ...]) of the last forward."""
    buf = (nf_op_time * capacity)()
    n = _lib.nf_get_op_times(model, buf, capacity)
    if n < 0:
        return int(-n), []
    return NF_OK, [(NF_OP_NAMES[e.kind], e.nano, e.layer, e.stream, e.grid, e.us) for e in buf[:n]]


def nf_op_gemm_bf16(a_ptr: int, b_ptr: int, c_ptr: int, M: int, N: int, K: int, sm_count: int = 0,
                    stream: int = 0) -> int:
    return _lib.nf_op_gemm_bf16(a_ptr, b_ptr, c_ptr, M, N, K, sm_count, stream)


def nf_op_decode_attention(model: int, q_ptr: int, out_ptr: int, io: nf_iter_io, layer: int, req_begin: int,
                           req_end: int, sm_count: int = 0, stream: int = 0) -> int:
    return _lib.nf_op_decode_attention(model, q_ptr, out_ptr, ctypes.byref(io), layer, req_begin, req_end, sm_count,
                                       stream)


def nf_op_prefill_attention(model: int, q_ptr: int, out_ptr: int, io: nf_iter_io, layer: int, num_decode: int,
                            prefill_len: int, sm_count: int = 0, stream: int = 0) -> int:
    return _lib.nf_op_prefill_attention(model, q_ptr, out_ptr, ctypes.byref(io), layer, num_decode, prefill_len,
                                        sm_count, stream)


def nf_op_wait_flag_test(flag_ptr: int, limit_ns: int, stream: int = 0) -> int:
    return _lib.nf_op_wait_flag_test(flag_ptr, limit_ns, stream)


def nf_op_persistent_wait_test(limit_ns: int, stream: int = 0) -> int:
    return _lib.nf_op_persistent_wait_test(limit_ns, stream)


def _i32_array(values) -> "ctypes.Array":
    vals = [int(v) for v in values]
    return (_i32 * max(1, len(vals)))(*vals)


def nf_sched_create(cfg: nf_sched_config):
    """Returns (status, scheduler handle)."""
    h = _vp()
    st = _lib.nf_sched_create(ctypes.byref(cfg), ctypes.byref(h))
    return st, h.value


def nf_sched_destroy(sched: int) -> None:
    _lib.nf_sched_destroy(sched)


def nf_sched_add_request(sched: int, prompt, max_new_tokens: int, eos_token: int = -1):
    """Returns (status, request id)."""
    arr = _i32_array(prompt)
    rid = _i64()
    st = _lib.nf_sched_add_request(sched, arr, len(prompt), max_new_tokens, eos_token, ctypes.byref(rid))
    return st, rid.value


def nf_sched_next(sched: int):
    """Returns (status, nf_sched_iter); the arrays it points to live until the next call."""
    it = nf_sched_iter()
    st = _lib.nf_sched_next(sched, ctypes.byref(it))
    return st, it


def nf_sched_complete(sched: int, iteration: int, next_token) -> int:
    arr = _i32_array(next_token)
    return _lib.nf_sched_complete(sched, iteration, arr, len(next_token))


def nf_sched_request_tokens(sched: int, rid: int, cap: int = 1 << 16):
    """Returns (status, generated tokens, finished)."""
    buf = (_i32 * max(1, cap))()
    n, fin = _i32(), _i32()
    st = _lib.nf_sched_request_tokens(sched, rid, buf, cap, ctypes.byref(n), ctypes.byref(fin))
    return st, list(buf[:min(n.value, cap)]), bool(fin.value)


def nf_sched_get_stats(sched: int):
    out = nf_sched_stats()
    st = _lib.nf_sched_get_stats(sched, ctypes.byref(out))
    return st, out
