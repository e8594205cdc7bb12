#!/usr/bin/env python
"""Throughput of one NanoFlow-style serving iteration on B200 (decode tokens/s).

A step is one call of nf_forward_iteration over the whole batch of the workload
(default: the Llama-3-8B-shaped layer with 512 decode requests, context U[1024,1536],
plus a 1024-token prefill chunk), with the plan chosen by nf_plan_iteration.

  python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

N > 1 (launched by torchrun): independent replicas, one per GPU, no collective on the
data path ("replicas only"); timing is the max over ranks. Rank 0 prints one JSON line.
--impl reference times the float64 CPU oracle on the host cores instead.
"""
from __future__ import annotations

import argparse
import json
import os
import statistics
import subprocess
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

METRIC = "decode tokens/s per B200 (Llama-3-8B shape); % of compute-bound optimum"
DEFAULT_WORKLOAD = "llama3_8b_layer"


def parse_args(argv=None):
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=400)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", default=DEFAULT_WORKLOAD)
    ap.add_argument("--nano", type=int, default=0, help="force the nano-batch count (0: planner)")
    ap.add_argument("--sm-attn", type=int, default=0, help="force the attention SM share (0: planner)")
    ap.add_argument("--template", type=int, default=-1)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-extras", action="store_true", help="skip e2e / sequential / op-timing passes")
    ap.add_argument("--cpu-sample", type=int, default=0, help="decode requests in the CPU oracle sample")
    ap.add_argument("--min-warmup-s", type=float, default=1.0,
                    help="the warm-up runs at least W steps and at least this many seconds")
    return ap.parse_args(argv)


# --------------------------------------------------------------------------- distributed plumbing

class Dist:
    def __init__(self):
        self.world = int(os.environ.get("WORLD_SIZE", "1"))
        self.rank = int(os.environ.get("RANK", "0"))
        self.local = int(os.environ.get("LOCAL_RANK", "0"))
        self.pg = None
        if self.world > 1:
            import datetime
            import torch
            import torch.distributed as dist
            backend = "nccl" if torch.cuda.is_available() else "gloo"
            if backend == "nccl":
                torch.cuda.set_device(self.local)
            dist.init_process_group(backend, timeout=datetime.timedelta(seconds=300))
            self.pg = dist

    def barrier(self):
        if self.pg is not None:
            self.pg.barrier()

    def max(self, x: float) -> float:
        if self.pg is None:
            return x
        import torch
        dev = f"cuda:{self.local}" if torch.cuda.is_available() else "cpu"
        t = torch.tensor([x], dtype=torch.float64, device=dev)
        self.pg.all_reduce(t, op=self.pg.ReduceOp.MAX)
        return float(t.item())

    def close(self):
        if self.pg is not None:
            self.pg.destroy_process_group()


# --------------------------------------------------------------------------- clocks

class ClockSampler:
    """nvidia-smi samples (50 ms) of SM clock and throttle reasons while running."""

    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.gpu = gpu_index
        self.proc = None
        self.lines = []
        self._t = None

    def start(self):
        try:
            self.proc = subprocess.Popen(["nvidia-smi", f"--id={self.gpu}", f"--query-gpu={self.FIELDS}",
                                          "--format=csv,noheader,nounits", "-lms", "50"],
                                         stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            self._t = threading.Thread(target=self._read, daemon=True)
            self._t.start()
        except Exception:
            self.proc = None

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append(line.strip())

    def stop(self) -> dict:
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except Exception:
            self.proc.kill()
        if self._t:
            self._t.join(timeout=2)
        sm, smax, reasons = [], [], set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for ln in self.lines:
            f = [x.strip() for x in ln.split(",")]
            if len(f) < 9:
                continue
            try:
                sm.append(float(f[1]))
                smax.append(float(f[2]))
            except ValueError:
                continue
            for name, v in zip(names, f[5:9]):
                if v.lower() == "active":
                    reasons.add(name)
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": max(smax) if smax else None,
                "reasons": sorted(reasons), "samples": len(sm)}


# --------------------------------------------------------------------------- work accounting

# DRAM bytes (read + write) per algorithmic byte of a kernel, from one ncu capture of that
# kernel as it stands; the bench scales it to its own launches (traffic grows with the pages
# read). Entries must be retaken whenever the kernel changes.
TRAFFIC_PER_ALGO_BYTE = {
    # all 512 requests of the Llama-3-8B layer on 148 SMs: 2,704,816,640 B read + 17,256,192 B written
    # for 2,684,391,424 algorithmic bytes (the ncu capture summarised under profiles/)
    "decode_attention": (1.0140, "ncu dram__bytes_read.sum + dram__bytes_write.sum, one full launch"),
}

def iteration_flops(work, batch):
    """GEMM FLOPs + attention matmul FLOPs of one iteration (compute-bound optimum numerator)."""
    s = work.shape
    T, R, C = batch.num_tokens, batch.num_decode, batch.prefill_len
    H, d, nq, nkv, F = s.hidden, s.head_dim, s.n_q_heads, s.n_kv_heads, s.ffn
    per_tok = 2 * H * ((nq + 2 * nkv) * d) + 2 * (nq * d) * H
    if s.n_experts:
        per_tok += s.top_k * (2 * H * 2 * F + 2 * F * H) + 2 * H * s.n_experts
    else:
        per_tok += 2 * H * 2 * F + 2 * F * H
    gemm = T * per_tok * s.n_layers
    keys = float(sum(int(c) + 1 for c in batch.ctx_lens))
    attn = s.n_layers * 4.0 * nq * d * (keys + C * (C + 1) / 2.0)
    lm = 2.0 * (R + (1 if C else 0)) * H * s.vocab if s.vocab else 0.0
    return gemm + attn + lm, gemm, attn, lm


def op_algorithmic(work, batch, plan, op, nano):
    """(bound, units per launch) of one op launch: FLOPs for GEMMs, bytes for decode attention."""
    s = work.shape
    t0, t1 = plan.tok_begin[nano], plan.tok_end[nano]
    M = t1 - t0
    H, d, nq, nkv, F = s.hidden, s.head_dim, s.n_q_heads, s.n_kv_heads, s.ffn
    if op == "qkv":
        return "tensor", 2.0 * M * (nq + 2 * nkv) * d * H
    if op == "o_proj":
        return "tensor", 2.0 * M * H * nq * d
    if op == "gate_up":
        return "tensor", 2.0 * M * 2 * F * H
    if op == "down":
        return "tensor", 2.0 * M * H * F
    if op == "moe":
        # router GEMM plus, for each of the top-k experts of every row, its gate/up and down GEMMs
        k = max(int(s.top_k), 1)
        return "tensor", 2.0 * M * H * s.n_experts + 2.0 * M * k * (2 * F * H + H * F)
    if op == "lm_head":
        return "tensor", 2.0 * (batch.num_decode + (1 if batch.prefill_len else 0)) * H * s.vocab
    if op == "decode_attention":
        # K and V of every KV head for the ctx + 1 keys of each decode request: (ctx + 1) * 4096 B at
        # the Llama-3-8B shape (8 KV heads x 128 x bf16 x 2)
        R = batch.num_decode
        r0, r1 = min(t0, R), min(t1, R)
        keys = sum(int(batch.ctx_lens[r]) + 1 for r in range(r0, r1))
        return "hbm", float(keys * 2 * nkv * d * 2)
    if op == "prefill_attention":
        C = batch.prefill_len
        return "tensor", 4.0 * nq * d * C * (C + 1) / 2.0
    return None, 0.0


def count_launches(work, plan, ctx_lens):
    """Kernels this library launches per iteration (checked against the ncu launch list)."""
    s = work.shape
    plan_ctx = list(ctx_lens)
    R = plan.num_decode
    tc = s.head_dim == 128 and s.n_kv_heads == 8 and s.n_q_heads in (32, 64)
    per_step = 1                          # residual set-up (or embedding)
    if R > 0:
        per_step += 1 if tc else 2        # decode schedule (+ split-item table on the warp-level path)
    for j in range(plan.n_nano):
        t0, t1 = plan.tok_begin[j], plan.tok_end[j]
        dec = 1 if min(t1, R) > min(t0, R) else 0
        # tensor-core decode: the attention kernel, and its split-KV merge pass when a request of the
        # nano-batch spans more than one chunk of 64 pages (1024 keys)
        split = any(-(-(int(c) + 1) // 16) > 64 for c in plan_ctx[min(t0, R):min(t1, R)])
        att = dec * ((2 if split else 1) if tc else 1) + (1 if t1 > R and plan.prefill_len else 0)
        ffn = 6 if s.n_experts else 2      # MoE: route+sort, gather, 2 grouped GEMMs, combine
        per_step += s.n_layers * (1 + att + 1 + ffn)
    if s.vocab:
        per_step += 3
    return per_step


# --------------------------------------------------------------------------- CPU oracle timing

def cpu_oracle_sample(work, batch, n_requests: int, repeats: int = 1):
    """Time the float64 oracle on the first n_requests decode rows (inputs pre-generated)."""
    import numpy as np
    from oracle.forward import iteration_forward, sub_batch
    from oracle.run import layer_weights_f64, make_kv
    from synth import bf16_to_f64
    from synth import weights as SW
    s = work.shape
    sb = sub_batch(batch, list(range(n_requests)), keep_prefill=False)
    wcache = {l: layer_weights_f64(s, l) for l in range(s.n_layers)}
    kw = {}
    if s.vocab:
        g = SW.global_specs(s)
        emb = bf16_to_f64(SW.host_rows(g["embed"], sb.tokens))
        kw = dict(embed_rows=lambda toks: emb, final_norm=bf16_to_f64(SW.host_tensor(g["final_norm"])),
                  lm_head=bf16_to_f64(SW.host_tensor(g["lm_head"])))
        x_in = None
    else:
        x_in = bf16_to_f64(SW.host_input_rows(s, np.arange(n_requests)))
    times = []
    for _ in range(repeats):
        kv = make_kv(s)
        for l in range(s.n_layers):   # pre-load the sample's pages (input regeneration is not timed)
            kv._load(l, sb.page_indices)
        t = time.perf_counter()
        iteration_forward(s, sb, lambda l: wcache[l], kv, x_in=x_in, **kw)
        times.append(time.perf_counter() - t)
    threads = os.cpu_count()
    try:
        from threadpoolctl import threadpool_info
        info = [p.get("num_threads") for p in threadpool_info() if p.get("internal_api") == "openblas"]
        if info:
            threads = max(info)
    except Exception:
        pass
    return times, threads


def workload_config(args, work, batch, world):
    """The workload keys of `config`, the same in both arms."""
    if work.ctx_lognormal_median > 0:
        ctx = f"lognormal median {work.ctx_lognormal_median:g}, sigma {work.ctx_lognormal_sigma:g}"
    else:
        ctx = f"uniform [{work.ctx_lo},{work.ctx_hi}]"
    return {"workload": args.workload, "decode_requests": batch.num_decode, "prefill_len": batch.prefill_len,
            "tokens": batch.num_tokens, "ctx": ctx, "parallelism": f"replicas x{world}"}


def run_reference(args, work, dist):
    if dist.rank != 0:
        return
    from synth.workloads import make_batch
    batch = make_batch(work)
    # each step is a bounded sample of decode requests, sized from a timed probe of 4 requests
    # so that the warm-up and timed steps together take about 90 s of host time
    probe, _ = cpu_oracle_sample(work, batch, min(4, batch.num_decode), repeats=1)
    per_req = probe[0] / min(4, batch.num_decode)
    n = args.cpu_sample or int(max(1, min(128, batch.num_decode, 90.0 / ((args.steps + args.warmup) * per_req))))
    cpu_oracle_sample(work, batch, n, repeats=max(1, args.warmup))  # warm-up
    times, threads = cpu_oracle_sample(work, batch, n, repeats=args.steps)
    tot = sum(times)
    value = n * len(times) / tot
    line = {"impl": "reference", "metric": METRIC, "value": value, "unit": "decode tokens/s",
            "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup, "ms_per_step": 1000 * tot / len(times),
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": workload_config(args, work, batch, dist.world),
            "cpu_baseline": {"value": value, "unit": "decode tokens/s", "cores": threads, "kind": "oracle",
                             "sample": f"{n} of {batch.num_decode} decode requests of {args.workload}, no prefill "
                                       "chunk, float64 numpy oracle, inputs pre-generated"},
            "e2e": {"value": value, "unit": "decode tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


# --------------------------------------------------------------------------- GPU arm

def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return d.get("hbm_gbs", 6650.0), d.get("bf16_tflops", 1590.0), d.get("bf16_tflops_sustained", 1400.0), "measured"
    return 6650.0, 1590.0, 1400.0, "fallback"


def run_ours(args, work, dist):
    import numpy as np
    import torch
    import intra_device_overlapped_b200 as nf
    from intra_device_overlapped_b200.harness import DeviceWorkload

    dev = f"cuda:{dist.local}"
    torch.cuda.set_device(dev)
    dw = DeviceWorkload(work, dev, keep_logits=False)
    b = dw.batch
    cost = dw.calibrate()
    forced = args.nano > 0 or args.sm_attn > 0 or args.template >= 0
    if forced:
        plan = dw.plan(nano=args.nano, sm_attn=args.sm_attn, template=args.template)
    else:  # the planner's candidates measured on this batch, fastest kept (nf_tune_plan)
        plan, _ = dw.tune(reps=5)
    stream = torch.cuda.current_stream(dev)

    # clocks are sampled (every 50 ms) from the start of the warm-up to the end of the timed region;
    # the warm-up runs at least W steps and at least one second, so that the record holds samples
    # under load even when the K timed steps take only milliseconds
    clocks = ClockSampler(dist.local)
    clocks.start()
    t_warm = time.perf_counter()
    nwarm = 0
    while nwarm < max(args.warmup, 3) or time.perf_counter() - t_warm < args.min_warmup_s:
        for _ in range(8):
            dw.forward(plan, stream)
        nwarm += 8
        torch.cuda.synchronize(dev)
    nf.check(dw.sync(), "warm-up")

    # ---- timed region: K iterations back to back (no per-op instrumentation inside it)
    dist.barrier()
    torch.cuda.synchronize(dev)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    torch.cuda.nvtx.range_push("timed")   # lets a profiler capture exactly the timed launches
    e0.record(stream)
    for _ in range(args.steps):
        dw.forward(plan, stream)
    e1.record(stream)
    torch.cuda.nvtx.range_pop()
    torch.cuda.synchronize(dev)
    dist.barrier()
    clk = clocks.stop()
    nf.check(dw.sync(), "timed steps")
    ms_total = dist.max(e0.elapsed_time(e1))

    # ---- the same K iterations again with per-op CUDA events on each op's stream (op times for the
    # roofline of the dominant kernel and the op shares)
    nf.check(nf.nf_set_timing(dw.model, True), "timing")
    for _ in range(args.steps):
        dw.forward(plan, stream)
    torch.cuda.synchronize(dev)
    nf.check(dw.sync(), "op-timing steps")
    st, op_times = nf.nf_get_op_times(dw.model, 1 << 20)
    nf.check(st, "op times")
    nf.check(nf.nf_set_timing(dw.model, False), "timing")
    ms_step = ms_total / args.steps
    R = b.num_decode
    value = dist.world * R * args.steps / (ms_total / 1000.0)

    flops, gemm_f, attn_f, lm_f = iteration_flops(work, b)
    hbm_gbs, bf16_tf, bf16_tf_sus, peak_src = load_peaks()
    t_opt_ms = flops / (bf16_tf * 1e12) * 1e3

    # per-op averages over the timed region
    agg = {}
    for (name, nano, layer, stream_id, grid, us) in op_times:
        bound, units = op_algorithmic(work, b, plan, name, nano) if nano >= 0 else op_algorithmic(work, b, plan, name, 0)
        a = agg.setdefault(name, {"launches": 0, "us": 0.0, "units": 0.0, "bound": bound})
        a["launches"] += 1
        a["us"] += us
        a["units"] += units
    dominant = max(agg, key=lambda k: agg[k]["us"]) if agg else None
    roofline = None
    if dominant:
        a = agg[dominant]
        avg_us = a["us"] / a["launches"]
        per_launch = a["units"] / a["launches"]
        if a["bound"] == "tensor":
            peak = bf16_tf
            achieved = per_launch / (avg_us * 1e-6) / 1e12
            unit = "TFLOP/s"
        else:
            peak = hbm_gbs
            achieved = per_launch / (avg_us * 1e-6) / 1e9
            unit = "GB/s"
        traffic, traffic_src = None, None
        if dominant in TRAFFIC_PER_ALGO_BYTE and a["bound"] == "hbm":
            ratio, traffic_src = TRAFFIC_PER_ALGO_BYTE[dominant]
            traffic = int(round(per_launch * ratio))
        roofline = {"kernel": dominant, "bound": a["bound"], "achieved": round(achieved, 1), "peak": peak,
                    "unit": unit, "frac": round(achieved / peak, 4), "traffic": traffic,
                    "traffic_unit": "bytes per launch", "traffic_source": traffic_src,
                    "avg_launch_us": round(avg_us, 2), "launches_per_step": a["launches"] / args.steps,
                    "peak_source": f"{peak_src} (burst)"}
    op_summary = {k: {"avg_us": round(v["us"] / v["launches"], 1), "launches": v["launches"],
                      "share": round(v["us"] / max(sum(x["us"] for x in agg.values()), 1e-9), 3)}
                  for k, v in agg.items()}

    extras = {}
    if not args.no_extras:
        # ---- the same plan replayed as a CUDA graph (nf_graph_create / nf_graph_launch) on a side stream,
        # timed like the headline
        side = torch.cuda.Stream(dev)
        torch.cuda.synchronize(dev)
        g = dw.graph(plan, side)
        t_warm = time.perf_counter()
        nw = 0
        while nw < max(args.warmup, 3) or time.perf_counter() - t_warm < args.min_warmup_s:
            for _ in range(8):
                nf.check(nf.nf_graph_launch(g, side.cuda_stream), "graph")
            nw += 8
            side.synchronize()
        g0, g1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        g0.record(side)
        for _ in range(args.steps):
            nf.check(nf.nf_graph_launch(g, side.cuda_stream), "graph")
        g1.record(side)
        torch.cuda.synchronize(dev)
        nf.check(dw.sync(), "graph steps")
        g_ms = g0.elapsed_time(g1) / args.steps
        extras["graph"] = {"ms_per_step": round(g_ms, 4),
                           "value": round(dist.world * R * 1000.0 / g_ms, 1), "unit": "decode tokens/s",
                           "how": "the tuned plan captured once as a CUDA graph (nf_graph_create) and replayed with "
                                  "nf_graph_launch, same warm-up and K steps as the headline"}

        # ---- the tuned plan with each layer as one persistent kernel (nf_forward_iteration_persistent):
        # operations scheduled on the device by completion counters instead of launches and events
        t_warm = time.perf_counter()
        nw = 0
        while nw < max(args.warmup, 3) or time.perf_counter() - t_warm < args.min_warmup_s:
            for _ in range(8):
                dw.forward(plan, stream, persistent=True)
            nw += 8
            torch.cuda.synchronize(dev)
        p0, p1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        p0.record(stream)
        for _ in range(args.steps):
            dw.forward(plan, stream, persistent=True)
        p1.record(stream)
        torch.cuda.synchronize(dev)
        nf.check(dw.sync(), "persistent steps")
        p_ms = p0.elapsed_time(p1) / args.steps
        extras["persistent"] = {"ms_per_step": round(p_ms, 4),
                                "value": round(dist.world * R * 1000.0 / p_ms, 1), "unit": "decode tokens/s",
                                "how": "the tuned plan with each layer as one persistent kernel "
                                       "(nf_forward_iteration_persistent: one-CTA GEMM tiles, device-side "
                                       "completion counters), same warm-up and K steps as the headline"}

        # ---- the same work without overlap: sequential plan, one nano-batch, every SM
        # timed exactly like the headline: the same warm-up (at least W steps and --min-warmup-s seconds of
        # this plan, so that the power-capped clock has settled on it), then K steps without per-op events
        seq_plan = dw.plan(nano=1, template=0)
        t_warm = time.perf_counter()
        nw = 0
        while nw < max(args.warmup, 3) or time.perf_counter() - t_warm < args.min_warmup_s:
            for _ in range(8):
                dw.forward(seq_plan, stream)
            nw += 8
            torch.cuda.synchronize(dev)
        s0, s1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        s0.record(stream)
        for _ in range(args.steps):
            dw.forward(seq_plan, stream)
        s1.record(stream)
        torch.cuda.synchronize(dev)
        seq_ms = s0.elapsed_time(s1) / args.steps
        # then the same steps again with per-op events (each op's time on all SMs)
        nf.check(nf.nf_set_timing(dw.model, True), "timing")
        nseq = max(3, args.steps // 2)
        for _ in range(nseq):
            dw.forward(seq_plan, stream)
        torch.cuda.synchronize(dev)
        st, seq_ops = nf.nf_get_op_times(dw.model, 1 << 20)
        nf.nf_set_timing(dw.model, False)
        iso = {}
        for (name, nano, layer, stream_id, grid, us) in seq_ops:
            iso[name] = iso.get(name, 0.0) + us / nseq
        att = ("decode_attention", "prefill_attention")
        extras["sequential"] = {"ms_per_step": round(seq_ms, 4),
                                "isolated_op_ms": {k: round(v / 1000, 4) for k, v in iso.items()},
                                "sum_isolated_gemm_ms": round(sum(v for k, v in iso.items() if k not in att) / 1000, 4),
                                "sum_isolated_attention_ms": round(sum(iso.get(k, 0.0) for k in att) / 1000, 4)}

        # ---- each op alone at the SM share the plan gave it: for every op, the grid it ran on in the
        # tuned plan (the one holding most of its time), then that op of the sequential iteration run
        # alone on that many SMs
        if plan.order_template != nf.NF_TEMPLATE_SEQUENTIAL:
            grid_time = {}
            for (name, nano, layer, stream_id, grid, us) in op_times:
                grid_time.setdefault(name, {}).setdefault(grid, 0.0)
                grid_time[name][grid] += us
            op_grid = {k: max(v, key=v.get) for k, v in grid_time.items()}
            share = {}
            for sms in sorted(set(op_grid.values())):
                sp = dw.plan(nano=1, template=0, sm_total=sms)
                for _ in range(2):
                    dw.forward(sp, stream)
                nf.check(nf.nf_set_timing(dw.model, True), "timing")
                nrep = max(3, args.steps // 4)
                for _ in range(nrep):
                    dw.forward(sp, stream)
                torch.cuda.synchronize(dev)
                st, sh_ops = nf.nf_get_op_times(dw.model, 1 << 20)
                nf.nf_set_timing(dw.model, False)
                for (name, nano, layer, stream_id, grid, us) in sh_ops:
                    if op_grid.get(name) == sms:
                        share[name] = share.get(name, 0.0) + us / nrep
            extras["sequential"]["isolated_op_ms_at_plan_share"] = {
                "sm_attn": plan.sm_attn, "sm_gemm": plan.sm_gemm, "grid_per_op": op_grid,
                "ops": {k: round(v / 1000, 4) for k, v in share.items()},
                "sum_ms": round(sum(share.values()) / 1000, 4)}

        # ---- KV offload beside the iteration: every step also copies the KV pages of two decode requests
        # (every layer) to pinned host memory on a low-priority stream, as a serving loop does for the
        # requests that finished; the timed region ends when both the iterations and the copies are done
        s = work.shape
        off_reqs = [0, 1] if R >= 2 else list(range(R))
        if off_reqs:
            pages = [int(pg) for r in off_reqs for pg in b.page_indices[b.page_indptr[r]:b.page_indptr[r + 1]]]
            page_elems = dw.kv[0].shape[1]
            host_kv = torch.empty((s.n_layers, len(pages), page_elems), dtype=torch.bfloat16).pin_memory()
            side = torch.cuda.Stream(dev, priority=0)
            side.wait_stream(stream)

            def offload():
                nf.check(nf.nf_offload_kv(dw.model, dw._kv_ptrs, b.num_pages, pages, 0, s.n_layers,
                                          host_kv.data_ptr(), side.cuda_stream), "offload")
            nw = 0
            t_warm = time.perf_counter()
            while nw < max(args.warmup, 3) or time.perf_counter() - t_warm < args.min_warmup_s:
                for _ in range(8):
                    offload()
                    dw.forward(plan, stream)
                nw += 8
                torch.cuda.synchronize(dev)
            o0, o1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            o0.record(stream)
            side.wait_stream(stream)
            for _ in range(args.steps):
                offload()
                dw.forward(plan, stream)
            stream.wait_stream(side)
            o1.record(stream)
            torch.cuda.synchronize(dev)
            nf.check(dw.sync(), "offload steps")
            off_ms = dist.max(o0.elapsed_time(o1)) / args.steps
            extras["kv_offload"] = {
                "requests_per_step": len(off_reqs), "pages_per_step": len(pages) * s.n_layers,
                "bytes_per_step": int(host_kv.numel() * 2), "ms_per_step": round(off_ms, 4),
                "slowdown": round(off_ms / ms_step - 1.0, 4),
                "how": "nf_offload_kv on a low-priority stream beside every iteration (gather kernel + D2H copy "
                       "per layer into pinned host memory)"}

        # ---- end to end through the C ABI with host buffers: every step copies its inputs from pinned
        # host memory to the device and reads its result back. As a serving loop does, the copies
        # of neighbouring steps overlap the compute of this one: two device input/output sets, the
        # H2D copies on one copy stream and the D2H reads on another, ordered by events. The timed
        # region runs from the first input copy to the end of the last result read.
        s = work.shape
        meta = (dw.positions, dw.ctx_len, dw.page_indptr, dw.page_indices)
        host_in = dw.hidden_in.cpu().pin_memory() if dw.hidden_in is not None else None
        host_tok = dw.tokens.cpu().pin_memory() if dw.tokens is not None else None
        host_meta = [t.cpu().pin_memory() for t in meta]
        host_out = torch.empty(tuple(dw.hidden_out.shape), dtype=dw.hidden_out.dtype).pin_memory()
        sets = []
        for _ in range(2):
            dmeta = [torch.empty_like(t) for t in meta]
            din = torch.empty_like(dw.hidden_in) if dw.hidden_in is not None else None
            dtok = torch.empty_like(dw.tokens) if dw.tokens is not None else None
            dout = torch.empty_like(dw.hidden_out)
            io_k = dw.make_io(hidden_in=din, hidden_out=dout)
            io_k.positions, io_k.ctx_len, io_k.page_indptr, io_k.page_indices = [t.data_ptr() for t in dmeta]
            if dtok is not None:
                io_k.token_ids = dtok.data_ptr()
            sets.append(dict(meta=dmeta, inp=din, tok=dtok, out=dout, io=io_k,
                             ev_in=torch.cuda.Event(), ev_done=torch.cuda.Event(), ev_out=torch.cuda.Event()))
        h2d = sum(t.numel() * t.element_size() for t in host_meta)
        h2d += host_in.numel() * host_in.element_size() if host_in is not None else 0
        h2d += host_tok.numel() * host_tok.element_size() if host_tok is not None else 0
        d2h = host_out.numel() * host_out.element_size()
        copy_in, copy_out = torch.cuda.Stream(dev), torch.cuda.Stream(dev)

        def e2e_step(k):
            b_ = sets[k % 2]
            with torch.cuda.stream(copy_in):
                copy_in.wait_event(b_["ev_done"])         # the step two back has finished reading this set
                for d_, h_ in zip(b_["meta"], host_meta):
                    d_.copy_(h_, non_blocking=True)
                if b_["inp"] is not None:
                    b_["inp"].copy_(host_in, non_blocking=True)
                if b_["tok"] is not None:
                    b_["tok"].copy_(host_tok, non_blocking=True)
                b_["ev_in"].record(copy_in)
            stream.wait_event(b_["ev_in"])
            stream.wait_event(b_["ev_out"])                # its previous result has been read back
            dw.forward(plan, stream, io=b_["io"])
            b_["ev_done"].record(stream)
            with torch.cuda.stream(copy_out):
                copy_out.wait_event(b_["ev_done"])
                host_out.copy_(b_["out"], non_blocking=True)
                b_["ev_out"].record(copy_out)

        # warmed up like the headline (at least W steps and --min-warmup-s seconds of these steps), so
        # that the power-capped clock has settled on this loop before it is timed
        k_run = 0
        t_warm = time.perf_counter()
        while k_run < max(args.warmup, 3) or time.perf_counter() - t_warm < args.min_warmup_s:
            for _ in range(8):
                e2e_step(k_run)
                k_run += 1
            torch.cuda.synchronize(dev)
        dist.barrier()
        t0 = torch.cuda.Event(enable_timing=True)
        t1 = torch.cuda.Event(enable_timing=True)
        t0.record(copy_in)
        for k in range(k_run, k_run + args.steps):
            e2e_step(k)
        t1.record(copy_out)
        torch.cuda.synchronize(dev)
        nf.check(dw.sync(), "e2e steps")
        e2e_ms = dist.max(t0.elapsed_time(t1))
        extras["e2e"] = {"value": dist.world * R * args.steps / (e2e_ms / 1000.0), "unit": "decode tokens/s",
                         "h2d_bytes_per_step": int(h2d), "d2h_bytes_per_step": int(d2h),
                         "copies": "pinned host <-> device every step, overlapping neighbouring steps' compute "
                                   "(two device buffer sets, separate H2D and D2H streams)"}

    cpu = None
    if dist.rank == 0 and dist.world == 1 and not args.no_cpu_baseline:
        n = args.cpu_sample or R
        times, threads = cpu_oracle_sample(work, b, n, repeats=1)
        cpu = {"value": n / times[0], "unit": "decode tokens/s", "cores": threads, "kind": "oracle",
               "sample": f"{n} of {R} decode requests of {args.workload}, no prefill chunk, float64 numpy oracle, "
                         f"inputs pre-generated, {times[0]:.1f} s"}

    line = {"metric": METRIC, "value": value, "unit": "decode tokens/s", "n_gpus": dist.world,
            "steps": args.steps, "warmup": max(args.warmup, 3), "warmup_steps_run": nwarm,
            "ms_per_step": round(ms_step, 4),
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
            "data": "synthetic (seeded random-init weights, seeded paged KV cache)",
            "config": {**workload_config(args, work, b, dist.world), "plan": plan.describe(),
                       "plan_choice": "forced on the command line" if forced else
                       "planner candidates timed on this batch (nf_tune_plan), fastest kept",
                       "l2": "working set (KV cache + weights) > 126 MB L2 on every step; no flush"},
            "frac_of_compute_optimum": round(t_opt_ms / ms_step, 4),
            "t_opt_ms": round(t_opt_ms, 4), "iteration_tflop": round(flops / 1e12, 4),
            # the same against the bf16 peak a GEMM sustains under the power cap (the timed steps run there)
            "frac_of_compute_optimum_sustained": round(flops / (bf16_tf_sus * 1e12) * 1e3 / ms_step, 4),
            "all_tokens_per_s": dist.world * b.num_tokens * args.steps / (ms_total / 1000.0),
            "ops": op_summary, "cost_model": {k: (round(v, 4) if isinstance(v, float) else v) for k, v in cost.items()},
            "roofline": roofline, "cpu_baseline": cpu, "clocks": clk,
            "gpu_launches": count_launches(work, plan, b.ctx_lens) * args.steps}
    line.update(extras)
    if "e2e" not in line:
        line["e2e"] = None
    if dist.rank == 0:
        print(json.dumps(line), flush=True)
    dw.close()


def main(argv=None):
    args = parse_args(argv)
    from synth.workloads import WORKLOADS
    work = WORKLOADS[args.workload]
    dist = Dist()
    try:
        if args.impl == "reference":
            run_reference(args, work, dist)
        else:
            run_ours(args, work, dist)
    finally:
        dist.close()


if __name__ == "__main__":
    main()
