"""Time one operation of the serving iteration alone, through the C ABI.

    python -m intra_device_overlapped_b200.opbench --op decode_attention --workload llama3_8b_layer \
        --requests 64 --sm 16 --reps 5

Ops: ``decode_attention`` (requests [0, --requests) of the workload's decode batch, KV read from the
paged pool), ``prefill_attention`` (the workload's prefill chunk), ``gemm`` (--m x --n x --k bf16,
random operands), ``iteration`` (whole serving iterations of the workload with a plan forced by
--nano / --template / --sm-attn, the sequential one by default; one iteration of the Llama-3-8B
layer launches the QKV, O, gate/up and down GEMMs in that order; --persistent runs each layer as
one persistent kernel instead). ``--sm`` is the persistent grid (0 = every SM). The printed line holds the mean
launch time over --reps launches (CUDA events on the launching stream, after --warmup launches) and
the algorithmic bytes or FLOPs of one launch, so that a profiler can target a small, known case.
--power-s S adds the op's steady state under load: S seconds of back-to-back launches after 1 s,
with the median SM clock and board power that nvidia-smi samples meanwhile.
"""
from __future__ import annotations

import argparse
import json

import numpy as np
import torch

from . import check, nf_op_decode_attention, nf_op_gemm_bf16, nf_op_prefill_attention


def _power(launch, seconds: float, stream) -> dict:
    """Steady state of `launch` run back to back: 1 s of warm-up, then `seconds` of launches while
    nvidia-smi samples the SM clock and the board power every 50 ms (medians reported)."""
    import statistics
    import subprocess
    import threading
    import time
    smi = subprocess.Popen(["nvidia-smi", "--id=0", "--query-gpu=clocks.sm,power.draw,clocks_event_reasons.active",
                            "--format=csv,noheader,nounits", "-lms", "50"], stdout=subprocess.PIPE, text=True)
    lines = []
    reader = threading.Thread(target=lambda: [lines.append(x.strip()) for x in smi.stdout], daemon=True)
    reader.start()
    try:
        t0 = time.time()
        while time.time() - t0 < 1.0:
            for _ in range(8):
                launch()
            torch.cuda.synchronize()
        mark = len(lines)
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        n = 0
        e0.record(stream)
        t0 = time.time()
        while time.time() - t0 < seconds:
            for _ in range(8):
                launch()
            n += 8
            torch.cuda.synchronize()
        e1.record(stream)
        torch.cuda.synchronize()
        rows = [x.split(",") for x in lines[mark:] if x.count(",") == 2]
    finally:
        smi.terminate()
    sm = [float(r[0]) for r in rows if r[0].strip()]
    pw = [float(r[1]) for r in rows if r[1].strip()]
    return {"steady_us": round(e0.elapsed_time(e1) * 1000.0 / max(n, 1), 2),
            "sm_mhz": statistics.median(sm) if sm else None, "power_w": statistics.median(pw) if pw else None,
            "samples": len(sm), "reasons": sorted({r[2].strip() for r in rows})}


def _time(launch, reps: int, warmup: int, stream) -> float:
    for _ in range(warmup):
        launch()
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for _ in range(reps):
        launch()
    e1.record(stream)
    torch.cuda.synchronize()
    return e0.elapsed_time(e1) * 1000.0 / reps


def main(argv=None) -> dict:
    ap = argparse.ArgumentParser()
    ap.add_argument("--op", choices=["decode_attention", "prefill_attention", "gemm", "iteration"], required=True)
    ap.add_argument("--nano", type=int, default=1)
    ap.add_argument("--template", type=int, default=0)
    ap.add_argument("--sm-attn", type=int, default=0)
    ap.add_argument("--persistent", action="store_true",
                    help="iteration: one persistent kernel per layer (nf_forward_iteration_persistent)")
    ap.add_argument("--workload", default="llama3_8b_layer")
    ap.add_argument("--layers", type=int, default=0, help="build only this many layers of the workload (0: all)")
    ap.add_argument("--requests", type=int, default=0, help="decode requests (0 = all)")
    ap.add_argument("--sm", type=int, default=0)
    ap.add_argument("--reps", type=int, default=5)
    ap.add_argument("--warmup", type=int, default=2)
    ap.add_argument("--m", type=int, default=1536)
    ap.add_argument("--n", type=int, default=4096)
    ap.add_argument("--k", type=int, default=4096)
    ap.add_argument("--power-s", type=float, default=0.0,
                    help="also run the op back to back for this many seconds (after 1 s) and report the median "
                         "SM clock and board power sampled by nvidia-smi")
    args = ap.parse_args(argv)
    dev = "cuda:0"
    torch.cuda.set_device(dev)
    stream = torch.cuda.current_stream(dev)
    out = {"op": args.op, "sm": args.sm}

    if args.op == "gemm":
        M, N, K = args.m, args.n, args.k
        g = torch.Generator(device=dev).manual_seed(0)
        a = torch.randn((M, K), device=dev, generator=g).to(torch.bfloat16)
        b = (torch.randn((N, K), device=dev, generator=g) * 0.02).to(torch.bfloat16)
        c = torch.empty((M, N), dtype=torch.float32, device=dev)
        launch = lambda: check(nf_op_gemm_bf16(a.data_ptr(), b.data_ptr(), c.data_ptr(), M, N, K, args.sm,
                                               stream.cuda_stream), "gemm")
        us = _time(launch, args.reps, args.warmup, stream)
        out.update({"shape": [M, N, K], "us": round(us, 2), "tflops": round(2.0 * M * N * K / us / 1e6, 1)})
        if args.power_s > 0:
            out["power"] = _power(launch, args.power_s, stream)
    else:
        from synth.workloads import WORKLOADS
        from .harness import DeviceWorkload
        w = WORKLOADS[args.workload]
        if args.layers > 0:
            from dataclasses import replace
            w = replace(w, shape=replace(w.shape, n_layers=min(args.layers, w.shape.n_layers)))
        dw = DeviceWorkload(w, dev, keep_logits=False)
        s, bt = w.shape, dw.batch
        q = torch.zeros((dw.T, s.n_q_heads, s.head_dim), dtype=torch.bfloat16, device=dev)
        o = torch.zeros_like(q)
        if args.op == "iteration":
            plan = dw.plan(nano=args.nano, template=args.template, sm_attn=args.sm_attn)
            launch = lambda: dw.forward(plan, stream, persistent=args.persistent)
            us = _time(launch, args.reps, args.warmup, stream)
            out.update({"workload": args.workload, "plan": plan.describe(), "persistent": args.persistent,
                        "us": round(us, 2)})
        elif args.op == "decode_attention":
            R = args.requests or bt.num_decode
            pages = sum(-(-(int(c) + 1) // s.page_size) for c in bt.ctx_lens[:R])
            nbytes = pages * 2 * s.n_kv_heads * s.page_size * s.head_dim * 2
            launch = lambda: check(nf_op_decode_attention(dw.model, q.data_ptr(), o.data_ptr(), dw.io, 0, 0, R,
                                                          args.sm, stream.cuda_stream), "decode")
            us = _time(launch, args.reps, args.warmup, stream)
            out.update({"workload": args.workload, "requests": R, "kv_bytes": nbytes, "us": round(us, 2),
                        "gbs": round(nbytes / us / 1e3, 1)})
        else:
            R, C = bt.num_decode, bt.prefill_len
            flops = 4.0 * s.n_q_heads * s.head_dim * C * (C + 1) / 2
            launch = lambda: check(nf_op_prefill_attention(dw.model, q.data_ptr(), o.data_ptr(), dw.io, 0, R, C,
                                                           args.sm, stream.cuda_stream), "prefill")
            us = _time(launch, args.reps, args.warmup, stream)
            out.update({"workload": args.workload, "chunk": C, "flops": flops, "us": round(us, 2),
                        "tflops": round(flops / us / 1e6, 2)})
        if args.power_s > 0:
            out["power"] = _power(launch, args.power_s, stream)
        check(dw.sync(), "status")
        dw.close()
    print(json.dumps(out), flush=True)
    return out


if __name__ == "__main__":
    main()
