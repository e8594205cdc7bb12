"""Time greedy serving of a synthetic request stream, with the CPU in lock step (lag 0) and one
iteration ahead of the GPU (lag 1).

    python -m intra_device_overlapped_b200.servebench --workload tiny_lm --requests 64 --new 32

Prompts are seeded uniform tokens with lengths U[1, chunk]; every request asks for --new tokens
(no end token, so both lags generate the same tokens). The model, its weights and the batch
limits (decode rows, prefill chunk) come from the workload; each run gets a KV pool of its own.
Prints one JSON line per lag: wall time, iterations, generated tokens per second, and the host
time spent forming and launching iterations.
"""
from __future__ import annotations

import argparse
import json

import numpy as np
import torch


def main(argv=None) -> list:
    from synth.workloads import TEST_WORKLOADS, WORKLOADS
    from .harness import DeviceWorkload
    from .serving import ServingSession
    ap = argparse.ArgumentParser()
    ap.add_argument("--workload", default="tiny_lm")
    ap.add_argument("--requests", type=int, default=64)
    ap.add_argument("--new", type=int, default=32)
    ap.add_argument("--pages", type=int, default=0, help="KV pool pages (0: enough for every running request)")
    ap.add_argument("--seed", type=int, default=11)
    args = ap.parse_args(argv)
    w = {**WORKLOADS, **TEST_WORKLOADS}[args.workload]
    dev = "cuda:0"
    dw = DeviceWorkload(w, dev, keep_logits=False)
    s = w.shape
    rng = np.random.default_rng(args.seed)
    prompts = [rng.integers(0, s.vocab, int(rng.integers(1, dw.C + 1))).tolist() for _ in range(args.requests)]
    per_req = (dw.C + args.new + 15) // 16
    pages = args.pages or per_req * (dw.R + 1)
    lines, streams = [], {}
    for lag in (0, 1, 0, 1):  # each lag twice: the first pair also warms up
        sess = ServingSession(dw.model, s, dev, num_pages=pages, max_running=dw.R, chunk_len=dw.C,
                              max_position=4096, lag=lag)
        ids = [sess.add(p, args.new) for p in prompts]
        torch.cuda.synchronize()
        st = sess.run()
        if dw.sync() != 0:
            raise RuntimeError("device status after serving")
        streams.setdefault(lag, [sess.tokens(i) for i in ids])
        sess.close()
        lines.append({"workload": args.workload, "lag": lag, "requests": args.requests, "new_tokens": args.new,
                      "iterations": st["launched"], "wall_ms": round(st["wall_s"] * 1e3, 2),
                      "ms_per_iteration": round(st["wall_s"] * 1e3 / max(st["launched"], 1), 4),
                      "generated_tokens_per_s": round(st["generated"] / st["wall_s"], 1),
                      "host_launch_ms": round(st["host_launch_s"] * 1e3, 2),
                      "discarded_tokens": st["discarded_tokens"]})
    if streams[0] != streams[1]:
        raise RuntimeError("lag 0 and lag 1 generated different tokens")
    for line in lines[2:]:
        print(json.dumps(line))
    dw.close()
    return lines


if __name__ == "__main__":
    main()
