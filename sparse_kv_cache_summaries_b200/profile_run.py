"""A short, fixed sequence of this library's kernels on one seeded workload, for profilers.

    python -m sparse_kv_cache_summaries_b200.profile_run [--workload llama8b_128k_b512]
        [--what build,step,dense,append] [--reps 3] [--summary-dtype fp32]

Runs each requested call `reps` times on the same device caches, with a write of a 256 MB buffer
between calls so that every launch starts with its inputs out of L2 (126 MB), then checks the
workspace status word and exits. Nothing is timed here: a profiler (ncu) captures the launches
it is told to. Order of the calls: build_summaries, decode_step, full_decode, append.
"""
from __future__ import annotations

import argparse

import torch

from sparse_kv_cache_summaries_b200 import compkv as ck
from sparse_kv_cache_summaries_b200 import synth

WHAT = ("build", "step", "dense", "append")


def main() -> None:
    ap = argparse.ArgumentParser()
    ap.add_argument("--workload", default="llama8b_128k_b512")
    ap.add_argument("--what", default=",".join(WHAT))
    ap.add_argument("--reps", type=int, default=3)
    ap.add_argument("--budget", type=int, default=None)
    ap.add_argument("--summary-dtype", default="fp32", choices=["fp32", "fp16"])
    args = ap.parse_args()
    what = [w for w in args.what.split(",") if w]
    for w in what:
        if w not in WHAT:
            raise SystemExit(f"unknown call {w!r}; choose from {WHAT}")

    wl = synth.WORKLOADS.get(args.workload) or {w.name: w for w in synth.grid_workloads()}[args.workload]
    budget = wl.budget if args.budget is None else args.budget
    dev = torch.device("cuda", 0)
    shape = ck.LayerShape(wl.batch, wl.n_q_heads, wl.n_kv_heads, wl.head_dim, wl.ctx_len,
                          wl.n_groups, summary_dtype=args.summary_dtype)
    q, K, V = synth.make_batch(wl)
    q, K, V = q.to(dev), K.to(dev), V.to(dev)
    summ = ck.empty_summaries(shape, dev)
    kb = ck.num_selected(shape, budget)
    sel = torch.empty((wl.batch, wl.n_kv_heads, max(kb, 1)), dtype=torch.int32, device=dev)
    out = torch.empty((wl.batch, wl.n_q_heads, wl.head_dim), dtype=torch.float32, device=dev)
    ws = ck.new_workspace(shape, budget, dev)
    dws = ck.new_full_workspace(shape, dev)
    flush = torch.empty(256 << 20, dtype=torch.uint8, device=dev)
    ck.build_summaries(shape, K, V, summ)
    pos = torch.full((wl.batch,), wl.ctx_len - 1, dtype=torch.int32, device=dev)
    k_new = K[:, :, -1].contiguous()
    v_new = V[:, :, -1].contiguous()
    torch.cuda.synchronize()

    for w in what:
        for _ in range(args.reps):
            flush.fill_(1)
            if w == "build":
                ck.build_summaries(shape, K, V, summ)
            elif w == "step":
                ck.decode_step(shape, q, K, V, summ, budget, sel, out, ws)
            elif w == "dense":
                ck.full_decode(shape, q, K, V, out, dws)
            elif w == "append":
                ck.append(shape, k_new, v_new, pos, summ)
            torch.cuda.synchronize()
    assert ck.read_device_status(ws) == 0
    print(f"profile_run ok: {wl.name}, calls {what} x {args.reps}")


if __name__ == "__main__":
    main()
