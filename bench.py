"""Benchmark of the CompKV decode step on B200 (one JSON line on rank 0).

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
                    [--workload llama8b_128k_b512]

A step is one whole decode step of one attention layer for the whole batch: compensation-aware
score + Top-K (compkv_score_select) and sparse compensated attention (compkv_sparse_decode), with
the block summaries prebuilt, on seeded synthetic caches (sparse_kv_cache_summaries_b200.synth).
The default workload is the Llama-3.1-8B layer at 128K context with a 512-token budget.

Timing: R = 4 independent caches (K, V, summaries) are resident in HBM and the steps rotate
through them, so the per-step working set (about 70 MB at 128K) times R exceeds the 126 MB L2.
Steps are replayed from CUDA graphs; the timed region is bracketed by a barrier and
torch.cuda.synchronize, timed with CUDA events on the launching stream, and the max over ranks
is taken. Several N run as independent replicas (weak scaling, no collective on the data path).

`--impl reference` times the fp64 CPU oracle on this host's cores instead (rank 0 only).
"""
from __future__ import annotations

import argparse
import hashlib
import json
import math
import os
import pathlib
import statistics
import sys
import threading
import time

ROOT = pathlib.Path(__file__).resolve().parent
sys.path.insert(0, str(ROOT))

METRIC = "decode attn steps/s & HBM GB/s (% of peak) at 128K ctx, 512-tok budget"
UNIT = "steps/s"
N_CACHES = 4
FALLBACK_HBM_GBS = 6650.0


def parse():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20000)
    ap.add_argument("--warmup", type=int, default=200)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--workload", default="llama8b_128k_b512")
    ap.add_argument("--budget", type=int, default=None)
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--dense-steps", type=int, default=200)
    ap.add_argument("--summary-dtype", default="fp32", choices=["fp32", "fp16"],
                    help="storage of the mean key / mean value summaries")
    return ap.parse_args()


def workload(name: str, budget):
    from sparse_kv_cache_summaries_b200 import synth
    if name in synth.WORKLOADS:
        wl = synth.WORKLOADS[name]
    else:
        grid = {w.name: w for w in synth.grid_workloads()}
        wl = grid[name]
    return wl if budget is None else wl.with_(budget=budget, name=f"{wl.name}_b{budget}")


def step_bytes(wl, summary_dtype: str = "fp32") -> dict:
    """Algorithmic bytes of one step: every block's summaries (mean key and mean value in the
    summary dtype, fp32 grouped variances, int32 count), bf16 K/V of the selected blocks, q in,
    out (fp32) out. Intermediates (workspace partials) are not counted."""
    esz = 2 if wl.dtype == "bf16" else 4
    ssz = 2 if summary_dtype == "fp16" else 4
    nb = wl.n_blocks
    kb = min(wl.budget // 16, nb)
    pairs = wl.batch * wl.n_kv_heads
    d, r = wl.head_dim, wl.n_groups
    summ = pairs * nb * (ssz * 2 * d + 4 * (r + 1))
    sel_kv = pairs * kb * 16 * d * esz * 2
    q = wl.batch * wl.n_q_heads * d * esz
    out = wl.batch * wl.n_q_heads * d * 4
    return {"step": summ + sel_kv + q + out, "summaries": summ, "selected_kv": sel_kv,
            "score_stream_kernel": summ + q, "dense": pairs * wl.ctx_len * d * esz * 2 + q + out}


def measured_peaks() -> dict:
    p = ROOT / "MEASURED_PEAKS.json"
    if p.exists():
        try:
            return json.loads(p.read_text())
        except Exception:
            pass
    return {}


def profile_traffic(kernel_key: str, wl_name: str, summary_dtype: str = "fp32") -> float | None:
    """DRAM bytes per launch from a committed ncu summary of the same kernel, workload and
    summary storage type, if its kernel source is unchanged."""
    f = ROOT / "profiles" / f"{kernel_key}_{wl_name}.json"
    if not f.exists():
        return None
    try:
        rec = json.loads(f.read_text())
        if rec.get("summary_dtype", "fp32") != summary_dtype:
            return None
        if rec.get("source_sha256") != source_hash(rec.get("sources", [])):
            return None
        return float(rec["dram_bytes_per_launch"])
    except Exception:
        return None


def source_hash(files) -> str:
    h = hashlib.sha256()
    for name in files:
        h.update((ROOT / name).read_bytes())
    return h.hexdigest()


class ClockSampler:
    """Samples SM clock and throttle reasons through NVML every 20 ms (read-only)."""

    REASONS = {"sw_power_cap": 0x4, "hw_slowdown": 0x8, "sw_thermal_slowdown": 0x20,
               "hw_thermal_slowdown": 0x40, "hw_power_brake": 0x80}

    def __init__(self, index: int):
        self.samples = []
        self.stop_ev = threading.Event()
        self.ok = False
        try:
            import pynvml
            pynvml.nvmlInit()
            self.nv = pynvml
            self.h = pynvml.nvmlDeviceGetHandleByIndex(index)
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self.h, pynvml.NVML_CLOCK_SM)
            self.ok = True
        except Exception:
            self.max_mhz = None
        self.th = threading.Thread(target=self._run, daemon=True)

    def _run(self):
        while not self.stop_ev.is_set():
            try:
                mhz = self.nv.nvmlDeviceGetClockInfo(self.h, self.nv.NVML_CLOCK_SM)
                rs = self.nv.nvmlDeviceGetCurrentClocksEventReasons(self.h)
                util = self.nv.nvmlDeviceGetUtilizationRates(self.h).gpu
                self.samples.append((time.perf_counter(), mhz, rs, util))
            except Exception:
                pass
            time.sleep(0.02)

    def start(self):
        if self.ok:
            self.th.start()
        return self

    def stop(self):
        self.stop_ev.set()
        if self.ok:
            self.th.join(timeout=1)

    def summary(self, t0: float, t1: float) -> dict:
        win = [s for s in self.samples if t0 <= s[0] <= t1]
        if len(win) < 3:   # the timed region was too short for the 20 ms sampler: widen it
            win = [s for s in self.samples if t0 - 0.5 <= s[0] <= t1 + 0.1]
        if not win:
            return {"sm_mhz": None, "sm_max_mhz": self.max_mhz, "reasons": [], "samples": 0}
        reasons = set()
        for s in win:
            for name, bit in self.REASONS.items():
                if s[2] & bit:
                    reasons.add(name)
        return {"sm_mhz": statistics.median(s[1] for s in win), "sm_max_mhz": self.max_mhz,
                "reasons": sorted(reasons), "samples": len(win)}


THROTTLE_REASONS = ("hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown")


def clocks_rejected(clocks: dict) -> bool:
    """True when a timed region's clock record cannot stand: a hardware or thermal slowdown was
    active, or the SM clock sat well below its maximum with no reason given (a clock lock left
    behind by another user). A power-cap slowdown alone is kept (it is normal under load)."""
    reasons = clocks.get("reasons") or []
    if any(r in reasons for r in THROTTLE_REASONS):
        return True
    mhz, mx = clocks.get("sm_mhz"), clocks.get("sm_max_mhz")
    return bool(mhz and mx and not reasons and mhz < 0.85 * mx)


def max_over_ranks(values, device=None):
    """Element-wise max of per-rank timings over the process group (identity when alone).
    NCCL on GPUs, gloo on CPU; every rank must call it with the same number of values."""
    import torch
    import torch.distributed as dist
    if not (dist.is_available() and dist.is_initialized()) or dist.get_world_size() == 1:
        return list(values)
    t = torch.tensor(list(values), dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return t.tolist()


def throughput(world: int, steps: int, ms_max: float) -> float:
    """Whole-job steps/s: every replica ran `steps` steps; the slowest rank sets the time."""
    return world * steps / (ms_max / 1e3)


# ---------------------------------------------------------------------------------- reference

def run_reference(args, rank: int):
    """fp64 oracle on the host cores, on a bounded sample of the same workload."""
    if rank != 0:
        return
    import numpy as np
    from threadpoolctl import threadpool_limits

    import oracle
    from sparse_kv_cache_summaries_b200 import synth
    wl = workload(args.workload, args.budget)
    res = cpu_oracle_sample(wl, target_s=60.0, max_units=args.steps)
    line = {"impl": "reference", "metric": METRIC, "value": res["steps_per_s"], "unit": UNIT,
            "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": 1e3 / res["steps_per_s"], "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": config_of(wl),
            "cpu_baseline": {"value": res["steps_per_s"], "unit": UNIT, "cores": res["cores"],
                             "kind": "oracle", "sample": res["sample"]},
            "e2e": {"value": res["steps_per_s"], "unit": UNIT, "h2d_bytes_per_step": 0,
                    "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)
    del np, threadpool_limits, oracle, synth


def cpu_oracle_sample(wl, target_s: float, max_units: int | None = None) -> dict:
    """Times the oracle's decode step (summaries prebuilt) one (sequence, kv-head) at a time, in
    order, until about `target_s` seconds of work; returns full steps per second."""
    import numpy as np
    from threadpoolctl import threadpool_limits

    import oracle
    from sparse_kv_cache_summaries_b200 import synth
    q, K, V = synth.make_sequence(wl, 0)
    pairs = wl.batch * wl.n_kv_heads
    G = wl.group_size
    with threadpool_limits(limits=1):
        summ = [oracle.block_summaries(K[g], V[g], 16, wl.n_groups) for g in range(wl.n_kv_heads)]
        done, t_total = 0, 0.0
        while t_total < target_s and (max_units is None or done < max_units):
            g = done % wl.n_kv_heads
            t0 = time.perf_counter()
            S = oracle.group_scores(q[g * G:(g + 1) * G], summ[g], oracle.default_scale(wl.head_dim))
            sel = oracle.select_blocks(S, oracle.n_select(wl.budget, 16, S.shape[0]))
            kg, vg = oracle.compkv._f64(K[g]), oracle.compkv._f64(V[g])
            for h in range(G):
                oracle.compensated_attention(q[g * G + h], kg, vg, summ[g], sel,
                                             oracle.default_scale(wl.head_dim), 16)
            t_total += time.perf_counter() - t0
            done += 1
    steps = done / pairs
    del np
    return {"steps_per_s": steps / t_total, "cores": 1, "seconds": t_total,
            "sample": f"{done} (sequence, kv-head) units = {steps:.3f} decode steps of "
                      f"{wl.name}, summaries prebuilt, numpy fp64, BLAS limited to 1 thread"}


def config_of(wl, summary_dtype: str = "fp32") -> dict:
    return {"workload": wl.name, "batch": wl.batch, "n_q_heads": wl.n_q_heads,
            "n_kv_heads": wl.n_kv_heads, "head_dim": wl.head_dim, "ctx_len": wl.ctx_len,
            "budget_tokens": wl.budget, "block_size": wl.block_size, "n_groups": wl.n_groups,
            "input_dtype": wl.dtype, "summary_dtype": summary_dtype,
            "l2": f"rotates {N_CACHES} independent caches; working set "
                  f"{N_CACHES} x step bytes > 126 MB L2",
            "graph": "CUDA graphs; streaming score kernel, then the select-and-attend kernel with programmatic dependent launch"}


# ---------------------------------------------------------------------------------- ours

def run_ours(args, rank: int, world: int, local_rank: int):
    import torch

    from sparse_kv_cache_summaries_b200 import build as B
    from sparse_kv_cache_summaries_b200 import compkv as ck
    from sparse_kv_cache_summaries_b200 import synth

    if rank == 0:
        B.build()
    if world > 1:
        import torch.distributed as dist
        dist.barrier()
    B.build()
    torch.cuda.set_device(local_rank)
    dev = torch.device("cuda", local_rank)
    wl = workload(args.workload, args.budget)
    shape = ck.LayerShape(wl.batch, wl.n_q_heads, wl.n_kv_heads, wl.head_dim, wl.ctx_len, wl.n_groups,
                          summary_dtype=args.summary_dtype)
    kb = ck.num_selected(shape, wl.budget)
    stream = torch.cuda.Stream(device=dev)

    caches = []
    build_times = []
    for i in range(N_CACHES):
        q, K, V = synth.make_batch(wl.with_(seed=wl.seed + 1000 * i + 97 * rank))
        c = {"q": q.to(dev), "K": K.to(dev), "V": V.to(dev)}
        c["summ"] = ck.empty_summaries(shape, dev)
        c["sel"] = torch.empty((wl.batch, wl.n_kv_heads, max(kb, 1)), dtype=torch.int32, device=dev)
        c["out"] = torch.empty((wl.batch, wl.n_q_heads, wl.head_dim), dtype=torch.float32, device=dev)
        c["ws"] = ck.new_workspace(shape, wl.budget, dev)
        c["dense_ws"] = ck.new_full_workspace(shape, dev)
        c["dense_out"] = torch.empty_like(c["out"])
        torch.cuda.synchronize()
        with torch.cuda.stream(stream):
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            ck.build_summaries(shape, c["K"], c["V"], c["summ"], stream=stream)   # warm
            e0.record(stream)
            ck.build_summaries(shape, c["K"], c["V"], c["summ"], stream=stream)
            e1.record(stream)
        stream.synchronize()
        build_times.append(e0.elapsed_time(e1))
        caches.append(c)
        del q, K, V

    def step(c):
        ck.decode_step(shape, c["q"], c["K"], c["V"], c["summ"], wl.budget, c["sel"], c["out"],
                       c["ws"], stream=stream)

    def stream_only(c):
        ck.score_stream(shape, c["q"], c["summ"], wl.budget, c["ws"], stream=stream)

    def score_only(c):
        ck.score_select(shape, c["q"], c["summ"], wl.budget, c["sel"], c["ws"], stream=stream)

    def sparse_only(c):
        ck.sparse_decode(shape, c["q"], c["K"], c["V"], c["summ"], c["sel"], wl.budget, c["out"],
                         c["ws"], stream=stream)

    def dense(c):
        ck.full_decode(shape, c["q"], c["K"], c["V"], c["dense_out"], c["dense_ws"], stream=stream)

    # warm every path once (plans, attributes), then capture graphs
    with torch.cuda.stream(stream):
        for c in caches:
            step(c)
            dense(c)
    stream.synchronize()

    def capture(fn, reps):
        g = torch.cuda.CUDAGraph()
        with torch.cuda.stream(stream):
            with torch.cuda.graph(g, stream=stream):
                for _ in range(reps):
                    for c in caches:
                        fn(c)
        return g

    UNROLL = 8
    paths = (("step", step), ("stream", stream_only), ("score", score_only), ("sparse", sparse_only))
    big = {name: capture(fn, UNROLL) for name, fn in paths}
    single = {k: [] for k in big}
    for name, fn in paths:
        for c in caches:
            g = torch.cuda.CUDAGraph()
            with torch.cuda.stream(stream):
                with torch.cuda.graph(g, stream=stream):
                    fn(c)
            single[name].append(g)
    per_big = UNROLL * N_CACHES

    def replay(name, n):
        full, rem = divmod(n, per_big)
        for _ in range(full):
            big[name].replay()
        for i in range(rem):
            single[name][i % N_CACHES].replay()

    def timed(name, n):
        torch.cuda.synchronize()
        if world > 1:
            torch.distributed.barrier()
        torch.cuda.synchronize()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        with torch.cuda.stream(stream):
            e0.record(stream)
            replay(name, n)
            e1.record(stream)
        stream.synchronize()
        torch.cuda.synchronize()
        if world > 1:
            torch.distributed.barrier()
        return e0.elapsed_time(e1)

    # a run whose clock record is rejected (on any rank) is measured once more
    for attempt in range(2):
        sampler = ClockSampler(local_rank).start()
        with torch.cuda.stream(stream):
            replay("step", args.warmup)
        stream.synchronize()
        t_wall0 = time.perf_counter()
        ms = timed("step", args.steps)
        t_wall1 = time.perf_counter()
        clocks = sampler.summary(t_wall0, t_wall1)
        rejected = max_over_ranks([1.0 if clocks_rejected(clocks) else 0.0], dev)[0] > 0
        if not rejected or attempt == 1:
            break
        sampler.stop()
    if attempt == 1:
        clocks["remeasured"] = "the first run's clock record was rejected"
    # per-kernel durations (same rotation, separately timed) for the roofline
    with torch.cuda.stream(stream):
        replay("stream", max(3, args.warmup // 4))
    ms_stream = timed("stream", args.steps)
    ms_score = timed("score", args.steps)
    ms_sparse = timed("sparse", args.steps)
    sampler.stop()

    ms, ms_stream, ms_score, ms_sparse = max_over_ranks([ms, ms_stream, ms_score, ms_sparse], dev)

    # dense baseline (same caches, same rotation, eager launches)
    nd = max(4, args.dense_steps)
    with torch.cuda.stream(stream):
        for c in caches:
            dense(c)
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    with torch.cuda.stream(stream):
        e0.record(stream)
        for i in range(nd):
            dense(caches[i % N_CACHES])
        e1.record(stream)
    stream.synchronize()
    ms_dense = e0.elapsed_time(e1) / nd

    # end to end through the public API: pinned host q in, fp32 out back, every step
    e2e = None
    if not args.no_e2e:
        q_host = [c["q"].cpu().pin_memory() for c in caches]
        out_host = torch.empty(caches[0]["out"].shape, dtype=torch.float32).pin_memory()
        q_dev = [torch.empty_like(c["q"]) for c in caches]
        n_e2e = min(args.steps, 5000)

        def e2e_step(i):
            c = caches[i % N_CACHES]
            qd = q_dev[i % N_CACHES]
            qd.copy_(q_host[i % N_CACHES], non_blocking=True)
            ck.decode_step(shape, qd, c["K"], c["V"], c["summ"], wl.budget, c["sel"], c["out"],
                           c["ws"], stream=stream)
            out_host.copy_(c["out"], non_blocking=True)

        with torch.cuda.stream(stream):
            for i in range(min(50, args.warmup + 8)):
                e2e_step(i)
        stream.synchronize()
        if world > 1:
            torch.distributed.barrier()
        torch.cuda.synchronize()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        with torch.cuda.stream(stream):
            e0.record(stream)
            for i in range(n_e2e):
                e2e_step(i)
            e1.record(stream)
        stream.synchronize()
        ms_e2e = max_over_ranks([e0.elapsed_time(e1)], dev)[0]
        e2e = {"value": throughput(world, n_e2e, ms_e2e), "unit": UNIT,
               "h2d_bytes_per_step": q_host[0].numel() * q_host[0].element_size(),
               "d2h_bytes_per_step": out_host.numel() * out_host.element_size(),
               "steps": n_e2e, "path": "compkv_decode_step via the Python binding, eager launches"}

    # incremental append of one token per sequence (timed on a copy of one cache's summaries)
    c0 = caches[0]
    sa = ck.Summaries(*(t.clone() for t in (c0["summ"].mean_k, c0["summ"].var_g,
                                            c0["summ"].mean_v, c0["summ"].count)))
    k_new = c0["K"][:, :, -1].contiguous()
    v_new = c0["V"][:, :, -1].contiguous()
    pos = torch.full((wl.batch,), wl.ctx_len - 1, dtype=torch.int32, device=dev)
    n_app = 200
    with torch.cuda.stream(stream):
        for _ in range(10):
            ck.append(shape, k_new, v_new, pos, sa, stream=stream)
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        for _ in range(n_app):
            ck.append(shape, k_new, v_new, pos, sa, stream=stream)
        e1.record(stream)
    stream.synchronize()
    append_us = e0.elapsed_time(e1) / n_app * 1e3
    del sa

    status = max(ck.read_device_status(c["ws"], stream) for c in caches)
    if rank != 0:
        return

    nbytes = step_bytes(wl, args.summary_dtype)
    peaks = measured_peaks()
    peak = float(peaks.get("hbm_gbs", FALLBACK_HBM_GBS))
    peak_src = "measured" if "hbm_gbs" in peaks else "fallback"
    sec_step = ms / 1e3 / args.steps
    us_stream = ms_stream / args.steps * 1e3
    us_score = ms_score / args.steps * 1e3
    us_sparse = ms_sparse / args.steps * 1e3
    gbs_step = nbytes["step"] / sec_step / 1e9
    achieved = nbytes["score_stream_kernel"] / (us_stream * 1e-6) / 1e9
    cpu = None
    if not args.no_cpu_baseline and world == 1:
        res = cpu_oracle_sample(wl, target_s=12.0)
        cpu = {"value": res["steps_per_s"], "unit": UNIT, "cores": res["cores"], "kind": "oracle",
               "sample": res["sample"]}
    line = {
        "metric": METRIC, "value": throughput(world, args.steps, ms), "unit": UNIT, "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms / args.steps,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f32",
        "data": "synthetic", "config": config_of(wl, args.summary_dtype),
        "hbm": {"gbs": gbs_step, "bytes_per_step": nbytes["step"], "peak_gbs": peak,
                "frac_of_" + peak_src: gbs_step / peak, "frac_of_nominal_8000": gbs_step / 8000.0},
        "roofline": {"kernel": "score_stream_kernel (scores, records and compensation partials "
                               "over every block's summaries)",
                     "bound": "hbm", "achieved": achieved, "peak": peak, "unit": "GB/s",
                     "frac": achieved / peak, "peak_source": peak_src,
                     "bytes_per_launch": nbytes["score_stream_kernel"], "us_per_launch": us_stream,
                     "traffic": profile_traffic("score_stream_kernel", wl.name, args.summary_dtype)},
        "kernels_us": {"score_stream": us_stream, "score_select": us_score,
                       "sparse_decode": us_sparse, "step": ms / args.steps * 1e3},
        "dense": {"ms_per_step": ms_dense, "steps_per_s": 1e3 / ms_dense,
                  "gbs": nbytes["dense"] / (ms_dense / 1e3) / 1e9,
                  "frac_of_" + peak_src: nbytes["dense"] / (ms_dense / 1e3) / 1e9 / peak,
                  "speedup_sparse_over_dense": ms_dense / (ms / args.steps)},
        "build_summaries_ms": statistics.median(build_times),
        "append_us": append_us,
        "e2e": e2e, "cpu_baseline": cpu, "gpu_launches": 2 * args.steps,
        "clocks": clocks, "device_status": status,
    }
    print(json.dumps(line), flush=True)


def main():
    args = parse()
    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))
    if args.impl == "reference":
        run_reference(args, rank)
        return
    if world > 1:
        import datetime

        import torch
        import torch.distributed as dist
        torch.cuda.set_device(local_rank)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=300),
                                device_id=torch.device("cuda", local_rank))
    try:
        run_ours(args, rank, world, local_rank)
    finally:
        if world > 1:
            import torch.distributed as dist
            dist.destroy_process_group()


if __name__ == "__main__":
    main()
