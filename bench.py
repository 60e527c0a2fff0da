"""Benchmark of the CompKV decode step on B200 (one JSON line on rank 0).

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
                    [--workload llama8b_128k_b512]

A step is one whole decode step of one attention layer for the whole batch: compensation-aware
score, Top-K and sparse compensated attention in one call (compkv_decode_step: the streaming score
kernel, then the select-and-attend kernel), with the block summaries prebuilt, on seeded synthetic
caches (sparse_kv_cache_summaries_b200.synth).
The default workload is the Llama-3.1-8B layer at 128K context with a 512-token budget.

Timing: R = 4 independent caches (K, V, summaries) are resident in HBM and the steps rotate
through them, so the per-step working set (about 70 MB at 128K) times R exceeds the 126 MB L2.
Steps are replayed from CUDA graphs. After a warm-up of at least --warmup steps and at least
WARMUP_S seconds, the timed region of exactly --steps steps is run many times (at least
MIN_REGIONS, and enough to fill MIN_WINDOW_S seconds); each region is bracketed by a barrier and
torch.cuda.synchronize and timed with CUDA events on the launching stream. The reported time per
step is the median region divided by --steps, then the max over ranks. NVML samples the SM clock
and the throttle reasons over the whole window of timed regions. Several N run as independent
replicas (weak scaling, no collective on the data path).

`--impl reference` times the fp64 CPU oracle on this host's cores instead (rank 0 only): whole
decode steps, BLAS threads = all cores, and it reports the number of steps it actually timed.
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
WARMUP_S = 0.5        # seconds of graph replays before the first timed region
MIN_REGIONS = 50      # timed regions of --steps steps, at least
MIN_WINDOW_S = 0.5    # ... and enough regions to fill this many seconds (clock sampling)
MAX_WINDOW_S = 20.0   # ... but no more than this many
KERNELS_PER_STEP = 2  # this library's kernels launched per decode step
STEP_GRAPH = ("CUDA graphs; streaming score kernel, then the select-and-attend kernel with "
              "programmatic dependent launch")


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
        """Median SM clock and the union of throttle reasons over the samples in [t0, t1]."""
        win = [s for s in self.samples if t0 <= s[0] <= t1]
        if not win:
            return {"sm_mhz": None, "sm_max_mhz": self.max_mhz, "reasons": [], "samples": 0,
                    "sampler_ok": self.ok}
        reasons = set()
        for s in win:
            for name, bit in self.REASONS.items():
                if s[2] & bit:
                    reasons.add(name)
        return {"sm_mhz": statistics.median(s[1] for s in win), "sm_max_mhz": self.max_mhz,
                "reasons": sorted(reasons), "samples": len(win), "sampler_ok": self.ok,
                "window_s": t1 - t0}


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
    """The fp64 oracle, as it stands, on this host's cores: whole decode steps of the same
    workload (summaries prebuilt), BLAS threads = all cores. It times `steps` steps, or as many
    whole steps as fit in about two minutes, and reports the count it actually timed."""
    if rank != 0:
        return
    wl = workload(args.workload, args.budget)
    res = cpu_oracle_steps(wl, steps=max(1, args.steps), warmup=min(args.warmup, 2),
                           threads=os.cpu_count() or 1, time_cap_s=120.0)
    line = {"impl": "reference", "metric": METRIC, "value": res["steps_per_s"], "unit": UNIT,
            "n_gpus": args.gpus, "steps": res["steps"], "warmup": res["warmup"],
            "ms_per_step": 1e3 / res["steps_per_s"], "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": config_of(wl),
            "cpu_baseline": {"value": res["steps_per_s"], "unit": UNIT, "cores": res["cores"],
                             "kind": "oracle", "sample": res["sample"]},
            "e2e": {"value": res["steps_per_s"], "unit": UNIT, "h2d_bytes_per_step": 0,
                    "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


def _oracle_unit(oracle, wl, q, K, V, summ, g):
    """The oracle's decode step for one (sequence, kv-head): score, Top-K, compensated attention
    of the kv-head's query heads (summaries prebuilt)."""
    G = wl.group_size
    s = oracle.default_scale(wl.head_dim)
    S = oracle.group_scores(q[g * G:(g + 1) * G], summ[g], s)
    sel = oracle.select_blocks(S, oracle.n_select(wl.budget, 16, S.shape[0]))
    kg, vg = oracle.compkv._f64(K[g]), oracle.compkv._f64(V[g])
    for h in range(G):
        oracle.compensated_attention(q[g * G + h], kg, vg, summ[g], sel, s, 16)


def _oracle_inputs(wl):
    import oracle
    from sparse_kv_cache_summaries_b200 import synth
    q, K, V = synth.make_sequence(wl, 0)
    summ = [oracle.block_summaries(K[g], V[g], 16, wl.n_groups) for g in range(wl.n_kv_heads)]
    return oracle, q, K, V, summ


def cpu_oracle_steps(wl, steps: int, warmup: int, threads: int, time_cap_s: float) -> dict:
    """Times whole decode steps of the oracle (every (sequence, kv-head) of sequence 0's layer,
    batch 1 shape; for B > 1 a step repeats it B times), up to `steps` or until `time_cap_s`."""
    from threadpoolctl import threadpool_limits
    oracle, q, K, V, summ = _oracle_inputs(wl)
    per_step = wl.batch * wl.n_kv_heads

    def one_step():
        for u in range(per_step):
            _oracle_unit(oracle, wl, q, K, V, summ, u % wl.n_kv_heads)

    with threadpool_limits(limits=threads):
        for _ in range(warmup):
            one_step()
        done, t_total = 0, 0.0
        while done < steps and (done == 0 or t_total < time_cap_s):
            t0 = time.perf_counter()
            one_step()
            t_total += time.perf_counter() - t0
            done += 1
    return {"steps_per_s": done / t_total, "steps": done, "warmup": warmup, "cores": threads,
            "seconds": t_total,
            "sample": f"{done} whole decode steps of {wl.name} ({per_step} (sequence, kv-head) "
                      f"units each), summaries prebuilt, numpy fp64, BLAS threads = {threads}"}


def cpu_oracle_sample(wl, target_s: float, threads: int = 1) -> dict:
    """Times the oracle's decode step (summaries prebuilt) one (sequence, kv-head) at a time, in
    order, until about `target_s` seconds of work; returns full steps per second."""
    from threadpoolctl import threadpool_limits
    oracle, q, K, V, summ = _oracle_inputs(wl)
    pairs = wl.batch * wl.n_kv_heads
    with threadpool_limits(limits=threads):
        done, t_total = 0, 0.0
        while t_total < target_s:
            t0 = time.perf_counter()
            _oracle_unit(oracle, wl, q, K, V, summ, done % wl.n_kv_heads)
            t_total += time.perf_counter() - t0
            done += 1
    steps = done / pairs
    return {"steps_per_s": steps / t_total, "cores": threads, "seconds": t_total,
            "sample": f"{done} (sequence, kv-head) units = {steps:.3f} decode steps of "
                      f"{wl.name}, summaries prebuilt, numpy fp64, BLAS threads = {threads}"}


def config_of(wl, summary_dtype: str = "fp32") -> dict:
    return {"workload": wl.name, "batch": wl.batch, "n_q_heads": wl.n_q_heads,
            "n_kv_heads": wl.n_kv_heads, "head_dim": wl.head_dim, "ctx_len": wl.ctx_len,
            "budget_tokens": wl.budget, "block_size": wl.block_size, "n_groups": wl.n_groups,
            "input_dtype": wl.dtype, "summary_dtype": summary_dtype,
            "l2": f"rotates {N_CACHES} independent caches; working set "
                  f"{N_CACHES} x step bytes > 126 MB L2",
            "graph": STEP_GRAPH}


# ---------------------------------------------------------------------------------- timing

def region_counts(est_region_ms: float, min_regions: int = MIN_REGIONS,
                  min_window_s: float = MIN_WINDOW_S, max_window_s: float = MAX_WINDOW_S) -> int:
    """How many timed regions to run: at least `min_regions`, and enough to fill `min_window_s`
    (so the clock sampler sees the load), but no more than `max_window_s` worth."""
    est = max(est_region_ms, 1e-3) / 1e3
    n = max(min_regions, math.ceil(min_window_s / est))
    cap = max(min_regions, int(max_window_s / est))
    return min(n, cap)


class GraphSet:
    """CUDA graphs of a per-cache step function: one graph of `chunk` steps over the rotating
    caches (replayed for long regions) and one graph per remainder length, so a region of n steps
    is n graph steps with no host launch between them."""

    def __init__(self, torch, stream, caches, fn, steps: int, chunk_cap: int = 256):
        self.torch, self.stream = torch, stream
        self.chunk = min(steps, chunk_cap)
        self.chunk -= self.chunk % len(caches) if self.chunk >= len(caches) else 0
        self.chunk = max(1, self.chunk)
        self.graphs = {}
        self._capture(caches, fn, self.chunk)
        rem = steps % self.chunk
        if rem:
            self._capture(caches, fn, rem)

    def _capture(self, caches, fn, n):
        torch = self.torch
        g = torch.cuda.CUDAGraph()
        with torch.cuda.stream(self.stream):
            with torch.cuda.graph(g, stream=self.stream):
                for i in range(n):
                    fn(caches[i % len(caches)])
        self.graphs[n] = g

    def replay(self, n: int):
        full, rem = divmod(n, self.chunk)
        for _ in range(full):
            self.graphs[self.chunk].replay()
        if rem:
            self.graphs[rem].replay()


def timed_regions(torch, stream, graphs: GraphSet, steps: int, world: int, device,
                  warmup_steps: int = 0, warmup_s: float = 0.0, regions: int | None = None):
    """Warm-up (at least `warmup_steps` steps and `warmup_s` seconds of replays), then `regions`
    timed regions of exactly `steps` steps each, every region bracketed by a barrier and a
    synchronize, timed with CUDA events on the launching stream. Every rank runs the same number
    of regions (the max over ranks of each rank's own count). Returns (per-region ms list, wall
    window (t0, t1))."""
    t_end = time.perf_counter() + warmup_s
    done = 0
    with torch.cuda.stream(stream):
        while done < warmup_steps or time.perf_counter() < t_end:
            graphs.replay(steps if steps <= 4096 else 4096)
            done += steps if steps <= 4096 else 4096
            stream.synchronize()

    def one():
        torch.cuda.synchronize()
        if world > 1:
            torch.distributed.barrier()
        torch.cuda.synchronize()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        with torch.cuda.stream(stream):
            e0.record(stream)
            graphs.replay(steps)
            e1.record(stream)
        stream.synchronize()
        return e0.elapsed_time(e1)

    if regions is None:
        probe = one()
        regions = region_counts(probe)
        regions = int(max_over_ranks([float(regions)], device)[0])
    t0 = time.perf_counter()
    times = [one() for _ in range(regions)]
    t1 = time.perf_counter()
    if world > 1:
        torch.distributed.barrier()
    return times, (t0, t1)


def region_stats(times_ms, steps: int) -> dict:
    """Median (the reported figure), min and max of the per-region times, per step in µs."""
    return {"regions": len(times_ms), "steps_per_region": steps,
            "median_us_per_step": statistics.median(times_ms) / steps * 1e3,
            "min_us_per_step": min(times_ms) / steps * 1e3,
            "max_us_per_step": max(times_ms) / steps * 1e3}


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
    for i in range(N_CACHES):
        q, K, V = synth.make_batch(wl.with_(seed=wl.seed + 1000 * i + 97 * rank))
        c = {"q": q.to(dev), "K": K.to(dev), "V": V.to(dev)}
        c["summ"] = ck.empty_summaries(shape, dev)
        c["sel"] = torch.empty((wl.batch, wl.n_kv_heads, max(kb, 1)), dtype=torch.int32, device=dev)
        c["out"] = torch.empty((wl.batch, wl.n_q_heads, wl.head_dim), dtype=torch.float32, device=dev)
        c["ws"] = ck.new_workspace(shape, wl.budget, dev)
        c["dense_ws"] = ck.new_full_workspace(shape, dev)
        c["dense_out"] = torch.empty_like(c["out"])
        with torch.cuda.stream(stream):
            ck.build_summaries(shape, c["K"], c["V"], c["summ"], stream=stream)
        stream.synchronize()
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

    def build(c):
        ck.build_summaries(shape, c["K"], c["V"], c["summ"], stream=stream)

    # warm every path once (plans, attributes), then capture graphs
    with torch.cuda.stream(stream):
        for c in caches:
            step(c)
            dense(c)
    stream.synchronize()
    steps = max(1, args.steps)
    g_step = GraphSet(torch, stream, caches, step, steps)

    # the headline: a run whose clock record is rejected (on any rank) is measured once more
    for attempt in range(2):
        sampler = ClockSampler(local_rank).start()
        times, (tw0, tw1) = timed_regions(torch, stream, g_step, steps, world, dev,
                                          warmup_steps=args.warmup, warmup_s=WARMUP_S)
        clocks = sampler.summary(tw0, tw1)
        sampler.stop()
        rejected = max_over_ranks([1.0 if clocks_rejected(clocks) else 0.0], dev)[0] > 0
        if not rejected or attempt == 1:
            break
    if attempt == 1:
        clocks["remeasured"] = "the first run's clock record was rejected"
    if clocks.get("samples", 0) < 3 and clocks.get("sampler_ok"):
        raise RuntimeError(f"clock sampler saw {clocks.get('samples')} samples in the timed window")
    stats = region_stats(times, steps)
    us_step = max_over_ranks([stats["median_us_per_step"]], dev)[0]

    # per-kernel durations for the roofline and the breakdown: same rotation, graphs, regions
    def per_step_us(fn, n, warm_s=0.2):
        gs = GraphSet(torch, stream, caches, fn, n)
        t, _ = timed_regions(torch, stream, gs, n, world, dev, warmup_steps=n, warmup_s=warm_s)
        return max_over_ranks([region_stats(t, n)["median_us_per_step"]], dev)[0]

    n_k = min(steps, 256)
    us_stream = per_step_us(stream_only, n_k)
    us_score = per_step_us(score_only, n_k)
    us_sparse = per_step_us(sparse_only, n_k)
    us_dense = per_step_us(dense, min(steps, 32))
    us_build = per_step_us(build, 4, warm_s=0.05)

    # end to end through the public API: pinned host q in, fp32 out back, every step
    e2e = None
    if not args.no_e2e:
        q_host = [c["q"].cpu().pin_memory() for c in caches]
        out_host = torch.empty(caches[0]["out"].shape, dtype=torch.float32).pin_memory()
        q_dev = [torch.empty_like(c["q"]) for c in caches]
        n_e2e = max(steps if steps <= 5000 else 5000, 1)

        def e2e_step(i):
            c = caches[i % N_CACHES]
            qd = q_dev[i % N_CACHES]
            qd.copy_(q_host[i % N_CACHES], non_blocking=True)
            ck.decode_step(shape, qd, c["K"], c["V"], c["summ"], wl.budget, c["sel"], c["out"],
                           c["ws"], stream=stream)
            out_host.copy_(c["out"], non_blocking=True)

        def e2e_region(n):
            torch.cuda.synchronize()
            if world > 1:
                torch.distributed.barrier()
            torch.cuda.synchronize()
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            with torch.cuda.stream(stream):
                e0.record(stream)
                for i in range(n):
                    e2e_step(i)
                e1.record(stream)
            stream.synchronize()
            return e0.elapsed_time(e1)

        with torch.cuda.stream(stream):
            t_end = time.perf_counter() + 0.2
            i = 0
            while i < 50 or time.perf_counter() < t_end:
                e2e_step(i)
                i += 1
        stream.synchronize()
        reg = region_counts(e2e_region(n_e2e), min_regions=5, min_window_s=0.3, max_window_s=5.0)
        reg = int(max_over_ranks([float(reg)], dev)[0])
        t_e2e = [e2e_region(n_e2e) for _ in range(reg)]
        ms_e2e = max_over_ranks([statistics.median(t_e2e)], dev)[0]
        e2e = {"value": throughput(world, n_e2e, ms_e2e), "unit": UNIT,
               "h2d_bytes_per_step": q_host[0].numel() * q_host[0].element_size(),
               "d2h_bytes_per_step": out_host.numel() * out_host.element_size(),
               "steps": n_e2e, "regions": reg,
               "path": "compkv_decode_step via the Python binding, eager launches; median region"}

    # incremental append of one token per sequence (on a copy of one cache's summaries): device
    # time per call from a graph of appends, and the host-bound eager rate through the binding
    c0 = caches[0]
    sa = ck.Summaries(*(t.clone() for t in (c0["summ"].mean_k, c0["summ"].var_g,
                                            c0["summ"].mean_v, c0["summ"].count)))
    k_new = c0["K"][:, :, -1].contiguous()
    v_new = c0["V"][:, :, -1].contiguous()
    pos = torch.full((wl.batch,), wl.ctx_len - 1, dtype=torch.int32, device=dev)

    def app(_c):
        ck.append(shape, k_new, v_new, pos, sa, stream=stream)

    append_us = per_step_us(app, 64, warm_s=0.05)
    n_app = 200
    with torch.cuda.stream(stream):
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        for _ in range(n_app):
            app(None)
        e1.record(stream)
    stream.synchronize()
    append_eager_us = e0.elapsed_time(e1) / n_app * 1e3
    del sa

    status = max(ck.read_device_status(c["ws"], stream) for c in caches)
    if rank != 0:
        return

    nbytes = step_bytes(wl, args.summary_dtype)
    peaks = measured_peaks()
    peak = float(peaks.get("hbm_gbs", FALLBACK_HBM_GBS))
    peak_src = "measured" if "hbm_gbs" in peaks else "fallback"
    gbs_step = nbytes["step"] / (us_step * 1e-6) / 1e9
    achieved = nbytes["score_stream_kernel"] / (us_stream * 1e-6) / 1e9
    cpu = None
    if not args.no_cpu_baseline and world == 1:
        allc = cpu_oracle_sample(wl, target_s=10.0, threads=os.cpu_count() or 1)
        one = cpu_oracle_sample(wl, target_s=10.0, threads=1)
        cpu = {"value": allc["steps_per_s"], "unit": UNIT, "cores": allc["cores"], "kind": "oracle",
               "sample": allc["sample"],
               "single_thread": {"value": one["steps_per_s"], "cores": 1, "sample": one["sample"]}}
    line = {
        "metric": METRIC, "value": throughput(world, steps, us_step * steps / 1e3), "unit": UNIT,
        "n_gpus": world, "steps": steps, "warmup": args.warmup, "ms_per_step": us_step / 1e3,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f32",
        "data": "synthetic", "config": config_of(wl, args.summary_dtype),
        "timing": {**stats, "reported": "median over the timed regions; max over ranks",
                   "warmup_s": WARMUP_S},
        "hbm": {"gbs": gbs_step, "bytes_per_step": nbytes["step"], "peak_gbs": peak,
                "frac_of_" + peak_src: gbs_step / peak, "frac_of_nominal_8000": gbs_step / 8000.0},
        "roofline": {"kernel": "score_stream_kernel (scores, records and compensation partials "
                               "over every block's summaries)",
                     "bound": "hbm", "achieved": achieved, "peak": peak, "unit": "GB/s",
                     "frac": achieved / peak, "peak_source": peak_src,
                     "bytes_per_launch": nbytes["score_stream_kernel"], "us_per_launch": us_stream,
                     "traffic": profile_traffic("score_stream_kernel", wl.name, args.summary_dtype)},
        "kernels_us": {"score_stream": us_stream, "score_select": us_score,
                       "sparse_decode": us_sparse, "step": us_step},
        "dense": {"ms_per_step": us_dense / 1e3, "steps_per_s": 1e6 / us_dense,
                  "gbs": nbytes["dense"] / (us_dense * 1e-6) / 1e9,
                  "frac_of_" + peak_src: nbytes["dense"] / (us_dense * 1e-6) / 1e9 / peak,
                  "speedup_sparse_over_dense": us_dense / us_step},
        "build_summaries_ms": us_build / 1e3,
        "append_us": append_us, "append_eager_us": append_eager_us,
        "e2e": e2e, "cpu_baseline": cpu, "gpu_launches": KERNELS_PER_STEP * steps * stats["regions"],
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
