"""Seeded synthetic decode workloads: a query per head and a long key/value cache.

This module draws numbers only. It holds none of the attention method's arithmetic (no
summaries, scores, selection or softmax), so the CUDA path and the fp64 oracle can both be fed
from it without sharing any of the method's code.

The caches are shaped like the long-context decode workloads that the CompKV write-up reports
on (CompKV review, "Summary": Llama-3.1-8B, 32K context and 512-token budget; Table 4:
128K context). The recipe below is a synthetic stand-in for the real activations of those
benchmarks (RULER, LongBench-Pro), which are not available here:

* q ~ N(0, 1) per query head, rounded to the cache dtype first.
* Keys: k = N(0, 1) noise + a per-block offset, one d-vector per (block, kv-head) shared by the
  block's tokens, drawn N(0, offset_var). ``offset_var`` is fixed, or drawn once per sequence
  from U(lo, hi).
* Planted blocks: a seeded set of blocks per kv-head has its key noise scaled by
  ``planted_std`` (high within-block variance).
* Outlier channels: ``outlier_channels`` seeded channels per kv-head have the whole key scaled
  by ``outlier_scale``.
* Needles: ``needles`` tokens get the key k = (L * sqrt(d) / |q_h|^2) q_h for a seeded query
  head h, so that head's scaled logit on it is L = ``needle_logit``.
* Values: v ~ N(0, 1).

Everything is drawn with numpy's PCG64, seeded with ``seed + b`` for sequence b, in the order
above, one kv-head at a time. The result is rounded to the cache dtype (bf16 round-to-nearest-
even, or fp32).
"""
from __future__ import annotations

import dataclasses
import math
from typing import Iterator

import numpy as np
import torch

__all__ = ["Workload", "WORKLOADS", "make_sequence", "make_batch", "grid_workloads"]


@dataclasses.dataclass(frozen=True)
class Workload:
    name: str
    batch: int
    n_q_heads: int
    n_kv_heads: int
    head_dim: int
    ctx_len: int
    budget: int
    dtype: str = "bf16"                 # "bf16" or "fp32": dtype of q, K and V
    seed: int = 0
    block_size: int = 16
    n_groups: int = 4                   # r, the number of key-variance channel groups
    offset_var: tuple = (0.5, 0.5)      # per-sequence U(lo, hi) variance of the block offsets
    outlier_channels: int = 4
    outlier_scale: float = 8.0
    planted: float = 0.01               # < 1: fraction of blocks per kv-head; >= 1: a count
    planted_std: float = 3.0
    needles: int = 8
    needle_logit: float = 10.0

    @property
    def group_size(self) -> int:
        return self.n_q_heads // self.n_kv_heads

    @property
    def n_blocks(self) -> int:
        return -(-self.ctx_len // self.block_size)

    @property
    def torch_dtype(self) -> torch.dtype:
        return {"bf16": torch.bfloat16, "fp32": torch.float32}[self.dtype]

    def planted_count(self) -> int:
        if self.planted >= 1:
            return int(self.planted)
        return int(round(self.planted * self.n_blocks))

    def with_(self, **kw) -> "Workload":
        return dataclasses.replace(self, **kw)


def _llama(ctx: int, budget: int, name: str) -> Workload:
    return Workload(name=name, batch=1, n_q_heads=32, n_kv_heads=8, head_dim=128,
                    ctx_len=ctx, budget=budget, dtype="bf16")


WORKLOADS: dict[str, Workload] = {
    # tiny correctness case: 1 q-head / 1 kv-head, d=64, 2048 tokens, budget 256, fp32
    "tiny": Workload(name="tiny", batch=1, n_q_heads=1, n_kv_heads=1, head_dim=64,
                     ctx_len=2048, budget=256, dtype="fp32", outlier_channels=0,
                     planted=4, needles=2),
    # Llama-3.1-8B-shaped decode layer (GQA 32/8, d=128) at 32K and 128K context
    "llama8b_32k_b512": _llama(32768, 512, "llama8b_32k_b512"),
    "llama8b_128k_b512": _llama(131072, 512, "llama8b_128k_b512"),
    # batched decode: 16 sequences of 64K, budget 1024, offset variance U(0.2, 1.0) per sequence
    "batched_16x64k_b1024": Workload(name="batched_16x64k_b1024", batch=16, n_q_heads=32,
                                     n_kv_heads=8, head_dim=128, ctx_len=65536, budget=1024,
                                     offset_var=(0.2, 1.0)),
}


def grid_workloads() -> Iterator[Workload]:
    """The 3 x 3 context-length x budget grid on the Llama layer shape."""
    for ctx in (32768, 65536, 131072):
        for budget in (512, 1024, 2048):
            yield _llama(ctx, budget, f"llama8b_{ctx // 1024}k_b{budget}")


def _round(x: np.ndarray, dtype: str) -> torch.Tensor:
    t = torch.from_numpy(np.ascontiguousarray(x, dtype=np.float32))
    return t.to(torch.bfloat16) if dtype == "bf16" else t.clone()


def make_sequence(wl: Workload, b: int = 0) -> tuple[torch.Tensor, torch.Tensor, torch.Tensor]:
    """Draw sequence ``b`` of a workload.

    Returns CPU tensors in ``wl.torch_dtype``: q [Hq, d], k [Hkv, T, d], v [Hkv, T, d].
    """
    rng = np.random.Generator(np.random.PCG64(wl.seed + b))
    Hq, Hkv, d, T, bs = wl.n_q_heads, wl.n_kv_heads, wl.head_dim, wl.ctx_len, wl.block_size
    nb = wl.n_blocks
    q = _round(rng.standard_normal((Hq, d), dtype=np.float32), wl.dtype)
    lo, hi = wl.offset_var
    off_var = lo if lo == hi else float(rng.uniform(lo, hi))
    k_out = torch.empty((Hkv, T, d), dtype=wl.torch_dtype)
    v_out = torch.empty((Hkv, T, d), dtype=wl.torch_dtype)
    k32 = np.empty((Hkv, T, d), dtype=np.float32)
    for g in range(Hkv):
        offsets = rng.standard_normal((nb, d), dtype=np.float32) * np.float32(math.sqrt(off_var))
        noise = rng.standard_normal((T, d), dtype=np.float32)
        n_pl = min(wl.planted_count(), nb)
        if n_pl:
            for j in rng.choice(nb, size=n_pl, replace=False):
                noise[j * bs:(j + 1) * bs] *= np.float32(wl.planted_std)
        kg = noise
        kg += np.repeat(offsets, bs, axis=0)[:T]
        if wl.outlier_channels:
            chans = rng.choice(d, size=wl.outlier_channels, replace=False)
            kg[:, chans] *= np.float32(wl.outlier_scale)
        k32[g] = kg
        v_out[g] = _round(rng.standard_normal((T, d), dtype=np.float32), wl.dtype)
    qf = q.to(torch.float32).numpy()
    for _ in range(wl.needles):
        h = int(rng.integers(Hq))
        t = int(rng.integers(T))
        qh = qf[h].astype(np.float64)
        k32[h // wl.group_size, t] = (wl.needle_logit * math.sqrt(d) / float(qh @ qh)) * qh
    for g in range(Hkv):
        k_out[g] = _round(k32[g], wl.dtype)
    return q, k_out, v_out


def make_batch(wl: Workload) -> tuple[torch.Tensor, torch.Tensor, torch.Tensor]:
    """All sequences of a workload: q [B, Hq, d], K [B, Hkv, T, d], V [B, Hkv, T, d] (CPU)."""
    q = torch.empty((wl.batch, wl.n_q_heads, wl.head_dim), dtype=wl.torch_dtype)
    K = torch.empty((wl.batch, wl.n_kv_heads, wl.ctx_len, wl.head_dim), dtype=wl.torch_dtype)
    V = torch.empty_like(K)
    for b in range(wl.batch):
        q[b], K[b], V[b] = make_sequence(wl, b)
    return q, K, V
