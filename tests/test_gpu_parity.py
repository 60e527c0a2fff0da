"""CUDA path (through the C ABI) vs the fp64 oracle, on the seeded synthetic workloads.

Sizes: the tiny case and shrunken Llama-layer caches that still span many 32-block tiles, several
cluster ranks and a ragged tail run on every (b, kv-head); the full-size workloads (32K and 128K
context, the 3 x 3 length/budget grid, the 16 x 64K batch) run in the launch configuration the
benchmark times (decode_step: the streaming score kernel, then the select-and-attend kernel with
programmatic dependent launch) and are checked on every kv-head of the Llama layer (the batched
workload: one kv-head of every sequence, all 8 kv-head indices covered), each pair computed by the
oracle one by one.
"""
import numpy as np
import pytest
import torch

import oracle
import parity as P
from sparse_kv_cache_summaries_b200 import compkv as ck
from sparse_kv_cache_summaries_b200 import synth

pytestmark = pytest.mark.gpu

TINY = synth.WORKLOADS["tiny"]
L32 = synth.WORKLOADS["llama8b_32k_b512"]
L128 = synth.WORKLOADS["llama8b_128k_b512"]
BATCH = synth.WORKLOADS["batched_16x64k_b1024"]


def all_pairs(wl):
    return [(b, g) for b in range(wl.batch) for g in range(wl.n_kv_heads)]


# ------------------------------------------------------------------ a0 summaries

@pytest.mark.parametrize("r", [1, 4, 64])
def test_summaries_tiny(r):
    wl = TINY.with_(n_groups=r)
    run = P.upload(wl)
    P.run_summaries(run)
    P.check_summaries(run, all_pairs(wl))


@pytest.mark.parametrize("r", [1, 2, 4, 128])
def test_summaries_llama_ragged(r):
    wl = L32.with_(ctx_len=4096 + 7, n_groups=r)
    run = P.upload(wl)
    P.run_summaries(run)
    P.check_summaries(run, all_pairs(wl))


def test_summaries_identical_keys_exact_zero():
    wl = L32.with_(ctx_len=512, needles=0)
    q, K, V = synth.make_batch(wl)
    K[:, :, 32:48] = K[:, :, 32:33]                 # block 2: 16 identical bf16 keys
    run = P.upload(wl, tensors=(q, K, V))
    P.run_summaries(run)
    assert torch.all(run.summ.var_g[:, :, 2] == 0)


def test_summaries_ragged_batch():
    wl = L32.with_(batch=3, ctx_len=2048, needles=2)
    run = P.upload(wl, ctx_lens=[2048, 1000, 17])
    P.run_summaries(run)
    P.check_summaries(run, all_pairs(wl))


# ------------------------------------------------------------------ a1-a3 decode step

@pytest.mark.parametrize("mode", ["compkv", "mass", "mass_comp"])
def test_decode_tiny(mode):
    run = P.run_step(P.upload(TINY), TINY.budget, mode)
    info = P.check_step(run, TINY.budget, mode, all_pairs(TINY))
    assert info["ties"] == 0


@pytest.mark.parametrize("mode", ["compkv", "mass", "mass_comp"])
def test_decode_llama_small_ragged_tail(mode):
    wl = L32.with_(ctx_len=8192 + 11)                # 513 blocks: several ranks, a partial block
    run = P.run_step(P.upload(wl), 512, mode)
    P.check_step(run, 512, mode, all_pairs(wl))


@pytest.mark.parametrize("G,d,dtype", [(1, 128, "bf16"), (2, 128, "bf16"), (8, 128, "bf16"),
                                       (4, 64, "bf16"), (8, 64, "bf16"), (4, 128, "fp32")])
def test_decode_head_layouts(G, d, dtype):
    wl = L32.with_(n_q_heads=2 * G, n_kv_heads=2, head_dim=d, ctx_len=4096 + 5, dtype=dtype,
                   outlier_channels=2, needles=3)
    run = P.run_step(P.upload(wl), 256, "compkv")
    P.check_summaries(run, all_pairs(wl))
    P.check_step(run, 256, "compkv", all_pairs(wl))


@pytest.mark.parametrize("budget", [512, 1024, 2048])   # Top-K lists of 32, 64 and 128 entries
def test_decode_fused_equals_separate_calls(budget):
    wl = L32.with_(ctx_len=16384)
    a = P.run_step(P.upload(wl), budget, "compkv", fused=True)
    b = P.run_step(P.upload(wl), budget, "compkv", fused=False)
    assert torch.equal(a.sel, b.sel)
    assert torch.equal(a.out, b.out)
    c = P.run_step(P.upload(wl), budget, "compkv", fused=True)
    assert torch.equal(a.out, c.out) and torch.equal(a.scores, c.scores)   # deterministic


# ------------------------------------------------------------------ edge cases

def test_budget_covers_everything_gives_dense():
    wl = L32.with_(ctx_len=2048 + 3)
    run = P.run_step(P.upload(wl), 1 << 20, "compkv")
    assert ck.num_selected(run.shape, 1 << 20) == run.shape.n_blocks
    ws = ck.new_full_workspace(run.shape)
    dense = torch.empty_like(run.out)
    ck.full_decode(run.shape, run.qd, run.Kd, run.Vd, dense, ws)
    torch.cuda.synchronize()
    P.check_dense(run, dense, all_pairs(wl))
    P.check_step(run, 1 << 20, "compkv", all_pairs(wl))
    assert torch.allclose(run.out, dense, rtol=2e-3, atol=1e-2)


@pytest.mark.parametrize("mode", ["compkv", "mass_comp"])
def test_budget_below_one_block_is_pure_compensation(mode):
    wl = L32.with_(ctx_len=4096)
    run = P.run_step(P.upload(wl), 15, mode)
    P.check_step(run, 15, mode, all_pairs(wl))


def test_all_equal_scores_pick_lowest_indices():
    wl = L32.with_(ctx_len=1024, needles=0, outlier_channels=0)
    q, K, V = synth.make_batch(wl)
    K[:] = K[:, :, :1]                               # every key identical: V = 0, S = 0 everywhere
    run = P.run_step(P.upload(wl, tensors=(q, K, V)), 256, "compkv")
    assert torch.equal(run.sel[0, :, :], torch.arange(16, dtype=torch.int32, device="cuda").expand(8, 16))
    P.check_step(run, 256, "compkv", all_pairs(wl))


def test_selection_held_by_one_rank():
    # every key identical: all scores tie and the Top-K_b is the K_b lowest block indices, all in
    # the first rank's chunk, so each rank's best few cannot settle the cut and the ranks' full
    # lists decide it
    wl = L32.with_(needles=0, outlier_channels=0)
    q, K, V = synth.make_batch(wl)
    K[:] = K[:, :, :1]
    run = P.run_step(P.upload(wl, tensors=(q, K, V)), 512, "compkv")
    assert torch.equal(run.sel[0], torch.arange(32, dtype=torch.int32, device="cuda").expand(8, 32))
    P.check_step(run, 512, "compkv", all_pairs(wl))
    sep = P.run_step(P.upload(wl, tensors=(q, K, V)), 512, "compkv", fused=False)
    assert torch.equal(run.sel, sep.sel) and torch.equal(run.out, sep.out)


@pytest.mark.parametrize("n_recent", [6, 40])
def test_selection_recent_window(n_recent):
    # keys of the last n_recent blocks pulled toward the group's mean query, so that the window
    # dominates the selection: 6 blocks fit in what the last rank sends in the one-round
    # exchange, 40 hold more of the Top-K_b than any rank sends
    wl = L32.with_(needles=0)
    q, K, V = synth.make_batch(wl)
    G = wl.group_size
    t0 = wl.ctx_len - 16 * n_recent
    for g in range(wl.n_kv_heads):
        qg = q[0, g * G:(g + 1) * G].float().mean(0)
        K[0, g, t0:] = (K[0, g, t0:].float() + 1.5 * qg).to(K.dtype)
    run = P.run_step(P.upload(wl, tensors=(q, K, V)), 512, "compkv")
    P.check_step(run, 512, "compkv", all_pairs(wl))
    if n_recent == 40:
        recent = (run.sel >= wl.n_blocks - n_recent).sum(-1)
        assert int(recent.min()) > 8      # more than one rank's list of the selection in the window
    sep = P.run_step(P.upload(wl, tensors=(q, K, V)), 512, "compkv", fused=False)
    assert torch.equal(run.sel, sep.sel) and torch.equal(run.out, sep.out)


def test_large_logits_do_not_overflow():
    wl = L32.with_(ctx_len=4096, needles=16, needle_logit=60.0)
    run = P.run_step(P.upload(wl), 512, "compkv")
    assert torch.isfinite(run.out).all()
    P.check_step(run, 512, "compkv", all_pairs(wl))


def test_ragged_batch_decode_and_dense():
    wl = L32.with_(batch=3, ctx_len=4096, needles=4)
    run = P.run_step(P.upload(wl, ctx_lens=[4096, 1500, 40]), 512, "compkv")
    P.check_step(run, 512, "compkv", all_pairs(wl))
    dense = torch.empty_like(run.out)
    ck.full_decode(run.shape, run.qd, run.Kd, run.Vd, dense, ck.new_full_workspace(run.shape),
                   ctx_lens=run.ctx_lens)
    torch.cuda.synchronize()
    P.check_dense(run, dense, all_pairs(wl))


# ------------------------------------------------------------------ a4 dense baseline

def test_dense_tiny_and_llama():
    for wl in (TINY, L32.with_(ctx_len=8192 + 9)):
        run = P.upload(wl)
        out = torch.empty((wl.batch, wl.n_q_heads, wl.head_dim), device="cuda")
        ws = ck.new_full_workspace(run.shape)
        for _ in range(2):                            # the merge ticket resets itself
            ck.full_decode(run.shape, run.qd, run.Kd, run.Vd, out, ws)
        torch.cuda.synchronize()
        P.check_dense(run, out, all_pairs(wl))


@pytest.mark.parametrize("G,d,dtype", [(1, 128, "bf16"), (2, 128, "bf16"), (8, 128, "bf16"),
                                       (4, 64, "bf16"), (8, 64, "bf16"), (4, 128, "fp32")])
def test_dense_head_layouts(G, d, dtype):
    # every head layout of both dense kernels (tensor cores for bf16, fp32 arithmetic for fp32),
    # with a ragged tail, more tiles per split than ring stages, and a repeated call (ticket reset)
    wl = L32.with_(n_q_heads=2 * G, n_kv_heads=2, head_dim=d, ctx_len=12288 + 21, dtype=dtype,
                   outlier_channels=2, needles=3)
    run = P.upload(wl)
    out = torch.empty((wl.batch, wl.n_q_heads, wl.head_dim), device="cuda")
    ws = ck.new_full_workspace(run.shape)
    for _ in range(2):
        ck.full_decode(run.shape, run.qd, run.Kd, run.Vd, out, ws)
    torch.cuda.synchronize()
    P.check_dense(run, out, all_pairs(wl))


# ------------------------------------------------------------------ full-size workloads

def _full(wl, pairs, budget=None, dense=False):
    run = P.upload(wl)
    budget = wl.budget if budget is None else budget
    P.run_step(run, budget, "compkv")
    P.check_summaries(run, pairs)
    info = P.check_step(run, budget, "compkv", pairs)
    if dense:
        out = torch.empty_like(run.out)
        ck.full_decode(run.shape, run.qd, run.Kd, run.Vd, out, ck.new_full_workspace(run.shape))
        torch.cuda.synchronize()
        P.check_dense(run, out, pairs)
    return info


def test_full_llama_32k():
    _full(L32, all_pairs(L32), dense=True)


def test_full_llama_128k():
    _full(L128, all_pairs(L128), dense=True)


@pytest.mark.parametrize("ctx", [32768, 65536, 131072])
def test_full_grid(ctx):
    wl = L32.with_(ctx_len=ctx)
    run = P.upload(wl)
    P.run_summaries(run)
    for budget in (512, 1024, 2048):
        P.run_step(run, budget, "compkv")
        P.check_step(run, budget, "compkv", all_pairs(wl))


def test_full_batched_16x64k():
    _full(BATCH, [(b, (3 * b) % BATCH.n_kv_heads) for b in range(BATCH.batch)])
