"""Incremental summary append (compkv_append) on the GPU.

Tokens appended one at a time must give the summaries that a rebuild over the longer sequence
gives (the review's FAQ: summaries "updated incrementally as new tokens enter the cache"), within
1e-6 of the largest value per tensor for the means and 1e-5 for the grouped variances (fp32
Welford over at most 16 tokens vs the build kernel's fp32 block sums); counts exactly. The fp64
oracle's append (pinned to its rebuild in oracle_checks.py) checks the first small case directly.
"""
import numpy as np
import pytest
import torch

import oracle
import parity as P
from sparse_kv_cache_summaries_b200 import compkv as ck
from sparse_kv_cache_summaries_b200 import synth

pytestmark = pytest.mark.gpu

L32 = synth.WORKLOADS["llama8b_32k_b512"]
MEAN_TOL, VAR_TOL = 1e-6, 1e-5


def _rel(a, b):
    a, b = a.double().cpu(), b.double().cpu()
    return float((a - b).abs().max() / b.abs().max().clamp_min(1e-30))


def _append_range(shape, K, V, summ, starts, stops, write_cache=None):
    """Appends tokens [starts[b], stops[b]) of each sequence, one token per call."""
    B = shape.batch
    pos = torch.zeros(B, dtype=torch.int32, device="cuda")
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    for step in range(max(e - s for s, e in zip(starts, stops))):
        t = [min(s + step, e - 1) for s, e in zip(starts, stops)]
        live = [s + step < e for s, e in zip(starts, stops)]
        if not all(live):  # sequences that are done get an out-of-range position (skipped)
            t = [ti if lv else shape.ctx_len for ti, lv in zip(t, live)]
        pos.copy_(torch.tensor(t, dtype=torch.int32))
        idx = torch.tensor([min(ti, shape.ctx_len - 1) for ti in t], device="cuda")
        k_new = K[torch.arange(B, device="cuda"), :, idx].contiguous()  # [B, Hkv, d]
        v_new = V[torch.arange(B, device="cuda"), :, idx].contiguous()
        if write_cache is None:
            ck.append(shape, k_new, v_new, pos, summ, status=status)
        else:
            ck.append(shape, k_new, v_new, pos, summ, write_cache[0], write_cache[1], status=status)
    torch.cuda.synchronize()
    return int(status.item())


def _build(shape, K, V, lens):
    s = ck.empty_summaries(shape)
    cl = torch.tensor(lens, dtype=torch.int32, device="cuda")
    ck.build_summaries(shape, K, V, s, cl)
    torch.cuda.synchronize()
    return s


def _check(a, b):
    assert torch.equal(a.count, b.count)
    assert _rel(a.mean_k, b.mean_k) <= MEAN_TOL
    assert _rel(a.mean_v, b.mean_v) <= MEAN_TOL
    assert _rel(a.var_g, b.var_g) <= VAR_TOL


def test_append_equals_rebuild_llama_layer():
    wl = L32.with_(ctx_len=4096 + 37)
    run = P.upload(wl)
    shape = run.shape
    T0, T1 = 4096 - 21, shape.ctx_len            # starts mid-block, crosses block boundaries
    summ = _build(shape, run.Kd, run.Vd, [T0])
    assert _append_range(shape, run.Kd, run.Vd, summ, [T0], [T1]) == 0
    _check(summ, _build(shape, run.Kd, run.Vd, [T1]))
    # the fp64 oracle's append, on one kv-head
    g = 3
    ref = oracle.block_summaries(run.K[0, g, :T0], run.V[0, g, :T0], 16, shape.n_groups)
    s = oracle.empty_summaries(shape.n_blocks, shape.head_dim, shape.n_groups)
    nb0 = ref.count.shape[0]
    s.count[:nb0], s.mean_k[:nb0], s.var_g[:nb0], s.mean_v[:nb0] = (ref.count, ref.mean_k,
                                                                     ref.var_g, ref.mean_v)
    for t in range(T0, T1):
        s = oracle.append_token(s, t, run.K[0, g, t], run.V[0, g, t], 16)
    got = summ.mean_k[0, g].cpu().double().numpy()
    assert np.abs(got - s.mean_k).max() <= 1e-5 * np.abs(s.mean_k).max()
    got = summ.var_g[0, g].cpu().double().numpy()
    assert np.abs(got - s.var_g).max() <= 1e-4 * np.abs(s.var_g).max()


@pytest.mark.parametrize("r,dtype,d", [(1, "fp32", 64), (4, "bf16", 128), (128, "bf16", 128)])
def test_append_from_empty_ragged_batch(r, dtype, d):
    wl = L32.with_(batch=3, n_q_heads=8, n_kv_heads=2, head_dim=d, ctx_len=96, n_groups=r,
                   dtype=dtype)
    run = P.upload(wl)
    shape = run.shape
    stops = [96, 53, 17]
    summ = ck.empty_summaries(shape)
    for t in (summ.mean_k, summ.var_g, summ.mean_v, summ.count):
        t.zero_()
    # sequences that are done are skipped through an out-of-range position, which is flagged
    assert _append_range(shape, run.Kd, run.Vd, summ, [0, 0, 0], stops) == 2
    _check(summ, _build(shape, run.Kd, run.Vd, stops))


def test_append_writes_the_cache_and_rejects_bad_positions():
    wl = L32.with_(ctx_len=256)
    run = P.upload(wl)
    shape = run.shape
    T0 = 200
    Kc, Vc = run.Kd.clone(), run.Vd.clone()
    Kc[:, :, T0:] = 0
    Vc[:, :, T0:] = 0
    summ = _build(shape, run.Kd, run.Vd, [T0])
    assert _append_range(shape, run.Kd, run.Vd, summ, [T0], [T0 + 20], write_cache=(Kc, Vc)) == 0
    assert torch.equal(Kc[:, :, :T0 + 20], run.Kd[:, :, :T0 + 20])
    assert torch.equal(Vc[:, :, :T0 + 20], run.Vd[:, :, :T0 + 20])
    assert not Kc[:, :, T0 + 20:].any()
    before = [t.clone() for t in (summ.mean_k, summ.var_g, summ.mean_v, summ.count)]
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    for bad in (-1, shape.ctx_len):
        pos = torch.tensor([bad], dtype=torch.int32, device="cuda")
        ck.append(shape, run.Kd[:, :, 0].contiguous(), run.Vd[:, :, 0].contiguous(), pos, summ,
                  status=status)
    torch.cuda.synchronize()
    assert status.item() == 2  # COMPKV_DEVERR_BAD_POSITION
    for a, b in zip(before, (summ.mean_k, summ.var_g, summ.mean_v, summ.count)):
        assert torch.equal(a, b)


def test_decode_step_on_appended_summaries():
    """A decode step over summaries grown by appends matches one over rebuilt summaries."""
    wl = L32.with_(ctx_len=2048 + 40)
    run = P.upload(wl)
    shape = run.shape
    T0 = 2048 - 7
    summ = _build(shape, run.Kd, run.Vd, [T0])
    assert _append_range(shape, run.Kd, run.Vd, summ, [T0], [shape.ctx_len]) == 0
    outs = []
    for s in (summ, _build(shape, run.Kd, run.Vd, [shape.ctx_len])):
        run.summ = s
        r = P.run_step(run, 256, "compkv")
        outs.append((r.sel.clone(), r.out.clone()))
    assert torch.equal(outs[0][0], outs[1][0])
    assert float((outs[0][1] - outs[1][1]).abs().max()) <= 1e-4
