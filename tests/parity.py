"""Helpers for the GPU-vs-oracle parity tests.

Tolerances (the bar the method's target sets: bf16 inputs with fp32 accumulation):
* summaries: max|gpu - ref| / max|ref| <= 1e-3 per tensor and (b, kv-head); counts exact;
* selection: the selected block set equals the oracle's Top-K_b, except blocks whose oracle
  score lies within 1e-5 (relative) of the K_b-th largest score (near-ties, logged);
* attention outputs: |gpu - ref| <= 1e-2 + 2e-3 |ref| elementwise (bf16 inputs, fp32 math), with
  the oracle run on the GPU's selection (identical to the oracle's own unless a near-tie
  swapped a block).
"""
from __future__ import annotations

import dataclasses

import numpy as np
import torch

import oracle
from sparse_kv_cache_summaries_b200 import compkv as ck
from sparse_kv_cache_summaries_b200 import synth

SUMM_TOL = 1e-3
TIE_RTOL = 1e-5
OUT_RTOL, OUT_ATOL = 2e-3, 1e-2
SCORE_RTOL = 1e-3      # GPU S_j vs oracle S_j, relative to the largest S of the kv-head


def layer_shape(wl: synth.Workload, **kw) -> ck.LayerShape:
    d = dict(batch=wl.batch, n_q_heads=wl.n_q_heads, n_kv_heads=wl.n_kv_heads,
             head_dim=wl.head_dim, ctx_len=wl.ctx_len, n_groups=wl.n_groups)
    d.update(kw)
    return ck.LayerShape(**d)


@dataclasses.dataclass
class GpuCase:
    wl: synth.Workload
    shape: ck.LayerShape
    q: torch.Tensor          # CPU copies (the generator's tensors)
    K: torch.Tensor
    V: torch.Tensor
    qd: torch.Tensor         # device copies
    Kd: torch.Tensor
    Vd: torch.Tensor
    ctx_lens: torch.Tensor | None
    summ: ck.Summaries | None = None
    sel: torch.Tensor | None = None
    scores: torch.Tensor | None = None
    out: torch.Tensor | None = None
    ws: torch.Tensor | None = None


def upload(wl: synth.Workload, ctx_lens=None, tensors=None, summary_dtype="fp32") -> GpuCase:
    q, K, V = tensors if tensors is not None else synth.make_batch(wl)
    shape = layer_shape(wl, summary_dtype=summary_dtype)
    cl = None if ctx_lens is None else torch.tensor(ctx_lens, dtype=torch.int32, device="cuda")
    return GpuCase(wl, shape, q, K, V, q.cuda(), K.cuda(), V.cuda(), cl)


def run_summaries(run: GpuCase) -> ck.Summaries:
    run.summ = ck.empty_summaries(run.shape)
    ck.build_summaries(run.shape, run.Kd, run.Vd, run.summ, run.ctx_lens)
    return run.summ


def run_step(run: GpuCase, budget: int, mode: str = "compkv", fused: bool = True) -> GpuCase:
    if run.summ is None:
        run_summaries(run)
    s = run.shape
    kb = ck.num_selected(s, budget)
    run.sel = torch.full((s.batch, s.n_kv_heads, max(kb, 1)), -7, dtype=torch.int32, device="cuda")
    run.scores = torch.zeros((s.batch, s.n_kv_heads, s.n_blocks), dtype=torch.float32, device="cuda")
    run.out = torch.full((s.batch, s.n_q_heads, s.head_dim), float("nan"), device="cuda")
    run.ws = ck.new_workspace(s, budget)
    if fused:
        ck.decode_step(s, run.qd, run.Kd, run.Vd, run.summ, budget, run.sel, run.out, run.ws, mode,
                       scores=run.scores)
    else:
        ck.score_select(s, run.qd, run.summ, budget, run.sel, run.ws, mode, scores=run.scores)
        ck.sparse_decode(s, run.qd, run.Kd, run.Vd, run.summ, run.sel, budget, run.out, run.ws, mode)
    torch.cuda.synchronize()
    assert ck.read_device_status(run.ws) == 0
    return run


def rel_err(a, b) -> float:
    a, b = np.asarray(a, np.float64), np.asarray(b, np.float64)
    den = np.max(np.abs(b))
    return float(np.max(np.abs(a - b)) / den) if den > 0 else float(np.max(np.abs(a - b)))


def check_summaries(run: GpuCase, pairs, tol=SUMM_TOL) -> dict:
    worst = {"mean_k": 0.0, "var_g": 0.0, "mean_v": 0.0}
    T = run.shape.ctx_len
    for b, g in pairs:
        Tb = T if run.ctx_lens is None else int(run.ctx_lens[b])
        ref = oracle.block_summaries(run.K[b, g, :Tb], run.V[b, g, :Tb], 16, run.shape.n_groups,
                                     run.shape.summary_dtype)
        nb = ref.count.shape[0]
        cnt = run.summ.count[b, g].cpu().numpy()
        assert np.array_equal(cnt[:nb], ref.count), (b, g)
        assert np.all(cnt[nb:] == 0)
        for name in worst:
            gpu = getattr(run.summ, name)[b, g, :nb].float().cpu().numpy()
            e = rel_err(gpu, getattr(ref, name))
            worst[name] = max(worst[name], e)
            assert e <= tol, (name, b, g, e)
    return worst


def check_selection(sel_gpu: np.ndarray, S_ref: np.ndarray, kb: int) -> int:
    """Returns the number of near-tie swaps (0 = bit-exact set)."""
    ref = set(oracle.select_blocks(S_ref, kb).tolist())
    got = set(int(j) for j in sel_gpu.tolist())
    assert len(got) == len(sel_gpu), "duplicate indices"
    assert list(sel_gpu) == sorted(sel_gpu), "not ascending"
    if got == ref:
        return 0
    thr = np.sort(S_ref)[::-1][kb - 1]
    diff = got ^ ref
    for j in diff:
        assert 0 <= j < S_ref.shape[0], j
        assert abs(S_ref[j] - thr) <= TIE_RTOL * abs(thr), (j, S_ref[j], thr)
    return len(diff) // 2


def check_step(run: GpuCase, budget: int, mode: str, pairs) -> dict:
    """Selection, scores and outputs of sampled (b, g) pairs against the oracle."""
    s = run.shape
    G = s.group_size
    info = {"ties": 0, "out_err": 0.0, "score_err": 0.0}
    sel_all = run.sel.cpu().numpy()
    sc_all = run.scores.cpu().numpy()
    out_all = run.out.cpu().numpy().astype(np.float64)
    selection = [[None] * s.n_kv_heads for _ in range(s.batch)]
    ref_scores = {}
    for b, g in pairs:
        Tb = s.ctx_len if run.ctx_lens is None else int(run.ctx_lens[b])
        summ = oracle.block_summaries(run.K[b, g, :Tb], run.V[b, g, :Tb], 16, s.n_groups,
                                      s.summary_dtype)
        S = oracle.group_scores(run.q[b, g * G:(g + 1) * G], summ, oracle.default_scale(s.head_dim),
                                mode)
        ref_scores[(b, g)] = S
        nb = S.shape[0]
        kb = oracle.n_select(budget, 16, nb)
        kb_gpu = ck.num_selected(s, budget)
        sel = sel_all[b, g, :kb_gpu]
        sel = sel[sel < nb]                      # ragged: slots past the sequence hold empty blocks
        assert len(sel) == kb, (len(sel), kb)
        if kb > 0:
            info["ties"] += check_selection(sel, S, kb)
        selection[b][g] = sel
        info["score_err"] = max(info["score_err"], rel_err(sc_all[b, g, :nb], S))
        assert rel_err(sc_all[b, g, :nb], S) <= SCORE_RTOL, (b, g)
    ctx = None if run.ctx_lens is None else run.ctx_lens.cpu().numpy()
    res = oracle.decode_step(run.q, run.K, run.V, budget, 16, s.n_groups, mode=mode, ctx_lens=ctx,
                             selection=selection, pairs=list(pairs), storage=s.summary_dtype)
    for b, g in pairs:
        ref = res.out[b, g * G:(g + 1) * G]
        got = out_all[b, g * G:(g + 1) * G]
        err = np.abs(got - ref)
        assert np.all(np.isfinite(got)), (b, g)
        bad = err > OUT_ATOL + OUT_RTOL * np.abs(ref)
        assert not bad.any(), (b, g, float(err.max()))
        info["out_err"] = max(info["out_err"], float(err.max()))
    return info


def check_dense(run: GpuCase, out: torch.Tensor, pairs) -> float:
    s = run.shape
    G = s.group_size
    ctx = None if run.ctx_lens is None else run.ctx_lens.cpu().numpy()
    ref = oracle.dense_step(run.q, run.K, run.V, ctx_lens=ctx, pairs=list(pairs))
    got = out.cpu().numpy().astype(np.float64)
    worst = 0.0
    for b, g in pairs:
        r = ref[b, g * G:(g + 1) * G]
        o = got[b, g * G:(g + 1) * G]
        err = np.abs(o - r)
        assert not (err > OUT_ATOL + OUT_RTOL * np.abs(r)).any(), (b, g, float(err.max()))
        worst = max(worst, float(err.max()))
    return worst
