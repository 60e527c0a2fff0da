"""CompKV decode step, restated plainly in numpy float64 (CPU).

TEST INFRASTRUCTURE ONLY. This is the checker, not the product: only ``tests/``,
``__graft_entry__.smoke()`` and the CPU-baseline leg of ``bench.py`` may import it. It shares
no code with the CUDA path and imports nothing from it.

Sources (cited below by tag):

* [Abstract]     CompKV: Compensation-Aware KV Selection for Long-Context LLM Inference,
                 abstract (arXiv 2609.26300), as reproduced on the shd-paper.top summary page.
* [Summary]      Evolve.pub review of the same paper, section "Summary" (Mean compensation,
                 exact KL identity, Section 3 Eq. 4-7, summaries, second-order mass estimate).
* [Claims]       same review, "Key claims under review".
* [Strengths]    same review, "Strengths" (Appendix A.1 exact log-partition KL identity,
                 A.2-A.3 mass-times-variance residual, A.5 mass Top-K as the special case).
* [FAQ]          same review, "Frequently asked questions" (what CompKV reads, the 2d+r+1
                 per-block summaries, updated incrementally).

The pages state the formulas in words only. The readings taken where they are silent
(numbered as in the design notes):

* R1  The exact log-partition identity is KL(q_S || p) = log Z - log Z_S, where q_S is the
      compensated token distribution (selected tokens keep their logits, every token of an
      omitted block gets the block-mean logit) and Z_S its partition function.
* R2  With delta_t = l_t - lbar_j, the residual of omitting block j is
      R_j = Z_j - n_j exp(lbar_j) = n_j exp(lbar_j) (mean_t exp(delta_t) - 1) >= 0, which to
      second order is (block mass) x (within-block logit variance) / 2.
* R3  Second-order mass estimate: m_j = n_j exp(lbar_j) (1 + V_j / 2). Per-head score:
      (m_j / sum_i m_i) * V_j / 2.
* R4  Grouped key variance: r contiguous channel groups of d / r channels; each group
      variance is the mean over its channels of the per-channel population variance. The
      logit-variance estimate is V_j = s^2 sum_g |q_{C_g}|^2 var_{j,g}.
* R5  The "+1" of 2d+r+1 is the block's token count n_j.
* R6  GQA: one selection per kv-head, on the sum over its query heads of the per-head scores.
* R7  Budget: K_b = min(floor(budget / block_size), N_b) blocks of exact attention; no forced
      sink or local blocks; compensation pseudo-tokens are not counted.
* R8  Ties: equal scores -> lower block index first; indices are returned ascending.
* R9  Softmax scale s = 1/sqrt(d); max-subtracted exponentials.
* R12 Removing compensation (App. A.5): the per-head score is the normalised mass
      m_j / sum_i m_i and omitted blocks contribute nothing; "mass_comp" selects by mass and
      still compensates.

Every function below is pinned by ``tests/test_oracle_pins.py`` against closed forms,
invariants, library routines and brute force.
"""
from __future__ import annotations

import itertools
import math
from dataclasses import dataclass

import numpy as np

MODES = ("compkv", "mass", "mass_comp")


def _f64(x) -> np.ndarray:
    """Upcast (numpy or torch, any float dtype) to a float64 numpy array."""
    if hasattr(x, "detach"):                 # a torch tensor: bf16/fp32 -> fp64 is exact
        x = x.detach().cpu().double().numpy()
    return np.asarray(x, dtype=np.float64)


def n_blocks(T: int, block_size: int) -> int:
    return -(-T // block_size)


def block_bounds(T: int, block_size: int, j: int) -> tuple[int, int]:
    """Token range [start, end) of block j: fixed-size token blocks [Abstract]."""
    return j * block_size, min((j + 1) * block_size, T)


def logsumexp(x: np.ndarray) -> float:
    x = np.asarray(x, dtype=np.float64)
    m = float(np.max(x))
    return m + math.log(float(np.sum(np.exp(x - m))))


# ----------------------------------------------------------------------------- summaries

@dataclass
class Summaries:
    """Per-block summaries of one (sequence, kv-head): 2d + r + 1 scalars per block [FAQ]."""
    count: np.ndarray    # [Nb]    n_j, tokens in block j (R5)
    mean_k: np.ndarray   # [Nb, d] mu_j, mean key
    var_g: np.ndarray    # [Nb, r] grouped key variance (R4)
    mean_v: np.ndarray   # [Nb, d] nu_j, mean value


def store(x: np.ndarray, storage: str) -> np.ndarray:
    """Storage rounding of a mean key / mean value: "fp32" keeps fp64 (the fp32 kernel's own
    rounding is inside the tolerances), "fp16" rounds to the nearest fp16 (IEEE, ties to even)."""
    if storage == "fp32":
        return x
    if storage == "fp16":
        return np.asarray(x, dtype=np.float64).astype(np.float16).astype(np.float64)
    raise ValueError(storage)


def block_summaries(k, v, block_size: int = 16, n_groups: int = 4,
                    storage: str = "fp32") -> Summaries:
    """Mean key, grouped key variance and mean value of every block [Summary; FAQ].

    k, v: [T, d] for one sequence and kv-head. Population (1/n) variances (R4), computed from
    the exact mean; `storage` rounds the stored means (the variance stays exact).
    """
    k, v = _f64(k), _f64(v)
    T, d = k.shape
    if d % n_groups:
        raise ValueError("n_groups must divide head_dim")
    nb = n_blocks(T, block_size)
    count = np.zeros(nb, dtype=np.int64)
    mean_k = np.zeros((nb, d))
    var_g = np.zeros((nb, n_groups))
    mean_v = np.zeros((nb, d))
    for j in range(nb):
        a, b = block_bounds(T, block_size, j)
        kb, vb = k[a:b], v[a:b]
        count[j] = b - a
        mu = kb.mean(axis=0)
        chan_var = ((kb - mu) ** 2).mean(axis=0)
        var_g[j] = chan_var.reshape(n_groups, d // n_groups).mean(axis=1)
        mean_k[j] = store(mu, storage)
        mean_v[j] = store(vb.mean(axis=0), storage)
    return Summaries(count, mean_k, var_g, mean_v)


def empty_summaries(nb: int, d: int, n_groups: int = 4) -> Summaries:
    """Summaries of nb blocks that hold no token yet (n = 0, all moments 0)."""
    return Summaries(np.zeros(nb, dtype=np.int64), np.zeros((nb, d)), np.zeros((nb, n_groups)),
                     np.zeros((nb, d)))


def append_token(summ: Summaries, t: int, k_t, v_t, block_size: int = 16,
                 storage: str = "fp32") -> Summaries:
    """The summaries of tokens [0, t] from those of [0, t) and token t (CompKV review, Frequently
    asked questions: the per-block summaries are "updated incrementally as new tokens enter the
    cache"). Returns a new Summaries; `summ` must have room for block t // block_size.

    Welford's update of the running mean and of the sum of squared deviations per channel,
        n' = n + 1,  mu' = mu + (k - mu) / n',  M2_c' = M2_c + (k_c - mu_c)(k_c - mu'_c),
    aggregated over each channel group. The grouped variance (R4: the mean over the group of the
    per-channel population variances) stays exactly updatable from (n, mu, var_g) alone, because
    the group's sum of M2_c is n |C| var_g. The mean value is a plain running mean.
    """
    k_t, v_t = _f64(k_t), _f64(v_t)
    j = t // block_size
    count, mean_k = summ.count.copy(), summ.mean_k.copy()
    var_g, mean_v = summ.var_g.copy(), summ.mean_v.copy()
    r = var_g.shape[1]
    d = mean_k.shape[1]
    gs = d // r
    n = int(count[j])
    n1 = n + 1
    mu = mean_k[j]
    mu1 = mu + (k_t - mu) / n1
    m2 = var_g[j] * (n * gs) + ((k_t - mu) * (k_t - mu1)).reshape(r, gs).sum(axis=1)
    var_g[j] = m2 / (n1 * gs)
    mean_k[j] = store(mu1, storage)
    mean_v[j] = store(mean_v[j] + (v_t - mean_v[j]) / n1, storage)
    count[j] = n1
    return Summaries(count, mean_k, var_g, mean_v)


# ----------------------------------------------------------------------------- scores

def default_scale(d: int) -> float:
    return 1.0 / math.sqrt(d)                                          # R9


def block_mean_logits(q, summ: Summaries, scale: float) -> np.ndarray:
    """lbar_j = s q . mu_j, the block-mean logit used by Mean compensation [Summary]."""
    return scale * (summ.mean_k @ _f64(q))


def logit_variance_estimate(q, summ: Summaries, scale: float) -> np.ndarray:
    """V_j = s^2 sum_g |q_{C_g}|^2 var_{j,g}: within-block logit variance from the grouped
    key variance (R4) [Summary: "grouped key variance (default r=4)"]."""
    q = _f64(q)
    r = summ.var_g.shape[1]
    q_norm2 = (q.reshape(r, -1) ** 2).sum(axis=1)
    return scale * scale * (summ.var_g @ q_norm2)


def second_order_log_mass(q, summ: Summaries, scale: float) -> np.ndarray:
    """log m_j, m_j = n_j exp(lbar_j) (1 + V_j/2): second-order mass estimate (R3) [Summary]."""
    lbar = block_mean_logits(q, summ, scale)
    vhat = logit_variance_estimate(q, summ, scale)
    return np.log(summ.count.astype(np.float64)) + lbar + np.log1p(vhat / 2.0)


def head_scores(q, summ: Summaries, scale: float, mode: str = "compkv") -> np.ndarray:
    """Per-block score of one query head.

    compkv: (m_j / sum_i m_i) * V_j / 2 -- mass times within-block logit variance, the
            estimate of the residual Mean compensation leaves (R2, R3) [Summary; Claims].
    mass, mass_comp: m_j / sum_i m_i -- attention-mass ranking, the rule that removing
            compensation recovers (R12) [Claims; Strengths, App. A.5].
    """
    if mode not in MODES:
        raise ValueError(mode)
    log_m = second_order_log_mass(q, summ, scale)
    mass = np.exp(log_m - logsumexp(log_m))
    if mode == "compkv":
        return mass * logit_variance_estimate(q, summ, scale) / 2.0
    return mass


def group_scores(q_group, summ: Summaries, scale: float, mode: str = "compkv") -> np.ndarray:
    """S_j = sum over the kv-head's query heads of the per-head scores (R6)."""
    q_group = _f64(q_group)
    return sum(head_scores(q_group[h], summ, scale, mode) for h in range(q_group.shape[0]))


def n_select(budget: int, block_size: int, nb: int) -> int:
    """K_b = min(floor(budget / block_size), N_b) (R7)."""
    return min(budget // block_size, nb)


def select_blocks(S, k_sel: int) -> np.ndarray:
    """Top-K blocks by score; ties to the lower index; returned ascending (R8) [Summary]."""
    S = np.asarray(S, dtype=np.float64)
    order = np.lexsort((np.arange(S.shape[0]), -S))   # by -S, then by index
    return np.sort(order[:k_sel])


# ----------------------------------------------------------------------------- attention

def token_logits(q, k, scale: float) -> np.ndarray:
    """l_t = s q . k_t for every cached token."""
    return scale * (_f64(k) @ _f64(q))


def compensated_attention(q, k, v, summ: Summaries, selected, scale: float,
                          block_size: int = 16, compensate: bool = True) -> np.ndarray:
    """Exact attention over the selected blocks plus Mean compensation, in one softmax.

    Every omitted block j enters as one term with logit lbar_j + log n_j and value nu_j, i.e.
    n_j pseudo-tokens at the block-mean logit carrying the mean value [Abstract; Summary; FAQ].
    """
    q, k, v = _f64(q), _f64(k), _f64(v)
    T = k.shape[0]
    nb = summ.count.shape[0]
    chosen = np.zeros(nb, dtype=bool)
    chosen[np.asarray(selected, dtype=np.int64)] = True
    logits, values = [], []
    lbar = block_mean_logits(q, summ, scale)
    for j in range(nb):
        a, b = block_bounds(T, block_size, j)
        if chosen[j]:
            logits.append(scale * (k[a:b] @ q))
            values.append(v[a:b])
        elif compensate:
            logits.append(np.array([lbar[j] + math.log(summ.count[j])]))
            values.append(summ.mean_v[j][None, :])
    lg = np.concatenate(logits)
    vals = np.concatenate(values, axis=0)
    w = np.exp(lg - lg.max())
    return (w[:, None] * vals).sum(axis=0) / w.sum()


def dense_attention(q, k, v, scale: float) -> np.ndarray:
    """Full softmax attention over all T tokens: the baseline the speedup is quoted against."""
    lg = token_logits(q, k, scale)
    w = np.exp(lg - lg.max())
    return (w[:, None] * _f64(v)).sum(axis=0) / w.sum()


def compensated_distribution(q, k, selected, scale: float, block_size: int = 16,
                             compensate: bool = True) -> np.ndarray:
    """The token distribution q_S that Mean compensation attends with (R1).

    Selected tokens keep e^{l_t}; each token of an omitted block gets e^{lbar_j} with lbar_j
    its block's mean logit (0 without compensation). Normalised over all T tokens.
    """
    lg = token_logits(q, k, scale)
    T = lg.shape[0]
    chosen = set(int(j) for j in selected)
    out = np.empty(T)
    for j in range(n_blocks(T, block_size)):
        a, b = block_bounds(T, block_size, j)
        if j in chosen:
            out[a:b] = lg[a:b]
        else:
            out[a:b] = lg[a:b].mean() if compensate else -np.inf
    m = out.max()
    w = np.exp(out - m)
    return w / w.sum()


def kl_divergence(p_from, p_to) -> float:
    """KL(p_from || p_to) by the token sum, skipping zero-mass tokens of p_from."""
    p_from, p_to = np.asarray(p_from), np.asarray(p_to)
    nz = p_from > 0
    return float(np.sum(p_from[nz] * (np.log(p_from[nz]) - np.log(p_to[nz]))))


def log_partitions(q, k, selected, scale: float, block_size: int = 16) -> tuple[float, float]:
    """(log Z, log Z_S): full and compensated partition functions (R1) [Strengths, App. A.1]."""
    lg = token_logits(q, k, scale)
    T = lg.shape[0]
    chosen = set(int(j) for j in selected)
    terms = []
    for j in range(n_blocks(T, block_size)):
        a, b = block_bounds(T, block_size, j)
        if j in chosen:
            terms.append(lg[a:b])
        else:
            terms.append(np.array([lg[a:b].mean() + math.log(b - a)]))
    return logsumexp(lg), logsumexp(np.concatenate(terms))


def block_residuals(q, k, scale: float, block_size: int = 16) -> tuple[np.ndarray, np.ndarray]:
    """Exact per-block mass and residual, normalised by Z: (Z_j / Z, R_j / Z) (R2).

    R_j = Z_j - n_j exp(lbar_j) is what Mean compensation misses when block j is omitted.
    """
    lg = token_logits(q, k, scale)
    T = lg.shape[0]
    logZ = logsumexp(lg)
    nb = n_blocks(T, block_size)
    mass = np.empty(nb)
    resid = np.empty(nb)
    for j in range(nb):
        a, b = block_bounds(T, block_size, j)
        mass[j] = np.exp(lg[a:b] - logZ).sum()
        resid[j] = mass[j] - (b - a) * math.exp(lg[a:b].mean() - logZ)
    return mass, resid


# ----------------------------------------------------------------------------- diagnostics

def average_ranks(x) -> np.ndarray:
    """Ranks 1..n of x ascending; tied values share the mean of their ranks."""
    x = np.asarray(x, dtype=np.float64)
    order = np.argsort(x, kind="stable")
    ranks = np.empty(x.shape[0])
    i = 0
    while i < x.shape[0]:
        j = i
        while j + 1 < x.shape[0] and x[order[j + 1]] == x[order[i]]:
            j += 1
        ranks[order[i:j + 1]] = (i + j) / 2.0 + 1.0
        i = j + 1
    return ranks


def rank_correlation(a, b) -> float:
    """Spearman's rank correlation: Pearson's correlation of the average ranks (the fidelity
    statistic the review quotes for App. B.2, 0.8604 on real activations)."""
    ra, rb = average_ranks(a), average_ranks(b)
    ra, rb = ra - ra.mean(), rb - rb.mean()
    den = math.sqrt(float((ra * ra).sum()) * float((rb * rb).sum()))
    return float((ra * rb).sum() / den) if den > 0 else 0.0


def residual_capture(score, resid, k_sel: int) -> float:
    """Share of the best achievable omitted-residual reduction that Top-K by `score` achieves:
    sum of resid over Top-K(score) / sum of resid over Top-K(resid) (review, App. B.2: 81.53%
    residual capture at r = 4 on real activations)."""
    resid = np.asarray(resid, dtype=np.float64)
    best = resid[select_blocks(resid, k_sel)].sum()
    got = resid[select_blocks(score, k_sel)].sum()
    return float(got / best) if best > 0 else 1.0


def group_residual_criterion(q_group, k, scale: float, block_size: int = 16) -> np.ndarray:
    """T_j = sum over the group's heads of R_{j,h} / Z_h: the first-order change of sum_h KL_h
    when block j is omitted under Mean compensation (readings 1 and 6). What the group score S_j
    estimates."""
    q_group = np.atleast_2d(_f64(q_group))
    k = _f64(k)
    return sum(block_residuals(q_group[h], k, scale, block_size)[1] for h in range(q_group.shape[0]))


def brute_force_best_subset(q_heads, k, k_sel: int, scale: float, block_size: int = 16,
                            compensate: bool = True) -> tuple[tuple, float]:
    """Enumerate every K_b-subset of blocks; return the one minimising sum_h KL(q_S^h || p^h).

    Tiny inputs only (all C(N_b, K_b) subsets). The KL is the token sum, not the identity.
    """
    q_heads = np.atleast_2d(_f64(q_heads))
    k = _f64(k)
    nb = n_blocks(k.shape[0], block_size)
    p = []
    for h in range(q_heads.shape[0]):
        lg = token_logits(q_heads[h], k, scale)
        w = np.exp(lg - lg.max())
        p.append(w / w.sum())
    best, best_val = None, math.inf
    for S in itertools.combinations(range(nb), k_sel):
        val = sum(kl_divergence(compensated_distribution(q_heads[h], k, S, scale, block_size,
                                                         compensate), p[h])
                  for h in range(q_heads.shape[0]))
        if val < best_val - 1e-15:
            best, best_val = S, val
    return best, best_val


# ----------------------------------------------------------------------------- decode step

@dataclass
class StepResult:
    out: np.ndarray            # [B, Hq, d]
    selected: list             # [B][Hkv] -> ascending block indices
    scores: list               # [B][Hkv] -> S_j over the sequence's blocks
    summaries: list            # [B][Hkv] -> Summaries


def decode_step(q, K, V, budget: int, block_size: int = 16, n_groups: int = 4,
                scale: float | None = None, mode: str = "compkv", ctx_lens=None,
                selection=None, pairs=None, summaries=None, storage: str = "fp32") -> StepResult:
    """One CompKV decode step for a batch, summaries -> score -> Top-K -> compensated attention.

    q [B, Hq, d]; K, V [B, Hkv, T, d]. ``ctx_lens`` gives each sequence's token count (default
    T). ``selection[b][g]`` overrides the selected blocks. ``pairs`` restricts the work to a list
    of (b, g) pairs (the other outputs stay NaN / None). ``summaries[b][g]`` reuses prebuilt ones.
    """
    if mode not in MODES:
        raise ValueError(mode)
    B, Hq, d = q.shape
    Hkv, T = K.shape[1], K.shape[2]
    G = Hq // Hkv
    s = default_scale(d) if scale is None else scale
    out = np.full((B, Hq, d), np.nan)
    sel = [[None] * Hkv for _ in range(B)]
    scr = [[None] * Hkv for _ in range(B)]
    summ_all = [[None] * Hkv for _ in range(B)]
    todo = pairs if pairs is not None else [(b, g) for b in range(B) for g in range(Hkv)]
    for b, g in todo:
        Tb = T if ctx_lens is None else int(ctx_lens[b])
        kb = _f64(K[b, g, :Tb])
        vb = _f64(V[b, g, :Tb])
        qg = _f64(q[b, g * G:(g + 1) * G])
        summ = (summaries[b][g] if summaries is not None
                else block_summaries(kb, vb, block_size, n_groups, storage))
        S = group_scores(qg, summ, s, mode)
        chosen = (np.asarray(selection[b][g]) if selection is not None
                  else select_blocks(S, n_select(budget, block_size, summ.count.shape[0])))
        for h in range(G):
            out[b, g * G + h] = compensated_attention(qg[h], kb, vb, summ, chosen, s, block_size,
                                                      compensate=(mode != "mass"))
        sel[b][g], scr[b][g], summ_all[b][g] = chosen, S, summ
    return StepResult(out, sel, scr, summ_all)


def dense_step(q, K, V, scale: float | None = None, ctx_lens=None, pairs=None) -> np.ndarray:
    """Full attention for every (sequence, query head): [B, Hq, d]."""
    B, Hq, d = q.shape
    Hkv, T = K.shape[1], K.shape[2]
    G = Hq // Hkv
    s = default_scale(d) if scale is None else scale
    out = np.full((B, Hq, d), np.nan)
    todo = pairs if pairs is not None else [(b, g) for b in range(B) for g in range(Hkv)]
    for b, g in todo:
        Tb = T if ctx_lens is None else int(ctx_lens[b])
        kb, vb = _f64(K[b, g, :Tb]), _f64(V[b, g, :Tb])
        for h in range(G):
            out[b, g * G + h] = dense_attention(_f64(q[b, g * G + h]), kb, vb, s)
    return out
