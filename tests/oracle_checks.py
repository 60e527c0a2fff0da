"""Pins of the fp64 oracle against what the CompKV write-up and the mathematics fix.

Each ``check_*`` raises AssertionError on a violation. They call the oracle through the module
object, so a test can plant a mistake in it (monkeypatch) and confirm that some pin fails.

What pins what (sources: CompKV abstract and the Evolve.pub review of CompKV):

* summaries      -> numpy mean/var per block (library), identical keys give exact zeros,
                    partial last block counts, hand-derived closed forms (golden files).
* append         -> token-by-token Welford appends equal the rebuilt summaries (review, FAQ).
* scores         -> golden closed forms; second-order behaviour: score x Zhat / R_j -> 1 as the
                    within-block spread eps -> 0 with error O(eps) (O(eps^2) for symmetric
                    spreads), and the mass estimate's error shrinks as eps^3 (eps^4).
* KL identity    -> token-sum KL(q_S || p) equals log Z - log Z_S (App. A.1).
* attention      -> dense limit (budget = T) equals dense attention, which equals torch's
                    scaled_dot_product_attention in fp64; the compensated output equals the
                    q_S-weighted token sum (a second, token-level form); a zero-residual block can
                    be omitted without changing the output.
* selection      -> brute force over all subsets: argmin KL is the Top-K by exact residual
                    (App. A.1); without compensation it is the Top-K by exact mass (App. A.5);
                    with two query heads of very different scales the normalised group score
                    picks the brute-force optimum of sum_h KL_h; ties go to the lower index.
"""
from __future__ import annotations

import json
import math
import pathlib

import numpy as np
import torch

import oracle.compkv as O

GOLDEN = pathlib.Path(__file__).parent / "golden"
_SAFE = {"sqrt": math.sqrt, "exp": math.exp, "log": math.log, "log1p": math.log1p,
         "cosh": math.cosh, "__builtins__": {}}


def ev(expr) -> float:
    """Evaluate a closed-form expression from a golden file."""
    return float(eval(str(expr), dict(_SAFE)))  # noqa: S307 - fixed, repo-owned expressions


def _close(a, b, rtol=1e-12, atol=1e-14, what=""):
    a, b = np.asarray(a, dtype=np.float64), np.asarray(b, dtype=np.float64)
    assert a.shape == b.shape, (what, a.shape, b.shape)
    assert np.allclose(a, b, rtol=rtol, atol=atol), (what, a, b)


def _rand_cache(rng, T, d, offset=0.7):
    k = rng.standard_normal((T, d)) + np.repeat(rng.standard_normal((-(-T // 16), d)) * offset,
                                                16, axis=0)[:T]
    v = rng.standard_normal((T, d))
    q = rng.standard_normal(d)
    return q, k, v


# ----------------------------------------------------------------------------- summaries

def check_summaries_library():
    rng = np.random.default_rng(1)
    T, d = 37, 8
    k, v = rng.standard_normal((T, d)), rng.standard_normal((T, d))
    for r in (1, 2, 4, 8):
        s = O.block_summaries(k, v, 16, r)
        assert list(s.count) == [16, 16, 5]
        for j, (a, b) in enumerate([(0, 16), (16, 32), (32, 37)]):
            _close(s.mean_k[j], np.mean(k[a:b], axis=0), what="mean_k")
            _close(s.mean_v[j], np.mean(v[a:b], axis=0), what="mean_v")
            var = np.var(k[a:b], axis=0, ddof=0)
            if r == d:
                _close(s.var_g[j], var, what="var_g r=d")
            if r == 1:
                _close(s.var_g[j], [var.mean()], what="var_g r=1")


def check_summaries_identical_keys():
    rng = np.random.default_rng(2)
    row = rng.standard_normal(8)
    k = np.tile(row, (32, 1))
    v = rng.standard_normal((32, 8))
    s = O.block_summaries(k, v, 16, 4)
    # the fp64 block mean of 16 equal values is within a few ulps of the value, so the
    # variance is zero up to (ulps * |k|)^2
    bound = (16 * np.finfo(np.float64).eps * np.max(np.abs(k))) ** 2
    assert np.all(s.var_g <= bound), s.var_g


def check_append_equals_rebuild():
    """Appending tokens one at a time (Welford) gives the block summaries of the longer sequence,
    from an empty cache and from a partly filled one (review, FAQ: summaries updated
    incrementally as new tokens enter the cache). Pinned to block_summaries (itself pinned to
    numpy), for several group counts and a partial last block."""
    rng = np.random.default_rng(41)
    for d, r, T0, T1 in ((8, 4, 0, 37), (16, 2, 21, 70), (16, 16, 16, 33), (12, 3, 5, 6)):
        _, k, v = _rand_cache(rng, T1, d, offset=2.0)
        k = k * 3.0 + 5.0  # a large common offset: a naive sum-of-squares update loses digits
        nb = -(-T1 // 16)
        s = O.empty_summaries(nb, d, r)
        if T0:
            base = O.block_summaries(k[:T0], v[:T0], 16, r)
            nb0 = base.count.shape[0]
            s.count[:nb0], s.mean_k[:nb0] = base.count, base.mean_k
            s.var_g[:nb0], s.mean_v[:nb0] = base.var_g, base.mean_v
        for t in range(T0, T1):
            s = O.append_token(s, t, k[t], v[t], 16)
        ref = O.block_summaries(k, v, 16, r)
        assert np.array_equal(s.count, ref.count), (s.count, ref.count)
        _close(s.mean_k, ref.mean_k, rtol=1e-12, atol=1e-12, what="append mean_k")
        _close(s.mean_v, ref.mean_v, rtol=1e-12, atol=1e-12, what="append mean_v")
        _close(s.var_g, ref.var_g, rtol=1e-10, atol=1e-12, what="append var_g")


def check_golden_two_blocks():
    g = json.loads((GOLDEN / "two_blocks_d2.json").read_text())
    E = g["expect"]
    scale = ev(g["scale"])
    q, k, v = np.array(g["q"]), np.array(g["k"]), np.array(g["v"])
    s = O.block_summaries(k, v, g["block_size"], g["n_groups"])
    _close(s.count, [ev(x) for x in E["count"]], what="count")
    _close(s.mean_k, [[ev(x) for x in r] for r in E["mean_k"]], what="mean_k")
    _close(s.var_g, [[ev(x) for x in r] for r in E["var_g"]], what="var_g")
    _close(s.mean_v, [[ev(x) for x in r] for r in E["mean_v"]], what="mean_v")
    _close(O.block_mean_logits(q, s, scale), [ev(x) for x in E["lbar"]], what="lbar")
    _close(O.logit_variance_estimate(q, s, scale), [ev(x) for x in E["vhat"]], what="vhat")
    _close(O.second_order_log_mass(q, s, scale), [ev(x) for x in E["log_mass"]], what="logm")
    _close(O.head_scores(q, s, scale, "compkv"), [ev(x) for x in E["score_compkv"]],
           what="score compkv")
    _close(O.head_scores(q, s, scale, "mass"), [ev(x) for x in E["score_mass"]], what="mass")
    sel_c = O.select_blocks(O.group_scores(q[None], s, scale, "compkv"), 1)
    sel_m = O.select_blocks(O.group_scores(q[None], s, scale, "mass"), 1)
    assert list(sel_c) == E["select_compkv_k1"] and list(sel_m) == E["select_mass_k1"]
    bs = g["block_size"]
    _close(O.compensated_attention(q, k, v, s, sel_c, scale, bs, True),
           [ev(x) for x in E["out_compkv_k1"]], what="out compkv")
    _close(O.compensated_attention(q, k, v, s, sel_m, scale, bs, False),
           [ev(x) for x in E["out_mass_k1"]], what="out mass")
    _close(O.compensated_attention(q, k, v, s, sel_m, scale, bs, True),
           [ev(x) for x in E["out_mass_comp_k1"]], what="out mass_comp")
    _close(O.compensated_attention(q, k, v, s, sel_c, scale, bs, True),
           O.dense_attention(q, k, v, scale), what="zero-residual block 1 -> dense")
    _, resid = O.block_residuals(q, k, scale, bs)
    _close(resid, [ev(x) for x in E["residual_over_Z"]], what="residual")
    logZ, _ = O.log_partitions(q, k, [0, 1], scale, bs)
    _close(logZ, ev(E["log_Z"]), what="logZ")
    d = json.loads((GOLDEN / "two_blocks_d2.json").read_text())
    r = d["expect"]["out_compkv_k1"]
    out = O.decode_step(torch.tensor(q)[None, None], torch.tensor(k)[None, None],
                        torch.tensor(v)[None, None], budget=bs, block_size=bs,
                        n_groups=g["n_groups"], scale=scale).out[0, 0]
    _close(out, [ev(x) for x in r], what="decode_step")


def check_golden_grouped_variance():
    g = json.loads((GOLDEN / "grouped_variance_d4.json").read_text())
    scale = ev(g["scale"])
    q, k, v = np.array(g["q"]), np.array(g["k"]), np.array(g["v"])
    for case in g["cases"]:
        s = O.block_summaries(k, v, g["block_size"], case["n_groups"])
        _close(s.var_g[0], [ev(x) for x in case["var_g"]], what=f"var_g r={case['n_groups']}")
        _close(O.logit_variance_estimate(q, s, scale)[0], ev(case["vhat"]), what="vhat")
    lg = O.token_logits(q, k, scale)
    _close(np.var(lg), ev(g["true_logit_variance"]), what="true V")


# ----------------------------------------------------------------------------- identities

def check_kl_identity():
    rng = np.random.default_rng(3)
    T, d, bs = 96 + 7, 8, 16
    q, k, v = _rand_cache(rng, T, d)
    q *= 2.0
    scale = 1 / math.sqrt(d)
    nb = O.n_blocks(T, bs)
    mass, resid = O.block_residuals(q, k, scale, bs)
    assert np.all(resid >= -1e-15) and abs(mass.sum() - 1) < 1e-12
    lg = O.token_logits(q, k, scale)
    p = np.exp(lg - O.logsumexp(lg))
    for trial in range(12):
        S = sorted(rng.choice(nb, size=int(rng.integers(0, nb + 1)), replace=False).tolist())
        qS = O.compensated_distribution(q, k, S, scale, bs)
        kl = O.kl_divergence(qS, p)
        logZ, logZS = O.log_partitions(q, k, S, scale, bs)
        assert logZS <= logZ + 1e-12
        assert kl >= -1e-14
        _close(kl, logZ - logZS, rtol=1e-10, atol=1e-13, what="KL identity")
        omitted = [j for j in range(nb) if j not in S]
        _close(kl, -math.log1p(-resid[omitted].sum()), rtol=1e-10, atol=1e-13,
               what="KL from residuals")


def check_second_form_and_dense_limit():
    rng = np.random.default_rng(4)
    T, d, bs = 80 + 9, 16, 16
    q, k, v = _rand_cache(rng, T, d)
    scale = 1 / math.sqrt(d)
    s = O.block_summaries(k, v, bs, 4)
    nb = O.n_blocks(T, bs)
    for trial in range(8):
        S = sorted(rng.choice(nb, size=int(rng.integers(1, nb + 1)), replace=False).tolist())
        for comp in (True, False):
            a = O.compensated_attention(q, k, v, s, S, scale, bs, comp)
            b = O.compensated_distribution(q, k, S, scale, bs, comp) @ v
            _close(a, b, rtol=1e-11, atol=1e-13, what="second form")
    dense = O.dense_attention(q, k, v, scale)
    _close(O.compensated_attention(q, k, v, s, list(range(nb)), scale, bs), dense,
           what="dense limit")
    ref = torch.nn.functional.scaled_dot_product_attention(
        torch.tensor(q)[None, None, None], torch.tensor(k)[None, None],
        torch.tensor(v)[None, None], scale=scale)[0, 0, 0].numpy()
    _close(dense, ref, rtol=1e-12, atol=1e-14, what="dense vs torch sdpa")
    # batch-level dense limit through the whole decode step
    qb = torch.tensor(rng.standard_normal((1, 4, d)))
    Kb = torch.tensor(rng.standard_normal((1, 2, T, d)))
    Vb = torch.tensor(rng.standard_normal((1, 2, T, d)))
    full = O.decode_step(qb, Kb, Vb, budget=T + bs, block_size=bs, n_groups=4).out
    _close(full, O.dense_step(qb, Kb, Vb), rtol=1e-11, what="decode_step dense limit")


def check_zero_residual_block():
    rng = np.random.default_rng(5)
    T, d, bs = 64, 8, 16
    q, k, v = _rand_cache(rng, T, d)
    k[16:32] = k[16]                       # block 1: identical keys
    v[16:32] *= 1000.0                     # arbitrary values
    scale = 1 / math.sqrt(d)
    s = O.block_summaries(k, v, bs, 4)
    _, resid = O.block_residuals(q, k, scale, bs)
    assert abs(resid[1]) < 1e-15, resid[1]
    sc = O.head_scores(q, s, scale, "compkv")
    assert sc[1] <= 1e-25 * sc.max(), sc          # zero up to fp64 rounding of the mean
    with_1 = O.compensated_attention(q, k, v, s, [0, 1], scale, bs)
    without_1 = O.compensated_attention(q, k, v, s, [0], scale, bs)
    assert np.max(np.abs(with_1 - without_1)) <= 1e-12 * np.max(np.abs(with_1)) + 1e-12


# ----------------------------------------------------------------------------- selection

def check_ties_and_order():
    S = np.array([1.0, 3.0, 3.0, 0.5, 3.0, 2.0])
    assert list(O.select_blocks(S, 2)) == [1, 2]
    assert list(O.select_blocks(S, 4)) == [1, 2, 4, 5]
    assert list(O.select_blocks(np.zeros(5), 3)) == [0, 1, 2]
    assert list(O.select_blocks(np.array([1.0, 2.0, 5.0, 3.0]), 3)) == [1, 2, 3]   # ascending
    assert O.n_select(512, 16, 8192) == 32 and O.n_select(100, 16, 4) == 4
    assert O.n_select(15, 16, 10) == 0


def _axis_blocks(eps, symmetric, nb=8, d=8, bs=16, seed=6):
    """Blocks whose key deviations lie on one coordinate axis each (diagonal covariance)."""
    rng = np.random.default_rng(seed)
    T = nb * bs - 5                            # ragged last block
    base = rng.standard_normal((nb, d)) * 0.5
    k = np.repeat(base, bs, axis=0)[:T].copy()
    spread = 0.3 + 1.7 * np.arange(nb) / nb    # distinct spreads -> distinct residuals
    for j in range(nb):
        a, b = j * bs, min((j + 1) * bs, T)
        n = b - a
        if symmetric:
            u = np.array([(1 if t % 2 == 0 else -1) for t in range(n)], dtype=float)
            if n % 2:
                u[-1] = 0.0
        else:
            u = np.array([2.0] + [-2.0 / (n - 1)] * (n - 1))   # mean 0, skewed
        k[a:b, j % d] += eps * spread[j] * u
    q = rng.standard_normal(d)
    v = rng.standard_normal((T, d))
    return q, k, v


def check_second_order_limit():
    d, bs = 8, 16
    scale = 1 / math.sqrt(d)
    for symmetric, order_ratio, mass_order in ((False, 2.0, 8.0), (True, 4.0, 16.0)):
        errs, merrs = [], []
        for eps in (0.08, 0.04, 0.02):
            q, k, v = _axis_blocks(eps, symmetric)
            s = O.block_summaries(k, v, bs, d)                   # r = d: exact for diagonal Cov
            lg = O.token_logits(q, k, scale)
            logZ = O.logsumexp(lg)
            mass, resid = O.block_residuals(q, k, scale, bs)
            log_m = O.second_order_log_mass(q, s, scale)
            logZhat = O.logsumexp(log_m)
            score = O.head_scores(q, s, scale, "compkv")
            ratio = score * math.exp(logZhat - logZ) / resid
            errs.append(np.max(np.abs(ratio - 1)))
            merrs.append(np.max(np.abs(np.exp(log_m - logZ) / mass - 1)))
            # exact V for diagonal covariance and r = d
            V_true = np.array([np.var(lg[j * bs:(j + 1) * bs]) for j in range(len(mass))])
            _close(O.logit_variance_estimate(q, s, scale), V_true, rtol=1e-9, atol=1e-15,
                   what="vhat == V for diagonal covariance, r = d")
            sel = O.select_blocks(score, 3)
            assert set(sel) == set(np.argsort(-resid)[:3]), (eps, sel)
        for a, b in zip(errs, errs[1:]):
            assert abs(a / b - order_ratio) < 0.25 * order_ratio, (symmetric, errs)
        for a, b in zip(merrs, merrs[1:]):
            assert abs(a / b - mass_order) < 0.3 * mass_order, (symmetric, merrs)
        assert errs[-1] < 0.05


def check_bruteforce_residual_topk():
    d, bs = 8, 16
    scale = 1 / math.sqrt(d)
    for seed, nb, kb in ((11, 8, 2), (12, 10, 3), (13, 12, 4)):
        rng = np.random.default_rng(seed)
        q, k, v = _rand_cache(rng, nb * bs, d, offset=0.6)
        k[: nb * bs // 2] *= 1.6
        best, val = O.brute_force_best_subset(q, k, kb, scale, bs, compensate=True)
        _, resid = O.block_residuals(q, k, scale, bs)
        assert set(best) == set(np.argsort(-resid)[:kb]), (seed, best)
        _close(val, -math.log1p(-(resid.sum() - np.sort(resid)[-kb:].sum())), rtol=1e-9,
               what="optimal KL")


def check_mass_only_reduction():
    d, bs = 8, 16
    scale = 1 / math.sqrt(d)
    for seed, nb, kb in ((21, 8, 2), (22, 10, 3)):
        rng = np.random.default_rng(seed)
        q, k, v = _rand_cache(rng, nb * bs, d, offset=0.9)
        best, val = O.brute_force_best_subset(q, k, kb, scale, bs, compensate=False)
        mass, _ = O.block_residuals(q, k, scale, bs)
        assert set(best) == set(np.argsort(-mass)[:kb]), (seed, best)
        _close(val, -math.log(np.sort(mass)[-kb:].sum()), rtol=1e-9, what="KL(p_S||p)")
        # the oracle's compensation-off score ranks by the second-order mass estimate; with a
        # small within-block spread that is the exact mass ranking
        k_small = np.repeat(k.reshape(nb, bs, d).mean(axis=1), bs, axis=0) \
            + 0.05 * (k - np.repeat(k.reshape(nb, bs, d).mean(axis=1), bs, axis=0))
        s = O.block_summaries(k_small, v, bs, 4)
        mass_s, _ = O.block_residuals(q, k_small, scale, bs)
        sel = O.select_blocks(O.group_scores(q[None], s, scale, "mass"), kb)
        assert set(sel) == set(np.argsort(-mass_s)[:kb])
        _close(O.head_scores(q, s, scale, "mass").sum(), 1.0, what="mass normalised")


def check_gqa_normalisation():
    """Two heads, one with ~e^6 larger logits: S must weight each head by its own Zhat."""
    d, bs, nb, kb = 8, 16, 8, 2
    scale = 1 / math.sqrt(d)
    rng = np.random.default_rng(31)
    base = rng.standard_normal((nb, d)) * 0.3
    k = np.repeat(base, bs, axis=0)
    eps = 0.05
    # head 0 looks along axis 0, head 1 along axis 1; blocks 0-3 spread on axis 0, 4-7 on axis 1
    qh = np.zeros((2, d))
    qh[0, 0], qh[1, 1] = 1.0, 1.0
    qh[0, 2], qh[1, 3] = 8.0, 0.3
    k[:, 2] = 1.0                          # head 0: every logit + s*8 -> Z^0 about 17x Z^1
    k[:, 3] = 0.0
    spread = np.array([3.0, 2.0, 1.5, 1.0, 2.5, 2.2, 1.2, 0.8])
    u = np.array([(1 if t % 2 == 0 else -1) for t in range(bs)], dtype=float)
    for j in range(nb):
        k[j * bs:(j + 1) * bs, 0 if j < 4 else 1] += eps * spread[j] * u
    v = rng.standard_normal((nb * bs, d))
    s = O.block_summaries(k, v, bs, d)
    S = O.group_scores(qh, s, scale, "compkv")
    best, _ = O.brute_force_best_subset(qh, k, kb, scale, bs, compensate=True)
    assert set(O.select_blocks(S, kb)) == set(best), (O.select_blocks(S, kb), best)
    # sensitivity: the unnormalised sum of m_j V_j / 2 picks head 0's blocks only
    raw = sum(np.exp(O.second_order_log_mass(qh[h], s, scale))
              * O.logit_variance_estimate(qh[h], s, scale) / 2 for h in range(2))
    assert set(O.select_blocks(raw, kb)) != set(best)


def check_fp16_storage():
    """fp16 storage rounds the stored means exactly as numpy's IEEE fp16 cast does (ties to even),
    leaves the variance (computed from the exact mean) and the counts untouched, and an append
    over fp16 storage works from the stored, rounded means."""
    rng = np.random.default_rng(8)
    _, k, v = _rand_cache(rng, 40, 8)
    a = O.block_summaries(k, v, 16, 2)
    h = O.block_summaries(k, v, 16, 2, storage="fp16")
    assert np.array_equal(h.mean_k, a.mean_k.astype(np.float16).astype(np.float64))
    assert np.array_equal(h.mean_v, a.mean_v.astype(np.float16).astype(np.float64))
    assert np.array_equal(h.var_g, a.var_g) and np.array_equal(h.count, a.count)
    assert np.float16(1.0 + 2.0 ** -11) == np.float16(1.0)          # tie rounds to even
    s = O.append_token(h, 40, k[0], v[0], 16, storage="fp16")
    mu = h.mean_k[2] + (k[0] - h.mean_k[2]) / (h.count[2] + 1)
    assert np.array_equal(s.mean_k[2], mu.astype(np.float16).astype(np.float64))


def _binary16_value(bits: int) -> float:
    """The value of an IEEE 754 binary16 bit pattern, decoded by its definition."""
    sign = -1.0 if bits >> 15 else 1.0
    e, f = (bits >> 10) & 0x1F, bits & 0x3FF
    if e == 0:
        return sign * math.ldexp(f, -24)          # subnormal: 2^-14 x f / 1024
    assert e != 0x1F, "no inf / NaN in these cases"
    return sign * math.ldexp(1024 + f, e - 25)    # 2^(e-15) x (1 + f / 1024)


def check_fp16_golden():
    """fp16 storage against hand-derived binary16 patterns (golden file): ties to even, just
    above a tie, the sign, an inexact decimal, the spacing of large values, the largest finite
    value and the subnormals."""
    g = json.loads((GOLDEN / "fp16_storage.json").read_text())
    for case in g["cases"]:
        m = ev(case["mean"])
        want = _binary16_value(int(case["bits"], 16))
        k = np.full((16, 2), m)
        k[:, 1] = -m
        v = np.full((16, 2), m)
        h = O.block_summaries(k, v, 16, 1, storage="fp16")
        assert h.mean_k[0, 0] == want and h.mean_k[0, 1] == -want, (case, h.mean_k[0], want)
        assert h.mean_v[0, 0] == want, (case, h.mean_v[0], want)
        assert h.count[0] == 16


def check_fidelity_statistics():
    """Spearman and residual capture: closed forms and textbook cases (App. B.2 statistics)."""
    x = np.array([3.0, 1.0, 4.0, 1.5, 9.0, 2.6])
    assert abs(O.rank_correlation(x, x) - 1.0) < 1e-15
    assert abs(O.rank_correlation(x, -x) + 1.0) < 1e-15
    assert abs(O.rank_correlation(x, np.exp(x)) - 1.0) < 1e-15          # monotone invariance
    # n = 4, one swapped pair: 1 - 6 sum d^2 / (n (n^2 - 1)) = 1 - 6*2/60 = 0.8
    assert abs(O.rank_correlation([1, 2, 3, 4], [1, 3, 2, 4]) - 0.8) < 1e-15
    # ties share the mean rank: ranks of [5, 7, 7, 9] are [1, 2.5, 2.5, 4]
    assert np.array_equal(O.average_ranks([5, 7, 7, 9]), [1, 2.5, 2.5, 4])
    # pearson of ranks [1, 2.5, 2.5, 4] vs [1, 2, 3, 4]: 4.5 / sqrt(4.5 * 5)
    assert abs(O.rank_correlation([5, 7, 7, 9], [1, 2, 3, 4]) - 4.5 / math.sqrt(22.5)) < 1e-15
    R = np.array([0.5, 0.1, 0.3, 0.05, 0.2])
    assert O.residual_capture(R, R, 2) == 1.0
    assert abs(O.residual_capture(-R, R, 2) - (0.1 + 0.05) / (0.5 + 0.3)) < 1e-15
    assert abs(O.residual_capture([0, 0, 0, 1, 1], R, 2) - (0.05 + 0.2) / 0.8) < 1e-15
    # the group criterion of one head is that head's normalised residual
    rng = np.random.default_rng(5)
    q, k, _ = _rand_cache(rng, 64, 8)
    _close(O.group_residual_criterion(q, k, 0.3), O.block_residuals(q, k, 0.3)[1], what="T_j")


ALL_CHECKS = [check_summaries_library, check_summaries_identical_keys, check_append_equals_rebuild,
              check_golden_two_blocks,
              check_golden_grouped_variance, check_kl_identity,
              check_second_form_and_dense_limit, check_zero_residual_block, check_ties_and_order,
              check_second_order_limit, check_bruteforce_residual_topk,
              check_mass_only_reduction, check_gqa_normalisation, check_fidelity_statistics,
              check_fp16_storage, check_fp16_golden]
