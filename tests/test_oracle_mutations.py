"""Plant plausible mistakes in the oracle and check that some pin catches each one.

Every mutation below is a slip a restatement of the method could make (a dropped term, a wrong
sign, scale or index, a transposed grouping, a wrong tie-break). The pins of oracle_checks.py
must not all pass on any of them. CPU only; the oracle is patched in this process only.
"""
import math

import numpy as np
import pytest

import oracle.compkv as O
import oracle_checks as C

_orig = {name: getattr(O, name) for name in (
    "block_summaries", "logit_variance_estimate", "second_order_log_mass", "head_scores",
    "compensated_attention", "select_blocks", "block_mean_logits", "dense_attention",
    "group_scores", "token_logits", "block_residuals", "log_partitions", "append_token", "rank_correlation",
    "residual_capture", "store")}


def _summaries_sample_var(k, v, block_size=16, n_groups=4):
    s = _orig["block_summaries"](k, v, block_size, n_groups)
    n = s.count.astype(float)[:, None]
    s.var_g = s.var_g * n / np.maximum(n - 1, 1)
    return s


def _summaries_interleaved(k, v, block_size=16, n_groups=4):
    k64 = np.asarray(C.np.asarray(k, dtype=float))
    s = _orig["block_summaries"](k, v, block_size, n_groups)
    T, d = k64.shape
    for j in range(s.count.shape[0]):
        kb = k64[j * block_size:(j + 1) * block_size]
        var = kb.var(axis=0)
        s.var_g[j] = var.reshape(d // n_groups, n_groups).mean(axis=0)
    return s


def _vhat_one_scale(q, summ, scale):
    return _orig["logit_variance_estimate"](q, summ, scale) / scale


def _logm_no_second_order(q, summ, scale):
    return np.log(summ.count.astype(float)) + O.block_mean_logits(q, summ, scale)


def _logm_no_count(q, summ, scale):
    return _orig["second_order_log_mass"](q, summ, scale) - np.log(summ.count.astype(float))


def _scores_unnormalised(q, summ, scale, mode="compkv"):
    log_m = O.second_order_log_mass(q, summ, scale)
    m = np.exp(log_m)
    return m * O.logit_variance_estimate(q, summ, scale) / 2 if mode == "compkv" else m


def _scores_full_variance(q, summ, scale, mode="compkv"):
    s = _orig["head_scores"](q, summ, scale, mode)
    return s * 2 if mode == "compkv" else s


def _attn_no_count(q, k, v, summ, selected, scale, block_size=16, compensate=True):
    saved = summ.count
    try:
        summ.count = np.ones_like(saved)
        # keep the selected blocks' token ranges (they do not use the count)
        return _orig["compensated_attention"](q, k, v, summ, selected, scale, block_size,
                                              compensate)
    finally:
        summ.count = saved


def _attn_shifted_value(q, k, v, summ, selected, scale, block_size=16, compensate=True):
    saved = summ.mean_v
    try:
        summ.mean_v = np.roll(saved, 1, axis=0)
        return _orig["compensated_attention"](q, k, v, summ, selected, scale, block_size,
                                              compensate)
    finally:
        summ.mean_v = saved


def _select_high_ties(S, k_sel):
    S = np.asarray(S, dtype=float)
    order = np.lexsort((-np.arange(S.shape[0]), -S))
    return np.sort(order[:k_sel])


def _select_unsorted(S, k_sel):
    S = np.asarray(S, dtype=float)
    return np.lexsort((np.arange(S.shape[0]), -S))[:k_sel]


def _lbar_sign(q, summ, scale):
    return -_orig["block_mean_logits"](q, summ, scale)


def _dense_scale2(q, k, v, scale):
    return _orig["dense_attention"](q, k, v, scale * scale)


def _group_first_head(q_group, summ, scale, mode="compkv"):
    q_group = np.atleast_2d(np.asarray(q_group, dtype=float))
    return O.head_scores(q_group[0], summ, scale, mode)


def _logits_no_scale(q, k, scale):
    return _orig["token_logits"](q, k, 1.0)


def _append_squared_new_mean(summ, t, k_t, v_t, block_size=16):
    """Welford slip: (k - mu')^2 instead of (k - mu)(k - mu')."""
    s = _orig["append_token"](summ, t, k_t, v_t, block_size)
    j = t // block_size
    n1 = s.count[j]
    if n1 > 1:
        k_t = np.asarray(k_t, dtype=float)
        r = s.var_g.shape[1]
        gs = s.mean_k.shape[1] // r
        mu = summ.mean_k[j]
        mu1 = s.mean_k[j]
        wrong = ((k_t - mu1) ** 2).reshape(r, gs).sum(1)
        right = ((k_t - mu) * (k_t - mu1)).reshape(r, gs).sum(1)
        s.var_g[j] = s.var_g[j] + (wrong - right) / (n1 * gs)
    return s


def _append_mean_over_n(summ, t, k_t, v_t, block_size=16):
    """Running-mean slip: divides by the old count."""
    s = _orig["append_token"](summ, t, k_t, v_t, block_size)
    j = t // block_size
    n = summ.count[j]
    if n > 0:
        v_t = np.asarray(v_t, dtype=float)
        s.mean_v[j] = summ.mean_v[j] + (v_t - summ.mean_v[j]) / n
    return s


def _spearman_on_values(a, b):
    """Pearson on raw values instead of ranks."""
    a, b = np.asarray(a, dtype=float), np.asarray(b, dtype=float)
    a, b = a - a.mean(), b - b.mean()
    return float((a * b).sum() / np.sqrt((a * a).sum() * (b * b).sum()))


def _capture_unnormalised(score, resid, k_sel):
    resid = np.asarray(resid, dtype=float)
    return float(resid[O.select_blocks(score, k_sel)].sum())


def _store_fp16_toward_zero(x, storage):
    """fp16 storage that truncates (rounds toward zero) instead of rounding to nearest even."""
    if storage != "fp16":
        return _orig["store"](x, storage)
    x = np.asarray(x, dtype=np.float64)
    h = x.astype(np.float16)
    over = np.abs(h.astype(np.float64)) > np.abs(x)
    h = np.where(over, np.nextafter(h, np.float16(0)), h)
    return h.astype(np.float64)


def _store_fp16_as_fp32(x, storage):
    """fp16 storage that keeps fp32 precision (the rounding step applied at the wrong width)."""
    if storage != "fp16":
        return _orig["store"](x, storage)
    return np.asarray(x, dtype=np.float64).astype(np.float32).astype(np.float64)


MUTATIONS = {
    "fp16_storage_toward_zero": ("store", _store_fp16_toward_zero),
    "fp16_storage_at_fp32": ("store", _store_fp16_as_fp32),
    "spearman_on_values": ("rank_correlation", _spearman_on_values),
    "capture_unnormalised": ("residual_capture", _capture_unnormalised),
    "append_squared_new_mean": ("append_token", _append_squared_new_mean),
    "append_mean_over_old_count": ("append_token", _append_mean_over_n),
    "sample_variance": ("block_summaries", _summaries_sample_var),
    "interleaved_groups": ("block_summaries", _summaries_interleaved),
    "vhat_missing_scale": ("logit_variance_estimate", _vhat_one_scale),
    "mass_without_second_order": ("second_order_log_mass", _logm_no_second_order),
    "mass_without_count": ("second_order_log_mass", _logm_no_count),
    "score_not_normalised": ("head_scores", _scores_unnormalised),
    "score_full_variance": ("head_scores", _scores_full_variance),
    "compensation_without_count": ("compensated_attention", _attn_no_count),
    "compensation_wrong_block_value": ("compensated_attention", _attn_shifted_value),
    "ties_to_higher_index": ("select_blocks", _select_high_ties),
    "selection_not_ascending": ("select_blocks", _select_unsorted),
    "mean_logit_sign": ("block_mean_logits", _lbar_sign),
    "dense_wrong_scale": ("dense_attention", _dense_scale2),
    "gqa_first_head_only": ("group_scores", _group_first_head),
    "logits_without_scale": ("token_logits", _logits_no_scale),
}


@pytest.mark.parametrize("name", sorted(MUTATIONS))
def test_mutation_is_caught(name, monkeypatch):
    attr, fn = MUTATIONS[name]
    monkeypatch.setattr(O, attr, fn)
    failed = []
    for check in C.ALL_CHECKS:
        try:
            check()
        except (AssertionError, ValueError, IndexError, FloatingPointError) as e:  # noqa: PERF203
            failed.append(check.__name__)
        except Exception as e:  # a crash also counts as caught, but say which
            failed.append(f"{check.__name__}:{type(e).__name__}")
    assert failed, f"mutation {name} passed every pin"


def test_unmutated_oracle_passes_every_pin():
    for check in C.ALL_CHECKS:
        check()
    assert math.isfinite(1.0)
