"""The seeded synthetic workloads: shapes, determinism and the planted structure (CPU)."""
import math

import numpy as np
import torch

from sparse_kv_cache_summaries_b200 import synth


def test_tiny_shapes_and_determinism():
    wl = synth.WORKLOADS["tiny"]
    q, k, v = synth.make_sequence(wl, 0)
    assert q.shape == (1, 64) and k.shape == (1, 2048, 64) and v.shape == (1, 2048, 64)
    assert q.dtype == torch.float32
    q2, k2, v2 = synth.make_sequence(wl, 0)
    assert torch.equal(q, q2) and torch.equal(k, k2) and torch.equal(v, v2)
    q3, _, _ = synth.make_sequence(wl, 1)
    assert not torch.equal(q, q3)


def test_tiny_needles_reach_target_logit():
    wl = synth.WORKLOADS["tiny"]
    q, k, _ = synth.make_sequence(wl, 0)
    logits = (k[0].double() @ q[0].double()) / math.sqrt(wl.head_dim)
    top = torch.sort(logits, descending=True).values[:2]
    assert torch.allclose(top, torch.full_like(top, wl.needle_logit), atol=1e-4), top


def test_planted_blocks_have_high_key_variance():
    wl = synth.WORKLOADS["tiny"]
    _, k, _ = synth.make_sequence(wl, 0)
    kb = k[0].reshape(wl.n_blocks, wl.block_size, wl.head_dim).double()
    var = kb.var(dim=1, unbiased=False).mean(dim=1)
    top = torch.sort(var, descending=True).values
    assert (top[:4] > 5.0).all() and (top[4:] < 2.5).all(), top[:6]


def test_llama_layer_is_bf16_with_outliers():
    wl = synth.WORKLOADS["llama8b_32k_b512"].with_(ctx_len=4096)
    q, k, v = synth.make_sequence(wl, 0)
    assert q.dtype == k.dtype == v.dtype == torch.bfloat16
    assert k.shape == (8, 4096, 128)
    ch_std = k.float().std(dim=1)                       # [Hkv, d]
    for g in range(8):
        big = (ch_std[g] > 5.0).sum().item()
        assert big == wl.outlier_channels, (g, big)


def test_grid_and_batched_configs():
    names = [w.name for w in synth.grid_workloads()]
    assert len(names) == 9 and "llama8b_128k_b2048" in names
    wl = synth.WORKLOADS["batched_16x64k_b1024"]
    assert wl.batch == 16 and wl.group_size == 4 and wl.n_blocks == 4096
    small = wl.with_(ctx_len=256, batch=2)
    q, K, V = synth.make_batch(small)
    assert K.shape == (2, 8, 256, 128)
    np.testing.assert_array_equal(K[1].float().numpy(), synth.make_sequence(small, 1)[1].float().numpy())
