"""fp16 storage of the mean key and mean value (LayerShape.summary_dtype = "fp16").

Parity: the CUDA path against the fp64 oracle with the same storage rounding (oracle.store:
IEEE fp16, ties to even, applied to the stored means; the variance stays exact), at the bars of
test_gpu_parity.py. Cost of the variant: the same inputs with fp32 and fp16 summaries, selection
overlap and output difference, printed and bounded.
"""
import numpy as np
import pytest
import torch

import parity as P
from sparse_kv_cache_summaries_b200 import compkv as ck
from sparse_kv_cache_summaries_b200 import synth

pytestmark = pytest.mark.gpu

TINY = synth.WORKLOADS["tiny"]
L32 = synth.WORKLOADS["llama8b_32k_b512"]
L128 = synth.WORKLOADS["llama8b_128k_b512"]


def all_pairs(wl):
    return [(b, g) for b in range(wl.batch) for g in range(wl.n_kv_heads)]


def test_fp16_summaries_tiny_and_ragged_tail():
    for wl in (TINY, L32.with_(ctx_len=8192 + 11)):
        run = P.upload(wl, summary_dtype="fp16")
        P.run_summaries(run)
        assert run.summ.mean_k.dtype == torch.float16
        P.check_summaries(run, all_pairs(wl))


@pytest.mark.parametrize("mode", ["compkv", "mass", "mass_comp"])
def test_fp16_decode_llama_ragged_tail(mode):
    wl = L32.with_(ctx_len=8192 + 11)
    run = P.upload(wl, summary_dtype="fp16")
    P.run_step(run, 512, mode)
    P.check_step(run, 512, mode, all_pairs(wl))


@pytest.mark.parametrize("G,d,dtype", [(1, 128, "bf16"), (8, 128, "bf16"), (4, 64, "bf16"),
                                       (8, 64, "bf16"), (4, 128, "fp32")])
def test_fp16_decode_head_layouts(G, d, dtype):
    wl = L32.with_(n_q_heads=2 * G, n_kv_heads=2, head_dim=d, ctx_len=4096 + 5, dtype=dtype,
                   outlier_channels=2, needles=3)
    run = P.upload(wl, summary_dtype="fp16")
    P.run_summaries(run)
    P.check_summaries(run, all_pairs(wl))
    P.run_step(run, 256, "compkv")
    P.check_step(run, 256, "compkv", all_pairs(wl))


def test_fp16_fused_equals_separate_and_is_deterministic():
    wl = L32.with_(ctx_len=16384)
    a = P.run_step(P.upload(wl, summary_dtype="fp16"), 512, "compkv", fused=True)
    b = P.run_step(P.upload(wl, summary_dtype="fp16"), 512, "compkv", fused=False)
    assert torch.equal(a.sel, b.sel) and torch.equal(a.out, b.out)
    c = P.run_step(P.upload(wl, summary_dtype="fp16"), 512, "compkv", fused=True)
    assert torch.equal(a.out, c.out) and torch.equal(a.scores, c.scores)


def test_fp16_append_equals_rebuild():
    wl = L32.with_(ctx_len=2048 + 19)
    run = P.upload(wl, summary_dtype="fp16")
    shape = run.shape
    T0 = 2048 - 13
    s = ck.empty_summaries(shape)
    ck.build_summaries(shape, run.Kd, run.Vd, s, torch.tensor([T0], dtype=torch.int32, device="cuda"))
    pos = torch.zeros(1, dtype=torch.int32, device="cuda")
    for t in range(T0, shape.ctx_len):
        pos.fill_(t)
        ck.append(shape, run.Kd[:, :, t].contiguous(), run.Vd[:, :, t].contiguous(), pos, s)
    ref = ck.empty_summaries(shape)
    ck.build_summaries(shape, run.Kd, run.Vd, ref)
    torch.cuda.synchronize()
    assert torch.equal(s.count, ref.count)
    for name in ("mean_k", "mean_v", "var_g"):
        a = getattr(s, name).double()
        b = getattr(ref, name).double()
        # each append rounds the running means to fp16: a few fp16 ulps after up to 16 appends
        assert float((a - b).abs().max() / b.abs().max()) <= 4e-3, name


def test_fp16_cost_against_fp32_full_128k():
    """The same 128K layer with fp32 and with fp16 summaries: the selections agree on most
    blocks, and the outputs agree within the output tolerance (sampled pairs against the oracle
    with fp16 storage too)."""
    tensors = synth.make_batch(L128)
    runs = {}
    for sd in ("fp32", "fp16"):
        run = P.upload(L128, tensors=tensors, summary_dtype=sd)
        runs[sd] = P.run_step(run, L128.budget, "compkv")
    a, b = runs["fp32"], runs["fp16"]
    overlap = np.mean([len(set(a.sel[0, g].tolist()) & set(b.sel[0, g].tolist())) / a.sel.shape[-1]
                       for g in range(L128.n_kv_heads)])
    diff = float((a.out - b.out).abs().max())
    print(f"fp16 vs fp32 summaries at 128K/512: selection overlap {overlap:.4f}, "
          f"max |out difference| {diff:.3e}")
    assert overlap >= 0.9
    assert diff <= P.OUT_ATOL
    P.check_step(b, L128.budget, "compkv", [(0, 0), (0, 5)])
