"""The allocation-free decode step (compkv_decode_step_static) through the C ABI.

Some callers cannot allocate device memory: an engine may own every allocation and hand this
library only its inputs and outputs, or allocating on the decode path may simply not be allowed.
For them the library keeps its scratch in a fixed device array of its own. This checks that the
entry point gives the same selection and outputs as the workspace-based compkv_decode_step, on two
calls in a row (the shared array keeps the first call's contents), and that a shape too large for
the array is refused before anything runs. It sorts last so a failure here leaves every other test
already run, and it passes both alone in a fresh process and after the rest of the suite.
"""
import ctypes

import pytest
import torch

import parity as P
from sparse_kv_cache_summaries_b200 import compkv as ck
from sparse_kv_cache_summaries_b200 import synth

pytestmark = pytest.mark.gpu


def test_static_scratch_step_matches_workspace_step():
    wl = synth.WORKLOADS["llama8b_32k_b512"].with_(ctx_len=16384 + 9)
    run = P.upload(wl)
    P.run_summaries(run)
    s = run.shape
    kb = ck.num_selected(s, wl.budget)
    ref_sel = torch.empty((1, s.n_kv_heads, kb), dtype=torch.int32, device="cuda")
    ref_out = torch.empty((1, s.n_q_heads, s.head_dim), device="cuda")
    ck.decode_step(s, run.qd, run.Kd, run.Vd, run.summ, wl.budget, ref_sel, ref_out,
                   ck.new_workspace(s, wl.budget))
    for _ in range(2):  # the second call runs on the scratch the first call left behind
        sel = torch.full_like(ref_sel, -1)
        out = torch.full_like(ref_out, float("nan"))
        ck.decode_step_static(s, run.qd, run.Kd, run.Vd, run.summ, wl.budget, sel, out)
        torch.cuda.synchronize()
        assert torch.equal(sel, ref_sel)
        assert ck.static_read_device_status() == 0
        err = (out - ref_out).abs()
        assert bool((err <= P.OUT_ATOL + P.OUT_RTOL * ref_out.abs()).all()), float(err.max())


def test_static_scratch_rejects_shapes_beyond_its_size():
    s = ck.LayerShape(batch=16, n_q_heads=32, n_kv_heads=8, head_dim=128, ctx_len=65536)
    assert ck.workspace_bytes(s, 1024) > 16 * 1024 * 1024
    dummy = torch.zeros(16, device="cuda")
    st = ck.lib().compkv_decode_step_static(ctypes.byref(s.c()), 0, 0, *[ctypes.c_void_p(dummy.data_ptr())] * 7,
                                            1024, 0.0, ctypes.c_void_p(dummy.data_ptr()), None,
                                            ctypes.c_void_p(dummy.data_ptr()), None)
    assert st == -4
