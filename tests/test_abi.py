"""The C-ABI library without a GPU: it loads, exports every function include/compkv.h declares,
and validates arguments on the host before any launch (no compute calls here)."""
import ctypes

import pytest

from sparse_kv_cache_summaries_b200 import build as B
from sparse_kv_cache_summaries_b200 import compkv as ck


@pytest.fixture(scope="module")
def lib():
    B.build()
    return ck.lib()


def test_exports_every_declared_function(lib):
    names = ck.header_functions()
    assert len(names) >= 12, names
    for name in names:
        assert hasattr(lib, name), f"{name} declared in include/compkv.h but not exported"


def test_version_and_status_strings(lib):
    assert ck.version() == 1
    assert ck.status_string(0) == "ok"
    assert "workspace" in ck.status_string(-4)
    assert ck.status_string(12345) == "unknown status"


def _shape(**kw):
    base = dict(batch=1, n_q_heads=32, n_kv_heads=8, head_dim=128, ctx_len=131072)
    base.update(kw)
    return ck.LayerShape(**base)


def test_num_selected_and_workspace(lib):
    s = _shape()
    assert ck.num_selected(s, 512) == 32
    assert ck.num_selected(s, 15) == 0
    assert ck.num_selected(_shape(ctx_len=100), 4096) == 7       # clamped to N_b
    ws = ck.workspace_bytes(s, 512)
    assert ws >= 256 + 8 * 4 * 130 * 4
    assert ck.full_workspace_bytes(s) > ws


@pytest.mark.parametrize("bad,status", [
    (dict(head_dim=96), -2), (dict(n_q_heads=12), -2), (dict(n_q_heads=24, n_kv_heads=8), -2),
    (dict(n_groups=3), -2), (dict(n_groups=256), -2), (dict(block_size=32), -2),
    (dict(batch=0), -1), (dict(ctx_len=0), -1),
])
def test_bad_shapes_rejected(lib, bad, status):
    s = _shape(**bad)
    assert lib.compkv_num_selected(ctypes.byref(s.c()), 512) == status
    assert ck.workspace_bytes(s, 512) == 0


def test_calls_validate_before_launch(lib):
    """Every rejected call returns before touching the device (fake pointers are never used)."""
    s = _shape().c()
    fake = ctypes.c_void_p(0x10000)          # 16-byte aligned, never dereferenced
    odd = ctypes.c_void_p(0x10008)           # 8-byte aligned only
    ws_need = lib.compkv_workspace_bytes(ctypes.byref(s), 512)
    # null query
    st = lib.compkv_score_select(ctypes.byref(s), 0, 0, None, fake, fake, fake, fake, 512, 0.0,
                                 fake, None, fake, ws_need, None)
    assert st == -1
    # misaligned q
    st = lib.compkv_score_select(ctypes.byref(s), 0, 0, odd, fake, fake, fake, fake, 512, 0.0,
                                 fake, None, fake, ws_need, None)
    assert st == -3
    # workspace too small
    st = lib.compkv_score_select(ctypes.byref(s), 0, 0, fake, fake, fake, fake, fake, 512, 0.0,
                                 fake, None, fake, ws_need - 1, None)
    assert st == -4
    # bad mode / dtype
    assert lib.compkv_score_select(ctypes.byref(s), 0, 7, fake, fake, fake, fake, fake, 512, 0.0,
                                   fake, None, fake, ws_need, None) == -1
    assert lib.compkv_score_select(ctypes.byref(s), 3, 0, fake, fake, fake, fake, fake, 512, 0.0,
                                   fake, None, fake, ws_need, None) == -1
    # mass-only selection with an empty budget has nothing to attend
    assert lib.compkv_score_select(ctypes.byref(s), 0, 1, fake, fake, fake, fake, fake, 8, 0.0,
                                   fake, None, fake, ws_need, None) == -1
    # negative budget
    assert lib.compkv_sparse_decode(ctypes.byref(s), 0, 0, fake, fake, fake, fake, fake, fake, fake,
                                    -16, 0.0, fake, fake, ws_need, None) == -1
    # decode_step checks K/V before launching score_select
    assert lib.compkv_decode_step(ctypes.byref(s), 0, 0, fake, None, fake, fake, fake, fake, fake,
                                  512, 0.0, fake, None, fake, fake, ws_need, None) == -1
    assert lib.compkv_decode_step(ctypes.byref(s), 0, 0, fake, odd, fake, fake, fake, fake, fake,
                                  512, 0.0, fake, None, fake, fake, ws_need, None) == -3
    # full decode
    fws = lib.compkv_full_workspace_bytes(ctypes.byref(s))
    assert lib.compkv_full_decode(ctypes.byref(s), 0, fake, fake, fake, None, 0.0, fake, fake,
                                  fws - 1, None) == -4
    assert lib.compkv_build_summaries(ctypes.byref(s), 0, fake, fake, None, fake, fake, odd, fake,
                                      None) == -3
    assert lib.compkv_read_device_status(None, None, None) == -1
